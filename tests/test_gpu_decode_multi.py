"""Multi-token decode: k tokens per row in one call give the same bits as k
single-token decode calls (the per-token arithmetic is the same and the state
stays f32 on chip), and match the float64 oracle, including a long-memory case
(decays near 1, write rates 1/2) where the state carries across the tokens."""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
import oracle
from gated_deltanet_mixer_gdn_b200 import synth

from _util import OUT_RMS_TOL, OUT_TOL, STATE_TOL, out_err, out_rms_err, state_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    return torch.device("cuda", 0)


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 8])
def test_decode_multi_equals_single_steps(dev, k):
    rows = 5
    case = synth.decode_case(5150 + k, rows=rows, steps=k)
    w = gdn.weights_to(case["weights"], dev)
    st1, cv1 = case["init_state"].to(dev), case["init_conv"].to(dev)
    st2, cv2 = st1.clone(), cv1.clone()
    outs = []
    for j in range(k):
        acts = {n: case[n][j].to(dev) for n in ("qkv", "z", "a", "b")}
        outs.append(gdn.decode(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st1, cv1))
    multi = {n: case[n].transpose(0, 1).contiguous().to(dev) for n in ("qkv", "z", "a", "b")}  # [rows, k, ...]
    out = gdn.decode_multi(multi["qkv"], multi["z"], multi["a"], multi["b"], w, st2, cv2)
    torch.cuda.synchronize(dev)
    assert torch.equal(out, torch.stack(outs, dim=1))
    assert torch.equal(st2, st1) and torch.equal(cv2, cv1)


def test_decode_multi_matches_oracle(dev):
    rows, k = 3, 4
    case = synth.decode_case(5160, rows=rows, steps=k)
    w = gdn.weights_to(case["weights"], dev)
    st, cv = case["init_state"].to(dev), case["init_conv"].to(dev)
    f = synth.to_f64
    st0, cv0 = f(case["init_state"]), f(case["init_conv"])
    multi = {n: case[n].transpose(0, 1).contiguous() for n in ("qkv", "z", "a", "b")}
    out = gdn.decode_multi(*(multi[n].to(dev) for n in ("qkv", "z", "a", "b")), w, st, cv)
    torch.cuda.synchronize(dev)
    wt = case["weights"]
    cu = np.arange(rows + 1) * k
    ref = oracle.mixer(case["dims"], cu, *(f(multi[n].reshape(rows * k, -1)) for n in ("qkv", "z", "a", "b")),
                       f(wt["conv_w"]), f(wt["A_log"]), f(wt["dt_bias"]), f(wt["norm_w"]), st0, cv0)
    y = ref["out"].reshape(rows * k, -1)
    assert out_err(out.reshape(rows * k, -1), y) <= OUT_TOL
    assert out_rms_err(out.reshape(rows * k, -1), y) <= OUT_RMS_TOL
    assert state_err(st, ref["state"]) <= STATE_TOL
    assert np.array_equal(cv.double().cpu().numpy().reshape(ref["conv"].shape), ref["conv"])


@pytest.mark.parametrize("k", [4, 8])
def test_decode_multi_long_memory_matches_oracle(dev, k):
    rows = 4
    case = synth.decode_case(5170 + k, rows=rows, steps=k)
    case["weights"]["A_log"] = torch.zeros_like(case["weights"]["A_log"])        # g = -softplus(a - 5)
    case["weights"]["dt_bias"] = torch.full_like(case["weights"]["dt_bias"], -5.0)
    case["b"] = torch.zeros_like(case["b"])                                      # beta = 1/2
    w = gdn.weights_to(case["weights"], dev)
    st, cv = case["init_state"].to(dev), case["init_conv"].to(dev)
    f = synth.to_f64
    st0, cv0 = f(case["init_state"]), f(case["init_conv"])
    multi = {n: case[n].transpose(0, 1).contiguous() for n in ("qkv", "z", "a", "b")}
    out = gdn.decode_multi(*(multi[n].to(dev) for n in ("qkv", "z", "a", "b")), w, st, cv)
    torch.cuda.synchronize(dev)
    wt = case["weights"]
    cu = np.arange(rows + 1) * k
    ref = oracle.mixer(case["dims"], cu, *(f(multi[n].reshape(rows * k, -1)) for n in ("qkv", "z", "a", "b")),
                       f(wt["conv_w"]), f(wt["A_log"]), f(wt["dt_bias"]), f(wt["norm_w"]), st0, cv0)
    y = ref["out"].reshape(rows * k, -1)
    assert out_err(out.reshape(rows * k, -1), y) <= OUT_TOL
    assert out_rms_err(out.reshape(rows * k, -1), y) <= OUT_RMS_TOL
    assert state_err(st, ref["state"]) <= STATE_TOL
