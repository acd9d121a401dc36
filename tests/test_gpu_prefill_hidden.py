"""Prefill from the hidden states (gdn_prefill_hidden: the load stage inside the
in_proj GEMM's epilogue) against the unfused pair gdn_in_proj + gdn_prefill.

The fused epilogue replays the load stage's arithmetic in the same order (the
projection rounded to bf16, the width-4 conv as the same chain of fused
multiply-adds, silu, the L2 norm summed in the order of the load stage's warp
reduction, the f16 hi/lo split, the gates), so outputs, final states and
histories must be bit-identical: across the fused tiles' 125-token steps, rows
that start and end inside a tile, rows with and without a history, in place,
rows shorter than the conv window, and packed rows (prefill_hidden_varlen against
in_proj + prefill_varlen).  One small case also goes through the oracle (projection,
then the mixer).
"""
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
    gdn.load_library()
    return torch.device("cuda", 0)


def _case(seed, B, T, hidden, init):
    dims = synth.MODEL
    gen = torch.Generator().manual_seed(seed)
    w = synth.draw_weights(gen, dims)
    n_in = dims.conv_channels + dims.value_width + 2 * dims.num_v_heads
    x = torch.randn((B, T, hidden), generator=gen).to(torch.bfloat16)
    w_in = (torch.randn((n_in, hidden), generator=gen) * hidden ** -0.5).to(torch.bfloat16)
    st = synth.draw_state(gen, B, dims) if init else None
    cv = synth.draw_history(gen, B, dims) if init else None
    return w, x, w_in, st, cv


def _unfused(dev, w, x, w_in, st, cv):
    B, T, hidden = x.shape
    qkv, z, a, b = gdn.in_proj(x.reshape(B * T, hidden), w_in)
    sh = lambda t: t.reshape(B, T, -1)
    return gdn.prefill(sh(qkv), sh(z), sh(a), sh(b), w, st, cv)


@pytest.mark.parametrize("B,T,hidden,init", [
    (1, 300, 256, False),   # three fused tiles, ragged last one, zero history
    (3, 130, 128, True),    # rows start and end inside tiles (tiles step 125 tokens)
    (5, 3, 64, True),       # rows of exactly the conv window
    (2, 2, 64, True),       # rows shorter than the conv window: history partly the initial one
    (1, 1, 64, False),
    (2, 1000, 512, True),   # several 64-token chunks per row; overlapped schedule
])
def test_bit_identical_to_unfused(dev, B, T, hidden, init):
    w, x, w_in, st, cv = _case(B * 1000 + T + hidden, B, T, hidden, init)
    wd = gdn.weights_to(w, dev)
    xd, wid = x.to(dev), w_in.to(dev)
    std = st.to(dev) if st is not None else None
    cvd = cv.to(dev) if cv is not None else None
    ref = _unfused(dev, wd, xd, wid, std, cvd)
    got = gdn.prefill_hidden(xd, wid, wd, std, cvd)
    torch.cuda.synchronize(dev)
    for g, r, name in zip(got, ref, ("out", "final_state", "final_conv")):
        assert torch.equal(g, r), f"{name} differs from in_proj + prefill"
    assert gdn.last_device_error() == 0


def test_in_place_states(dev):
    B, T, hidden = 2, 700, 256
    w, x, w_in, st, cv = _case(77, B, T, hidden, True)
    wd = gdn.weights_to(w, dev)
    xd, wid = x.to(dev), w_in.to(dev)
    ref = _unfused(dev, wd, xd, wid, st.to(dev), cv.to(dev))
    std, cvd = st.to(dev), cv.to(dev)
    out, fs, fc = gdn.prefill_hidden(xd, wid, wd, std, cvd, in_place=True)
    torch.cuda.synchronize(dev)
    assert fs.data_ptr() == std.data_ptr() and fc.data_ptr() == cvd.data_ptr()
    assert torch.equal(out, ref[0]) and torch.equal(std, ref[1]) and torch.equal(cvd, ref[2])


@pytest.mark.parametrize("lengths,init", [
    ([0, 1, 2, 3, 130, 300, 5], True),     # empty and short rows, rows across tiles
    ([64, 200, 1], False),
    ([700, 0, 450], True),
])
def test_varlen_bit_identical_to_unfused(dev, lengths, init):
    hidden = 256
    total = sum(lengths)
    w, x, w_in, st, cv = _case(sum(lengths) + len(lengths), 1, total, hidden, False)
    gen = torch.Generator().manual_seed(len(lengths) * 7)
    N = len(lengths)
    st = synth.draw_state(gen, N, synth.MODEL) if init else None
    cv = synth.draw_history(gen, N, synth.MODEL) if init else None
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    wd = gdn.weights_to(w, dev)
    xd, wid = x[0].to(dev), w_in.to(dev)
    std = st.to(dev) if st is not None else None
    cvd = cv.to(dev) if cv is not None else None
    qkv, z, a, b = gdn.in_proj(xd, wid)
    ref = gdn.prefill_varlen(cu, qkv, z, a, b, wd, std, cvd)
    got = gdn.prefill_hidden_varlen(cu, xd, wid, wd, std, cvd)
    torch.cuda.synchronize(dev)
    for g, r, name in zip(got, ref, ("out", "final_state", "final_conv")):
        assert torch.equal(g, r), f"{name} differs from in_proj + prefill_varlen"
    # in place
    std2, cvd2 = (st.to(dev), cv.to(dev)) if init else (None, None)
    if init:
        gdn.prefill_hidden_varlen(cu, xd, wid, wd, std2, cvd2, in_place=True)
        torch.cuda.synchronize(dev)
        assert torch.equal(std2, ref[1]) and torch.equal(cvd2, ref[2])
    assert gdn.last_device_error() == 0


def test_layer_shape_bit_identical(dev):
    """One row of 8192 tokens through the 27B layer's in_proj (5120 -> 16480)."""
    w, x, w_in, st, cv = _case(5, 1, 8192, 5120, True)
    wd = gdn.weights_to(w, dev)
    xd, wid = x.to(dev), w_in.to(dev)
    ref = _unfused(dev, wd, xd, wid, st.to(dev), cv.to(dev))
    got = gdn.prefill_hidden(xd, wid, wd, st.to(dev), cv.to(dev))
    torch.cuda.synchronize(dev)
    for g, r in zip(got, ref):
        assert torch.equal(g, r)
    assert gdn.last_device_error() == 0


def test_against_oracle(dev):
    """Projection in float64, rounded to bf16 (the activations' dtype between in_proj and
    the mixer), then the oracle's mixer; the fused path within the mixer's bars."""
    B, T, hidden = 2, 200, 256
    dims = synth.MODEL
    w, x, w_in, st, cv = _case(31, B, T, hidden, True)
    out, fs, fc = gdn.prefill_hidden(x.to(dev), w_in.to(dev), gdn.weights_to(w, dev), st.to(dev), cv.to(dev))
    torch.cuda.synchronize(dev)
    proj = oracle.projection(x.reshape(B * T, hidden).double().numpy(), w_in.double().numpy())
    proj = torch.from_numpy(proj).to(torch.bfloat16).double().numpy()
    C, VD, Vh = dims.conv_channels, dims.value_width, dims.num_v_heads
    qkv, z, b, a = proj[:, :C], proj[:, C:C + VD], proj[:, C + VD:C + VD + Vh], proj[:, C + VD + Vh:]
    f = synth.to_f64
    ref = oracle.mixer(dims, np.arange(B + 1) * T, qkv, z, a, b, f(w["conv_w"]), f(w["A_log"]),
                       f(w["dt_bias"]), f(w["norm_w"]), st.numpy().astype(np.float64),
                       cv.numpy().astype(np.float64))
    assert out_err(out, ref["out"]) <= OUT_TOL
    assert out_rms_err(out, ref["out"]) <= OUT_RMS_TOL
    assert state_err(fs, ref["state"]) <= STATE_TOL
    # the history holds the projection's bf16 values: the GPU's f32 sum and the float64 one
    # may round to neighbouring bf16 values (one unit in the last place is <= 2^-7 relative)
    fc64 = fc.double().cpu().numpy().reshape(ref["conv"].shape)
    assert np.all(np.abs(fc64 - ref["conv"]) <= 2.0 ** -7 * np.abs(ref["conv"]))
