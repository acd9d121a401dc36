"""The mixer followed by out_proj in one call (gdn_prefill_out): the gated-norm
output times out_proj (Qwen/Qwen3.8-27B architecture page, module tree:
out_proj 5120x6144), with each recurrence segment's projection overlapped with
the later segments' recurrence.  Compared with the float64 oracle (mixer, then
projection of its output) and, bit for bit, with prefill followed by out_proj."""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
import oracle
from gated_deltanet_mixer_gdn_b200 import synth

from _util import check_outputs, oracle_prefill, to_dev

pytestmark = pytest.mark.gpu

HIDDEN = 5120


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    gdn.load_library()


def _w_out(seed, dev):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((HIDDEN, 6144), generator=g) * 6144 ** -0.5).to(torch.bfloat16).to(dev)


@pytest.mark.parametrize("B,T,overlapped", [(2, 300, False), (1, 2048, True)])
def test_prefill_out_against_oracle_and_unfused(B, T, overlapped):
    case = synth.dense_case(5100 + T, B=B, T=T, init=True)
    w, acts, st, cv = to_dev(case)
    w_out = _w_out(T, "cuda")
    assert (gdn.prefill_schedule(B, T)[0] > 1) == overlapped
    out, fs, fc = gdn.prefill_out(acts["qkv"], acts["z"], acts["a"], acts["b"], w, w_out, st, cv)
    y, fs2, fc2 = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    ref_pair = gdn.out_proj(y.reshape(B * T, -1), w_out)
    torch.cuda.synchronize()
    assert torch.equal(out.reshape(B * T, -1), ref_pair), "not the bits of prefill + out_proj"
    assert torch.equal(fs, fs2) and torch.equal(fc, fc2)
    ref = oracle_prefill(case)
    ref_out = oracle.projection(ref["out"], w_out.double().cpu().numpy())
    check_outputs(f"prefill + out_proj B={B} T={T}", out.reshape(B * T, -1), ref_out, fs, ref["state"], fc,
                  ref["conv"])
    assert gdn.last_device_error() == 0
