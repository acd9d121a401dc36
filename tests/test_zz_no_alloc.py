"""gdn_prefill_noalloc: the prefill for callers that cannot call cudaMalloc
(an engine plugin whose host owns every device allocation, or a path that
must not take an allocation's implicit device synchronisation).  Its scratch is
a fixed device array inside the library, so the test checks that two calls in
a row, with different inputs, give the same results as gdn_prefill with a
caller-allocated workspace, that each call leaves the device's free memory
unchanged, and that a request beyond the fixed capacity is refused.  The file sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import synth

from _util import OUT_RMS_TOL, OUT_TOL, STATE_TOL, out_err, out_rms_err, state_err

pytestmark = pytest.mark.gpu

GDN_ERR_WORKSPACE = -4


def _noalloc_fn():
    lib = gdn.load_library()
    fn = lib.gdn_prefill_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(gdn._DimsC), ctypes.POINTER(gdn._WeightsC), i32, i32,
                   vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    return fn


def _call_noalloc(fn, B, T, w, acts, st, cv, out, fs, fc):
    dc = gdn._dims_c(synth.MODEL)
    wc = gdn._weights_c(w, out.device)
    p = gdn._ptr
    return fn(ctypes.byref(dc), ctypes.byref(wc), B, T, p(acts["qkv"]), p(acts["z"]), p(acts["a"]), p(acts["b"]),
              p(st), p(cv), p(out), p(fs), p(fc), gdn._stream(out.device))


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    return torch.device("cuda", 0)


def test_noalloc_two_calls_match_workspace_entry_point(dev):
    fn = _noalloc_fn()
    for call, (seed, B, T) in enumerate(((9001, 2, 300), (9002, 3, 129))):
        case = synth.dense_case(seed, B=B, T=T, init=True)
        w = gdn.weights_to(case["weights"], dev)
        acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
        st = case["init_state"].to(dev)
        cv = case["init_conv"].to(dev)
        ref_out, ref_st, ref_cv = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
        out = torch.empty_like(ref_out)
        fs = torch.empty_like(ref_st)
        fc = torch.empty_like(ref_cv)
        # the library is loaded (the reference call above ran the same kernels), so the call
        # itself must leave the device's free memory exactly as it was
        torch.cuda.synchronize(dev)
        free_before = torch.cuda.mem_get_info(dev)[0]
        status = _call_noalloc(fn, B, T, w, acts, st, cv, out, fs, fc)
        assert status == 0, gdn.status_string(status)
        torch.cuda.synchronize(dev)
        assert torch.cuda.mem_get_info(dev)[0] == free_before, f"call {call} changed the free device memory"
        ref64 = ref_out.double().cpu().numpy()
        assert out_err(out, ref64) <= OUT_TOL, f"call {call}"
        assert out_rms_err(out, ref64) <= OUT_RMS_TOL, f"call {call}"
        assert state_err(fs, ref_st.double().cpu().numpy()) <= STATE_TOL, f"call {call}"
        assert torch.equal(fc, ref_cv), f"call {call}"


def test_noalloc_rejects_requests_beyond_its_scratch(dev):
    fn = _noalloc_fn()
    case = synth.dense_case(9003, B=1, T=4)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    out = torch.empty((1, 4, 6144), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, 48, 128, 128), dtype=torch.float32, device=dev)
    fc = torch.empty((1, 3, 10240), dtype=torch.float32, device=dev)
    # 1 row of 1217 tokens needs more than the 64 MiB of fixed scratch (1216 is the most
    # one row gets); refused before any launch
    lib = gdn.load_library()
    size = lib.gdn_prefill_workspace_size
    size.restype = ctypes.c_size_t
    dc = gdn._dims_c(synth.MODEL)
    assert size(ctypes.byref(dc), 1, 1216) <= 64 * 1024 * 1024 < size(ctypes.byref(dc), 1, 1217)
    status = _call_noalloc(fn, 1, 1217, w, acts, None, None, out, fs, fc)
    assert status == GDN_ERR_WORKSPACE
