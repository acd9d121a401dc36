"""Host-side checks of the C ABI that need no GPU: the library loads and exports
every function include/gdn.h declares, the workspace queries, and argument
validation (all rejected before any CUDA call is made)."""
import ctypes
import os
import re

import pytest

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gdn.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert set(names) == set(gdn.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.gdn_version() >= 100
    assert gdn.status_string(0) == "ok"
    assert "workspace" in gdn.status_string(-4)


def _dims(kh=16, vh=48, d=128, w=4):
    return gdn._DimsC(kh, vh, d, w)


def test_workspace_sizes(lib):
    d = _dims()
    one = lib.gdn_prefill_workspace_size(ctypes.byref(d), 1, 1)
    big = lib.gdn_prefill_workspace_size(ctypes.byref(d), 2, 1000)
    # per token: q, k and their residual parts (f16), v (f16), gates; per 64-token chunk
    # and value head a 33,296-byte record of the chunked form
    assert one > 0 and big >= 2000 * (4 * 16 * 128 * 2 + 48 * 128 * 2 + 2 * 48 * 4) + 2 * 16 * 48 * 33280
    # packed rows are planned for the most chunks N rows of 2000 tokens can have
    assert lib.gdn_prefill_varlen_workspace_size(ctypes.byref(d), 2, 2000) >= big
    assert lib.gdn_prefill_varlen_workspace_size(ctypes.byref(d), 3, 2000) >= \
        lib.gdn_prefill_varlen_workspace_size(ctypes.byref(d), 2, 2000)
    assert lib.gdn_prefill_workspace_size(ctypes.byref(_dims(d=64)), 1, 10) == 0
    assert lib.gdn_prefill_workspace_size(ctypes.byref(d), -1, 10) == 0


def test_unsupported_dims_rejected(lib):
    w = gdn._WeightsC(16, 16, 16, 16)
    for bad, code in ((_dims(d=64), -2), (_dims(w=3), -2), (_dims(kh=5, vh=48), -2), (_dims(kh=1, vh=16), -2),
                      (_dims(kh=0), -1)):
        st = lib.gdn_decode(ctypes.byref(bad), ctypes.byref(w), 1, *([None] * 7), None)
        assert st == code


def test_invalid_arguments_rejected(lib):
    d = _dims()
    w = gdn._WeightsC(16, 16, 16, 16)
    # null weights
    assert lib.gdn_decode(ctypes.byref(d), None, 1, *([None] * 7), None) == -1
    # null buffers with rows > 0
    assert lib.gdn_decode(ctypes.byref(d), ctypes.byref(w), 2, *([None] * 7), None) == -1
    # misaligned state pointer
    assert lib.gdn_decode(ctypes.byref(d), ctypes.byref(w), 2, 16, 16, 16, 16, 8, 16, 16, None) == -1
    # rows < 0
    assert lib.gdn_decode(ctypes.byref(d), ctypes.byref(w), -1, *([None] * 7), None) == -1
    # varlen: cu_seqlens not starting at 0 / decreasing / wrong total
    for cu, total in (([1, 5], 5), ([0, 5, 3], 3), ([0, 4], 5)):
        arr = (ctypes.c_int32 * len(cu))(*cu)
        st = lib.gdn_prefill_varlen(ctypes.byref(d), ctypes.byref(w), len(cu) - 1, arr, 16, total,
                                    16, 16, 16, 16, None, None, 16, None, None, 16, 1 << 30, None)
        assert st == -1
    # prefill: negative T
    assert lib.gdn_prefill(ctypes.byref(d), ctypes.byref(w), 1, -3, *([16] * 4), None, None, 16, None, None,
                           16, 1 << 30, None) == -1


def test_projection_and_hidden_arguments_checked_on_host(lib):
    d = _dims()
    w = gdn._WeightsC(16, 16, 16, 16)
    # contraction width not a multiple of 64: unsupported, before any CUDA call
    assert lib.gdn_in_proj(ctypes.byref(d), 8, 100, 16, 16, 16, 16, 16, 16, None) == -2
    assert lib.gdn_out_proj(ctypes.byref(d), -8, 128, 16, 16, 16, None) == -1
    assert lib.gdn_prefill_hidden(ctypes.byref(d), ctypes.byref(w), 1, 8, 100, 16, 16, None, None, 16, None,
                                  None, 16, 1 << 30, None) == -2
    # negative sizes, null hidden states, null weights
    assert lib.gdn_prefill_hidden(ctypes.byref(d), ctypes.byref(w), -1, 8, 128, 16, 16, None, None, 16, None,
                                  None, 16, 1 << 30, None) == -1
    assert lib.gdn_prefill_hidden(ctypes.byref(d), ctypes.byref(w), 1, 8, 128, None, 16, None, None, 16, None,
                                  None, 16, 1 << 30, None) == -1
    assert lib.gdn_prefill_hidden(ctypes.byref(d), None, 1, 8, 128, 16, 16, None, None, 16, None,
                                  None, 16, 1 << 30, None) == -1
    # misaligned hidden states
    assert lib.gdn_prefill_hidden(ctypes.byref(d), ctypes.byref(w), 1, 8, 128, 8, 16, None, None, 16, None,
                                  None, 16, 1 << 30, None) == -1
    # the hidden-state prefill's workspace holds the prefill's, z and the staged histories
    ws = lib.gdn_prefill_hidden_workspace_size(ctypes.byref(d), 2, 1000)
    assert ws >= lib.gdn_prefill_workspace_size(ctypes.byref(d), 2, 1000) + 2000 * 6144 * 2 + 2 * 3 * 10240 * 4
    # head counts the fused tiles do not cover (odd value-head count) take the unfused launches:
    # room for qkv, z, a, b as well
    d_odd = _dims(kh=1, vh=3)
    C_odd = (2 + 3) * 128
    assert lib.gdn_prefill_hidden_workspace_size(ctypes.byref(d_odd), 4, 2) >= \
        lib.gdn_prefill_workspace_size(ctypes.byref(d_odd), 4, 2) + 8 * (C_odd + 3 * 128 + 6) * 2
    # packed rows: the packed prefill's workspace, z and the staged histories
    assert lib.gdn_prefill_hidden_varlen_workspace_size(ctypes.byref(d), 3, 1000) >= \
        lib.gdn_prefill_varlen_workspace_size(ctypes.byref(d), 3, 1000) + 1000 * 6144 * 2 + 3 * 3 * 10240 * 4
    for cu, total in (([1, 5], 5), ([0, 5, 3], 3), ([0, 4], 5)):
        arr = (ctypes.c_int32 * len(cu))(*cu)
        assert lib.gdn_prefill_hidden_varlen(ctypes.byref(d), ctypes.byref(w), len(cu) - 1, arr, 16, total, 128,
                                             16, 16, None, None, 16, None, None, 16, 1 << 30, None) == -1
    # the schedule query: null outputs, negative sizes
    seg, lau = ctypes.c_int32(-7), ctypes.c_int32(-7)
    assert lib.gdn_prefill_schedule(ctypes.byref(d), 1, 8192, 0, None, None) == -1
    assert lib.gdn_prefill_schedule(ctypes.byref(d), -1, 8192, 0, ctypes.byref(seg), ctypes.byref(lau)) == -1
    assert lib.gdn_prefill_schedule(ctypes.byref(d), 0, 8192, 0, ctypes.byref(seg), ctypes.byref(lau)) == 0
    assert (seg.value, lau.value) == (0, 0)


def test_slot_tables_checked_on_host(lib):
    # a slot twice, a slot past the pool, a negative slot, an empty pool: refused before any launch
    d = _dims()
    w = gdn._WeightsC(16, 16, 16, 16)
    for slots, pool in (([0, 0], 4), ([0, 4], 4), ([-1, 2], 4), ([0, 1], 0)):
        arr = (ctypes.c_int32 * 2)(*slots)
        assert lib.gdn_decode_slots(ctypes.byref(d), ctypes.byref(w), 2, arr, 16, pool, *([16] * 4), 16, 16, 16,
                                    None) == -1
        cu = (ctypes.c_int32 * 3)(0, 3, 5)
        assert lib.gdn_prefill_varlen_slots(ctypes.byref(d), ctypes.byref(w), 2, cu, 16, 5, arr, 16, pool,
                                            *([16] * 4), 16, 16, 16, 16, 1 << 30, None) == -1


def test_binding_refuses_cpu_tensors():
    import torch
    from gated_deltanet_mixer_gdn_b200 import synth
    case = synth.dense_case(1, 1, 4)
    with pytest.raises(gdn.GdnError):
        gdn.prefill(case["qkv"], case["z"], case["a"], case["b"], case["weights"])


def test_schedule_for_a_given_sm_count(lib):
    """The segment planner of the dense prefill, on the host for a given SM count: the recurrence
    runs on CTA pairs when 2 rows x heads fit the SMs, overlaps only when its CTAs leave 32 SMs and
    rows hold 16 chunks, and one call launches 2 + 2 x segments kernels."""
    def plan(B, T, nsm, from_hidden=False):
        return gdn.prefill_schedule(B, T, from_hidden, nsm=nsm)

    # B200 (148 SMs): one row on pairs (96 CTAs) overlaps in 3 segments; two rows on one CTA per
    # head (96 CTAs) in 5; three rows (144 CTAs) leave too few SMs; short rows stay plain
    assert plan(1, 8192, 148) == (3, 8)
    assert plan(2, 65536, 148) == (5, 12)
    assert plan(3, 8192, 148) == (1, 4)
    assert plan(1, 15 * 64, 148) == (1, 4)
    # 100 SMs: one row still fits as pairs (96) but then leaves only 4 SMs: plain; 95 SMs: one CTA
    # per head (48) and overlap
    assert plan(1, 8192, 100) == (1, 4)
    assert plan(1, 8192, 95) == (4, 10)
    # the fused in_proj path launches the same number (its GEMM replaces the load stage)
    assert plan(1, 8192, 148, from_hidden=True) == (3, 8)
    for B, T in ((1, 1), (1, 64), (2, 4096), (4, 8192), (1, 65536)):
        s, n = plan(B, T, 148)
        assert 1 <= s <= 8 and n == 2 + 2 * s
    assert plan(0, 8192, 148) == (0, 0) and plan(1, 0, 148) == (0, 0)
    d = _dims()
    seg, lau = ctypes.c_int32(-7), ctypes.c_int32(-7)
    assert lib.gdn_prefill_schedule_nsm(ctypes.byref(d), 1, 8192, 0, 0, ctypes.byref(seg), ctypes.byref(lau)) == -1
    assert lib.gdn_prefill_schedule_nsm(ctypes.byref(d), -1, 8192, 0, 148, ctypes.byref(seg), ctypes.byref(lau)) == -1
    assert lib.gdn_prefill_schedule_nsm(ctypes.byref(d), 1, 8192, 0, 148, None, None) == -1
