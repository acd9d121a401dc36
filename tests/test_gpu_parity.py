"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Every test draws seeded synthetic inputs, runs the B200 kernels through the
Python binding of include/gdn.h, runs the float64 oracle on the same bits, and
compares element by element: outputs within 2e-2 relative error (elements
below the output RMS measured against the RMS), final states within 1e-3
relative Frobenius error per row, conv histories bit-exact.
"""
import math

import numpy as np
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import synth

from _util import (OUT_RMS_TOL, OUT_TOL, STATE_TOL, check_outputs, conv_exact, group_case, oracle_prefill,
                   out_err, out_rms_err, record, state_err, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    gdn.load_library()


def _check_prefill(case, res, ref, name="prefill"):
    out, fs, fc = res
    r = check_outputs(name, out, ref["out"], fs, ref["state"], fc, ref["conv"])
    assert gdn.last_device_error() == 0
    return r


# ---------------------------------------------------------------- decode

def test_decode_small_chain():
    case = synth.decode_case(101, rows=5, steps=4)
    w, _, st, cv = to_dev(case)
    st_ref, cv_ref = case["init_state"], case["init_conv"]
    for s in range(4):
        acts = {k: case[k][s] for k in ("qkv", "z", "a", "b")}
        out = gdn.decode(*(acts[k].cuda() for k in ("qkv", "z", "a", "b")), w, st, cv)
        ref = oracle_prefill(case, cu=np.arange(6), init_state=st_ref, init_conv=cv_ref, acts=acts)
        assert out_err(out, ref["out"]) <= OUT_TOL
        assert state_err(st, ref["state"]) <= STATE_TOL
        assert conv_exact(cv, ref["conv"])
        st_ref, cv_ref = ref["state"], ref["conv"]
    assert gdn.last_device_error() == 0


def test_decode_batch_all_steps_every_group():
    """The decode batch exactly as benchmarked (64 rows x 128 steps, seed of the decode
    workload): every step's output, the final states and histories.  Row r is compared on
    the 3 value heads of q/k head r % 16, so every q/k group of the 64-row persistent grid is
    checked on 4 rows; the oracle runs each row's 128 tokens as one chain (decode = prefill
    token by token)."""
    case = synth.config(1)
    steps, rows = case["qkv"].shape[0], case["qkv"].shape[1]
    w, _, st, cv = to_dev(case)
    outs = torch.empty((steps, rows, 6144), dtype=torch.bfloat16, device="cuda")
    for s in range(steps):
        gdn.decode(*(case[k][s].cuda() for k in ("qkv", "z", "a", "b")), w, st, cv, out=outs[s])
    torch.cuda.synchronize()
    outs, st, cv = outs.cpu(), st.cpu(), cv.cpu()
    worst = {"out": 0.0, "out_rms": 0.0, "state": 0.0}
    for kap in range(16):
        R = [r for r in range(rows) if r % 16 == kap]
        sub = group_case(case, kap)
        acts = {k: sub[k][:, R].transpose(0, 1).reshape(len(R) * steps, -1) for k in ("qkv", "z", "a", "b")}
        ref = oracle_prefill(sub, cu=np.arange(len(R) + 1) * steps, init_state=sub["init_state"][R],
                             init_conv=sub["init_conv"][R], acts=acts)
        y = outs[:, R].index_select(2, sub["z_channels"]).transpose(0, 1).reshape(len(R) * steps, -1)
        e_out, e_rms = out_err(y, ref["out"]), out_rms_err(y, ref["out"])
        e_st = state_err(st[R].index_select(1, sub["heads"]), ref["state"])
        worst = {"out": max(worst["out"], e_out), "out_rms": max(worst["out_rms"], e_rms),
                 "state": max(worst["state"], e_st)}
        assert e_out <= OUT_TOL and e_rms <= OUT_RMS_TOL, f"group {kap}: output {e_out:.3e} / rms {e_rms:.3e}"
        assert e_st <= STATE_TOL, f"group {kap}: state {e_st:.3e}"
        assert conv_exact(cv[R].index_select(2, sub["channels"]), ref["conv"]), f"group {kap}: history"
    record("decode batch 64x128, all groups", **worst)
    assert gdn.last_device_error() == 0


def test_decode_split_groups_bit_identical():
    """Batches small enough for one CTA per value head in one wave (at most 3 rows here) run
    each q/k group as a cluster of one-value-head CTAs (the first shifts the shared q/k
    history once the others hold it); the results are the same bits as the persistent
    grouping: 6 rows at once against 3 + 2 + 1, over 3 steps."""
    case = synth.decode_case(777, rows=6, steps=3)
    w, _, st, cv = to_dev(case)
    st2, cv2 = st.clone(), cv.clone()
    for s in range(3):
        acts = [case[k][s].cuda() for k in ("qkv", "z", "a", "b")]
        o_all = gdn.decode(*acts, w, st, cv)
        parts = []
        for lo, hi in ((0, 3), (3, 5), (5, 6)):
            parts.append(gdn.decode(*(t[lo:hi] for t in acts), w, st2[lo:hi], cv2[lo:hi]))
        torch.cuda.synchronize()
        assert torch.equal(o_all, torch.cat(parts))
    assert torch.equal(st, st2) and torch.equal(cv, cv2)
    assert gdn.last_device_error() == 0


def test_decode_zero_rows_is_noop():
    case = synth.decode_case(3, rows=1, steps=1)
    w, _, st, cv = to_dev(case)
    e = torch.empty((0, 10240), dtype=torch.bfloat16, device="cuda")
    out = gdn.decode(e, e.new_empty((0, 6144)), e.new_empty((0, 48)), e.new_empty((0, 48)), w,
                     st[:0], cv[:0])
    assert out.shape == (0, 6144)


# ---------------------------------------------------------------- dense prefill

def test_prefill_small_config():
    case = synth.config(0)  # B=1, T=256, zero initial state
    w, acts, _, _ = to_dev(case)
    res = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w)
    torch.cuda.synchronize()
    _check_prefill(case, res, oracle_prefill(case), "prefill B=1 T=256 (all heads)")


# one row: the recurrence on CTA pairs (each 64 of a head's value channels); two rows: one CTA
# per (row, value head)
@pytest.mark.parametrize("B", [1, 2])
@pytest.mark.parametrize("T", [1, 2, 3, 63, 64, 65, 127, 200])
def test_prefill_ragged_lengths_with_state(T, B):
    case = synth.dense_case(500 + T + (1000 if B == 1 else 0), B=B, T=T, init=True)
    w, acts, st, cv = to_dev(case)
    res = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    torch.cuda.synchronize()
    _check_prefill(case, res, oracle_prefill(case))


def test_prefill_long_memory_family():
    """g ~ -7e-3 per token: the state carries across many chunks."""
    case = synth.dense_case(77, B=1, T=600, init=True, long_memory=True)
    w, acts, st, cv = to_dev(case)
    res = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    torch.cuda.synchronize()
    _check_prefill(case, res, oracle_prefill(case), "prefill long-memory T=600")


@pytest.mark.parametrize("B", [1, 2])
def test_prefill_in_place_state(B):
    case = synth.dense_case(78 if B == 2 else 178, B=B, T=130, init=True)
    ref = oracle_prefill(case)
    w, acts, st, cv = to_dev(case)
    out, fs, fc = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv, in_place=True)
    torch.cuda.synchronize()
    assert fs.data_ptr() == st.data_ptr() and fc.data_ptr() == cv.data_ptr()
    _check_prefill(case, (out, fs, fc), ref)


def test_prefill_no_decay_no_write_keeps_state_exactly():
    case = synth.dense_case(79, B=1, T=100, init=True)
    case["a"] = torch.full_like(case["a"], -math.inf)
    case["b"] = torch.full_like(case["b"], -math.inf)
    w, acts, st, cv = to_dev(case)
    _, fs, _ = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    torch.cuda.synchronize()
    assert torch.equal(fs, st)


def test_prefill_zero_tokens_copies_state():
    case = synth.dense_case(80, B=2, T=0, init=True)
    w, acts, st, cv = to_dev(case)
    out, fs, fc = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(fs, st) and torch.equal(fc, cv)


# ---------------------------------------------------------------- varlen prefill

def test_varlen_ragged_rows():
    lengths = [0, 1, 3, 70, 130, 64, 2]
    case = synth.prefill_case(81, lengths, init=True)
    w, acts, st, cv = to_dev(case)
    res = gdn.prefill_varlen(case["cu_seqlens"], acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    torch.cuda.synchronize()
    _check_prefill(case, res, oracle_prefill(case))


@pytest.mark.parametrize("n", [1500, 2100])
def test_varlen_many_short_rows(n):
    """Thousands of packed rows of 0-5 tokens and one of 200: the recurrence launches rows
    longest first (a device-side sort up to 2048 rows, the identity above), which must not
    change any row's result.  Oracle on value head 0 (zero initial state and history)."""
    rng = np.random.default_rng(n)
    lengths = [int(x) for x in rng.integers(0, 6, n)]
    lengths[n // 3] = 200
    case = synth.prefill_case(900 + n, lengths, init=False)
    w, acts, _, _ = to_dev(case)
    out, fs, fc = gdn.prefill_varlen(case["cu_seqlens"], acts["qkv"], acts["z"], acts["a"], acts["b"], w)
    torch.cuda.synchronize()
    ref = oracle_prefill(case, heads=(0, 1))
    assert out_err(out[:, :128], ref["out"]) <= OUT_TOL
    assert out_rms_err(out[:, :128], ref["out"]) <= OUT_RMS_TOL
    assert state_err(fs[:, 0:1], ref["state"]) <= STATE_TOL
    assert conv_exact(fc, ref["conv"])
    assert gdn.last_device_error() == 0


def test_varlen_zero_initial_state():
    case = synth.prefill_case(82, [5, 90, 33], init=False)
    w, acts, _, _ = to_dev(case)
    res = gdn.prefill_varlen(case["cu_seqlens"], acts["qkv"], acts["z"], acts["a"], acts["b"], w)
    torch.cuda.synchronize()
    _check_prefill(case, res, oracle_prefill(case))


# ---------------------------------------------------------------- cross-path agreement

def test_split_prefill_equals_single_and_oracle():
    case = synth.dense_case(83, B=1, T=300, init=True)
    ref = oracle_prefill(case)
    w, acts, st, cv = to_dev(case)
    o1, s1, c1 = gdn.prefill(*(acts[k][:, :170].contiguous() for k in ("qkv", "z", "a", "b")), w, st, cv)
    o2, s2, c2 = gdn.prefill(*(acts[k][:, 170:].contiguous() for k in ("qkv", "z", "a", "b")), w, s1, c1)
    torch.cuda.synchronize()
    _check_prefill(case, (torch.cat([o1, o2], 1), s2, c2), ref)


def test_decode_after_prefill_equals_oracle():
    case = synth.dense_case(84, B=3, T=90, init=True)
    T0 = 80
    w, acts, st, cv = to_dev(case)
    _, s, c = gdn.prefill(*(acts[k][:, :T0].contiguous() for k in ("qkv", "z", "a", "b")), w, st, cv)
    outs = [gdn.decode(*(acts[k][:, t].contiguous() for k in ("qkv", "z", "a", "b")), w, s, c)
            for t in range(T0, 90)]
    torch.cuda.synchronize()
    ref = oracle_prefill(case)
    y = torch.stack(outs, 1)
    assert out_err(y, ref["out"].reshape(3, 90, -1)[:, T0:]) <= OUT_TOL
    assert state_err(s, ref["state"]) <= STATE_TOL
    assert conv_exact(c, ref["conv"])


# ---------------------------------------------------------------- benchmark-sized workloads

def test_chunked_prefill_8192_and_split():
    case = synth.config(2)  # B=1, T=8192, zero initial state
    ref = oracle_prefill(case)
    w, acts, _, _ = to_dev(case)
    res = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w)
    torch.cuda.synchronize()
    _check_prefill(case, res, ref, "prefill B=1 T=8192 (all heads)")
    o1, s1, c1 = gdn.prefill(*(acts[k][:, :4096].contiguous() for k in ("qkv", "z", "a", "b")), w)
    o2, s2, c2 = gdn.prefill(*(acts[k][:, 4096:].contiguous() for k in ("qkv", "z", "a", "b")), w, s1, c1)
    torch.cuda.synchronize()
    _check_prefill(case, (torch.cat([o1, o2], 1), s2, c2), ref, "prefill 4096+4096 split (all heads)")


GROUPS = (0, 5, 10, 15)


def test_varlen_benchmark_rows_sampled_groups():
    """The 8-row varlen workload (lengths U[512,16384]); oracle on the 12 value heads of
    q/k heads 0, 5, 10 and 15."""
    case = synth.config(3)
    sub = group_case(case, GROUPS)
    ref = oracle_prefill(sub)
    w, acts, st, cv = to_dev(case)
    out, fs, fc = gdn.prefill_varlen(case["cu_seqlens"], acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    torch.cuda.synchronize()
    zc, hs, ch = sub["z_channels"].cuda(), sub["heads"].cuda(), sub["channels"].cuda()
    check_outputs("varlen 8 rows (groups 0,5,10,15)", out.index_select(1, zc), ref["out"], fs.index_select(1, hs),
                  ref["state"], fc.index_select(2, ch), ref["conv"])
    assert gdn.last_device_error() == 0


def test_long_context_two_rows_then_decode_sampled_groups():
    """Two rows of 65,536 tokens from zero state, returning final states, then 256 decode
    steps per row from those states; oracle on the 12 value heads of q/k heads 0, 5, 10 and
    15 (and the history of their channels).  The oracle continues from its own states."""
    case = synth.config(4)
    sub = group_case(case, GROUPS)
    w, acts, _, _ = to_dev(case)
    out, fs, fc = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w)
    torch.cuda.synchronize()
    ref = oracle_prefill(sub)
    zc, hs, ch = sub["z_channels"].cuda(), sub["heads"].cuda(), sub["channels"].cuda()
    o2 = out.reshape(2 * 65536, -1).index_select(1, zc)
    check_outputs("long context 2x65536 (groups 0,5,10,15)", o2, ref["out"], fs.index_select(1, hs), ref["state"],
                  fc.index_select(2, ch), ref["conv"])
    # 256 decode steps from the GPU's final state; the oracle runs them as one 256-token chain per row
    dec = case["decode"]
    steps = dec["qkv"].shape[0]
    outs = torch.empty((steps, 2, 6144), dtype=torch.bfloat16, device="cuda")
    for s in range(steps):
        gdn.decode(*(dec[k][s].cuda() for k in ("qkv", "z", "a", "b")), w, fs, fc, out=outs[s])
    torch.cuda.synchronize()
    idx = {"qkv": sub["channels"], "z": sub["z_channels"], "a": sub["heads"], "b": sub["heads"]}
    chain = {k: dec[k].index_select(-1, idx[k]).transpose(0, 1).reshape(2 * steps, -1) for k in idx}
    r = oracle_prefill(sub, cu=np.array([0, steps, 2 * steps]), init_state=ref["state"], init_conv=ref["conv"],
                       acts=chain)
    y = outs.index_select(2, zc).transpose(0, 1).reshape(2 * steps, -1)
    check_outputs("decode 256 steps after long context (groups 0,5,10,15)", y, r["out"], fs.index_select(1, hs),
                  r["state"], fc.index_select(2, ch), r["conv"])
    assert gdn.last_device_error() == 0
