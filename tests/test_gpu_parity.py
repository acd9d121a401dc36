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

from _util import (OUT_RMS_TOL, OUT_TOL, STATE_TOL, conv_exact, group_case, oracle_prefill, out_err,
                   out_rms_err, state_err, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    gdn.load_library()


def _check_prefill(case, res, ref):
    out, fs, fc = res
    e_out = out_err(out, ref["out"])
    e_rms = out_rms_err(out, ref["out"])
    e_st = state_err(fs, ref["state"])
    assert e_out <= OUT_TOL, f"output error {e_out:.3e}"
    assert e_rms <= OUT_RMS_TOL, f"output rms error {e_rms:.3e}"
    assert e_st <= STATE_TOL, f"state error {e_st:.3e}"
    assert conv_exact(fc, ref["conv"]), "conv history not bit-exact"
    assert gdn.last_device_error() == 0
    return e_out, e_st


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


def test_decode_batch_shape_sampled_heads():
    """64 rows x 16 steps at the decode batch's shapes; oracle on 6 value heads
    (two whole q/k groups) of every row."""
    case = synth.decode_case(1235, rows=64, steps=16)
    w, _, st, cv = to_dev(case)
    outs = []
    for s in range(16):
        outs.append(gdn.decode(*(case[k][s].cuda() for k in ("qkv", "z", "a", "b")), w, st, cv))
    heads = (3, 9)
    st_ref, cv_ref = case["init_state"], case["init_conv"]
    errs = []
    for s in range(16):
        acts = {k: case[k][s] for k in ("qkv", "z", "a", "b")}
        ref = oracle_prefill(case, cu=np.arange(65), init_state=st_ref, init_conv=cv_ref, acts=acts, heads=heads)
        full_state = st_ref if isinstance(st_ref, np.ndarray) else st_ref.numpy().astype(np.float64)
        full_state = full_state.copy()
        full_state[:, heads[0]:heads[1]] = ref["state"]
        errs.append(out_err(outs[s][:, heads[0] * 128:heads[1] * 128], ref["out"]))
        st_ref, cv_ref = full_state, ref["conv"]
    assert max(errs) <= OUT_TOL
    assert state_err(st[:, heads[0]:heads[1]], st_ref[:, heads[0]:heads[1]]) <= STATE_TOL
    assert conv_exact(cv, cv_ref)


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
    _check_prefill(case, res, oracle_prefill(case))


@pytest.mark.parametrize("T", [1, 2, 3, 63, 64, 65, 127, 200])
def test_prefill_ragged_lengths_with_state(T):
    case = synth.dense_case(500 + T, B=2, T=T, init=True)
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
    _check_prefill(case, res, oracle_prefill(case))


def test_prefill_in_place_state():
    case = synth.dense_case(78, B=2, T=130, init=True)
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
    _check_prefill(case, res, ref)
    o1, s1, c1 = gdn.prefill(*(acts[k][:, :4096].contiguous() for k in ("qkv", "z", "a", "b")), w)
    o2, s2, c2 = gdn.prefill(*(acts[k][:, 4096:].contiguous() for k in ("qkv", "z", "a", "b")), w, s1, c1)
    torch.cuda.synchronize()
    _check_prefill(case, (torch.cat([o1, o2], 1), s2, c2), ref)


def test_varlen_benchmark_rows_sampled_group():
    """The 8-row varlen workload (lengths U[512,16384]); oracle on the 3 value
    heads of q/k head 7."""
    case = synth.config(3)
    sub = group_case(case, 7)
    ref = oracle_prefill(sub)
    w, acts, st, cv = to_dev(case)
    out, fs, fc = gdn.prefill_varlen(case["cu_seqlens"], acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    torch.cuda.synchronize()
    zc, hs, ch = sub["z_channels"].cuda(), sub["heads"].cuda(), sub["channels"].cuda()
    assert out_err(out.index_select(1, zc), ref["out"]) <= OUT_TOL
    assert out_rms_err(out.index_select(1, zc), ref["out"]) <= OUT_RMS_TOL
    assert state_err(fs.index_select(1, hs), ref["state"]) <= STATE_TOL
    assert conv_exact(fc.index_select(2, ch), ref["conv"])


def test_long_context_two_rows_then_decode_sampled_group():
    """Two rows of 65,536 tokens from zero state, returning final states, then
    256 decode steps per row from those states; oracle on the 3 value heads of
    q/k head 15 (and the history of their channels)."""
    case = synth.config(4)
    sub = group_case(case, 15)
    w, acts, _, _ = to_dev(case)
    out, fs, fc = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w)
    torch.cuda.synchronize()
    ref = oracle_prefill(sub)
    zc, hs, ch = sub["z_channels"].cuda(), sub["heads"].cuda(), sub["channels"].cuda()
    o2 = out.reshape(2 * 65536, -1).index_select(1, zc)
    assert out_err(o2, ref["out"]) <= OUT_TOL
    assert out_rms_err(o2, ref["out"]) <= OUT_RMS_TOL
    assert state_err(fs.index_select(1, hs), ref["state"]) <= STATE_TOL
    assert conv_exact(fc.index_select(2, ch), ref["conv"])
    # 256 decode steps from the GPU's final state; the oracle continues from its own
    dec = case["decode"]
    outs = [gdn.decode(*(dec[k][s].cuda() for k in ("qkv", "z", "a", "b")), w, fs, fc) for s in range(256)]
    torch.cuda.synchronize()
    st_ref, cv_ref = ref["state"], ref["conv"]
    errs = []
    for s in range(256):
        step = {"qkv": dec["qkv"][s].index_select(-1, sub["channels"]), "z": dec["z"][s].index_select(-1, sub["z_channels"]),
                "a": dec["a"][s].index_select(-1, sub["heads"]), "b": dec["b"][s].index_select(-1, sub["heads"])}
        r = oracle_prefill(sub, cu=np.arange(3), init_state=st_ref, init_conv=cv_ref, acts=step)
        errs.append(out_err(outs[s].index_select(1, zc), r["out"]))
        st_ref, cv_ref = r["state"], r["conv"]
    assert max(errs) <= OUT_TOL
    assert state_err(fs.index_select(1, hs), st_ref) <= STATE_TOL
    assert conv_exact(fc.index_select(2, ch), cv_ref)
