"""Slot-indexed state pool (decode_rows / prefill_slots on a server's fixed rows):
decode and packed prefill on pool rows named by a slot table match the float64
oracle run from those pool rows, give the same bits as the dense entry points on
the gathered rows, and leave every other pool row untouched."""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import synth

from _util import check_outputs, oracle_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    return torch.device("cuda", 0)


def _pool(seed, P, dev):
    g = torch.Generator().manual_seed(seed)
    st = (torch.randn((P, 48, 128, 128), generator=g) * 0.05).to(dev)
    cv = torch.randn((P, 3, 10240), generator=g).to(dev)
    return st, cv


def test_decode_slots_match_dense_decode(dev):
    P, slots = 7, [5, 0, 3]
    st_pool, cv_pool = _pool(11, P, dev)
    case = synth.decode_case(4321, rows=len(slots), steps=2)
    w = gdn.weights_to(case["weights"], dev)
    idx = torch.tensor(slots, device=dev, dtype=torch.long)
    dense_st, dense_cv = st_pool[idx].clone(), cv_pool[idx].clone()
    before_st, before_cv = st_pool.clone(), cv_pool.clone()
    for step in range(2):
        acts = {k: case[k][step].to(dev) for k in ("qkv", "z", "a", "b")}
        ref = gdn.decode(acts["qkv"], acts["z"], acts["a"], acts["b"], w, dense_st, dense_cv)
        out = gdn.decode_slots(slots, acts["qkv"], acts["z"], acts["a"], acts["b"], w, st_pool, cv_pool)
        torch.cuda.synchronize(dev)
        assert torch.equal(out, ref), f"step {step}"
    assert torch.equal(st_pool[idx], dense_st) and torch.equal(cv_pool[idx], dense_cv)
    rest = torch.tensor([r for r in range(P) if r not in slots], device=dev, dtype=torch.long)
    assert torch.equal(st_pool[rest], before_st[rest]) and torch.equal(cv_pool[rest], before_cv[rest])


def test_prefill_varlen_slots_match_varlen(dev):
    P, slots, lengths = 8, [6, 1, 4], [100, 200, 1]
    st_pool, cv_pool = _pool(12, P, dev)
    case = synth.prefill_case(4322, lengths, init=False)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    cu = case["cu_seqlens"]
    idx = torch.tensor(slots, device=dev, dtype=torch.long)
    init_st, init_cv = st_pool[idx].clone(), cv_pool[idx].clone()
    before_st, before_cv = st_pool.clone(), cv_pool.clone()
    ref_out, ref_st, ref_cv = gdn.prefill_varlen(cu, acts["qkv"], acts["z"], acts["a"], acts["b"], w, init_st, init_cv)
    out = gdn.prefill_varlen_slots(cu, slots, acts["qkv"], acts["z"], acts["a"], acts["b"], w, st_pool, cv_pool)
    torch.cuda.synchronize(dev)
    assert torch.equal(out, ref_out)
    assert torch.equal(st_pool[idx], ref_st) and torch.equal(cv_pool[idx], ref_cv)
    rest = torch.tensor([r for r in range(P) if r not in slots], device=dev, dtype=torch.long)
    assert torch.equal(st_pool[rest], before_st[rest]) and torch.equal(cv_pool[rest], before_cv[rest])


def test_decode_slots_against_oracle(dev):
    """decode_rows on a pool: 3 successive steps of 3 rows on pool rows 5, 0, 3, compared with
    the float64 oracle run from those pool rows (the 3 tokens of a row as one chain, all 48
    value heads); the pool rows no slot names stay bit-identical."""
    P, slots, steps = 7, [5, 0, 3], 3
    st_pool, cv_pool = _pool(13, P, dev)
    case = synth.decode_case(4323, rows=len(slots), steps=steps)
    w = gdn.weights_to(case["weights"], dev)
    idx = torch.tensor(slots, dtype=torch.long)
    init_st, init_cv = st_pool.cpu()[idx], cv_pool.cpu()[idx]
    before_st, before_cv = st_pool.clone(), cv_pool.clone()
    outs = [gdn.decode_slots(torch.tensor(slots, dtype=torch.int32, device=dev),
                             *(case[k][s].to(dev) for k in ("qkv", "z", "a", "b")), w, st_pool, cv_pool)
            for s in range(steps)]
    torch.cuda.synchronize(dev)
    acts = {k: case[k].transpose(0, 1).reshape(len(slots) * steps, -1) for k in ("qkv", "z", "a", "b")}
    ref = oracle_prefill(case, cu=np.arange(len(slots) + 1) * steps, init_state=init_st, init_conv=init_cv,
                         acts=acts)
    y = torch.stack(outs, 1).reshape(len(slots) * steps, -1)
    check_outputs("decode_slots 3 rows x 3 steps", y, ref["out"], st_pool[idx.to(dev)], ref["state"],
                  cv_pool[idx.to(dev)], ref["conv"])
    rest = torch.tensor([r for r in range(P) if r not in slots], device=dev, dtype=torch.long)
    assert torch.equal(st_pool[rest], before_st[rest]) and torch.equal(cv_pool[rest], before_cv[rest])
    assert gdn.last_device_error() == 0


def test_prefill_varlen_slots_against_oracle(dev):
    """prefill_slots on a pool: rows of 100, 200, 1 and 70 tokens starting from pool rows 6, 1,
    4 and 2 (nonzero states and histories), compared element by element with the float64
    oracle on the gathered rows; untouched pool rows stay bit-identical."""
    P, slots, lengths = 8, [6, 1, 4, 2], [100, 200, 1, 70]
    st_pool, cv_pool = _pool(14, P, dev)
    case = synth.prefill_case(4324, lengths, init=False)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    idx = torch.tensor(slots, dtype=torch.long)
    init_st, init_cv = st_pool.cpu()[idx], cv_pool.cpu()[idx]
    before_st, before_cv = st_pool.clone(), cv_pool.clone()
    out = gdn.prefill_varlen_slots(case["cu_seqlens"], slots, acts["qkv"], acts["z"], acts["a"], acts["b"], w,
                                   st_pool, cv_pool)
    torch.cuda.synchronize(dev)
    ref = oracle_prefill(case, init_state=init_st, init_conv=init_cv)
    check_outputs("prefill_varlen_slots 4 rows", out, ref["out"], st_pool[idx.to(dev)], ref["state"],
                  cv_pool[idx.to(dev)], ref["conv"])
    rest = torch.tensor([r for r in range(P) if r not in slots], device=dev, dtype=torch.long)
    assert torch.equal(st_pool[rest], before_st[rest]) and torch.equal(cv_pool[rest], before_cv[rest])
    assert gdn.last_device_error() == 0
