"""Slot-indexed state pool: decode and packed prefill on pool rows named by a
slot table give the same bits as the dense entry points on the gathered rows,
and leave every other pool row untouched."""
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import synth

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
