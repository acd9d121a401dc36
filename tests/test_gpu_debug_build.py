"""The debug build of the library (libgdn_b200_debug.so, compiled with
-DGDN_DEBUG) in place of a memory checker: every kernel checks the indices of
the global-memory accesses it computes (tokens against the token count,
records against the chunks planned, state and history rows against the rows
or the pool) and records a failed check in the device error word instead of
touching memory.  The checks change no arithmetic, so on small cases of every
entry-point family the debug build must give the same bits as the release
build, with the error word still 0.  The debug build runs in a child process
(the binding loads one library per process)."""
import os
import subprocess
import sys

import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import build as gdn_build
from gated_deltanet_mixer_gdn_b200 import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_cases(dev):
    """Small cases of every entry point; returns {name: tensor} on the CPU."""
    res = {}
    case = synth.dense_case(6100, B=2, T=130, init=True)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    st, cv = case["init_state"].to(dev), case["init_conv"].to(dev)
    o, s, c = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st, cv)
    res.update(prefill_out=o, prefill_state=s, prefill_conv=c)
    g = torch.Generator().manual_seed(1)
    w_out = (torch.randn((512, 6144), generator=g) * 0.01).to(torch.bfloat16).to(dev)
    res["prefill_out_proj"] = gdn.prefill_out(acts["qkv"], acts["z"], acts["a"], acts["b"], w, w_out, st, cv)[0]
    vc = synth.prefill_case(6101, [0, 1, 3, 70, 130, 2], init=True)
    va = {k: vc[k].to(dev) for k in ("qkv", "z", "a", "b")}
    o, s, c = gdn.prefill_varlen(vc["cu_seqlens"], va["qkv"], va["z"], va["a"], va["b"], gdn.weights_to(vc["weights"], dev),
                                 vc["init_state"].to(dev), vc["init_conv"].to(dev))
    res.update(varlen_out=o, varlen_state=s, varlen_conv=c)
    dc = synth.decode_case(6102, rows=3, steps=3)
    dw = gdn.weights_to(dc["weights"], dev)
    ds, dv = dc["init_state"].to(dev), dc["init_conv"].to(dev)
    res["decode_out"] = torch.stack([gdn.decode(*(dc[k][t].to(dev) for k in ("qkv", "z", "a", "b")), dw, ds, dv)
                                     for t in range(3)])
    res.update(decode_state=ds, decode_conv=dv)
    mk = {k: dc[k].transpose(0, 1).contiguous().to(dev) for k in ("qkv", "z", "a", "b")}
    ms, mv = dc["init_state"].to(dev), dc["init_conv"].to(dev)
    res["multi_out"] = gdn.decode_multi(mk["qkv"], mk["z"], mk["a"], mk["b"], dw, ms, mv)
    res.update(multi_state=ms, multi_conv=mv)
    pool_s = (torch.randn((5, 48, 128, 128), generator=g) * 0.05).to(dev)
    pool_c = torch.randn((5, 3, 10240), generator=g).to(dev)
    res["slots_out"] = gdn.decode_slots([4, 1, 2], *(dc[k][0].to(dev) for k in ("qkv", "z", "a", "b")), dw, pool_s,
                                        pool_c)
    sc = synth.prefill_case(6103, [40, 0, 65], init=False)
    sa = {k: sc[k].to(dev) for k in ("qkv", "z", "a", "b")}
    res["varlen_slots_out"] = gdn.prefill_varlen_slots(sc["cu_seqlens"], [0, 3, 2], sa["qkv"], sa["z"], sa["a"],
                                                       sa["b"], gdn.weights_to(sc["weights"], dev), pool_s, pool_c)
    res.update(pool_state=pool_s, pool_conv=pool_c)
    torch.cuda.synchronize(dev)
    return {k: v.cpu() for k, v in res.items()}


CHILD = """
import sys, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import gated_deltanet_mixer_gdn_b200 as gdn
from test_gpu_debug_build import run_cases
assert gdn.LIB_PATH.endswith("libgdn_b200_debug.so"), gdn.LIB_PATH
res = run_cases(torch.device("cuda", 0))
res["error_word"] = torch.tensor([gdn.last_device_error()])
torch.save(res, {out!r})
"""


def test_debug_build_same_bits_no_failed_check(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    lib = gdn_build.build(debug=True)
    out = str(tmp_path / "debug.pt")
    env = dict(os.environ, GDN_B200_LIBRARY=lib)
    subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), out=out)],
                   env=env, check=True, timeout=600)
    dbg = torch.load(out)
    assert int(dbg.pop("error_word")[0]) == 0, "an index check of the debug build failed"
    rel = run_cases(torch.device("cuda", 0))
    assert gdn.last_device_error() == 0
    assert set(rel) == set(dbg)
    for k in rel:
        assert torch.equal(rel[k], dbg[k]), f"{k}: the debug build's bits differ"
