"""The library's calls inside CUDA graphs: the dense prefill whose schedule forks onto the
library's internal streams (captured through the event fork / join on the capturing stream),
and the small-batch decode launched as thread-block clusters.  Replays give the same bits as
eager calls."""
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    gdn.load_library()
    return torch.device("cuda", 0)


def test_overlapped_prefill_in_a_graph(dev):
    B, T = 1, 2048
    assert gdn.prefill_schedule(B, T)[0] > 1  # the overlapped schedule on internal streams
    case = synth.dense_case(4711, B, T, init=True)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    st0, cv0 = case["init_state"].to(dev), case["init_conv"].to(dev)
    ref = gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st0, cv0)  # eager (also warms up)
    out = torch.empty_like(ref[0])
    fs = torch.empty_like(ref[1])
    fc = torch.empty_like(ref[2])
    s = torch.cuda.Stream(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, st0, cv0, out=out, final_state=fs,
                    final_conv=fc)
    for _ in range(2):
        out.zero_()
        fs.zero_()
        g.replay()
        torch.cuda.synchronize(dev)
        assert torch.equal(out, ref[0]) and torch.equal(fs, ref[1]) and torch.equal(fc, ref[2])
    assert gdn.last_device_error() == 0


def test_small_batch_decode_in_a_graph(dev):
    rows, steps = 2, 4
    case = synth.decode_case(4712, rows=rows, steps=steps)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    st, cv = case["init_state"].to(dev), case["init_conv"].to(dev)
    st_e, cv_e = st.clone(), cv.clone()
    ref = [gdn.decode(*(acts[k][j] for k in ("qkv", "z", "a", "b")), w, st_e, cv_e) for j in range(steps)]
    out = torch.empty((steps, rows, 6144), dtype=torch.bfloat16, device=dev)
    st_g, cv_g = st.clone(), cv.clone()
    s = torch.cuda.Stream(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for j in range(steps):
            gdn.decode(*(acts[k][j] for k in ("qkv", "z", "a", "b")), w, st_g, cv_g, out=out[j])
    st_g.copy_(st)
    cv_g.copy_(cv)
    g.replay()
    torch.cuda.synchronize(dev)
    assert torch.equal(out, torch.stack(ref)) and torch.equal(st_g, st_e) and torch.equal(cv_g, cv_e)
    assert gdn.last_device_error() == 0
