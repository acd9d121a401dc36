"""The projections around the mixer (in_proj, out_proj) on the tensor cores
against the float64 definition y = x W^T: every element within the bf16
rounding of the output (plus the f32 accumulation), small shapes with ragged
tiles and the 27B layer's full shapes on sampled rows."""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
import oracle
from gated_deltanet_mixer_gdn_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 5e-3  # |y - y_ref| / max(|y_ref|, rms(y_ref)); bf16 rounding of the output is <= 2^-9 relative


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    return torch.device("cuda", 0)


def _draw(seed, shape, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _err(y, ref):
    y = y.double().cpu().numpy()
    rms = max(np.sqrt(np.mean(ref * ref)), 1e-30)
    return float((np.abs(y - ref) / np.maximum(np.abs(ref), rms)).max())


def _split(full, dims):
    C, VD, Vh = dims.conv_channels, dims.value_width, dims.num_v_heads
    return full[:, :C], full[:, C:C + VD], full[:, C + VD + Vh:], full[:, C + VD:C + VD + Vh]  # qkv, z, a, b


@pytest.mark.parametrize("T,hidden", [(300, 512), (1, 64), (129, 192)])
def test_in_proj_small(dev, T, hidden):
    dims = synth.MODEL
    N = dims.conv_channels + dims.value_width + 2 * dims.num_v_heads
    x = _draw(T * 7 + hidden, (T, hidden))
    w = _draw(T * 11 + hidden, (N, hidden), hidden ** -0.5)
    outs = gdn.in_proj(x.to(dev), w.to(dev))
    torch.cuda.synchronize(dev)
    ref = oracle.projection(x.double().numpy(), w.double().numpy())
    for got, want in zip(outs, _split(ref, dims)):
        assert _err(got, want) <= TOL


@pytest.mark.parametrize("T,hidden", [(130, 320), (64, 256)])
def test_out_proj_small(dev, T, hidden):
    K = synth.MODEL.value_width
    y = _draw(T + hidden, (T, K))
    w = _draw(T * 3 + hidden, (hidden, K), K ** -0.5)
    out = gdn.out_proj(y.to(dev), w.to(dev))
    torch.cuda.synchronize(dev)
    assert _err(out, oracle.projection(y.double().numpy(), w.double().numpy())) <= TOL


def test_full_layer_shapes_sampled_rows(dev):
    """in_proj 8192 x 5120 -> 16480 and out_proj 8192 x 6144 -> 5120, checked on 40 rows."""
    dims = synth.MODEL
    T, hidden = 8192, 5120
    N = dims.conv_channels + dims.value_width + 2 * dims.num_v_heads
    x = _draw(1, (T, hidden))
    w_in = _draw(2, (N, hidden), hidden ** -0.5)
    w_out = _draw(3, (hidden, dims.value_width), dims.value_width ** -0.5)
    xd, wid, wod = x.to(dev), w_in.to(dev), w_out.to(dev)
    qkv, z, a, b = gdn.in_proj(xd, wid)
    o = gdn.out_proj(z.contiguous(), wod)  # any [T, 6144] bf16 input
    torch.cuda.synchronize(dev)
    rows = np.unique(np.concatenate([np.random.default_rng(0).integers(0, T, 38), [0, T - 1]]))
    ref = oracle.projection(x[rows].double().numpy(), w_in.double().numpy())
    for got, want in zip((qkv, z, a, b), _split(ref, dims)):
        assert _err(got[rows], want) <= TOL
    ref_o = oracle.projection(z[rows].double().cpu().numpy(), w_out.double().numpy())
    assert _err(o[rows], ref_o) <= TOL
