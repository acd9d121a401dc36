"""Seeded synthetic inputs for the Gated DeltaNet mixer.

This module only draws random tensors; it contains none of the mixer's
arithmetic.  It is the one piece of code shared by the CPU oracle's tests and
the CUDA path's tests and benchmark, so both sides see identical bits.

Shapes follow the Qwen3.8-27B Gated DeltaNet layer (Qwen3.8 27B model card,
"Gated DeltaNet" bullet; Qwen/Qwen3.8-27B architecture page, "Module tree",
``linear_attn``): 16 query/key heads and 48 value heads of width 128, a width-4
depthwise conv over the 10240 projected qkv channels, z of width 6144 and the
two 48-wide gate inputs a and b.

Draw order (all draws in float32 from one ``torch.Generator``; bf16 tensors are
the round-to-nearest-even cast of those draws):
conv_w, A_log, dt_bias, norm_w, per-row initial state, per-row conv history,
then the activations qkv, z, a, b.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Dims:
    """Mixer dimensions (defaults: the 27B model's GDN layer)."""

    num_k_heads: int = 16
    num_v_heads: int = 48
    head_dim: int = 128
    conv_width: int = 4

    @property
    def conv_channels(self) -> int:
        return (2 * self.num_k_heads + self.num_v_heads) * self.head_dim

    @property
    def value_width(self) -> int:
        return self.num_v_heads * self.head_dim


MODEL = Dims()


def _normal(gen: torch.Generator, shape, std: float, mean: float = 0.0) -> torch.Tensor:
    return torch.randn(shape, generator=gen, dtype=torch.float32) * std + mean


def draw_weights(gen: torch.Generator, dims: Dims = MODEL, long_memory: bool = False) -> Dict[str, torch.Tensor]:
    """conv_w ~ N(0, 0.5) (bf16), A_log = log U(1, 16), dt_bias ~ N(0, 0.5), norm_w ~ N(0, 0.1).

    ``long_memory`` replaces the gate parameters by A_log = 0, dt_bias = -5 so
    that the per-token decay g is about -7e-3 and the state remembers across
    many chunks (a test-only family).
    """
    conv_w = _normal(gen, (dims.conv_channels, dims.conv_width), 0.5).to(torch.bfloat16)
    A_log = torch.log(torch.rand((dims.num_v_heads,), generator=gen, dtype=torch.float32) * 15.0 + 1.0)
    dt_bias = _normal(gen, (dims.num_v_heads,), 0.5)
    norm_w = _normal(gen, (dims.head_dim,), 0.1)
    if long_memory:
        A_log = torch.zeros_like(A_log)
        dt_bias = torch.full_like(dt_bias, -5.0)
    return {"conv_w": conv_w, "A_log": A_log, "dt_bias": dt_bias, "norm_w": norm_w}


def draw_state(gen: torch.Generator, rows: int, dims: Dims = MODEL, std: float = 0.05) -> torch.Tensor:
    return _normal(gen, (rows, dims.num_v_heads, dims.head_dim, dims.head_dim), std)


def draw_history(gen: torch.Generator, rows: int, dims: Dims = MODEL, std: float = 1.0) -> torch.Tensor:
    return _normal(gen, (rows, dims.conv_width - 1, dims.conv_channels), std)


def draw_activations(gen: torch.Generator, lead: Sequence[int], dims: Dims = MODEL,
                     a_std: float = 1.0) -> Dict[str, torch.Tensor]:
    lead = tuple(lead)
    qkv = _normal(gen, lead + (dims.conv_channels,), 1.0).to(torch.bfloat16)
    z = _normal(gen, lead + (dims.value_width,), 1.0).to(torch.bfloat16)
    a = _normal(gen, lead + (dims.num_v_heads,), a_std).to(torch.bfloat16)
    b = _normal(gen, lead + (dims.num_v_heads,), 1.0).to(torch.bfloat16)
    return {"qkv": qkv, "z": z, "a": a, "b": b}


def prefill_case(seed: int, lengths: Sequence[int], dims: Dims = MODEL, init: bool = False,
                 long_memory: bool = False) -> Dict[str, object]:
    """A packed (varlen) prefill problem: rows of the given lengths.

    Returns weights, ``cu_seqlens`` (int32, N+1), packed activations
    [sum(lengths), ...], and per-row initial state / history (None = zeros).
    """
    gen = torch.Generator().manual_seed(seed)
    w = draw_weights(gen, dims, long_memory=long_memory)
    n = len(lengths)
    state = draw_state(gen, n, dims) if init else None
    hist = draw_history(gen, n, dims) if init else None
    total = int(sum(lengths))
    act = draw_activations(gen, (total,), dims, a_std=0.25 if long_memory else 1.0)
    cu = torch.zeros(n + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(list(lengths), dtype=torch.int64), 0).to(torch.int32)
    return {"dims": dims, "weights": w, "cu_seqlens": cu, "lengths": list(lengths),
            "init_state": state, "init_conv": hist, **act}


def dense_case(seed: int, B: int, T: int, dims: Dims = MODEL, init: bool = False,
               long_memory: bool = False) -> Dict[str, object]:
    """A dense [B, T] prefill problem (activations shaped [B, T, ...])."""
    gen = torch.Generator().manual_seed(seed)
    w = draw_weights(gen, dims, long_memory=long_memory)
    state = draw_state(gen, B, dims) if init else None
    hist = draw_history(gen, B, dims) if init else None
    act = draw_activations(gen, (B, T), dims, a_std=0.25 if long_memory else 1.0)
    return {"dims": dims, "weights": w, "B": B, "T": T, "init_state": state, "init_conv": hist, **act}


def decode_case(seed: int, rows: int, steps: int, dims: Dims = MODEL) -> Dict[str, object]:
    """``steps`` successive single-token steps for ``rows`` rows, each row with
    its own initial f32 state ~ N(0, 0.05) and conv history ~ N(0, 1).
    Activations are shaped [steps, rows, ...]."""
    gen = torch.Generator().manual_seed(seed)
    w = draw_weights(gen, dims)
    state = draw_state(gen, rows, dims)
    hist = draw_history(gen, rows, dims)
    act = draw_activations(gen, (steps, rows), dims)
    return {"dims": dims, "weights": w, "rows": rows, "steps": steps,
            "init_state": state, "init_conv": hist, **act}


def varlen_lengths(seed: int, n: int = 8, lo: int = 512, hi: int = 16384) -> List[int]:
    """Row lengths uniform on the integers [lo, hi], drawn from the seed."""
    gen = torch.Generator().manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen)]


# The five benchmark-shaped workloads.  Seed = 1234 + index.
CONFIG_NAMES = {
    0: "prefill B=1 T=256, zero initial state",
    1: "decode 64 rows x 128 steps, random initial state and history",
    2: "chunked prefill B=1 T=8192, zero initial state (and split 4096+4096)",
    3: "varlen prefill 8 rows, lengths U[512,16384], random initial state and history",
    4: "long-context prefill B=2 T=65536, zero initial state, then 256 decode steps",
}


def config(index: int, dims: Dims = MODEL) -> Dict[str, object]:
    seed = 1234 + index
    if index == 0:
        return dense_case(seed, 1, 256, dims)
    if index == 1:
        return decode_case(seed, 64, 128, dims)
    if index == 2:
        return dense_case(seed, 1, 8192, dims)
    if index == 3:
        lengths = varlen_lengths(seed)
        return prefill_case(seed + 100000, lengths, dims, init=True)
    if index == 4:
        case = dense_case(seed, 2, 65536, dims)
        gen = torch.Generator().manual_seed(seed + 100000)
        case["decode"] = draw_activations(gen, (256, 2), dims)
        return case
    raise ValueError(f"no config {index}")


def to_f64(t: Optional[torch.Tensor]):
    """Exact widening to a float64 numpy array (None passes through)."""
    if t is None:
        return None
    return t.to(torch.float64).numpy()
