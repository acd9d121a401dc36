"""B200-native Gated DeltaNet token mixer.

Python binding of the C ABI in ``include/gdn.h`` (``libgdn_b200.so``, built for
sm_100a by ``build.py``).  This module only marshals torch CUDA tensors into
pointers, allocates outputs and the workspace through torch, and passes the
current CUDA stream; every step of the mixer runs in the library's kernels.
There is no CPU path: if the library is missing the calls raise.

    weights = {"conv_w": bf16 [C,4], "A_log": f32 [Vh], "dt_bias": f32 [Vh], "norm_w": f32 [128]}
    out, state, conv = prefill(qkv, z, a, b, weights)               # qkv [B,T,C] ...
    out, state, conv = prefill_varlen(cu_seqlens, qkv, z, a, b, weights, state0, conv0)
    out = decode(qkv, z, a, b, weights, state, conv)                 # state, conv updated in place
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Dict, Optional, Sequence

import torch

from .synth import Dims, MODEL

_PKG = os.path.dirname(os.path.abspath(__file__))
# GDN_B200_LIBRARY selects another build of the library (the debug build, libgdn_b200_debug.so)
LIB_PATH = os.environ.get("GDN_B200_LIBRARY") or os.path.join(_PKG, "libgdn_b200.so")

EXPORTS = ("gdn_prefill_workspace_size", "gdn_prefill", "gdn_prefill_out_workspace_size", "gdn_prefill_out",
           "gdn_prefill_schedule", "gdn_prefill_schedule_nsm", "gdn_prefill_varlen_workspace_size",
           "gdn_prefill_varlen", "gdn_decode", "gdn_decode_multi", "gdn_decode_slots", "gdn_prefill_varlen_slots",
           "gdn_in_proj", "gdn_out_proj", "gdn_prefill_hidden_workspace_size", "gdn_prefill_hidden",
           "gdn_prefill_hidden_varlen_workspace_size", "gdn_prefill_hidden_varlen",
           "gdn_prefill_noalloc", "gdn_last_device_error", "gdn_set_decode_wait_limit", "gdn_test_decode_stop_copies_at",
           "gdn_status_string",
           "gdn_version")

GDN_OK = 0


class GdnError(RuntimeError):
    pass


class _DimsC(ctypes.Structure):
    _fields_ = [("num_k_heads", ctypes.c_int32), ("num_v_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("conv_width", ctypes.c_int32)]


class _WeightsC(ctypes.Structure):
    _fields_ = [("conv_w", ctypes.c_void_p), ("A_log", ctypes.c_void_p),
                ("dt_bias", ctypes.c_void_p), ("norm_w", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()


def load_library() -> ctypes.CDLL:
    """Load libgdn_b200.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise GdnError(f"{LIB_PATH} is missing: build it first (python -m gated_deltanet_mixer_gdn_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        dp, wp = ctypes.POINTER(_DimsC), ctypes.POINTER(_WeightsC)
        L.gdn_prefill_workspace_size.restype = sz
        L.gdn_prefill_workspace_size.argtypes = [dp, i32, i32]
        L.gdn_prefill_varlen_workspace_size.restype = sz
        L.gdn_prefill_varlen_workspace_size.argtypes = [dp, i32, i32]
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_prefill_out_workspace_size.restype = sz
        L.gdn_prefill_out_workspace_size.argtypes = [dp, i32, i32]
        L.gdn_prefill_out.restype = ctypes.c_int
        L.gdn_prefill_out.argtypes = [dp, wp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.gdn_prefill_schedule.restype = ctypes.c_int
        L.gdn_prefill_schedule.argtypes = [dp, i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
        L.gdn_prefill_schedule_nsm.restype = ctypes.c_int
        L.gdn_prefill_schedule_nsm.argtypes = [dp, i32, i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
        L.gdn_prefill.argtypes = [dp, wp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.gdn_prefill_varlen.restype = ctypes.c_int
        L.gdn_prefill_varlen.argtypes = [dp, wp, i32, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.gdn_decode.restype = ctypes.c_int
        L.gdn_decode.argtypes = [dp, wp, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.gdn_in_proj.restype = ctypes.c_int
        L.gdn_in_proj.argtypes = [dp, i32, i32, vp, vp, vp, vp, vp, vp, vp]
        L.gdn_prefill_hidden_workspace_size.restype = sz
        L.gdn_prefill_hidden_workspace_size.argtypes = [dp, i32, i32]
        L.gdn_prefill_hidden.restype = ctypes.c_int
        L.gdn_prefill_hidden.argtypes = [dp, wp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.gdn_prefill_hidden_varlen_workspace_size.restype = sz
        L.gdn_prefill_hidden_varlen_workspace_size.argtypes = [dp, i32, i32]
        L.gdn_prefill_hidden_varlen.restype = ctypes.c_int
        L.gdn_prefill_hidden_varlen.argtypes = [dp, wp, i32, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                                sz, vp]
        L.gdn_out_proj.restype = ctypes.c_int
        L.gdn_out_proj.argtypes = [dp, i32, i32, vp, vp, vp, vp]
        L.gdn_decode_multi.restype = ctypes.c_int
        L.gdn_decode_multi.argtypes = [dp, wp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.gdn_decode_slots.restype = ctypes.c_int
        L.gdn_decode_slots.argtypes = [dp, wp, i32, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.gdn_prefill_varlen_slots.restype = ctypes.c_int
        L.gdn_prefill_varlen_slots.argtypes = [dp, wp, i32, vp, vp, i32, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp,
                                               vp, sz, vp]
        L.gdn_last_device_error.restype = ctypes.c_int
        L.gdn_last_device_error.argtypes = []
        L.gdn_set_decode_wait_limit.restype = ctypes.c_int
        L.gdn_set_decode_wait_limit.argtypes = [ctypes.c_uint64]
        L.gdn_test_decode_stop_copies_at.restype = ctypes.c_int
        L.gdn_test_decode_stop_copies_at.argtypes = [ctypes.c_int32]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_version.restype = ctypes.c_int
        _lib = L
        return L


def status_string(status: int) -> str:
    return load_library().gdn_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != GDN_OK:
        raise GdnError(f"{what} failed: {status_string(status)} ({status})")


def _dims_c(dims: Dims) -> _DimsC:
    return _DimsC(dims.num_k_heads, dims.num_v_heads, dims.head_dim, dims.conv_width)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, device: torch.device) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _weights_c(weights: Dict[str, torch.Tensor], device: torch.device) -> _WeightsC:
    cw = _need(weights["conv_w"], torch.bfloat16, "conv_w", device)
    al = _need(weights["A_log"], torch.float32, "A_log", device)
    dt = _need(weights["dt_bias"], torch.float32, "dt_bias", device)
    nw = _need(weights["norm_w"], torch.float32, "norm_w", device)
    return _WeightsC(cw.data_ptr(), al.data_ptr(), dt.data_ptr(), nw.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _device_of(qkv: torch.Tensor) -> torch.device:
    if not qkv.is_cuda:
        raise GdnError("the mixer runs on the GPU only: pass CUDA tensors")
    return qkv.device


def prefill(qkv, z, a, b, weights, init_state=None, init_conv=None, *, out=None, final_state=None,
            final_conv=None, dims: Dims = MODEL, in_place: bool = False):
    """Dense prefill of B rows x T tokens.  qkv [B,T,C], z [B,T,Vh*D], a/b [B,T,Vh] bf16.
    Returns (out bf16 [B,T,Vh*D], final_state f32 [B,Vh,D,D], final_conv f32 [B,W-1,C]).
    ``in_place`` writes the final state and history over the initial ones."""
    dev = _device_of(qkv)
    L = load_library()
    B, T = int(qkv.shape[0]), int(qkv.shape[1])
    C, VD, Vh, D, Wm = dims.conv_channels, dims.value_width, dims.num_v_heads, dims.head_dim, dims.conv_width - 1
    _need(qkv, torch.bfloat16, "qkv", dev)
    _need(z, torch.bfloat16, "z", dev)
    _need(a, torch.bfloat16, "a", dev)
    _need(b, torch.bfloat16, "b", dev)
    if tuple(qkv.shape) != (B, T, C) or tuple(z.shape) != (B, T, VD) or tuple(a.shape) != (B, T, Vh) \
            or tuple(b.shape) != (B, T, Vh):
        raise ValueError("prefill: shape mismatch")
    if init_state is not None:
        _need(init_state, torch.float32, "init_state", dev)
    if init_conv is not None:
        _need(init_conv, torch.float32, "init_conv", dev)
    if out is None:
        out = torch.empty((B, T, VD), dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = init_state if (in_place and init_state is not None) else \
            torch.empty((B, Vh, D, D), dtype=torch.float32, device=dev)
    if final_conv is None:
        final_conv = init_conv if (in_place and init_conv is not None) else \
            torch.empty((B, Wm, C), dtype=torch.float32, device=dev)
    dc = _dims_c(dims)
    ws_bytes = L.gdn_prefill_workspace_size(ctypes.byref(dc), B, T)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    st = L.gdn_prefill(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), B, T,
                       _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), _ptr(init_state), _ptr(init_conv),
                       _ptr(out), _ptr(final_state), _ptr(final_conv), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "gdn_prefill")
    return out, final_state, final_conv


def prefill_out(qkv, z, a, b, weights, w_out, init_state=None, init_conv=None, *, out=None, final_state=None,
                final_conv=None, dims: Dims = MODEL, in_place: bool = False):
    """Dense prefill followed by out_proj in one call: qkv [B,T,C], z [B,T,Vh*D], a/b [B,T,Vh] bf16,
    w_out bf16 [hidden, Vh*D].  Returns (out bf16 [B,T,hidden], final_state, final_conv); the same
    bits as prefill followed by out_proj."""
    dev = _device_of(qkv)
    L = load_library()
    B, T = int(qkv.shape[0]), int(qkv.shape[1])
    C, VD, Vh, D, Wm = dims.conv_channels, dims.value_width, dims.num_v_heads, dims.head_dim, dims.conv_width - 1
    for t, dt, nm in ((qkv, torch.bfloat16, "qkv"), (z, torch.bfloat16, "z"), (a, torch.bfloat16, "a"),
                      (b, torch.bfloat16, "b"), (w_out, torch.bfloat16, "w_out")):
        _need(t, dt, nm, dev)
    hidden = int(w_out.shape[0])
    if tuple(qkv.shape) != (B, T, C) or tuple(z.shape) != (B, T, VD) or tuple(a.shape) != (B, T, Vh) \
            or tuple(b.shape) != (B, T, Vh) or tuple(w_out.shape) != (hidden, VD):
        raise ValueError("prefill_out: shape mismatch")
    if init_state is not None:
        _need(init_state, torch.float32, "init_state", dev)
    if init_conv is not None:
        _need(init_conv, torch.float32, "init_conv", dev)
    if out is None:
        out = torch.empty((B, T, hidden), dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = init_state if (in_place and init_state is not None) else \
            torch.empty((B, Vh, D, D), dtype=torch.float32, device=dev)
    if final_conv is None:
        final_conv = init_conv if (in_place and init_conv is not None) else \
            torch.empty((B, Wm, C), dtype=torch.float32, device=dev)
    dc = _dims_c(dims)
    ws_bytes = L.gdn_prefill_out_workspace_size(ctypes.byref(dc), B, T)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    st = L.gdn_prefill_out(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), B, T, hidden,
                           _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), _ptr(init_state), _ptr(init_conv), _ptr(w_out),
                           _ptr(out), _ptr(final_state), _ptr(final_conv), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "gdn_prefill_out")
    return out, final_state, final_conv


def prefill_schedule(B: int, T: int, from_hidden: bool = False, dims: Dims = MODEL, nsm: int | None = None):
    """(segments, launches) of a dense prefill of B x T tokens that returns its final state, on
    the current device (or, with nsm, on a device of nsm SMs, without one): recurrence segments
    of the overlapped schedule (1: plain) and the number of kernels the call launches (prefill,
    or prefill_hidden with from_hidden)."""
    L = load_library()
    dc = _dims_c(dims)
    seg, lau = ctypes.c_int32(0), ctypes.c_int32(0)
    if nsm is None:
        _check(L.gdn_prefill_schedule(ctypes.byref(dc), int(B), int(T), int(bool(from_hidden)), ctypes.byref(seg),
                                      ctypes.byref(lau)), "gdn_prefill_schedule")
    else:
        _check(L.gdn_prefill_schedule_nsm(ctypes.byref(dc), int(B), int(T), int(bool(from_hidden)), int(nsm),
                                          ctypes.byref(seg), ctypes.byref(lau)), "gdn_prefill_schedule_nsm")
    return seg.value, lau.value


def prefill_varlen(cu_seqlens, qkv, z, a, b, weights, init_state=None, init_conv=None, *, out=None,
                   final_state=None, final_conv=None, dims: Dims = MODEL, cu_seqlens_dev=None,
                   in_place: bool = False):
    """Packed prefill of N rows.  cu_seqlens: N+1 int32 (host tensor, list, or CUDA
    tensor).  qkv [total,C], z [total,Vh*D], a/b [total,Vh].
    Returns (out [total,Vh*D], final_state [N,Vh,D,D], final_conv [N,W-1,C])."""
    dev = _device_of(qkv)
    L = load_library()
    if isinstance(cu_seqlens, torch.Tensor):
        cu_host = cu_seqlens.detach().to("cpu", torch.int32).contiguous()
    else:
        cu_host = torch.tensor(list(cu_seqlens), dtype=torch.int32)
    N = int(cu_host.numel()) - 1
    total = int(qkv.shape[0])
    C, VD, Vh, D, Wm = dims.conv_channels, dims.value_width, dims.num_v_heads, dims.head_dim, dims.conv_width - 1
    for t, dt, nm in ((qkv, torch.bfloat16, "qkv"), (z, torch.bfloat16, "z"), (a, torch.bfloat16, "a"),
                      (b, torch.bfloat16, "b")):
        _need(t, dt, nm, dev)
    if tuple(qkv.shape) != (total, C) or tuple(z.shape) != (total, VD) or tuple(a.shape) != (total, Vh) \
            or tuple(b.shape) != (total, Vh):
        raise ValueError("prefill_varlen: shape mismatch")
    if cu_seqlens_dev is None:
        cu_seqlens_dev = cu_host.to(dev, non_blocking=False)
    _need(cu_seqlens_dev, torch.int32, "cu_seqlens_dev", dev)
    if out is None:
        out = torch.empty((total, VD), dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = init_state if (in_place and init_state is not None) else \
            torch.empty((N, Vh, D, D), dtype=torch.float32, device=dev)
    if final_conv is None:
        final_conv = init_conv if (in_place and init_conv is not None) else \
            torch.empty((N, Wm, C), dtype=torch.float32, device=dev)
    dc = _dims_c(dims)
    ws_bytes = L.gdn_prefill_varlen_workspace_size(ctypes.byref(dc), N, total)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    st = L.gdn_prefill_varlen(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), N,
                              ctypes.c_void_p(cu_host.data_ptr()), _ptr(cu_seqlens_dev), total,
                              _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), _ptr(init_state), _ptr(init_conv),
                              _ptr(out), _ptr(final_state), _ptr(final_conv), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "gdn_prefill_varlen")
    return out, final_state, final_conv


def decode(qkv, z, a, b, weights, state, conv, *, out=None, dims: Dims = MODEL):
    """One token for each of `rows` rows.  qkv [rows,C], z [rows,Vh*D], a/b [rows,Vh] bf16;
    state f32 [rows,Vh,D,D] and conv f32 [rows,W-1,C] are updated in place.  Returns out."""
    dev = _device_of(qkv)
    L = load_library()
    rows = int(qkv.shape[0])
    for t, dt, nm in ((qkv, torch.bfloat16, "qkv"), (z, torch.bfloat16, "z"), (a, torch.bfloat16, "a"),
                      (b, torch.bfloat16, "b"), (state, torch.float32, "state"), (conv, torch.float32, "conv")):
        _need(t, dt, nm, dev)
    if out is None:
        out = torch.empty((rows, dims.value_width), dtype=torch.bfloat16, device=dev)
    dc = _dims_c(dims)
    st = L.gdn_decode(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), rows,
                      _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), _ptr(state), _ptr(conv), _ptr(out), _stream(dev))
    _check(st, "gdn_decode")
    return out


def decode_multi(qkv, z, a, b, weights, state, conv, *, out=None, dims: Dims = MODEL):
    """k successive tokens for each of `rows` rows in one call.  qkv [rows,k,C],
    z [rows,k,Vh*D], a/b [rows,k,Vh] bf16; state f32 [rows,Vh,D,D] and conv f32
    [rows,W-1,C] are updated in place.  Returns out [rows,k,Vh*D]."""
    dev = _device_of(qkv)
    L = load_library()
    rows, k = int(qkv.shape[0]), int(qkv.shape[1])
    for t, dt, nm in ((qkv, torch.bfloat16, "qkv"), (z, torch.bfloat16, "z"), (a, torch.bfloat16, "a"),
                      (b, torch.bfloat16, "b"), (state, torch.float32, "state"), (conv, torch.float32, "conv")):
        _need(t, dt, nm, dev)
    if out is None:
        out = torch.empty((rows, k, dims.value_width), dtype=torch.bfloat16, device=dev)
    dc = _dims_c(dims)
    st = L.gdn_decode_multi(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), rows, k,
                            _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), _ptr(state), _ptr(conv), _ptr(out), _stream(dev))
    _check(st, "gdn_decode_multi")
    return out


def in_proj(x, w_in, *, dims: Dims = MODEL, out=None):
    """x bf16 [T, hidden] times the stacked in_proj weights w_in bf16 [C + Vh*D + 2*Vh, hidden]
    (qkv, z, b, a rows).  Returns (qkv [T,C], z [T,Vh*D], a [T,Vh], b [T,Vh])."""
    dev = _device_of(x)
    L = load_library()
    _need(x, torch.bfloat16, "x", dev)
    _need(w_in, torch.bfloat16, "w_in", dev)
    T, hidden = int(x.shape[0]), int(x.shape[1])
    C, VD, Vh = dims.conv_channels, dims.value_width, dims.num_v_heads
    if tuple(w_in.shape) != (C + VD + 2 * Vh, hidden):
        raise ValueError("in_proj: w_in shape")
    qkv, z, a, b = out if out is not None else (
        torch.empty((T, C), dtype=torch.bfloat16, device=dev), torch.empty((T, VD), dtype=torch.bfloat16, device=dev),
        torch.empty((T, Vh), dtype=torch.bfloat16, device=dev), torch.empty((T, Vh), dtype=torch.bfloat16, device=dev))
    dc = _dims_c(dims)
    st = L.gdn_in_proj(ctypes.byref(dc), T, hidden, _ptr(x), _ptr(w_in), _ptr(qkv), _ptr(z), _ptr(b), _ptr(a),
                       _stream(dev))
    _check(st, "gdn_in_proj")
    return qkv, z, a, b


def prefill_hidden(x, w_in, weights, init_state=None, init_conv=None, *, out=None, final_state=None,
                   final_conv=None, dims: Dims = MODEL, in_place: bool = False):
    """Dense prefill from the layer's hidden states: x bf16 [B,T,hidden] through the stacked in_proj
    weights w_in (rows of qkv, z, b, a) into the mixer, the load stage running inside the in_proj GEMM.
    Returns (out bf16 [B,T,Vh*D] before out_proj, final_state f32 [B,Vh,D,D], final_conv f32 [B,W-1,C]);
    the same results, bit for bit, as in_proj followed by prefill."""
    dev = _device_of(x)
    L = load_library()
    _need(x, torch.bfloat16, "x", dev)
    _need(w_in, torch.bfloat16, "w_in", dev)
    B, T, hidden = int(x.shape[0]), int(x.shape[1]), int(x.shape[2])
    C, VD, Vh, D, Wm = dims.conv_channels, dims.value_width, dims.num_v_heads, dims.head_dim, dims.conv_width - 1
    if tuple(w_in.shape) != (C + VD + 2 * Vh, hidden):
        raise ValueError("prefill_hidden: w_in shape")
    if init_state is not None:
        _need(init_state, torch.float32, "init_state", dev)
    if init_conv is not None:
        _need(init_conv, torch.float32, "init_conv", dev)
    if out is None:
        out = torch.empty((B, T, VD), dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = init_state if (in_place and init_state is not None) else \
            torch.empty((B, Vh, D, D), dtype=torch.float32, device=dev)
    if final_conv is None:
        final_conv = init_conv if (in_place and init_conv is not None) else \
            torch.empty((B, Wm, C), dtype=torch.float32, device=dev)
    dc = _dims_c(dims)
    ws_bytes = L.gdn_prefill_hidden_workspace_size(ctypes.byref(dc), B, T)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    st = L.gdn_prefill_hidden(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), B, T, hidden,
                              _ptr(x), _ptr(w_in), _ptr(init_state), _ptr(init_conv), _ptr(out),
                              _ptr(final_state), _ptr(final_conv), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "gdn_prefill_hidden")
    return out, final_state, final_conv


def prefill_hidden_varlen(cu_seqlens, x, w_in, weights, init_state=None, init_conv=None, *, out=None,
                          final_state=None, final_conv=None, dims: Dims = MODEL, cu_seqlens_dev=None,
                          in_place: bool = False):
    """Packed prefill from hidden states: x bf16 [total, hidden] holds the rows given by cu_seqlens
    (int32 [N+1]); the load stage runs inside the in_proj GEMM.  Returns (out bf16 [total, Vh*D],
    final_state f32 [N,Vh,D,D], final_conv f32 [N,W-1,C]); the same bits as in_proj followed by
    prefill_varlen."""
    dev = _device_of(x)
    L = load_library()
    _need(x, torch.bfloat16, "x", dev)
    _need(w_in, torch.bfloat16, "w_in", dev)
    cu_host = torch.as_tensor(cu_seqlens, dtype=torch.int32).cpu().contiguous()
    N = int(cu_host.numel()) - 1
    total, hidden = int(x.shape[0]), int(x.shape[1])
    if N < 0 or int(cu_host[-1]) != total:
        raise ValueError("prefill_hidden_varlen: cu_seqlens must end at the token count")
    C, VD, Vh, D, Wm = dims.conv_channels, dims.value_width, dims.num_v_heads, dims.head_dim, dims.conv_width - 1
    if tuple(w_in.shape) != (C + VD + 2 * Vh, hidden):
        raise ValueError("prefill_hidden_varlen: w_in shape")
    cu_dev = cu_seqlens_dev if cu_seqlens_dev is not None else cu_host.to(dev)
    if init_state is not None:
        _need(init_state, torch.float32, "init_state", dev)
    if init_conv is not None:
        _need(init_conv, torch.float32, "init_conv", dev)
    if out is None:
        out = torch.empty((total, VD), dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = init_state if (in_place and init_state is not None) else \
            torch.empty((N, Vh, D, D), dtype=torch.float32, device=dev)
    if final_conv is None:
        final_conv = init_conv if (in_place and init_conv is not None) else \
            torch.empty((N, Wm, C), dtype=torch.float32, device=dev)
    dc = _dims_c(dims)
    ws_bytes = L.gdn_prefill_hidden_varlen_workspace_size(ctypes.byref(dc), N, total)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    st = L.gdn_prefill_hidden_varlen(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), N,
                                     ctypes.c_void_p(cu_host.data_ptr()), _ptr(cu_dev), total, hidden, _ptr(x),
                                     _ptr(w_in), _ptr(init_state), _ptr(init_conv), _ptr(out), _ptr(final_state),
                                     _ptr(final_conv), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "gdn_prefill_hidden_varlen")
    return out, final_state, final_conv


def out_proj(y, w_out, *, dims: Dims = MODEL, out=None):
    """y bf16 [T, Vh*D] times w_out bf16 [hidden, Vh*D]^T.  Returns out [T, hidden]."""
    dev = _device_of(y)
    L = load_library()
    _need(y, torch.bfloat16, "y", dev)
    _need(w_out, torch.bfloat16, "w_out", dev)
    T, hidden = int(y.shape[0]), int(w_out.shape[0])
    if out is None:
        out = torch.empty((T, hidden), dtype=torch.bfloat16, device=dev)
    dc = _dims_c(dims)
    st = L.gdn_out_proj(ctypes.byref(dc), T, hidden, _ptr(y), _ptr(w_out), _ptr(out), _stream(dev))
    _check(st, "gdn_out_proj")
    return out


def _slot_tables(slots, n, dev):
    if isinstance(slots, torch.Tensor):
        host = slots.detach().to("cpu", torch.int32).contiguous()
    else:
        host = torch.tensor(list(slots), dtype=torch.int32)
    if host.numel() != n:
        raise ValueError("one slot per row")
    return host, host.to(dev)


def decode_slots(slots, qkv, z, a, b, weights, state_pool, conv_pool, *, out=None, dims: Dims = MODEL):
    """One token for each of `rows` rows, row r on pool row slots[r] (int32, host or CUDA
    tensor or list).  state_pool f32 [P,Vh,D,D] and conv_pool f32 [P,W-1,C] are updated in
    place.  Returns out [rows,Vh*D]."""
    dev = _device_of(qkv)
    L = load_library()
    rows = int(qkv.shape[0])
    for t, dt, nm in ((qkv, torch.bfloat16, "qkv"), (z, torch.bfloat16, "z"), (a, torch.bfloat16, "a"),
                      (b, torch.bfloat16, "b"), (state_pool, torch.float32, "state_pool"),
                      (conv_pool, torch.float32, "conv_pool")):
        _need(t, dt, nm, dev)
    host, devs = _slot_tables(slots, rows, dev)
    if out is None:
        out = torch.empty((rows, dims.value_width), dtype=torch.bfloat16, device=dev)
    dc = _dims_c(dims)
    st = L.gdn_decode_slots(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), rows,
                            ctypes.c_void_p(host.data_ptr()), _ptr(devs), int(state_pool.shape[0]),
                            _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), _ptr(state_pool), _ptr(conv_pool), _ptr(out),
                            _stream(dev))
    _check(st, "gdn_decode_slots")
    return out


def prefill_varlen_slots(cu_seqlens, slots, qkv, z, a, b, weights, state_pool, conv_pool, *, out=None,
                         dims: Dims = MODEL):
    """Packed prefill of N rows, row n starting from and updating pool row slots[n] in place.
    Returns out [total,Vh*D]."""
    dev = _device_of(qkv)
    L = load_library()
    if isinstance(cu_seqlens, torch.Tensor):
        cu_host = cu_seqlens.detach().to("cpu", torch.int32).contiguous()
    else:
        cu_host = torch.tensor(list(cu_seqlens), dtype=torch.int32)
    N = int(cu_host.numel()) - 1
    total = int(qkv.shape[0])
    for t, dt, nm in ((qkv, torch.bfloat16, "qkv"), (z, torch.bfloat16, "z"), (a, torch.bfloat16, "a"),
                      (b, torch.bfloat16, "b"), (state_pool, torch.float32, "state_pool"),
                      (conv_pool, torch.float32, "conv_pool")):
        _need(t, dt, nm, dev)
    host, devs = _slot_tables(slots, N, dev)
    cu_dev = cu_host.to(dev)
    if out is None:
        out = torch.empty((total, dims.value_width), dtype=torch.bfloat16, device=dev)
    dc = _dims_c(dims)
    ws_bytes = L.gdn_prefill_varlen_workspace_size(ctypes.byref(dc), N, total)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    st = L.gdn_prefill_varlen_slots(ctypes.byref(dc), ctypes.byref(_weights_c(weights, dev)), N,
                                    ctypes.c_void_p(cu_host.data_ptr()), _ptr(cu_dev), total,
                                    ctypes.c_void_p(host.data_ptr()), _ptr(devs), int(state_pool.shape[0]),
                                    _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), _ptr(state_pool), _ptr(conv_pool),
                                    _ptr(out), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "gdn_prefill_varlen_slots")
    return out


def last_device_error() -> int:
    """The device error word (0, or the code of the first bounded wait that ran out); cleared by reading."""
    return load_library().gdn_last_device_error()


DECODE_WAIT_LIMIT_DEFAULT_NS = 2_000_000_000


def set_decode_wait_limit(ns: int = DECODE_WAIT_LIMIT_DEFAULT_NS) -> None:
    """Bound of every wait inside the decode kernels on the current device (default 2 s)."""
    _check(load_library().gdn_set_decode_wait_limit(int(ns)), "gdn_set_decode_wait_limit")


def weights_to(weights: Dict[str, torch.Tensor], device) -> Dict[str, torch.Tensor]:
    return {k: v.to(device).contiguous() for k, v in weights.items()}


__all__ = ["prefill", "prefill_out", "prefill_schedule", "prefill_varlen", "decode", "decode_multi", "decode_slots", "in_proj", "out_proj", "prefill_hidden", "prefill_hidden_varlen", "prefill_varlen_slots", "last_device_error", "set_decode_wait_limit", "status_string", "load_library",
           "GdnError", "Dims", "MODEL", "LIB_PATH", "EXPORTS", "weights_to"]
