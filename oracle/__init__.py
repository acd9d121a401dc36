"""CPU oracle of the Gated DeltaNet token mixer (float64).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py`` — never by the product package.
The arithmetic lives in ``gdn_oracle.c`` (plain C, token-by-token); this module
only builds it with gcc and marshals numpy arrays into it.  ``chunked.py``
holds the chunk-64 WY restatement of the same recurrence, used only to check
that algebra against the token-by-token definition.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants and brute force (the channel order and the
q/k-head grouping are conventions the pages never fix: parity unpinned for
those two readings).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None
_lock = threading.Lock()

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into libgdn_oracle.so next to it (gcc, -O3 -fopenmp)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            d, i, i64p = ctypes.c_double, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)
            L.oracle_silu.restype = d
            L.oracle_silu.argtypes = [d]
            L.oracle_sigmoid.restype = d
            L.oracle_sigmoid.argtypes = [d]
            L.oracle_softplus.restype = d
            L.oracle_softplus.argtypes = [d]
            L.oracle_gates.argtypes = [d, d, d, d, _dp, _dp]
            L.oracle_conv_tap.restype = d
            L.oracle_conv_tap.argtypes = [i, _dp, _dp]
            L.oracle_causal_conv.argtypes = [i, i, _dp, _dp, _dp]
            L.oracle_l2norm.argtypes = [i, _dp, d, _dp]
            L.oracle_delta_rule_step.argtypes = [i, i, _dp, _dp, _dp, d, d, _dp, _dp]
            L.oracle_delta_rule.argtypes = [i, i, i, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
            L.oracle_gated_rmsnorm.argtypes = [i, _dp, _dp, _dp, d, _dp]
            L.oracle_mixer.restype = i
            L.oracle_mixer.argtypes = [i, i, i, i, i, i64p, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                       _dp, _dp, i, i, d, _dp, _dp, _dp, i]
            L.oracle_max_threads.restype = i
            _lib = L
    return _lib


def _c(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(x: Optional[np.ndarray]):
    return None if x is None else x.ctypes.data_as(_dp)


EPS = 1e-6  # Qwen/Qwen3.8-27B architecture page, header table: "RMSNorm · eps 1e-06"


# ---- stage functions ---------------------------------------------------------

def silu(x: float) -> float:
    return lib().oracle_silu(float(x))


def sigmoid(x: float) -> float:
    return lib().oracle_sigmoid(float(x))


def softplus(x: float) -> float:
    return lib().oracle_softplus(float(x))


def gates(A_log: float, dt_bias: float, a: float, b: float):
    g, beta = ctypes.c_double(), ctypes.c_double()
    lib().oracle_gates(float(A_log), float(dt_bias), float(a), float(b), ctypes.byref(g), ctypes.byref(beta))
    return g.value, beta.value


def causal_conv(xbar: np.ndarray, w: np.ndarray) -> np.ndarray:
    """One channel: xbar = [W-1 history values (oldest first), L inputs]; returns L pre-silu values."""
    xbar, w = _c(xbar), _c(w)
    W = w.shape[0]
    L = xbar.shape[0] - (W - 1)
    out = np.zeros(L)
    lib().oracle_causal_conv(L, W, _p(xbar), _p(w), _p(out))
    return out


def l2norm(x: np.ndarray, eps: float = EPS) -> np.ndarray:
    x = _c(x)
    y = np.zeros_like(x)
    lib().oracle_l2norm(x.shape[0], _p(x), eps, _p(y))
    return y


def delta_rule(q, k, v, g, beta, S0):
    """Recurrence on prepared inputs. q,k [T,Dk]; v [T,Dv]; g,beta [T]; S0 [Dv,Dk].
    Returns (o [T,Dv], S_T [Dv,Dk])."""
    q, k, v, g, beta = _c(q), _c(k), _c(v), _c(g), _c(beta)
    S = _c(S0).copy()
    T, Dk = k.shape
    Dv = v.shape[1]
    o = np.zeros((T, Dv))
    lib().oracle_delta_rule(T, Dk, Dv, _p(q), _p(k), _p(v), _p(g), _p(beta), _p(S), _p(o))
    return o, S


def gated_rmsnorm(o, z, w, eps: float = EPS):
    o, z, w = _c(o), _c(z), _c(w)
    y = np.zeros_like(o)
    lib().oracle_gated_rmsnorm(o.shape[0], _p(o), _p(z), _p(w), eps, _p(y))
    return y


# ---- whole mixer -------------------------------------------------------------

def mixer(dims, cu_seqlens, qkv, z, a, b, conv_w, A_log, dt_bias, norm_w,
          init_state=None, init_conv=None, heads=None, nthreads: int = 0,
          want_out: bool = True, want_state: bool = True, want_conv: bool = True):
    """Packed prefill of N rows (decode = rows of length 1), all inputs as float64
    arrays (exact widening of the bf16/f32 tensors the GPU sees).

    ``heads`` = (h_lo, h_hi) restricts the value heads computed (outputs then
    cover only those heads).  Returns dict(out [total, H*D], state [N, H, D, D],
    conv [N, W-1, C]) in float64.
    """
    Kh, Vh, D, W = dims.num_k_heads, dims.num_v_heads, dims.head_dim, dims.conv_width
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    total = int(cu[-1])
    C = (2 * Kh + Vh) * D
    h_lo, h_hi = (0, Vh) if heads is None else heads
    H = h_hi - h_lo
    widths = (C, Vh * D, Vh, Vh)
    arrs = [np.ascontiguousarray(_c(x).reshape(-1, wd)[:total]) for x, wd in zip((qkv, z, a, b), widths)]
    cw, al, dt, nw = _c(conv_w), _c(A_log), _c(dt_bias), _c(norm_w)
    s0 = None if init_state is None else _c(init_state)
    c0 = None if init_conv is None else _c(init_conv)
    out = np.zeros((total, H * D)) if want_out else None
    st = np.zeros((N, H, D, D)) if want_state else None
    cv = np.zeros((N, W - 1, C)) if want_conv else None
    rc = lib().oracle_mixer(Kh, Vh, D, W, N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                            *[_p(x) for x in arrs], _p(cw), _p(al), _p(dt), _p(nw), _p(s0), _p(c0),
                            h_lo, h_hi, EPS, _p(out), _p(st), _p(cv), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_mixer failed with status {rc}")
    return {"out": out, "state": st, "conv": cv}


# ---- the projections around the mixer ------------------------------------------

def projection(x, w):
    """x [T, K] times w [N, K] transposed, in float64: the plain definition of a
    linear layer y = x W^T (the module tree's in_proj / out_proj, row-major
    weights [out_features][in_features]); numpy's matmul is the step."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def max_threads() -> int:
    return lib().oracle_max_threads()
