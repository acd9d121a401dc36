"""Chunked (WY / UT-transform) restatement of the gated delta rule, float64 numpy.

TEST INFRASTRUCTURE ONLY.  The pages give the recurrence token by token (Qwen3.8
27B model card, "Gated DeltaNet" bullet) and no chunked algorithm.  This module
writes the chunk-C form derived from that recurrence, step by step, so that a
test can check the derivation against the token-by-token oracle before any GPU
code relies on it.  It works on prepared inputs (q already L2-normalised and
scaled, k normalised, v, g = log-decay, beta = write rate) of one value head.

Derivation.  Inside a chunk let G_i = g_1 + ... + g_i (inclusive) and
gamma_i = exp(G_i).  Unrolling S_i = exp(g_i) S_{i-1} + u_i k_i^T gives
S_i = gamma_i S0 + sum_{j<=i} (gamma_i / gamma_j) u_j k_j^T.  Putting that into
u_i = beta_i (v_i - exp(g_i) S_{i-1} k_i) gives the unit lower-triangular system

    (I + A) U = diag(beta) V - diag(beta * gamma) K S0^T,
    A_ij = beta_i * exp(G_i - G_j) * (k_i . k_j)   for j < i, else 0,

so with T = (I + A)^-1:  U = T diag(beta) V - T diag(beta gamma) K S0^T = U~ - W S0^T.
The outputs and the carried state follow by substitution:

    O   = diag(gamma) Q S0^T + (tril_incl(Q K^T) * E) U,  E_ij = exp(G_i - G_j), j <= i
    S_C = gamma_C S0 + U^T diag(exp(G_C - G)) K.

Ratios of gammas are always formed as exp of a difference over j <= i only,
never as a quotient, so nothing overflows when the decay is strong.
"""
from __future__ import annotations

import numpy as np


def chunk_step(q, k, v, g, beta, S0):
    """One chunk.  q,k [n,Dk]; v [n,Dv]; g,beta [n]; S0 [Dv,Dk] -> (O [n,Dv], S [Dv,Dk])."""
    n = k.shape[0]
    G = np.cumsum(g)
    i_idx, j_idx = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    lower = j_idx < i_idx
    lower_incl = j_idx <= i_idx
    diff = np.where(lower_incl, G[:, None] - G[None, :], -np.inf)  # mask before exp
    E = np.exp(diff)                                               # 0 above the diagonal
    A = np.where(lower, beta[:, None] * E * (k @ k.T), 0.0)
    T = np.linalg.inv(np.eye(n) + A)
    U_tilde = T @ (beta[:, None] * v)
    W = T @ ((beta * np.exp(G))[:, None] * k)
    U = U_tilde - W @ S0.T
    O = np.exp(G)[:, None] * (q @ S0.T) + (np.where(lower_incl, q @ k.T, 0.0) * E) @ U
    S = np.exp(G[-1]) * S0 + U.T @ (np.exp(G[-1] - G)[:, None] * k)
    return O, S


def delta_rule_chunked(q, k, v, g, beta, S0, chunk: int = 64):
    """Whole sequence in chunks of ``chunk`` tokens (last chunk may be shorter)."""
    T = k.shape[0]
    S = np.array(S0, dtype=np.float64, copy=True)
    O = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        O[c0:c1], S = chunk_step(q[c0:c1], k[c0:c1], v[c0:c1], g[c0:c1], beta[c0:c1], S)
    return O, S
