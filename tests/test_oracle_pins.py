"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a closed form, an invariant the method
implies, a library routine that a special case reduces to, or a brute-force
expansion written independently here.  Together they are meant to catch a
dropped term, a wrong sign, an index slip or a transposed operand anywhere in
the oracle.  No GPU needed.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import chunked
from gated_deltanet_mixer_gdn_b200 import synth

RNG = np.random.default_rng(20261202)


# ---- scalar pieces -------------------------------------------------------------

@pytest.mark.parametrize("x", [-40.0, -3.5, -1e-3, 0.0, 0.7, 5.0, 30.0, 700.0])
def test_softplus_matches_logaddexp(x):
    assert oracle.softplus(x) == pytest.approx(np.logaddexp(0.0, x), rel=1e-15, abs=1e-300)


def test_softplus_identities():
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    for x in (0.3, 2.0, 17.0):
        # log(1+e^x) - log(1+e^-x) = x
        assert oracle.softplus(x) - oracle.softplus(-x) == pytest.approx(x, rel=1e-14)
    assert oracle.softplus(-math.inf) == 0.0


def test_sigmoid_and_silu():
    from scipy.special import expit
    for x in (-20.0, -1.0, 0.0, 0.25, 9.0):
        assert oracle.sigmoid(x) == pytest.approx(expit(x), rel=1e-15)
        assert oracle.sigmoid(x) + oracle.sigmoid(-x) == pytest.approx(1.0, rel=1e-15)
        # silu(x) - silu(-x) = x, silu(0) = 0
        assert oracle.silu(x) - oracle.silu(-x) == pytest.approx(x, rel=1e-14, abs=1e-15)
    assert oracle.silu(0.0) == 0.0
    assert oracle.sigmoid(-math.inf) == 0.0


def test_gates_closed_forms():
    g, beta = oracle.gates(0.0, 0.0, 0.0, 0.0)
    assert g == pytest.approx(-math.log(2.0), rel=1e-15) and beta == 0.5
    g, _ = oracle.gates(math.log(3.0), 1.0, -1.0, 0.0)  # a + dt_bias = 0
    assert g == pytest.approx(-3.0 * math.log(2.0), rel=1e-14)
    g, _ = oracle.gates(math.log(16.0), 0.0, 50.0, 0.0)  # softplus(50) = 50 to 1e-22
    assert g == pytest.approx(-800.0, rel=1e-14)
    g, beta = oracle.gates(0.5, 0.0, -math.inf, -math.inf)
    assert g == 0.0 and beta == 0.0  # no decay, no write


# ---- conv and L2 norm ----------------------------------------------------------------

def test_conv_is_valid_cross_correlation():
    xbar = RNG.standard_normal(3 + 17)
    w = RNG.standard_normal(4)
    assert np.allclose(oracle.causal_conv(xbar, w), np.correlate(xbar, w, mode="valid"), rtol=0, atol=1e-13)


def test_conv_tap_order():
    xbar = RNG.standard_normal(3 + 9)
    # tap 3 is the current token: one-hot there is the identity on the inputs
    assert np.array_equal(oracle.causal_conv(xbar, [0, 0, 0, 1.0]), xbar[3:])
    # tap 0 is three tokens back: the output is the history followed by the inputs, delayed
    assert np.array_equal(oracle.causal_conv(xbar, [1.0, 0, 0, 0]), xbar[:9])


def test_l2norm():
    x = RNG.standard_normal(128) * 3.0
    y = oracle.l2norm(x, eps=0.0)
    assert np.linalg.norm(y) == pytest.approx(1.0, rel=1e-15)
    assert np.allclose(y * np.linalg.norm(x), x, rtol=1e-14)
    # eps enters under the square root of the squared norm
    y = oracle.l2norm(np.array([3.0, 4.0]), eps=11.0)
    assert np.allclose(y, [0.5, 4.0 / 6.0], rtol=1e-15)


# ---- the recurrence ----------------------------------------------------------------

def _unit_rows(T, D):
    k = RNG.standard_normal((T, D))
    return k / np.linalg.norm(k, axis=1, keepdims=True)


def test_identity_no_decay_no_write():
    T, D = 9, 6
    q, k, v = RNG.standard_normal((T, D)), _unit_rows(T, D), RNG.standard_normal((T, D))
    S0 = RNG.standard_normal((D, D))
    o, S = oracle.delta_rule(q, k, v, np.zeros(T), np.zeros(T), S0)
    assert np.array_equal(S, S0)
    assert np.allclose(o, q @ S0.T, rtol=0, atol=1e-13)


def test_delta_rule_projection():
    # beta = 1, |k| = 1: after the step the state maps k exactly to v, whatever S_{t-1} and alpha
    D = 8
    S = RNG.standard_normal((D, D))
    for t in range(6):
        q, k, v = RNG.standard_normal((1, D)), _unit_rows(1, D), RNG.standard_normal((1, D))
        g = -abs(RNG.standard_normal()) * 2.0
        _, S = oracle.delta_rule(q, k, v, np.array([g]), np.ones(1), S)
        assert np.allclose(S @ k[0], v[0], rtol=0, atol=1e-12)


def test_decay_only_closed_form():
    T, D = 11, 5
    q, k, v = RNG.standard_normal((T, D)), _unit_rows(T, D), RNG.standard_normal((T, D))
    g = -RNG.uniform(0.0, 2.0, T)
    S0 = RNG.standard_normal((D, D))
    o, S = oracle.delta_rule(q, k, v, g, np.zeros(T), S0)
    G = np.cumsum(g)
    assert np.allclose(S, math.exp(G[-1]) * S0, rtol=1e-13, atol=0)
    assert np.allclose(o, np.exp(G)[:, None] * (q @ S0.T), rtol=1e-13, atol=1e-300)


def test_single_token_from_zero_state():
    D = 7
    q, k, v = RNG.standard_normal((1, D)), _unit_rows(1, D), RNG.standard_normal((1, D))
    beta = 0.37
    o, S = oracle.delta_rule(q, k, v, np.array([-0.4]), np.array([beta]), np.zeros((D, D)))
    assert np.allclose(o[0], beta * v[0] * float(k[0] @ q[0]), rtol=1e-14)
    assert np.allclose(S, beta * np.outer(v[0], k[0]), rtol=1e-14)


@pytest.mark.parametrize("D,Dv,T", [(2, 2, 1), (2, 3, 4), (3, 2, 6), (4, 4, 5)])
def test_brute_force_product_form(D, Dv, T):
    """S_T = S0 P_1...P_T + sum_t beta_t v_t k_t^T P_{t+1}...P_T with
    P_t = alpha_t (I - beta_t k_t k_t^T), evaluated as explicit matrix products."""
    q, k, v = RNG.standard_normal((T, D)), RNG.standard_normal((T, D)), RNG.standard_normal((T, Dv))
    g, beta = -RNG.uniform(0, 1.5, T), RNG.uniform(0, 1, T)
    S0 = RNG.standard_normal((Dv, D))
    o, S = oracle.delta_rule(q, k, v, g, beta, S0)
    P = [math.exp(g[t]) * (np.eye(D) - beta[t] * np.outer(k[t], k[t])) for t in range(T)]

    def state_after(n):
        acc = S0.copy()
        for t in range(n):
            acc = acc @ P[t]
        for t in range(n):
            term = beta[t] * np.outer(v[t], k[t])
            for s in range(t + 1, n):
                term = term @ P[s]
            acc = acc + term
        return acc

    assert np.allclose(S, state_after(T), rtol=1e-12, atol=1e-12)
    for t in range(T):
        assert np.allclose(o[t], state_after(t + 1) @ q[t], rtol=1e-12, atol=1e-12)


def test_state_rows_are_independent():
    T, D = 7, 6
    q, k, v = RNG.standard_normal((T, D)), _unit_rows(T, D), RNG.standard_normal((T, D))
    g, beta = -RNG.uniform(0, 1, T), RNG.uniform(0, 1, T)
    S0 = RNG.standard_normal((D, D))
    o1, S1 = oracle.delta_rule(q, k, v, g, beta, S0)
    S0b = S0.copy()
    S0b[2] += RNG.standard_normal(D)
    o2, S2 = oracle.delta_rule(q, k, v, g, beta, S0b)
    changed_rows = np.nonzero(np.any(S1 != S2, axis=1))[0]
    assert list(changed_rows) == [2]
    assert list(np.nonzero(np.any(o1 != o2, axis=0))[0]) == [2]


# ---- the chunked restatement against the definition -----------------------------------

@pytest.mark.parametrize("chunk", [1, 7, 16, 64])
@pytest.mark.parametrize("long_memory", [False, True])
def test_chunked_form_equals_recurrence(chunk, long_memory):
    T, D = 150, 16
    q, k, v = RNG.standard_normal((T, D)) / 4, _unit_rows(T, D), RNG.standard_normal((T, D))
    g = -RNG.uniform(0.001, 0.01, T) if long_memory else -RNG.uniform(0.03, 60.0, T)
    beta = RNG.uniform(0, 1, T)
    S0 = RNG.standard_normal((D, D)) * 0.05
    o_ref, S_ref = oracle.delta_rule(q, k, v, g, beta, S0)
    o, S = chunked.delta_rule_chunked(q, k, v, g, beta, S0, chunk=chunk)
    scale = max(1.0, np.abs(o_ref).max())
    assert np.abs(o - o_ref).max() <= 1e-12 * scale
    assert np.abs(S - S_ref).max() <= 1e-12 * max(1.0, np.abs(S_ref).max())


# ---- gated RMSNorm ------------------------------------------------------------------

def test_gated_norm_limits():
    o = RNG.standard_normal(128)
    z = np.full(128, 40.0)  # silu(40) = 40 to 1e-16 relative
    y = oracle.gated_rmsnorm(o, z, np.zeros(128), eps=0.0)
    assert np.allclose(y, 40.0 * o / np.sqrt(np.mean(o * o)), rtol=1e-14)
    z = RNG.standard_normal(128)
    w = RNG.standard_normal(128) * 0.1
    y1 = oracle.gated_rmsnorm(o, z, w, eps=0.0)
    y2 = oracle.gated_rmsnorm(o * 1234.5, z, w, eps=0.0)
    assert np.allclose(y1, y2, rtol=1e-13)
    # w = -1 switches the head off (zero-centred weight: scale is 1 + w)
    assert np.all(oracle.gated_rmsnorm(o, z, -np.ones(128)) == 0.0)
    # constant o = c: rms = |c|, y = sign(c) * (1 + w) * silu(z) up to eps
    y = oracle.gated_rmsnorm(np.full(128, -2.0), z, w, eps=0.0)
    from scipy.special import expit
    assert np.allclose(y, -(1 + w) * z * expit(z), rtol=1e-14)


# ---- the whole mixer ------------------------------------------------------------------

TINY = synth.Dims(num_k_heads=2, num_v_heads=6, head_dim=8, conv_width=4)


def _mixer(case, cu=None, **kw):
    w = case["weights"]
    f = synth.to_f64
    cu = case["cu_seqlens"].numpy() if cu is None else cu
    return oracle.mixer(case["dims"], cu, f(case["qkv"]), f(case["z"]), f(case["a"]), f(case["b"]),
                        f(w["conv_w"]), f(w["A_log"]), f(w["dt_bias"]), f(w["norm_w"]),
                        f(case["init_state"]), f(case["init_conv"]), **kw)


def _compose_by_hand(case):
    """Mixer rebuilt in numpy from the pinned stage functions: pins the wiring
    (channel split [q|k|v], value head h reading q/k head h // (Vh/Kh))."""
    d = case["dims"]
    Kh, Vh, D, W = d.num_k_heads, d.num_v_heads, d.head_dim, d.conv_width
    f = synth.to_f64
    w = {k: f(x) for k, x in case["weights"].items()}
    qkv, z, a, b = f(case["qkv"]), f(case["z"]), f(case["a"]), f(case["b"])
    cu = case["cu_seqlens"].numpy()
    outs, states = [], []
    for n in range(len(cu) - 1):
        t0, t1 = cu[n], cu[n + 1]
        hist = np.zeros((W - 1, qkv.shape[1])) if case["init_conv"] is None else f(case["init_conv"])[n]
        xbar = np.concatenate([hist, qkv[t0:t1]], 0)
        conv = np.stack([oracle.causal_conv(xbar[:, ch], w["conv_w"][ch]) for ch in range(qkv.shape[1])], 1)
        act = np.vectorize(oracle.silu)(conv)
        out = np.zeros((t1 - t0, Vh * D))
        st = []
        for h in range(Vh):
            kap = h // (Vh // Kh)
            qh = act[:, kap * D:(kap + 1) * D]
            kh = act[:, Kh * D + kap * D: Kh * D + (kap + 1) * D]
            vh = act[:, 2 * Kh * D + h * D: 2 * Kh * D + (h + 1) * D]
            qn = np.stack([oracle.l2norm(r) for r in qh]) / math.sqrt(D)
            kn = np.stack([oracle.l2norm(r) for r in kh])
            gb = [oracle.gates(w["A_log"][h], w["dt_bias"][h], a[t, h], b[t, h]) for t in range(t0, t1)]
            g = np.array([x[0] for x in gb])
            beta = np.array([x[1] for x in gb])
            S0 = np.zeros((D, D)) if case["init_state"] is None else f(case["init_state"])[n, h]
            o, S = oracle.delta_rule(qn, kn, vh, g, beta, S0)
            for t in range(t1 - t0):
                out[t, h * D:(h + 1) * D] = oracle.gated_rmsnorm(o[t], z[t0 + t, h * D:(h + 1) * D], w["norm_w"])
            st.append(S)
        outs.append(out)
        states.append(np.stack(st))
    return np.concatenate(outs, 0), np.stack(states)


def test_mixer_equals_composed_stages():
    case = synth.prefill_case(7, [5, 1, 9], TINY, init=True)
    res = _mixer(case)
    out, st = _compose_by_hand(case)
    assert np.allclose(res["out"], out, rtol=1e-13, atol=1e-13)
    assert np.allclose(res["state"], st, rtol=1e-13, atol=1e-13)


def test_mixer_history_is_exact_copy():
    case = synth.prefill_case(8, [0, 1, 2, 3, 6], TINY, init=True)
    res = _mixer(case)
    qkv, hist, cu = synth.to_f64(case["qkv"]), synth.to_f64(case["init_conv"]), case["cu_seqlens"].numpy()
    for n in range(5):
        xbar = np.concatenate([hist[n], qkv[cu[n]:cu[n + 1]]], 0)
        assert np.array_equal(res["conv"][n], xbar[-3:])


def test_mixer_split_equals_single_call():
    case = synth.prefill_case(9, [23], TINY, init=True)
    full = _mixer(case)
    first = dict(case)
    cut = 10
    first_part = {**case, "cu_seqlens": torch.tensor([0, cut], dtype=torch.int32)}
    r1 = _mixer(first_part)
    second = {**case, "qkv": case["qkv"][cut:], "z": case["z"][cut:], "a": case["a"][cut:], "b": case["b"][cut:],
              "cu_seqlens": torch.tensor([0, 23 - cut], dtype=torch.int32),
              "init_state": torch.from_numpy(r1["state"]), "init_conv": torch.from_numpy(r1["conv"])}
    r2 = _mixer(second)
    assert np.allclose(np.concatenate([r1["out"], r2["out"]]), full["out"], rtol=1e-12, atol=1e-12)
    assert np.allclose(r2["state"], full["state"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(r2["conv"], full["conv"])
    del first


def test_mixer_decode_chain_equals_prefill():
    case = synth.prefill_case(10, [12], TINY, init=True)
    full = _mixer(case)
    st, cv = case["init_state"], case["init_conv"]
    outs = []
    for t in range(12):
        step = {**case, "qkv": case["qkv"][t:t + 1], "z": case["z"][t:t + 1], "a": case["a"][t:t + 1],
                "b": case["b"][t:t + 1], "cu_seqlens": torch.tensor([0, 1], dtype=torch.int32),
                "init_state": st, "init_conv": cv}
        r = _mixer(step)
        outs.append(r["out"])
        st, cv = torch.from_numpy(r["state"]), torch.from_numpy(r["conv"])
    assert np.allclose(np.concatenate(outs), full["out"], rtol=1e-12, atol=1e-12)
    assert np.allclose(st.numpy(), full["state"], rtol=1e-12, atol=1e-12)


def test_mixer_no_decay_no_write_keeps_state():
    case = synth.prefill_case(11, [4, 6], TINY, init=True)
    case["a"] = torch.full_like(case["a"], -math.inf)   # softplus(-inf) = 0: g = 0
    case["b"] = torch.full_like(case["b"], -math.inf)   # sigmoid(-inf) = 0: beta = 0
    res = _mixer(case)
    assert np.array_equal(res["state"], synth.to_f64(case["init_state"]))


def test_mixer_head_subset():
    case = synth.prefill_case(12, [7, 3], TINY, init=True)
    full = _mixer(case)
    part = _mixer(case, heads=(2, 5))
    D = TINY.head_dim
    assert np.array_equal(part["out"], full["out"][:, 2 * D:5 * D])
    assert np.array_equal(part["state"], full["state"][:, 2:5])


def test_group_case_reproduces_full_mixer_heads():
    """The one-q/k-head sub-problem used by the full-size parity tests gives
    exactly the full mixer's outputs, states and history for that group."""
    from _util import group_case
    case = synth.prefill_case(13, [9, 4], TINY, init=True)
    full = _mixer(case)
    sub = group_case(case, 1)
    part = _mixer(sub)
    D = TINY.head_dim
    hs = sub["heads"].numpy()
    assert np.array_equal(part["out"], full["out"][:, hs[0] * D:(hs[-1] + 1) * D])
    assert np.array_equal(part["state"], full["state"][:, hs])
    assert np.array_equal(part["conv"], full["conv"][:, :, sub["channels"].numpy()])


def test_projection_is_the_linear_layer_definition():
    """y[t][n] = sum_k x[t][k] w[n][k]: against an explicit triple loop on a tiny
    case, the identity weight, and a one-hot row of the weight."""
    import oracle
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 4))
    w = rng.standard_normal((5, 4))
    y = oracle.projection(x, w)
    ref = np.zeros((3, 5))
    for t in range(3):
        for n in range(5):
            for k in range(4):
                ref[t, n] += x[t, k] * w[n, k]
    assert y.shape == (3, 5) and np.allclose(y, ref, rtol=0, atol=1e-12)
    assert np.array_equal(oracle.projection(x, np.eye(4)), x)
    w1 = np.zeros((2, 4))
    w1[1, 2] = 1.0
    assert np.array_equal(oracle.projection(x, w1)[:, 1], x[:, 2]) and not oracle.projection(x, w1)[:, 0].any()
