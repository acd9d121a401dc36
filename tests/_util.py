"""Shared helpers of the tests: run the oracle on a synthetic case, move a case
to the GPU, and the parity measures with their bars.

Bars (stated for the GDN path): outputs within 2e-2 maximum relative error,
each element's error divided by max(|y_ref|, rms(y_ref)) so that elements near
zero are measured against the output RMS; final states
||S - S_ref||_F / ||S_ref||_F <= 1e-3 per row; conv histories bit-exact.
Two aggregate output checks ride along: rms(y - y_ref) / rms(y_ref) <= 5e-3
and, recorded only, max|y - y_ref| / rms(y_ref) (dominated by the bf16
rounding of the largest outputs, whose magnitude reaches ~40x the RMS).

With GDN_PARITY_LOG=<path> in the environment, every parity check appends one
JSON line (test name, the measured errors, the bars) to that file, so the
margins of each workload can be collected from a GPU run.
"""
import json
import os

import numpy as np
import torch

import oracle
from gated_deltanet_mixer_gdn_b200 import synth

OUT_TOL = 2e-2
OUT_RMS_TOL = 5e-3
STATE_TOL = 1e-3


def oracle_prefill(case, cu=None, heads=None, nthreads=0, init_state=None, init_conv=None, acts=None):
    """Oracle on a synth case (dense cases are flattened to packed rows)."""
    d = case["dims"]
    f = synth.to_f64
    w = case["weights"]
    acts = acts or {k: case[k] for k in ("qkv", "z", "a", "b")}
    if cu is None:
        if "cu_seqlens" in case:
            cu = case["cu_seqlens"].numpy()
        else:
            B, T = acts["qkv"].shape[0], acts["qkv"].shape[1]
            cu = np.arange(B + 1, dtype=np.int64) * T
    flat = {k: v.reshape(-1, v.shape[-1]) for k, v in acts.items()}
    st = case["init_state"] if init_state is None else init_state
    cv = case["init_conv"] if init_conv is None else init_conv
    return oracle.mixer(d, cu, f(flat["qkv"]), f(flat["z"]), f(flat["a"]), f(flat["b"]),
                        f(w["conv_w"]), f(w["A_log"]), f(w["dt_bias"]), f(w["norm_w"]),
                        None if st is None else (st.numpy() if isinstance(st, torch.Tensor) else st).astype(np.float64),
                        None if cv is None else (cv.numpy() if isinstance(cv, torch.Tensor) else cv).astype(np.float64),
                        heads=heads, nthreads=nthreads)


def _as64(y, shape):
    y = y.float().cpu().numpy().astype(np.float64) if isinstance(y, torch.Tensor) else y
    return y.reshape(shape)


def out_err(y, y_ref):
    """max_i |y_i - y_ref_i| / max(|y_ref_i|, rms(y_ref))"""
    y = _as64(y, y_ref.shape)
    if y_ref.size == 0:
        return 0.0
    rms = max(np.sqrt(np.mean(y_ref * y_ref)), 1e-30)
    return float((np.abs(y - y_ref) / np.maximum(np.abs(y_ref), rms)).max())


def out_rms_err(y, y_ref):
    """rms(y - y_ref) / rms(y_ref)"""
    y = _as64(y, y_ref.shape)
    if y_ref.size == 0:
        return 0.0
    return float(np.sqrt(np.mean((y - y_ref) ** 2)) / max(np.sqrt(np.mean(y_ref * y_ref)), 1e-30))


def record(name, **values):
    """Append the measured errors of one parity check to $GDN_PARITY_LOG (if set)."""
    path = os.environ.get("GDN_PARITY_LOG")
    if not path:
        return
    line = {"check": name, **{k: float(v) if isinstance(v, (float, np.floating)) else v for k, v in values.items()},
            "bars": {"out": OUT_TOL, "out_rms": OUT_RMS_TOL, "state": STATE_TOL}}
    with open(path, "a") as f:
        f.write(json.dumps(line) + "\n")


def check_outputs(name, out, ref_out, fs=None, ref_state=None, fc=None, ref_conv=None):
    """Assert the output, state and history bars; record the measured errors."""
    e_out, e_rms, e_max = out_err(out, ref_out), out_rms_err(out, ref_out), out_maxabs_over_rms(out, ref_out)
    e_st = state_err(fs, ref_state) if fs is not None else None
    record(name, out=e_out, out_rms=e_rms, out_maxabs_over_rms=e_max, state=e_st)
    assert e_out <= OUT_TOL, f"{name}: output error {e_out:.3e}"
    assert e_rms <= OUT_RMS_TOL, f"{name}: output rms error {e_rms:.3e}"
    if fs is not None:
        assert e_st <= STATE_TOL, f"{name}: state error {e_st:.3e}"
    if fc is not None:
        assert conv_exact(fc, ref_conv), f"{name}: conv history not bit-exact"
    return e_out, e_st


def out_maxabs_over_rms(y, y_ref):
    y = _as64(y, y_ref.shape)
    if y_ref.size == 0:
        return 0.0
    return float(np.abs(y - y_ref).max() / max(np.sqrt(np.mean(y_ref * y_ref)), 1e-30))


def state_err(S, S_ref):
    """Worst per-row relative Frobenius error; S, S_ref [N, H, D, D]."""
    S = S.double().cpu().numpy() if isinstance(S, torch.Tensor) else S
    S = S.reshape(S_ref.shape)
    errs = []
    for n in range(S_ref.shape[0]):
        den = np.linalg.norm(S_ref[n])
        num = np.linalg.norm(S[n] - S_ref[n])
        errs.append(num / den if den > 0 else num)
    return float(max(errs)) if errs else 0.0


def conv_exact(cv, cv_ref):
    cv = cv.double().cpu().numpy() if isinstance(cv, torch.Tensor) else cv
    return bool(np.array_equal(cv.reshape(cv_ref.shape), cv_ref))


def to_dev(case, device="cuda"):
    w = {k: v.to(device) for k, v in case["weights"].items()}
    acts = {k: case[k].to(device) for k in ("qkv", "z", "a", "b")}
    st = None if case["init_state"] is None else case["init_state"].to(device)
    cv = None if case["init_conv"] is None else case["init_conv"].to(device)
    return w, acts, st, cv


def group_case(case, kappa):
    """The sub-problem of q/k head(s) `kappa` (an int or a list): their q and k
    channels, the channels, z, gates and parameters of their value heads, as a
    case with len(kappa) q/k heads.  The mixer computes each value head from
    exactly these inputs, so the oracle on this case gives those heads' outputs
    and states (and the history of these channels) at a fraction of the cost."""
    d = case["dims"]
    groups = [kappa] if isinstance(kappa, int) else list(kappa)
    G, D = d.num_v_heads // d.num_k_heads, d.head_dim
    heads = [kp * G + j for kp in groups for j in range(G)]
    ch = [kp * D + c for kp in groups for c in range(D)]
    ch += [d.num_k_heads * D + kp * D + c for kp in groups for c in range(D)]
    ch += [2 * d.num_k_heads * D + h * D + c for h in heads for c in range(D)]
    ch = torch.tensor(ch)
    zc = torch.tensor([h * D + c for h in heads for c in range(D)])
    hs = torch.tensor(heads)
    sub = dict(case)
    sub["dims"] = synth.Dims(num_k_heads=len(groups), num_v_heads=G * len(groups), head_dim=D,
                             conv_width=d.conv_width)
    w = case["weights"]
    sub["weights"] = {"conv_w": w["conv_w"][ch], "A_log": w["A_log"][hs], "dt_bias": w["dt_bias"][hs],
                      "norm_w": w["norm_w"]}
    for k, idx in (("qkv", ch), ("z", zc), ("a", hs), ("b", hs)):
        sub[k] = case[k].index_select(-1, idx).contiguous()
    if case.get("init_state") is not None:
        sub["init_state"] = case["init_state"][:, hs].contiguous()
    if case.get("init_conv") is not None:
        sub["init_conv"] = case["init_conv"].index_select(-1, ch).contiguous()
    sub["channels"], sub["z_channels"], sub["heads"] = ch, zc, hs
    return sub
