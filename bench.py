"""Benchmark of the B200 Gated DeltaNet mixer.

Default workload (N=1): the decode batch — 64 rows x 128 successive single-token
steps with the 27B model's GDN shapes, each row with its own f32 state
[48,128,128] ~ N(0,0.05) and conv history ~ N(0,1).  One bench step = that
whole pass (128 decode launches, 8192 row-tokens).  Metric: row-tokens/s.
A second measured object, "prefill", times the chunked prefill (one row of
8192 tokens from zero state, and the 8-row varlen workload) in tokens/s
against the tensor roofline; a third, "decode_multi", the same decode batch
with 4 tokens per row per call (gdn_decode_multi); a fourth, "projections",
the in_proj / out_proj GEMMs around the mixer at the layer's shapes; a fifth,
"prefill_from_hidden", one row of 8192 tokens from the hidden states with the
load stage inside the in_proj GEMM, beside in_proj followed by the prefill.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N>1) every rank runs its own replica of the workload (the rows
are independent: weak scaling, no collective on the data path); the time is
the max over ranks.  ``--impl reference`` times the float64 CPU oracle on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_mixer_gdn_b200 import synth  # noqa: E402

ROWS, DECODE_STEPS = 64, 128
STATE_BYTES_PER_ROW_TOKEN = 2 * 48 * 128 * 128 * 4          # f32 state read + write
PREFILL_T = 8192
PREFILL_FLOP_PER_TOKEN = 7602176                               # chunk-64 contraction FLOPs, 48 heads
PREFILL_BYTES_PER_TOKEN = 10240 * 2 + 6144 * 2 + 2 * 48 * 2 + 6144 * 2


def decode_traffic():
    """DRAM bytes per decode launch from the committed ncu record, if it was taken
    on the decode kernel's current source; else None."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", "gdn_decode_kernel_traffic.json")
    src = os.path.join(ROOT, "gated_deltanet_mixer_gdn_b200", "csrc", "decode.cuh")
    if not os.path.exists(rec):
        return None
    with open(rec) as f:
        d = json.load(f)
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    return d.get("bytes_per_launch") if d.get("decode_cuh_sha256") == h else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        finally:
            os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- oracle timing

def oracle_decode_sample(case, steps: int, rows: int):
    """Time the float64 oracle on `rows` rows x `steps` decode tokens (all 48 heads)."""
    import numpy as np
    import oracle
    f = synth.to_f64
    w = case["weights"]
    st = f(case["init_state"][:rows])
    cv = f(case["init_conv"][:rows])
    cu = np.arange(rows + 1)
    t0 = time.perf_counter()
    for s in range(steps):
        r = oracle.mixer(case["dims"], cu, f(case["qkv"][s, :rows]), f(case["z"][s, :rows]), f(case["a"][s, :rows]),
                         f(case["b"][s, :rows]), f(w["conv_w"]), f(w["A_log"]), f(w["dt_bias"]), f(w["norm_w"]),
                         st, cv)
        st, cv = r["state"], r["conv"]
    return time.perf_counter() - t0


def cpu_baseline_line(case, budget_s: float = 15.0):
    import oracle
    oracle.build()
    rows = 16
    dt = oracle_decode_sample(case, 1, rows)  # also warms up
    steps = max(1, min(DECODE_STEPS, int(budget_s / max(dt, 1e-3))))
    dt = oracle_decode_sample(case, steps, rows)
    return {"value": rows * steps / dt, "unit": "row-tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{rows} rows x {steps} decode tokens of the 64x128 decode batch (all 48 heads), f64"}


DECODE_METRIC = "GDN decode row-tokens/s (64-row batch, 128 steps)"


def decode_config(world):
    return {"workload": "decode 64 rows x 128 steps, Qwen3.8-27B GDN layer shapes (16 qk / 48 v heads, dim 128), "
                        "per-row f32 state", "rows": ROWS, "tokens_per_row": DECODE_STEPS,
            "parallelism": f"replicas x{world}", "l2": "inputs larger than L2 (402.7 MB of state per step)"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    case = synth.config(1)
    import oracle
    oracle.build()
    rows, steps = 16, 4
    for _ in range(args.warmup):
        oracle_decode_sample(case, steps, rows)
    t = 0.0
    for _ in range(args.steps):
        t += oracle_decode_sample(case, steps, rows)
    value = rows * steps * args.steps / t
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value,
            "unit": "row-tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(1),
            "cpu_baseline": {"value": value, "unit": "row-tokens/s", "cores": oracle.max_threads(),
                             "kind": "oracle", "sample": f"{rows} rows x {steps} tokens per step, all 48 heads"},
            "e2e": {"value": value, "unit": "row-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------- our path

def run_ours(args, world, rank, local):
    import gated_deltanet_mixer_gdn_b200 as gdn
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    case = synth.config(1)
    w = gdn.weights_to(case["weights"], dev)
    qkv = case["qkv"].to(dev)
    z = case["z"].to(dev)
    a = case["a"].to(dev)
    b = case["b"].to(dev)
    state0 = case["init_state"].to(dev)
    conv0 = case["init_conv"].to(dev)
    state = state0.clone()
    conv = conv0.clone()
    out = torch.empty((DECODE_STEPS, ROWS, 6144), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)

    def one_pass():
        for s in range(DECODE_STEPS):
            gdn.decode(qkv[s], z[s], a[s], b[s], w, state, conv, out=out[s])

    # capture the 128-launch pass in a CUDA graph (inputs already resident)
    with torch.cuda.stream(stream):
        one_pass()  # warm, loads the library
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        one_pass()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    t_ms = e0.elapsed_time(e1)
    t_max = max_over_ranks(t_ms, world)
    clocks = clk.summary()
    launches = args.steps * DECODE_STEPS
    per_launch_s = t_ms / 1000.0 / launches
    value = world * ROWS * DECODE_STEPS * args.steps / (t_max / 1000.0)
    achieved = ROWS * STATE_BYTES_PER_ROW_TOKEN / per_launch_s / 1e9

    # ---- end to end through the public API with host buffers
    pin = {k: case[k].pin_memory() for k in ("qkv", "z", "a", "b")}
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in pin.items()}
    host_out = torch.empty((DECODE_STEPS, ROWS, 6144), dtype=torch.bfloat16).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = host_out.numel() * host_out.element_size()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 5))
    # A serving loop: the inputs of a group of G decode steps go host -> device on a copy stream
    # while the previous group computes, and each group's outputs go back on another stream while
    # the next group computes (every byte of every step still crosses inside the timed region).
    # Device inputs and outputs are double-buffered across passes, so the next pass's first
    # copies run during this pass's last group.
    G = 16
    groups = DECODE_STEPS // G
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    bufs = [(dev_in, out), ({k: torch.empty_like(v) for k, v in dev_in.items()}, torch.empty_like(out))]
    ev_in = [torch.cuda.Event() for _ in range(groups)]
    ev_out = [torch.cuda.Event() for _ in range(groups)]
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]   # a pass's decodes done with its buffers
    ev_read = [torch.cuda.Event(), torch.cuda.Event()]   # a pass's outputs copied to the host
    barrier(world)
    torch.cuda.synchronize(dev)
    e2.record(stream)
    h2d_stream.wait_event(e2)
    for p in range(e2e_steps):
        din, dout = bufs[p % 2]
        if p >= 2:
            h2d_stream.wait_event(ev_used[p % 2])   # the pass before the last consumed din
            stream.wait_event(ev_read[p % 2])       # and its outputs have left dout
        for g in range(groups):
            sl = slice(g * G, (g + 1) * G)
            with torch.cuda.stream(h2d_stream):
                for k in din:
                    din[k][sl].copy_(pin[k][sl], non_blocking=True)
                ev_in[g].record(h2d_stream)
            stream.wait_event(ev_in[g])
            with torch.cuda.stream(stream):
                for s in range(g * G, (g + 1) * G):
                    gdn.decode(din["qkv"][s], din["z"][s], din["a"][s], din["b"][s], w, state, conv, out=dout[s])
                ev_out[g].record(stream)
            d2h_stream.wait_event(ev_out[g])
            with torch.cuda.stream(d2h_stream):
                host_out[sl].copy_(dout[sl], non_blocking=True)
        ev_used[p % 2].record(stream)
        ev_read[p % 2].record(d2h_stream)
    stream.wait_stream(d2h_stream)
    stream.wait_stream(h2d_stream)
    e3.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    t_e2e = max_over_ranks(e2.elapsed_time(e3), world)
    e2e_value = world * ROWS * DECODE_STEPS * e2e_steps / (t_e2e / 1000.0)

    line = None
    if rank == 0:
        line = {
            "metric": DECODE_METRIC,
            "value": value, "unit": "row-tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_max / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": decode_config(world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": decode_traffic(),
                         "kernel": "gdn_decode_kernel", "peak_source": peaks["source"],
                         "algorithmic_bytes_per_launch": ROWS * STATE_BYTES_PER_ROW_TOKEN},
            "e2e": {"value": e2e_value, "unit": "row-tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "clocks": clocks,
            "gpu_launches": launches,
        }
    return line, case


def bench_decode_multi(args, local, k=4):
    """The same 64-row, 128-token decode batch with k tokens per row per call
    (gdn_decode_multi): 128 / k launches per pass, the state read and written once
    per launch.  CUDA events on the launching stream around a captured pass."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    case = synth.config(1)
    w = gdn.weights_to(case["weights"], dev)
    # [steps, rows, ...] -> per launch [rows, k, ...]
    acts = {n: case[n].to(dev).view(DECODE_STEPS // k, k, ROWS, -1).transpose(1, 2).contiguous()
            for n in ("qkv", "z", "a", "b")}
    state = case["init_state"].to(dev)
    conv = case["init_conv"].to(dev)
    out = torch.empty((DECODE_STEPS // k, ROWS, k, 6144), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)

    def one_pass():
        for s in range(DECODE_STEPS // k):
            gdn.decode_multi(acts["qkv"][s], acts["z"][s], acts["a"][s], acts["b"][s], w, state, conv, out=out[s])

    with torch.cuda.stream(stream):
        one_pass()
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        one_pass()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    t = e0.elapsed_time(e1) / 1000.0
    launches = args.steps * (DECODE_STEPS // k)
    achieved = ROWS * STATE_BYTES_PER_ROW_TOKEN / (t / launches) / 1e9  # state bytes per launch / launch time
    return {"workload": f"decode 64 rows x 128 tokens, {k} tokens per row per call", "tokens_per_call": k,
            "value": ROWS * DECODE_STEPS * args.steps / t, "unit": "row-tokens/s",
            "us_per_launch": t / launches * 1e6,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                         "algorithmic_bytes_per_launch": ROWS * STATE_BYTES_PER_ROW_TOKEN},
            "gpu_launches": launches}


def bench_projections(args, local, T=8192):
    """The projections around the mixer at the 27B layer's shapes: in_proj
    [T,5120] x [16480,5120]^T and out_proj [T,6144] x [5120,6144]^T (bf16, f32
    accumulation), random inputs; CUDA events on the launching stream, L2 flushed
    between calls."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    d = synth.MODEL
    H = 5120
    N = d.conv_channels + d.value_width + 2 * d.num_v_heads
    g = torch.Generator(device=dev).manual_seed(7)
    x = torch.randn((T, H), generator=g, device=dev).to(torch.bfloat16)
    w_in = (torch.randn((N, H), generator=g, device=dev) * H ** -0.5).to(torch.bfloat16)
    y = torch.randn((T, d.value_width), generator=g, device=dev).to(torch.bfloat16)
    w_out = (torch.randn((H, d.value_width), generator=g, device=dev) * d.value_width ** -0.5).to(torch.bfloat16)
    outs = gdn.in_proj(x, w_in)
    o = gdn.out_proj(y, w_out)
    stream = torch.cuda.Stream(dev)
    res = {}
    for name, call, flop, shape in (
            ("in_proj", lambda: gdn.in_proj(x, w_in, out=outs), 2 * T * N * H, f"[{T},{H}] x [{N},{H}]^T"),
            ("out_proj", lambda: gdn.out_proj(y, w_out, out=o), 2 * T * H * d.value_width,
             f"[{T},{d.value_width}] x [{H},{d.value_width}]^T")):
        t, n = _time_prefill(call, dev, stream, max(3, args.warmup), max(5, args.steps))
        tf = flop / t / 1e12
        res[name] = {"workload": shape + " bf16, f32 accumulation", "ms": t * 1000.0, "tflops": tf,
                     "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                  "frac": tf / peaks["bf16_tflops"], "peak_source": peaks["source"],
                                  # the launches run back to back for several ms, under the power cap:
                                  # against the seconds-long cuBLAS figure as well
                                  "peak_sustained": peaks["bf16_tflops_sustained"],
                                  "frac_sustained": tf / peaks["bf16_tflops_sustained"]},
                     "gpu_launches": n}
    return res


def prefill_launches(B, T, from_hidden=False):
    """Kernels one dense prefill call (final state returned) launches, from the library's own
    schedule (load stage, history writer, WY records and recurrence per segment)."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    return gdn.prefill_schedule(B, T, from_hidden)[1]


def prefill_launches_varlen():
    """Kernels one packed (varlen) prefill call launches: load stage, history writer, chunk
    offsets and row order, WY records, recurrence."""
    return 5


def bench_hidden(args, local, T=8192):
    """Prefill of one row of T tokens from the layer's hidden states [T,5120]: the load
    stage inside the in_proj GEMM (gdn_prefill_hidden) against in_proj followed by the
    prefill (both on the same inputs, bit-identical results)."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    dev = torch.device("cuda", local)
    d = synth.MODEL
    H = 5120
    N = d.conv_channels + d.value_width + 2 * d.num_v_heads
    g = torch.Generator(device=dev).manual_seed(11)
    w = gdn.weights_to(synth.draw_weights(torch.Generator().manual_seed(11), d), dev)
    x = torch.randn((1, T, H), generator=g, device=dev).to(torch.bfloat16)
    w_in = (torch.randn((N, H), generator=g, device=dev) * H ** -0.5).to(torch.bfloat16)
    out = torch.empty((1, T, d.value_width), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, d.num_v_heads, 128, 128), dtype=torch.float32, device=dev)
    fc = torch.empty((1, 3, d.conv_channels), dtype=torch.float32, device=dev)
    proj = gdn.in_proj(x[0], w_in)
    stream = torch.cuda.Stream(dev)

    def unfused():
        gdn.in_proj(x[0], w_in, out=proj)
        q, z, a, b = (t.unsqueeze(0) for t in proj)
        gdn.prefill(q, z, a, b, w, out=out, final_state=fs, final_conv=fc)

    reps = max(5, args.steps)
    tf, nf = _time_prefill(lambda: gdn.prefill_hidden(x, w_in, w, out=out, final_state=fs, final_conv=fc),
                           dev, stream, max(3, args.warmup), reps)
    tu, nu = _time_prefill(unfused, dev, stream, max(3, args.warmup), reps)
    return {"workload": f"prefill B=1 T={T} from hidden states [{T},{H}] (in_proj 5120->{N} + mixer), "
                        "zero initial state",
            "fused": {"value": T / tf, "unit": "tokens/s", "ms": tf * 1000.0,
                      "gpu_launches": prefill_launches(1, T, True) * nf},
            "unfused": {"value": T / tu, "unit": "tokens/s", "ms": tu * 1000.0,
                        "gpu_launches": (1 + prefill_launches(1, T)) * nu},
            "l2": "flushed (256 MiB write) before each timed call"}


def bench_prefill_out(args, local, T=8192):
    """The mixer followed by out_proj (hidden 5120) for one row of T tokens: gdn_prefill_out (each
    segment's projection overlapped with the later segments' recurrence) against gdn_prefill
    followed by gdn_out_proj (bit-identical results)."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    dev = torch.device("cuda", local)
    case = synth.config(2) if T == 8192 else synth.dense_case(1236, 1, T)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    g = torch.Generator(device=dev).manual_seed(13)
    w_out = (torch.randn((5120, 6144), generator=g, device=dev) * 6144 ** -0.5).to(torch.bfloat16)
    out = torch.empty((1, T, 5120), dtype=torch.bfloat16, device=dev)
    y = torch.empty((1, T, 6144), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, 48, 128, 128), dtype=torch.float32, device=dev)
    fc = torch.empty((1, 3, 10240), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    warm, reps = max(3, args.warmup), max(5, args.steps)
    tf, nf = _time_prefill(lambda: gdn.prefill_out(acts["qkv"], acts["z"], acts["a"], acts["b"], w, w_out, out=out,
                                                   final_state=fs, final_conv=fc), dev, stream, warm, reps)

    def pair():
        gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, out=y, final_state=fs, final_conv=fc)
        gdn.out_proj(y[0], w_out, out=out[0])

    tu, nu = _time_prefill(pair, dev, stream, warm, reps)
    segs = gdn.prefill_schedule(1, T)[0]
    return {"workload": f"prefill B=1 T={T} then out_proj [{T},6144] x [5120,6144]^T, zero initial state",
            "fused": {"value": T / tf, "unit": "tokens/s", "ms": tf * 1000.0,
                      "gpu_launches": (prefill_launches(1, T) + segs) * nf},
            "unfused": {"value": T / tu, "unit": "tokens/s", "ms": tu * 1000.0,
                        "gpu_launches": (prefill_launches(1, T) + 1) * nu},
            "l2": "flushed (256 MiB write) before each timed call"}


def _time_prefill(call, dev, stream, warmup, reps):
    """Median seconds of `call` (CUDA events on `stream`), L2 flushed before each timed call."""
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > L2, written between iterations
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            call()
        torch.cuda.synchronize(dev)
        pt = []
        for _ in range(reps):
            flush.fill_(1)
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            call()
            s1.record(stream)
            s1.synchronize()
            pt.append(s0.elapsed_time(s1) / 1000.0)
    return statistics.median(pt), len(pt)


def prefill_line(tokens, sec, workload, launches, peaks):
    tf = tokens * PREFILL_FLOP_PER_TOKEN / sec / 1e12
    return {"workload": workload, "value": tokens / sec, "unit": "tokens/s", "ms": sec * 1000.0,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / peaks["bf16_tflops"], "peak_source": peaks["source"],
                         "scope": "whole call (every kernel of the prefill)",
                         "algorithmic_flop_per_token": PREFILL_FLOP_PER_TOKEN},
            "l2": "flushed (256 MiB write) before each timed call", "gpu_launches": launches}


def oracle_prefill_sample(case, rows, tokens):
    """Seconds the float64 oracle takes for the first `tokens` tokens of each of the given rows
    (all 48 heads, the rows' initial state and history)."""
    import numpy as np
    import oracle
    f = synth.to_f64
    w = case["weights"]
    if "cu_seqlens" in case:
        cu = case["cu_seqlens"].tolist()
        spans = [(cu[r], min(cu[r + 1], cu[r] + tokens)) for r in rows]
        take = lambda t: torch.cat([t[a:b] for a, b in spans])  # noqa: E731
    else:
        spans = [(0, tokens)] * len(rows)
        take = lambda t: t[list(rows), :tokens].reshape(-1, t.shape[-1])  # noqa: E731
    lens = [b - a for a, b in spans]
    cu_s = np.concatenate([[0], np.cumsum(lens)])
    st = None if case["init_state"] is None else f(case["init_state"][list(rows)])
    cv = None if case["init_conv"] is None else f(case["init_conv"][list(rows)])
    acts = {k: f(take(case[k])) for k in ("qkv", "z", "a", "b")}
    t0 = time.perf_counter()
    oracle.mixer(case["dims"], cu_s, acts["qkv"], acts["z"], acts["a"], acts["b"], f(w["conv_w"]), f(w["A_log"]),
                 f(w["dt_bias"]), f(w["norm_w"]), st, cv)
    return time.perf_counter() - t0, int(sum(lens))


def prefill_cpu_baseline(case, rows, tokens, what):
    import oracle
    oracle.build()
    dt, n = oracle_prefill_sample(case, rows, tokens)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{what}: {n} tokens ({len(rows)} row(s), up to {tokens} tokens each), all 48 heads, f64 "
                      f"({dt:.1f} s)"}


def prefill_e2e(args, dev, case, w, seg=2048):
    """One row of T tokens through the public API from pinned host buffers, as a serving loop
    streams a long prompt: the row is cut into segments of `seg` tokens; segment k+1's inputs
    go host -> device on a copy stream while segment k runs (each segment's prefill continues
    from the state and history the previous one left), and each segment's output goes back on
    another stream; the final state and history come back after the last segment.  Every input
    and output byte crosses inside the timed region."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    T = case["qkv"].shape[1]
    nseg = T // seg
    pin = {k: case[k][0].pin_memory() for k in ("qkv", "z", "a", "b")}
    din = {k: torch.empty_like(v, device=dev) for k, v in pin.items()}
    host_out = torch.empty((T, 6144), dtype=torch.bfloat16).pin_memory()
    host_st = torch.empty((1, 48, 128, 128), dtype=torch.float32).pin_memory()
    host_cv = torch.empty((1, 3, 10240), dtype=torch.float32).pin_memory()
    dout = torch.empty((T, 6144), dtype=torch.bfloat16, device=dev)
    st = [torch.empty((1, 48, 128, 128), dtype=torch.float32, device=dev) for _ in range(2)]
    cv = [torch.empty((1, 3, 10240), dtype=torch.float32, device=dev) for _ in range(2)]
    h2d_bytes = sum(v.numel() * v.element_size() for v in pin.values())
    d2h_bytes = host_out.numel() * 2 + host_st.numel() * 4 + host_cv.numel() * 4
    comp, h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nseg)]
    ev_out = [torch.cuda.Event() for _ in range(nseg)]

    def one_pass():
        h2d.wait_stream(comp)
        for k in range(nseg):
            sl = slice(k * seg, (k + 1) * seg)
            with torch.cuda.stream(h2d):
                for n in din:
                    din[n][sl].copy_(pin[n][sl], non_blocking=True)
                ev_in[k].record(h2d)
            comp.wait_event(ev_in[k])
            with torch.cuda.stream(comp):
                acts = [din[n][sl].unsqueeze(0) for n in ("qkv", "z", "a", "b")]
                gdn.prefill(*acts, w, None if k == 0 else st[(k - 1) % 2], None if k == 0 else cv[(k - 1) % 2],
                            out=dout[sl].unsqueeze(0), final_state=st[k % 2], final_conv=cv[k % 2])
                ev_out[k].record(comp)
            d2h.wait_event(ev_out[k])
            with torch.cuda.stream(d2h):
                host_out[sl].copy_(dout[sl], non_blocking=True)
        with torch.cuda.stream(d2h):
            host_st.copy_(st[(nseg - 1) % 2], non_blocking=True)
            host_cv.copy_(cv[(nseg - 1) % 2], non_blocking=True)
        comp.wait_stream(d2h)

    one_pass()
    torch.cuda.synchronize(dev)
    reps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(reps):
        one_pass()
    e1.record(comp)
    torch.cuda.synchronize(dev)
    sec = e0.elapsed_time(e1) / 1000.0 / reps
    return {"value": T / sec, "unit": "tokens/s", "ms": sec * 1000.0, "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes, "segments": nseg,
            "how": f"{nseg} segments of {seg} tokens, copies overlapped with the previous segment's prefill"}


def bench_prefill(args, world, rank, local, T, full=True):
    """Chunked prefill.  Top level: one row of T tokens from zero state (the 8192-token
    workload), with its roofline, the oracle timed on a sample of it, and the end-to-end number
    through the public API from host buffers.  Nested beside it (full=True): the 256-token row,
    the 4096 + 4096 split run carrying state, the 8-row varlen workload and the 2 x 65,536
    long-context rows."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    stream = torch.cuda.Stream(dev)
    warm, reps = max(3, args.warmup), max(5, args.steps)
    pcase = synth.config(2) if T == 8192 else synth.dense_case(1236, 1, T)
    pw = gdn.weights_to(pcase["weights"], dev)
    a1 = {k: pcase[k].to(dev) for k in ("qkv", "z", "a", "b")}
    pout = torch.empty((1, T, 6144), dtype=torch.bfloat16, device=dev)
    pst = torch.empty((1, 48, 128, 128), dtype=torch.float32, device=dev)
    pcv = torch.empty((1, 3, 10240), dtype=torch.float32, device=dev)
    t1, n1 = _time_prefill(lambda: gdn.prefill(a1["qkv"], a1["z"], a1["a"], a1["b"], pw, out=pout, final_state=pst,
                                               final_conv=pcv), dev, stream, warm, reps)
    res = prefill_line(T, t1, f"prefill B=1 T={T}, zero initial state, final state returned",
                       prefill_launches(1, T) * n1, peaks)
    res["metric"] = "GDN prefill tokens/s"
    if T % 2048 == 0:
        res["e2e"] = prefill_e2e(args, dev, pcase, pw)
    if not full:
        return res
    if world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = prefill_cpu_baseline(pcase, [0], T, f"prefill B=1 T={T}")
    configs = {}
    # 4096 + 4096: the second half continues from the state and history the first half left
    h = T // 2
    halves = [{k: a1[k][:, i * h:(i + 1) * h].contiguous() for k in a1} for i in range(2)]
    sst = torch.empty_like(pst)
    scv = torch.empty_like(pcv)

    def split():
        gdn.prefill(halves[0]["qkv"], halves[0]["z"], halves[0]["a"], halves[0]["b"], pw, out=pout[:, :h],
                    final_state=sst, final_conv=scv)
        gdn.prefill(halves[1]["qkv"], halves[1]["z"], halves[1]["a"], halves[1]["b"], pw, sst, scv, out=pout[:, h:],
                    final_state=pst, final_conv=pcv)

    ts, ns = _time_prefill(split, dev, stream, warm, reps)
    configs["split"] = prefill_line(T, ts, f"prefill B=1 T={T} as {h} + {h} tokens, state and history carried",
                                    2 * prefill_launches(1, h) * ns, peaks)
    # the 256-token row (latency)
    c0 = synth.config(0)
    w0 = gdn.weights_to(c0["weights"], dev)
    a0 = {k: c0[k].to(dev) for k in ("qkv", "z", "a", "b")}
    o0 = torch.empty((1, 256, 6144), dtype=torch.bfloat16, device=dev)
    s0 = torch.empty_like(pst)
    v0 = torch.empty_like(pcv)
    t0, n0 = _time_prefill(lambda: gdn.prefill(a0["qkv"], a0["z"], a0["a"], a0["b"], w0, out=o0, final_state=s0,
                                               final_conv=v0), dev, stream, warm, reps)
    configs["t256"] = prefill_line(256, t0, "prefill B=1 T=256, zero initial state (latency)",
                                   prefill_launches(1, 256) * n0, peaks)
    configs["t256"]["us"] = t0 * 1e6
    if world == 1 and not args.no_cpu_baseline:
        configs["t256"]["cpu_baseline"] = prefill_cpu_baseline(c0, [0], 256, "prefill B=1 T=256")
    if T == 8192:
        vcase = synth.config(3)
        vw = gdn.weights_to(vcase["weights"], dev)
        av = {k: vcase[k].to(dev) for k in ("qkv", "z", "a", "b")}
        cu, cud = vcase["cu_seqlens"], vcase["cu_seqlens"].to(dev)
        st0, cv0 = vcase["init_state"].to(dev), vcase["init_conv"].to(dev)
        total = int(cu[-1])
        vout = torch.empty((total, 6144), dtype=torch.bfloat16, device=dev)
        vst = torch.empty_like(st0)
        vcv = torch.empty_like(cv0)
        t2, n2 = _time_prefill(lambda: gdn.prefill_varlen(cu, av["qkv"], av["z"], av["a"], av["b"], vw, st0, cv0,
                                                          out=vout, final_state=vst, final_conv=vcv,
                                                          cu_seqlens_dev=cud),
                               dev, stream, warm, reps)
        configs["varlen8"] = prefill_line(total, t2, f"varlen prefill 8 rows ({total} tokens, lengths "
                                          "U[512,16384]), random initial state and history",
                                          prefill_launches_varlen() * n2, peaks)
        if world == 1 and not args.no_cpu_baseline:
            configs["varlen8"]["cpu_baseline"] = prefill_cpu_baseline(vcase, list(range(8)), 16384,
                                                                      "varlen prefill 8 rows")
        del av, st0, cv0, vout, vst, vcv
        if not args.no_long:
            configs["long2"] = bench_long_context(args, local, lambda *a: prefill_line(*a, peaks))
    res["configs"] = configs
    return res


def bench_long_context(args, local, line):
    """Long-context prefill: 2 rows x 65536 tokens from zero state, returning the final
    states (overlapped schedule); then 256 decode steps per row from those states."""
    import gated_deltanet_mixer_gdn_b200 as gdn
    dev = torch.device("cuda", local)
    case = synth.config(4)
    w = gdn.weights_to(case["weights"], dev)
    acts = {k: case[k].to(dev) for k in ("qkv", "z", "a", "b")}
    B, T = acts["qkv"].shape[0], acts["qkv"].shape[1]
    out = torch.empty((B, T, 6144), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((B, 48, 128, 128), dtype=torch.float32, device=dev)
    fc = torch.empty((B, 3, 10240), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    reps = max(3, min(args.steps, 5))
    t, n = _time_prefill(lambda: gdn.prefill(acts["qkv"], acts["z"], acts["a"], acts["b"], w, out=out, final_state=fs,
                                             final_conv=fc), dev, stream, 3, reps)
    res = line(B * T, t, f"long-context prefill B={B} T={T}, zero initial state, final states returned",
               prefill_launches(B, T) * n)
    if not args.no_cpu_baseline:
        res["cpu_baseline"] = prefill_cpu_baseline(case, [0, 1], T, f"long-context prefill B={B} T={T}")
    # 256 decode steps per row from the prefill's states (2 rows: launch-latency bound, reported)
    steps = case["decode"]["qkv"].shape[0]
    dq = {k: case["decode"][k].to(dev) for k in ("qkv", "z", "a", "b")}
    dout = torch.empty((steps, B, 6144), dtype=torch.bfloat16, device=dev)
    st, cv = fs.clone(), fc.clone()

    def steps_pass():
        for s in range(steps):
            gdn.decode(dq["qkv"][s], dq["z"][s], dq["a"][s], dq["b"][s], w, st, cv, out=dout[s])

    # the 256 launches as one captured graph (as a serving loop would replay them), from the
    # prefill's states each time
    with torch.cuda.stream(stream):
        steps_pass()
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        steps_pass()
    with torch.cuda.stream(stream):
        st.copy_(fs)
        cv.copy_(fc)
        graph.replay()
        st.copy_(fs)
        cv.copy_(fc)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    td = e0.elapsed_time(e1) / 1000.0
    res["decode_after"] = {"workload": f"{steps} decode steps x {B} rows from the prefill's states (CUDA graph)",
                           "value": B * steps / td, "unit": "row-tokens/s", "us_per_step": td / steps * 1e6,
                           "gpu_launches": steps}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "hidden", "multi"],
                    help="decode: the 64-row decode batch (default line); prefill: only the chunked prefill; "
                         "hidden: only the prefill from hidden states (fused in_proj + load stage); "
                         "multi: only the multi-token decode (4 tokens per call; a small case for profiling)")
    ap.add_argument("--prefill-T", type=int, default=PREFILL_T, help="tokens of the prefill measurement")
    ap.add_argument("--headline-only", action="store_true",
                    help="only the decode batch line (headline and e2e; a small case for profiling)")
    ap.add_argument("--no-long", action="store_true",
                    help="with --workload prefill: skip the 2 x 65,536-token leg")
    ap.add_argument("--prefill-only", action="store_true",
                    help="with --workload prefill: only the one-row prefill (a small case for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        if args.workload == "multi":
            multi = bench_decode_multi(args, local)
            if rank == 0:
                print(json.dumps({"metric": "GDN multi-token decode row-tokens/s", **multi}))
            return 0
        if args.workload == "hidden":
            hid = bench_hidden(args, local)
            if rank == 0:
                print(json.dumps({"metric": "GDN prefill from hidden states tokens/s", **hid}))
            return 0
        if args.workload == "prefill":
            pre = bench_prefill(args, world, rank, local, args.prefill_T, full=not args.prefill_only)
            if rank == 0:
                print(json.dumps(pre))
            return 0
        line, case = run_ours(args, world, rank, local)
        if args.headline_only:
            if rank == 0:
                print(json.dumps(line))
            return 0
        pre = bench_prefill(args, world, rank, local, args.prefill_T)
        multi = bench_decode_multi(args, local)
        proj = bench_projections(args, local)
        hid = bench_hidden(args, local)
        pout = bench_prefill_out(args, local)
        if rank == 0:
            line["prefill"] = pre
            line["prefill_out_proj"] = pout
            line["decode_multi"] = multi
            line["projections"] = proj
            line["prefill_from_hidden"] = hid
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline_line(case)
            print(json.dumps(line))
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
