#!/usr/bin/env python
"""Benchmark of the token-choice MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config mixtral|switch|deepseekmoe|deepseek_v3|tiny]

One step = one forward of the whole layer (route, capacity, dispatch, expert
FFNs, combine, losses) over one batch of T synthetic tokens.  The default
workload is the Mixtral-shaped layer (T=8192, d=4096, E=8 SwiGLU experts with
d_ff=14336, top-2, cf=1.25): it is the layer the headline targets name.  With
N > 1 (torchrun, one process per GPU) every rank runs an independent replica
on its own batch: the layer needs no exchange between GPUs, so the scaling is
weak and no collective touches the data path; the per-step time is the max
over ranks.

Rank 0 prints one JSON line.  `value` is device-timed (CUDA events, inputs
resident in HBM); `e2e` repeats the measurement through HostStream: every
step's input is copied in from pinned host memory and its output and losses
copied back inside the timed region, the copies of neighbouring steps
overlapping a step's kernels;
`roofline` covers the dominant stage (the expert FFN: two grouped tcgen05
GEMMs) from its own CUDA events in the same timed region; `cpu_baseline` times
the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from moe_inputs import CONFIGS, generate, seed_for  # noqa: E402

METRIC = "MoE layer fwd tokens/s on 1 B200; grouped-GEMM % BF16 peak; dispatch % HBM BW"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20   # written between cold stage timings: twice the 126 MB L2
def route_kernels(shape) -> int:
    """Kernels of the router: bf16 layers with up to 16 experts run one kernel,
    wider ones three (split, logits, select); the fp32 layer one."""
    if shape.dtype != 1:
        return 1
    return 1 if shape.E <= 16 else 3


def kernels_per_step(shape) -> int:
    """Kernels of ours one moe_forward launches: the router (route_kernels),
    capacity 2 (histograms and the loss phase sums; placement with the
    totals and the losses),
    dispatch 1, expert FFN (bf16: the two grouped GEMMs; fp32: two, plus two
    for shared experts), combine 1 (0 for a top-1 layer without shared
    experts: GEMM2 writes y); the score-ordered capacity adds three launches
    and a losses launch."""
    ffn = 2 if shape.dtype == 1 else (4 if shape.n_shared else 2)
    extra = 4 if shape.priority == 2 else 0
    combine = 0 if shape.k == 1 and shape.n_shared == 0 else 1   # top-1: in GEMM2's epilogue
    return route_kernels(shape) + 2 + 1 + ffn + combine + extra
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) of the expert-FFN stage (GEMM1 + GEMM2) per launch, from one ncu
# capture of the same workload, valid only for the GEMM source it was taken on.
GEMM_SOURCE = os.path.join(ROOT, "mixture_experts_layer_54_b200", "csrc", "ffn_tcgen05.cu")
MEASURED_TRAFFIC = {
    ("mixtral", "2672a43efa7fa1986e967ab95bf785cfbe76a776dc5d64b52997fef08a675984"): 5.612e9,
}


def measured_traffic(config: str):
    import hashlib
    try:
        with open(GEMM_SOURCE, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return MEASURED_TRAFFIC.get((config, sha))


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="mixtral", choices=sorted(CONFIGS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-layer", action="store_true",
                    help="skip the Switch, DeepSeekMoE and DeepSeek-V3 shaped layers that the "
                         "default (Mixtral-shaped) run also times")
    ap.add_argument("--stage", choices=["route", "ffn", "forward"], default=None,
                    help="time one stage alone on the workload's tensors (profiling aid; "
                         "prints its own JSON line, not the benchmark line)")
    ap.add_argument("--experts", type=int, default=None,
                    help="with --stage ffn: this many experts, tokens scaled so that each "
                         "expert keeps its rows (a smaller device footprint, same GEMM shapes)")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, device) -> float:
    """Slowest rank's time (every rank calls this the same number of times)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        self.gpu = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        time.sleep(0.1)
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [s.strip() for s in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, flag in zip(names, f[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ work accounting

def perm_rows(shape) -> int:
    """Rows of the permuted buffers: kept slots plus per-expert padding to 128."""
    C = shape.T if math.isinf(shape.cf) else min(shape.T, math.ceil(shape.cf * shape.T * shape.k
                                                                    / shape.E))
    kept = min(shape.T * shape.k, C * shape.E)
    return (kept + shape.E * 127 + 127) // 128 * 128


def layer_work(shape, counts, kept_total, dropped_tokens):
    """Algorithmic FLOPs and bytes of one step (no padding rows, no dense E-way
    work), per stage."""
    T, d, E, k, F = shape.T, shape.d, shape.E, shape.k, shape.d_ff
    b = 2 if shape.dtype == 1 else 4
    m = 3 if shape.act == 1 else 2
    S, Fs = shape.n_shared, shape.d_ff_shared
    N = kept_total
    ffn_flops = 2.0 * m * N * d * F + 2.0 * m * S * T * d * Fs
    w_bytes = (E * m * d * F + S * m * d * Fs) * b
    ffn_bytes = w_bytes + (N + (T if S else 0)) * d * b * 2 + (N + S * T) * F * b * 2
    routed_tokens = T - dropped_tokens
    return {
        "route": {"bytes": T * d * b + d * E * 4 + T * k * 8 + math.ceil(T / 32) * (E + 1) * 4,
                  "flops": 2.0 * T * d * E},
        "dispatch": {"bytes": routed_tokens * d * b + N * d * b + T * k * 9},
        # the dispatch fused into GEMM1 instead: the row table (cleared, one entry per kept slot)
        "dispatch_rows": {"bytes": perm_rows(shape) * 4 + T * k * 9 + N * 4},
        "expert_ffn": {"flops": ffn_flops, "bytes": ffn_bytes},
        "combine": {"bytes": N * d * b + (T * d * b if S else 0) + T * d * b + T * k * 9},
        "capacity": {"bytes": T * k * 4 * 3 + T * k + T},
        "losses": {"bytes": math.ceil(T / 32) * (E + 1) * 4 + E * 4},
    }


# ------------------------------------------------------------ oracle timing

def oracle_inputs(inp):
    import numpy as np

    def host(t):
        if t is None:
            return None
        t = t.detach().contiguous().cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()
    return {k: host(getattr(inp, k)) for k in
            ("x", "W_r", "logit_bias", "select_bias", "W1", "W3", "W2", "Ws1", "Ws3", "Ws2")}


def time_oracle(shape, h, n_tokens):
    """Oracle routing, capacity and losses over all T tokens plus the expert
    FFNs of the first n_tokens tokens; returns (t_route_s, t_ffn_s)."""
    import numpy as np
    import oracle
    t0 = time.perf_counter()
    r = oracle.route(h["x"], h["W_r"], shape.k, shape.score, shape.renorm, h["logit_bias"],
                     h["select_bias"])
    cap = oracle.capacity_walk(r.topk, shape.E, shape.cf, shape.priority)
    oracle.losses(r.scores, cap.counts, r.lse, shape.k, shape.score)
    t1 = time.perf_counter()
    tokens = np.arange(n_tokens, dtype=np.int32)
    oracle.ffn_tokens(h["x"], r.topk, r.gates, cap.keep, h["W1"], h["W3"], h["W2"], shape.act,
                      h["Ws1"], h["Ws3"], h["Ws2"], tokens)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def size_oracle_sample(shape, h, seconds):
    """Tokens whose FFNs take about `seconds` on the host cores (probed on one
    token per host thread, so the probe itself keeps every core busy)."""
    import oracle
    probe = min(shape.T, max(4, oracle.num_threads()))
    _, tp = time_oracle(shape, h, probe)
    per = max(tp / probe, 1e-6)
    return int(max(4, min(shape.T, seconds / per)))


def graph_time_us(fn, n=20):
    """Device time of one call of fn: n calls captured in a CUDA graph,
    replayed once between CUDA events (after three eager warm-up calls)."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        for _ in range(n):
            fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()
    torch.cuda.synchronize()
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / n


def next_rows(moe, shape, inp, staged, seq_len):
    """Device times of the rows past the forward, on the same batch: the
    batch-prioritized capacity (from the router's scores), the sequence-wise
    balance loss and one loss-free bias step."""
    import dataclasses
    cfg2 = moe.moe_config(dataclasses.replace(shape, priority=2))
    cfg = moe.moe_config(shape)
    _, _, _, _, scores = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, inp.select_bias,
                                       want_scores=True)
    ws2 = moe.workspace(moe.moe_stage_workspace_size(cfg2), inp.x.device)
    cap = moe.moe_capacity_scored(cfg2, staged.topk, scores, ws=ws2)
    t_cap = graph_time_us(lambda: moe.moe_capacity_scored(cfg2, staged.topk, scores, ws=ws2))
    loss, per = moe.moe_seq_balance_loss(cfg, seq_len, staged.topk, staged.partials)
    t_seq = graph_time_us(lambda: moe.moe_seq_balance_loss(cfg, seq_len, staged.topk,
                                                           staged.partials, per, loss))
    bias = torch.zeros(shape.E, dtype=torch.float32, device=inp.x.device)
    t_bias = graph_time_us(lambda: moe.moe_bias_update(cfg, staged.counts, 1e-3, bias))
    torch.cuda.synchronize()
    return {"capacity_scored": {"us": round(t_cap, 2), "launches": 6,
                                "n_dropped": int(cap.n_dropped.item())},
            "seq_balance_loss": {"us": round(t_seq, 2), "seq_len": seq_len, "launches": 2,
                                 "value": round(float(loss.item()), 6)},
            "bias_update": {"us": round(t_bias, 2), "launches": 1}}


def fused_dispatch(moe, cfg, inp, staged):
    """The dispatch fused into GEMM1 (row table + rows gathered from x) and the
    combine's gate fused into GEMM2 (gated rows to a [T k, d] buffer, then an
    ordered sum), against the permuted copy + expert FFN + combine that the
    step runs; same batch, same box, each from a captured graph."""
    R = moe.moe_perm_rows(cfg)
    dev = inp.x.device
    rows = torch.empty((R,), dtype=torch.int32, device=dev)
    Y = torch.empty_like(staged.Y_perm)
    Ysh = None if staged.Y_sh is None else torch.empty_like(staged.Y_sh)
    Yslot = torch.empty((cfg.T * cfg.k, cfg.d), dtype=staged.y.dtype, device=dev)
    y = torch.empty_like(staged.y)
    w = (inp.W1, inp.W3, inp.W2)
    ws = (inp.Ws1, inp.Ws3, inp.Ws2)

    def dispatch_fused():
        moe.moe_dispatch_rows(cfg, staged.topk, staged.pos, staged.keep, staged.offsets, rows)
        moe.moe_expert_ffn_gather(cfg, inp.x, rows, staged.offsets, *w, *ws, ws=staged.ws,
                                  Y_perm=Y, Y_shared=Ysh)

    def dispatch_unfused():
        moe.moe_dispatch(cfg, inp.x, staged.topk, staged.pos, staged.keep, staged.offsets,
                         staged.x_perm)
        moe.moe_expert_ffn(cfg, staged.x_perm, staged.offsets, *w, inp.x, *ws, ws=staged.ws,
                           Y_perm=Y, Y_shared=Ysh)

    def unfused():
        dispatch_unfused()
        moe.moe_combine(cfg, Y, Ysh, staged.gates, staged.topk, staged.pos, staged.keep,
                        staged.offsets, y=y)

    def combine_fused():
        moe.moe_dispatch(cfg, inp.x, staged.topk, staged.pos, staged.keep, staged.offsets,
                         staged.x_perm, src_slot=rows)
        moe.moe_expert_ffn_slots(cfg, staged.x_perm, inp.x, rows, staged.offsets, staged.kept,
                                 staged.gates, *w, *ws, ws=staged.ws, Y_slot=Yslot, Y_shared=Ysh)
        moe.moe_combine_slots(cfg, Yslot, Ysh, staged.keep, y=y)

    def both_fused():
        moe.moe_dispatch_rows(cfg, staged.topk, staged.pos, staged.keep, staged.offsets, rows)
        moe.moe_expert_ffn_slots(cfg, None, inp.x, rows, staged.offsets, staged.kept,
                                 staged.gates, *w, *ws, ws=staged.ws, Y_slot=Yslot, Y_shared=Ysh)
        moe.moe_combine_slots(cfg, Yslot, Ysh, staged.keep, y=y)

    t = {name: graph_time_us(fn, n=5) for name, fn in
         [("dispatch_fused", dispatch_fused), ("dispatch_unfused", dispatch_unfused),
          ("unfused", unfused), ("combine_fused", combine_fused), ("both_fused", both_fused)]}
    if moe.moe_device_status(staged.ws) != 0:
        raise SystemExit("device status set by a fused variant")
    return {"us": round(t["dispatch_fused"], 1), "unfused_us": round(t["dispatch_unfused"], 1),
            "launches": 3,
            "dispatch_and_ffn": {"fused_us": round(t["dispatch_fused"], 1),
                                 "unfused_us": round(t["dispatch_unfused"], 1)},
            "dispatch_ffn_combine": {"unfused_us": round(t["unfused"], 1),
                                     "combine_fused_us": round(t["combine_fused"], 1),
                                     "both_fused_us": round(t["both_fused"], 1)},
            "note": "dispatch fused: moe_dispatch_rows + moe_expert_ffn_gather (cp.async row "
                    "gathers) vs moe_dispatch + moe_expert_ffn; combine fused: "
                    "moe_expert_ffn_slots (gate in GEMM2's epilogue) + moe_combine_slots"}


def cpu_baseline(shape, inp, seconds):
    import oracle
    h = oracle_inputs(inp)
    n = size_oracle_sample(shape, h, seconds)
    t_route, t_ffn = time_oracle(shape, h, n)
    per_token = t_route / shape.T + t_ffn / n
    return {"value": 1.0 / per_token, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"routing, capacity and losses over all {shape.T} tokens "
                       f"({t_route:.2f} s) plus expert FFNs of {n} tokens ({t_ffn:.2f} s), "
                       f"per-token cost extrapolated to the full batch")}


def workload_name(shape):
    act = "SwiGLU" if shape.act == 1 else "GELU"
    sh = f" + {shape.n_shared} shared (d_ff={shape.d_ff_shared})" if shape.n_shared else ""
    sc = "sigmoid+selection bias" if shape.score == 1 else "softmax"
    cf = "no capacity" if math.isinf(shape.cf) else f"cf={shape.cf}"
    return (f"{shape.name} MoE layer fwd: T={shape.T} d={shape.d} E={shape.E} {act} experts "
            f"d_ff={shape.d_ff}{sh}, top-{shape.k} {sc}, {cf}")


# ------------------------------------------------------------ reference arm

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    shape = CONFIGS[args.config]
    inp = generate(shape, device="cpu")
    h = oracle_inputs(inp)
    # at least four tokens per host thread (the oracle's FFN loop runs OpenMP
    # over tokens), else too few tokens leave cores idle and understate it
    n = max(size_oracle_sample(shape, h, 1.0), min(shape.T, 4 * oracle.num_threads()))
    for _ in range(args.warmup):
        time_oracle(shape, h, n)
    tr = tf = 0.0
    for _ in range(args.steps):
        a, b = time_oracle(shape, h, n)
        tr += a
        tf += b
    per_token = (tr / args.steps) / shape.T + (tf / args.steps) / n
    value = 1.0 / per_token
    sample = (f"each step: oracle routing, capacity and losses over all {shape.T} tokens plus "
              f"expert FFNs of {n} tokens, per-token cost extrapolated to the full batch")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * shape.T / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_name(shape), "global_batch": shape.T,
                       "parallelism": "none (host cores)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ our arm

def time_layer_graph(moe, shape, inp, dev, steps, warmup, local):
    """Graph-timed forwards of one layer (inputs resident).

    value: `steps` calls of moe_forward (the public one-call API) captured
    once in a CUDA graph with events only before the first and after the last,
    replayed once between synchronises while clocks are sampled.
    stages: the same number of forwards as the six per-stage calls (route,
    capacity, dispatch, expert FFN, combine, losses) with events between the
    stages, captured and replayed separately; events between kernels keep the
    next kernel from starting early, so the stages add up to a little more
    than the forward."""
    cfg = moe.moe_config(shape)
    fwd = moe.MoEForward(cfg, dev)
    w = moe.weights_struct(inp.W_r, inp.W1, inp.W2, inp.W3, inp.logit_bias, inp.select_bias,
                           inp.Ws1, inp.Ws3, inp.Ws2)
    staged = moe.StagedForward(cfg, dev)
    wargs = (inp.x, inp.W_r, inp.W1, inp.W2, inp.W3, inp.logit_bias, inp.select_bias, inp.Ws1,
             inp.Ws3, inp.Ws2)
    nst = len(moe.StagedForward.STAGES)
    for _ in range(max(warmup, 3)):
        fwd(inp.x, w)
        staged(*wargs)
    torch.cuda.synchronize()
    for ws in (fwd.ws, staged.ws):
        status = moe.moe_device_status(ws)
        if status != 0:
            raise SystemExit(f"device status {status} after warm-up ({shape.name}): a bounded "
                             "wait gave up; not timing a failing kernel")
    if steps is None:   # enough steps for about a quarter of a second
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(3):
            fwd(inp.x, w)
        e1.record()
        torch.cuda.synchronize()
        per = e0.elapsed_time(e1) / 3 / 1e3
        steps = int(min(max(0.25 / max(per, 1e-6), 20), 2000))

    # ---- the forward, K calls in one graph ----
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        ev[0].record()
        for _ in range(steps):
            fwd(inp.x, w)
        ev[1].record()
    torch.cuda.synchronize()
    barrier(dev)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        graph.replay()
        torch.cuda.synchronize()
    barrier(dev)
    status = moe.moe_device_status(fwd.ws)
    if status != 0:
        raise SystemExit(f"device status {status} in the timed region ({shape.name})")
    total_ms = ev[0].elapsed_time(ev[1])
    del graph

    # ---- the per-stage calls, with events between the stages ----
    events = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(nst + 1)]
              for _ in range(steps)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        for i in range(steps):
            staged(*wargs, events=events[i])
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    if moe.moe_device_status(staged.ws) != 0:
        raise SystemExit(f"device status set in the per-stage replay ({shape.name})")
    stage_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in events) / steps for i in range(nst)]
    staged_total = events[0][0].elapsed_time(events[-1][-1]) / steps
    del graph
    if not torch.equal(fwd.y, staged.y):
        raise SystemExit(f"the forward and the per-stage calls disagree ({shape.name})")
    return {"staged": staged, "fwd": fwd, "steps": steps, "ms_per_step": total_ms / steps,
            "staged_ms_per_step": staged_total,
            "stage_ms": dict(zip(moe.StagedForward.STAGES, stage_ms)),
            "kept": int(staged.kept.sum().item()),
            "dropped_tokens": int(staged.dropped.sum().item()),
            "status": status, "clocks": clk.summary()}


def summarize_layer(shape, ms_per_step, stage_ms, kept, dropped_tokens, steps, peaks, world=1):
    """Per-stage rates, the expert FFN against the bf16 peak, and the layer
    roofline (slower of its FLOPs at the bf16 peak and its bytes at the HBM
    copy bandwidth) for one graph-timed layer."""
    work = layer_work(shape, None, kept, dropped_tokens)
    stages = {}
    for name, ms in stage_ms.items():
        entry = {"us": round(ms * 1e3, 2)}
        if "bytes" in work[name]:
            entry["GB/s"] = round(work[name]["bytes"] / (ms / 1e3) / 1e9, 1)
            entry["hbm_frac"] = round(entry["GB/s"] / peaks["hbm_gbs"], 3)
        if "flops" in work[name]:
            entry["TFLOP/s"] = round(work[name]["flops"] / (ms / 1e3) / 1e12, 1)
        stages[name] = entry
    ffn = work["expert_ffn"]
    ach = ffn["flops"] / (stage_ms["expert_ffn"] / 1e3) / 1e12
    # A timed region long enough for the 1 kW power cap to settle (>= 0.2 s)
    # is compared with the sustained matmul figure, a shorter one with the
    # burst figure; both fractions are reported.
    region_s = ms_per_step * steps / 1e3
    peak_kind = "sustained" if region_s >= 0.2 else "burst"
    peak = peaks["bf16_tflops_sustained" if peak_kind == "sustained" else "bf16_tflops"]
    t_flop = ffn["flops"] / (peak * 1e12)
    all_bytes = sum(work[n].get("bytes", 0) for n in stage_ms)
    t_byte = all_bytes / (peaks["hbm_gbs"] * 1e9)
    ffn_t_byte = ffn["bytes"] / (peaks["hbm_gbs"] * 1e9)
    return {
        "stages": stages,
        "expert_ffn": {"TFLOP/s": round(ach, 1), "peak_TFLOP/s": peak, "peak_kind": peak_kind,
                       "frac_of_peak": round(ach / peak, 4),
                       "GB/s": round(ffn["bytes"] / (stage_ms["expert_ffn"] / 1e3) / 1e9, 1),
                       "hbm_frac": round(ffn_t_byte / (stage_ms["expert_ffn"] / 1e3), 4),
                       "bound": "tensor" if ffn["flops"] / (peak * 1e12) >= ffn_t_byte else "hbm",
                       "flops": ffn["flops"], "algorithmic_bytes": ffn["bytes"]},
        "layer_roofline": {"t_flop_us": round(t_flop * 1e6, 1), "t_byte_us": round(t_byte * 1e6, 1),
                           "bound": "tensor" if t_flop >= t_byte else "hbm",
                           "frac": round(max(t_flop, t_byte) / (ms_per_step / 1e3), 4)},
        "timed_region_s": round(region_s, 3),
        "roofline_peak": (peak, peak_kind, ach),
    }


def per_layer(moe, dev, local, peaks, names, warmup):
    """The other model-shaped layers, graph-timed one after another in the
    same run (each layer's tensors freed before the next is drawn)."""
    out = {}
    for name in names:
        shape = CONFIGS[name]
        inp = generate(shape, device=dev)
        r = time_layer_graph(moe, shape, inp, dev, None, warmup, local)
        sm = summarize_layer(shape, r["ms_per_step"], r["stage_ms"], r["kept"],
                             r["dropped_tokens"], r["steps"], peaks)
        sm.pop("roofline_peak")
        clk = r["clocks"]
        out[name] = {"workload": workload_name(shape),
                     "value": round(shape.T / (r["ms_per_step"] / 1e3), 1), "unit": UNIT,
                     "ms_per_step": round(r["ms_per_step"], 4), "steps": r["steps"],
                     "staged_ms_per_step": round(r["staged_ms_per_step"], 4),
                     "kept_assignments": r["kept"], "dropped_tokens": r["dropped_tokens"],
                     "gpu_launches": kernels_per_step(shape) * r["steps"],
                     "clocks": {"sm_mhz": clk["sm_mhz"], "reasons": clk["reasons"],
                                "samples": clk["samples"]},
                     "traffic": measured_traffic(name), **sm}
        r.pop("staged")
        r.pop("fwd")
        del r, inp
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import mixture_experts_layer_54_b200 as moe

    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    shape = CONFIGS[args.config]
    inp = generate(shape, device=dev, seed=seed_for(shape) + 1000 * rank)
    cfg = moe.moe_config(shape)

    # ---- device-timed region: the K steps, captured once in a CUDA graph with
    # timing events between the stages, replayed once between barriers ----
    r = time_layer_graph(moe, shape, inp, dev, args.steps, args.warmup, local)
    staged, status, clocks = r["staged"], r["status"], r["clocks"]
    kept_total, dropped_tokens = r["kept"], r["dropped_tokens"]
    ms_per_step = max_over_ranks(r["ms_per_step"], dev)

    # ---- end to end: pinned host input in, result out, inside the timed region.
    # Batches stream through HostStream (public API): each step copies its x
    # in and its y and losses out, overlapped with the neighbouring steps'
    # kernels; the region ends when the last step's outputs are on the host ----
    w = moe.weights_struct(inp.W_r, inp.W1, inp.W2, inp.W3, inp.logit_bias, inp.select_bias,
                           inp.Ws1, inp.Ws3, inp.Ws2)
    hs = moe.HostStream(cfg, dev, w)
    x_host = inp.x.cpu().pin_memory()
    y_host = [torch.empty(x_host.shape, dtype=x_host.dtype).pin_memory() for _ in range(2)]
    loss_host = [torch.empty((2,), dtype=torch.float32).pin_memory() for _ in range(2)]
    for i in range(max(args.warmup, 3)):
        hs.submit(x_host, y_host[i % 2], loss_host[i % 2])
    hs.drain()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize()
    e0.record()
    hs.start_after(e0)
    for i in range(args.steps):
        hs.submit(x_host, y_host[i % 2], loss_host[i % 2])
    hs.drain()
    e1.record()
    torch.cuda.synchronize()
    barrier(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    if not torch.equal(y_host[(args.steps - 1) % 2], hs.fwd[(args.steps - 1) % 2].y.cpu()):
        raise SystemExit("e2e: the host copy of y differs from the device result")
    del hs

    extra = next_rows(moe, shape, inp, staged, seq_len=min(shape.T, 1024)) \
        if shape.T % 32 == 0 and shape.T > 0 else None
    if extra is not None:
        extra["fused_dispatch"] = fused_dispatch(moe, cfg, inp, staged)
    peaks, peak_src = load_peaks()
    layers = None
    if world == 1 and not args.no_per_layer and args.config == "mixtral":
        del staged, inp, w
        r.pop("staged")
        r.pop("fwd")
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        layers = per_layer(moe, dev, local, peaks, ["switch", "deepseekmoe", "deepseek_v3"],
                           args.warmup)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    tokens = shape.T * world
    value = tokens / (ms_per_step / 1e3)
    sm = summarize_layer(shape, ms_per_step, r["stage_ms"], kept_total, dropped_tokens,
                         args.steps, peaks, world)
    peak, peak_kind, ach = sm["roofline_peak"]
    ffn = sm["expert_ffn"]
    roofline = {"bound": "tensor", "achieved": round(ach, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                "traffic": measured_traffic(args.config),
                "traffic_unit": "bytes per launch (ncu dram read + write, GEMM1 + GEMM2)",
                "algorithmic_bytes": ffn["algorithmic_bytes"],
                "kernel": "moe_expert_ffn: grouped tcgen05 GEMM1 (act fused) + GEMM2",
                "flops_per_launch": ffn["flops"],
                "peak_source": (f"measured bf16 {peak_kind} (MEASURED_PEAKS.json)"
                                if peak_src == "measured" else
                                f"fallback bf16 {peak_kind}: MEASURED_PEAKS.json absent, the "
                                "profiling recipe's figures"),
                "timed_region_s": sm["timed_region_s"],
                "frac_of_burst": round(ach / peaks["bf16_tflops"], 4),
                "frac_of_sustained": round(ach / peaks["bf16_tflops_sustained"], 4)}
    b = 2 if shape.dtype == 1 else 4
    h2d = shape.T * shape.d * b
    d2h = shape.T * shape.d * b + 8
    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if shape.dtype == 1 else "f32", "data": "synthetic",
            "config": {"workload": workload_name(shape), "global_batch": tokens,
                       "tokens_per_gpu": shape.T, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (expert weights "
                             f"{(shape.E * (3 if shape.act == 1 else 2) * shape.d * shape.d_ff * b) / 1e9:.2f} GB)",
                       "kept_assignments": kept_total, "dropped_tokens": dropped_tokens},
            "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": kernels_per_step(shape) * args.steps,
            "timing": "device: one CUDA graph of K moe_forward calls; stages: a second graph "
                      "of the per-stage calls with events between them; e2e: HostStream "
                      "(copies of step i +- 1 overlap step i's kernels)",
            "roofline": roofline, "layer_roofline": sm["layer_roofline"], "stages": sm["stages"],
            "staged_ms_per_step": round(r["staged_ms_per_step"], 4),
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
            "device_status": status,
            "next_rows": extra}
    if layers is not None:
        line["per_layer"] = layers
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape, generate(shape, device=dev), args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_stage(args):
    """The router alone on the workload's tokens and router weights: the same
    seeded draw with the experts narrowed to 64 columns, so the expert weights
    take no room.  W warm-up calls, then K calls between CUDA events."""
    import mixture_experts_layer_54_b200 as moe
    from moe_inputs import shrink
    device = torch.device("cuda", 0)
    shape = CONFIGS[args.config]
    small = shrink(shape, d_ff=64, d_ff_shared=64 if shape.n_shared else shape.d_ff_shared)
    inp = generate(small, device)
    cfg = moe.moe_config(small)
    ws = moe.workspace(moe.moe_stage_workspace_size(cfg), device)
    call = lambda: moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, inp.select_bias, ws=ws)
    for _ in range(max(args.warmup, 1)):
        call()
    torch.cuda.synchronize()
    # warm: a graph of K back-to-back calls (x stays in L2 when it fits)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        call()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(args.steps):
                call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph.replay()
    torch.cuda.synchronize()
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    warm_us = e0.elapsed_time(e1) * 1e3 / args.steps
    del graph
    # cold: each call timed alone after writing a buffer larger than L2
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    cold = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        cold.append((a, b))
    torch.cuda.synchronize()
    cold_us = sorted(a.elapsed_time(b) * 1e3 for a, b in cold)[len(cold) // 2]
    if moe.moe_device_status(ws) != 0:
        raise SystemExit("device status set: a bounded wait expired")
    x_bytes = inp.x.numel() * inp.x.element_size()
    peaks, _ = load_peaks()
    print(json.dumps({"stage": "route", "workload": workload_name(shape), "calls": args.steps,
                      "us_per_call": round(cold_us, 2), "x_bytes": x_bytes,
                      "GB/s": round(x_bytes / cold_us / 1e3, 1),
                      "hbm_frac": round(x_bytes / cold_us / 1e3 / peaks["hbm_gbs"], 3),
                      "warm_us_per_call": round(warm_us, 2),
                      "timing": "us_per_call: median of K calls each timed alone (CUDA events) "
                                "after an L2 flush; warm: a graph of K back-to-back calls"}))


def run_stage_ffn(args):
    """The expert FFN (the two grouped GEMMs) alone: route, capacity and
    dispatch once, then W warm-up calls and K calls of moe_expert_ffn between
    CUDA events.  --experts E keeps the layer's per-expert GEMM shapes with E
    experts (T scaled by E / E_layer)."""
    import mixture_experts_layer_54_b200 as moe
    from moe_inputs import shrink
    device = torch.device("cuda", 0)
    shape = CONFIGS[args.config]
    if args.experts:
        E = args.experts
        shape = shrink(shape, E=E, T=max(shape.T * E // shape.E, 1), k=min(shape.k, E))
    inp = generate(shape, device)
    cfg = moe.moe_config(shape)
    topk, gates, _, _, _ = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, inp.select_bias)
    cap = moe.moe_capacity(cfg, topk)
    x_perm = moe.moe_dispatch(cfg, inp.x, topk, cap.pos, cap.keep, cap.offsets)
    Y, Ysh, ws = moe.moe_expert_ffn(cfg, x_perm, cap.offsets, inp.W1, inp.W3, inp.W2, inp.x,
                                    inp.Ws1, inp.Ws3, inp.Ws2)
    call = lambda: moe.moe_expert_ffn(cfg, x_perm, cap.offsets, inp.W1, inp.W3, inp.W2, inp.x,
                                      inp.Ws1, inp.Ws3, inp.Ws2, ws=ws, Y_perm=Y, Y_shared=Ysh)
    for _ in range(max(args.warmup, 1)):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    if moe.moe_device_status(ws) != 0:
        raise SystemExit("device status set: a bounded wait expired")
    us = e0.elapsed_time(e1) * 1e3 / args.steps
    kept = int(cap.kept.sum().item())
    work = layer_work(shape, None, kept, 0)["expert_ffn"]
    peaks, _ = load_peaks()
    w_bytes = sum(t.numel() * t.element_size() for t in
                  (inp.W1, inp.W3, inp.W2, inp.Ws1, inp.Ws3, inp.Ws2) if t is not None)
    print(json.dumps({"stage": "expert_ffn", "workload": workload_name(shape), "calls": args.steps,
                      "us_per_call": round(us, 2), "kept_assignments": kept,
                      "TFLOP/s": round(work["flops"] / us / 1e6, 1),
                      "frac_of_burst": round(work["flops"] / us / 1e6 / peaks["bf16_tflops"], 3),
                      "weight_bytes": w_bytes, "algorithmic_bytes": work["bytes"],
                      "GB/s": round(work["bytes"] / us / 1e3, 1),
                      "hbm_frac": round(work["bytes"] / us / 1e3 / peaks["hbm_gbs"], 3),
                      "timing": "back-to-back calls, CUDA events (launch gaps included)"}))


def run_stage_forward(args):
    """The whole layer through moe_forward, eagerly: W warm-up calls, then K
    calls between CUDA events (launch gaps included).  The small command the
    kernel launch list is taken from."""
    import mixture_experts_layer_54_b200 as moe
    device = torch.device("cuda", 0)
    shape = CONFIGS[args.config]
    inp = generate(shape, device)
    cfg = moe.moe_config(shape)
    fwd = moe.MoEForward(cfg, device)
    w = moe.weights_struct(inp.W_r, inp.W1, inp.W2, inp.W3, inp.logit_bias, inp.select_bias,
                           inp.Ws1, inp.Ws3, inp.Ws2)
    for _ in range(max(args.warmup, 1)):
        fwd(inp.x, w)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fwd(inp.x, w)
    e1.record()
    torch.cuda.synchronize()
    if moe.moe_device_status(fwd.ws) != 0:
        raise SystemExit("device status set: a bounded wait expired")
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"stage": "forward", "workload": workload_name(shape), "calls": args.steps,
                      "ms_per_call": round(ms, 4), "tokens/s": round(shape.T / ms * 1e3, 1),
                      "kernels_per_call": kernels_per_step(shape),
                      "timing": "back-to-back eager calls, CUDA events (launch gaps included)"}))


def main(argv=None):
    args = parse(argv)
    if args.stage == "ffn":
        run_stage_ffn(args)
        return
    if args.stage == "forward":
        run_stage_forward(args)
        return
    if args.stage:
        run_stage(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
