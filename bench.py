#!/usr/bin/env python
"""Throughput of the B200 quantized MoE FFN layer.

One step = one full layer forward (router logits, top-k, Q8_0 activation
quantization, batch-union grouping, gate/up + SwiGLU, down + weighted combine)
on a fresh batch of synthetic tokens. Consecutive steps rotate over several
layer replicas (distinct expert weights), so the expert bytes a step touches are
never left in L2 by the previous steps. The timed region replays a CUDA graph of
the steps (launch overhead removed), bracketed by a barrier and a device
synchronize on both sides; multi-GPU runs are weak-scaled (each rank its own
tokens and replicas, no data-path collective) and report the max over ranks.
The line also carries the metric's prefill half ("prefill"): the OLMoE-shaped
packed-int4 layer on 4096 tokens per GPU, whose experts run as tensor-core GEMMs
(fp16 operands holding the integer codes), with its tensor roofline against the fp16 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload olmoe_int8:1]
  python bench.py --impl reference ...   (the CPU oracle as the reference arm)
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth as S  # noqa: E402

METRIC = "MoE-layer tok/s (decode b=1, prefill 4k); HBM GB/s and int8 TC % of peak"
DEFAULT_WORKLOAD = "olmoe_int8:1"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------- helpers
def parse_workload(spec: str):
    name, _, t = spec.partition(":")
    cfg = S.CONFIGS[name]
    T = int(t) if t else cfg.tokens[0]
    return cfg, T


def workload_desc(cfg, T, top_p=0.0):
    return (f"{cfg.name} T={T}: H{cfg.H} E{cfg.E} I{cfg.I} top-{cfg.top_k} {cfg.score}"
            f"{' renorm' if cfg.renormalize else ''}{f' rsf {cfg.rsf}' if cfg.rsf != 1 else ''}"
            f"{f' adaptive top-p {top_p:g}' if 0 < top_p < 1 else ''}, "
            f"{cfg.wtype} {cfg.wscale} experts, {cfg.act} activations"
            f"{f', shared I{cfg.shared_I}' if cfg.shared_I else ''}")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def blob_row_bytes(cfg, K, I_rows):
    kb = K * {"int8": 8, "int4": 4, "int2": 2}[cfg.wtype] // 8
    sb = (K // 32) * 2 if cfg.wscale == "g32_f16" else 4
    return I_rows * (kb + sb)


def gateup_bytes(cfg, T, n_active):
    """Algorithmic bytes of the gate/up stage: each unique expert's gate/up codes+scales once,
    the shared expert's, q_x read and q_h (+ scales) written."""
    P = T * cfg.top_k
    b = n_active * blob_row_bytes(cfg, cfg.H, 2 * cfg.I)
    if cfg.shared_I:
        b += blob_row_bytes(cfg, cfg.H, 2 * cfg.shared_I)
    b += T * cfg.H + (T * (cfg.H // 32) * 2 if cfg.act == "g32_f16" else T * 4)
    b += P * cfg.I + (P * (cfg.I // 32) * 2 if cfg.act == "g32_f16" else P * 4)
    if cfg.shared_I:
        b += T * cfg.shared_I
    return b


def expert_bytes(cfg, T, n_active):
    """Algorithmic bytes of the expert kernel: the unique experts' blobs (gate/up and down,
    codes and scales) and the shared expert's; activations and h stay on chip or in L2."""
    b = n_active * (blob_row_bytes(cfg, cfg.H, 2 * cfg.I) + blob_row_bytes(cfg, cfg.I, cfg.H))
    if cfg.shared_I:
        b += blob_row_bytes(cfg, cfg.H, 2 * cfg.shared_I) + blob_row_bytes(cfg, cfg.shared_I, cfg.H)
    return b


def layer_bytes(cfg, T, n_active):
    """Algorithmic bytes of one layer forward: unique experts' blobs (gate/up and down), the
    shared expert, the router weight, x in and y out (fp32)."""
    b = n_active * (blob_row_bytes(cfg, cfg.H, 2 * cfg.I) + blob_row_bytes(cfg, cfg.I, cfg.H))
    if cfg.shared_I:
        b += blob_row_bytes(cfg, cfg.H, 2 * cfg.shared_I) + blob_row_bytes(cfg, cfg.shared_I, cfg.H)
    b += cfg.E * cfg.H * 4 + 2 * T * cfg.H * 4
    return b


def layer_int_ops(cfg, T, pairs=None):
    """pairs: routed (token, expert) pairs computed (T * k, or fewer with adaptive top-p)."""
    pairs = T * cfg.top_k if pairs is None else pairs
    return 2 * (pairs * 3 * cfg.H * cfg.I + T * 3 * cfg.H * cfg.shared_I)


def step_plan(steps: int, period: int, event_steps: int):
    """How the timed steps are replayed: CUDA graphs of G steps with no event nodes, n_main
    replays of the G-step graph and then one graph of the rem remaining steps (n_main * G + rem
    = steps). The Ge steps with per-stage event nodes (which cut the programmatic edges and add
    ~3 us per stage) are a separate graph replayed after the timed region, never inside it."""
    if steps < 1 or period < 1:
        raise ValueError("steps and period must be >= 1")
    G = min(steps, period)
    n_main, rem = divmod(steps, G)
    Ge = max(1, min(G, event_steps))
    return G, n_main, rem, Ge


def timed_replays(steps: int, period: int, event_steps: int):
    """The graph replays of the timed region, in order: (graph, steps it runs, instrumented).
    None of them carries event nodes, whatever the step counts."""
    G, n_main, rem, _ = step_plan(steps, period, event_steps)
    plan = [("graph", G, False)] * n_main
    if rem:
        plan.append(("graph_rem", rem, False))
    return plan


def expert_set_bytes(cfg) -> int:
    """Blob bytes of one layer's experts (routed and shared: codes and scales)."""
    b = cfg.E * (blob_row_bytes(cfg, cfg.H, 2 * cfg.I) + blob_row_bytes(cfg, cfg.I, cfg.H))
    if cfg.shared_I:
        b += blob_row_bytes(cfg, cfg.H, 2 * cfg.shared_I) + blob_row_bytes(cfg, cfg.shared_I, cfg.H)
    return b


def line_config(cfg, T, args, world=1):
    """The `config` object of the JSON line: the workload and how it is stepped. Both arms
    print the same object for the same arguments."""
    G, n_main, rem, Ge = step_plan(args.steps, args.period, args.event_steps)
    R = args.replicas
    return {"workload": workload_desc(cfg, T, args.top_p), "T": T, "replicas": R,
            "l2": f"inputs larger than L2: {R} layer replicas rotate "
                  f"({R * expert_set_bytes(cfg) / 1e9:.2f} GB of expert blobs)",
            "graph": f"timed steps replayed as CUDA graphs of {G} steps ({n_main} x {G}"
                     f"{f' + {rem}' if rem else ''}) with no event nodes; per-stage events come "
                     f"from {Ge} further steps replayed after the timed region",
            "accumulate": "int32 dots, fp32 scales",
            "parallelism": f"dp{world} (weak: independent tokens per GPU)"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 20 ms while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.samples = []
        self.proc = None
        self.window = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.perf_counter(), line.strip()))

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        t0, t1 = self.window if self.window else (0, float("inf"))
        inside = [s for ts, s in self.samples if t0 <= ts <= t1]
        note = "samples inside the timed region"
        if not inside and self.samples:
            # region shorter than one sampling period: keep the samples bracketing it
            near = sorted(self.samples, key=lambda p: min(abs(p[0] - t0), abs(p[0] - t1)))[:2]
            inside = [s for _, s in near]
            note = "timed region shorter than the 20 ms sampling period: nearest samples"
        sm, mx, reasons = [], [], set()
        for s in inside:
            f = [v.strip() for v in s.split(",")]
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except (ValueError, IndexError):
                continue
            for name, v in zip(self.REASONS, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "note": note}


# --------------------------------------------------------------------- oracle
def oracle_sampler(cfg, T, top_p=0.0, seed_base=7_000_000):
    """Prepare the oracle for timing on host cores: experts of a token sample, pre-quantized.
    Returns (run_units(n_units) -> tokens processed, unit description, cores)."""
    import oracle as O
    from concurrent.futures import ThreadPoolExecutor

    cores = os.cpu_count() or 1
    wbits = {"int8": 8, "int4": 4, "int2": 2}[cfg.wtype]
    wg32 = cfg.wscale == "g32_f16"
    ag32 = cfg.act == "g32_f16"
    n_tok = 64
    case = S.Case.make(cfg, n_tok, seed=seed_base + T)
    x = case.x()
    Wr, bias = case.router_w(), case.bias()
    L = O.router_logits(x, Wr)
    idx, _ = O.route(L, bias, cfg.score, cfg.top_k, cfg.renormalize, cfg.rsf, top_p=top_p)
    experts = {}
    shared = None
    if cfg.shared_I:
        shared = O.QExperts.quantize(case.shared_gate_up()[None], case.shared_down()[None], wbits, wg32)
    per_tok = cfg.top_k + (1 if shared is not None else 0)
    pool = ThreadPoolExecutor(cores)

    def ensure(e):
        if e not in experts:
            experts[e] = O.QExperts.quantize(case.gate_up(e)[None], case.down(e)[None], wbits, wg32)
        return experts[e]

    # pre-quantize the experts of the first tokens (input preparation, not timed)
    for e in sorted(set(int(v) for v in idx[:16].reshape(-1)) - {-1}):
        ensure(e)
    cursor = [0]

    def run_units(n_units):
        """Oracle work for n_units (token, expert) units starting at the cursor: per token the
        router logits, top-k, activation quantization, its expert FFNs and the combine."""
        units = []
        while len(units) < n_units:
            t = (cursor[0] // per_tok) % 16
            u = cursor[0] % per_tok
            units.append((t, u))
            cursor[0] += 1
        toks = sorted(set(t for t, _ in units))
        Lt = O.router_logits(x[toks], Wr)
        it, wt = O.route(Lt, bias, cfg.score, cfg.top_k, cfg.renormalize, cfg.rsf, top_p=top_p)
        qx, sx = O.quantize_act(x[toks], ag32)
        pos = {t: i for i, t in enumerate(toks)}

        def one(tu):
            t, u = tu
            i = pos[t]
            if u < cfg.top_k:
                if it[i, u] < 0:                 # slot dropped by adaptive top-p
                    return i, 0.0
                r = O.expert_ffn(experts[int(it[i, u])], 0, qx[i], sx[i], ag32)
                return i, wt[i, u] * r["ye"]
            r = O.expert_ffn(shared, 0, qx[i], sx[i], ag32)
            return i, r["ye"]

        y = np.zeros((len(toks), cfg.H))
        for i, v in pool.map(one, units):
            y[i] += v
        return n_units / per_tok

    desc = (f"(token, expert) units of {cfg.name}: per token its router logits, top-{cfg.top_k}, "
            f"Q8_0 quantization, {per_tok} expert FFNs (fp64 down) and the combine; "
            f"16 tokens cycled, {cores} threads over units")
    return run_units, desc, cores


def time_oracle(cfg, T, top_p=0.0, budget_s=45.0):
    run_units, desc, cores = oracle_sampler(cfg, T, top_p)
    per_tok = cfg.top_k + (1 if cfg.shared_I else 0)
    t0 = time.perf_counter()
    run_units(per_tok)
    t1 = time.perf_counter() - t0
    # about budget_s of CPU work (the first, single-token call sizes it)
    n = max(per_tok, int(budget_s / max(t1, 1e-4)) * per_tok)
    n = min(n, 100_000 * per_tok)
    t0 = time.perf_counter()
    toks = run_units(n)
    el = time.perf_counter() - t0
    return {"value": toks / el, "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"{toks:g} tokens = {n} {desc}; {el:.1f} s"}


def reference_arm(args, cfg, T):
    """The oracle as the reference implementation, on host cores: K timed steps, each a
    bounded sample of the workload (whole (token, expert) units), so the run stays short."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    run_units, desc, cores = oracle_sampler(cfg, T, args.top_p)
    per_tok = cfg.top_k + (1 if cfg.shared_I else 0)
    t0 = time.perf_counter()
    run_units(1)
    t_unit = max(time.perf_counter() - t0, 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    units = int(max(1, min(per_tok * T, budget / t_unit)))
    for _ in range(args.warmup):
        run_units(units)
    t0 = time.perf_counter()
    toks = 0.0
    for _ in range(args.steps):
        toks += run_units(units)
    el = time.perf_counter() - t0
    value = toks / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": line_config(cfg, T, args, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps, each {units} {desc} "
                                   f"({units / per_tok:g} tokens per step)"},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- GPU arm
PREFILL_WORKLOAD = "olmoe_int4:4096"


def rank_seeds(rank: int, replicas: int, batches: int):
    """Weak scaling: every rank its own layer replicas (expert weights) and token batches --
    seeds disjoint across ranks, so no rank's inputs repeat another's."""
    return ([1000 * rank + r for r in range(replicas)],
            [90_000_000 + 1_000_000 * rank + s for s in range(batches)])


def max_over_ranks(ms: float, world: int, device) -> float:
    """The timed duration of the slowest rank (every rank calls this, in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank_step: int, world: int, steps: int, ms_max: float) -> float:
    """Tokens per second of all ranks together over the slowest rank's timed region."""
    return world * tokens_per_rank_step * steps / (ms_max / 1e3)


def prefill_arm(args, dev, world, M, torch, dist):
    """The metric's "prefill 4k" half: the OLMoE-shaped packed-int4 layer (group-32 scales) on
    T = 4096 fresh tokens per GPU (every expert > 64 pairs: the tensor-core GEMMs). Eager steps
    timed with CUDA events (max over ranks); the GEMM kernels' share from stage events."""
    cfg, T = parse_workload(args.prefill_workload)
    rank = int(os.environ.get("RANK", "0"))
    rcfg = M.RouteCfg(score=cfg.score, top_k=cfg.top_k, renormalize=cfg.renormalize,
                      routed_scaling_factor=cfg.rsf, act=cfg.act)
    case = S.Case.make(cfg, T, replica=1000 * rank + 7)
    gu = torch.empty((cfg.E, 2 * cfg.I, cfg.H), dtype=torch.float32, device=dev)
    case.gate_up_gpu(gu)
    dn = torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.float32, device=dev)
    case.down_gpu(dn)
    blob = M.ExpertBlob.quantize(gu, dn, cfg.wtype, cfg.wscale)
    del gu, dn
    shared = None
    if cfg.shared_I:
        sgu = torch.empty((1, 2 * cfg.shared_I, cfg.H), dtype=torch.float32, device=dev)
        sdn = torch.empty((1, cfg.H, cfg.shared_I), dtype=torch.float32, device=dev)
        case.shared_gate_up_gpu(sgu)
        case.shared_down_gpu(sdn)
        shared = M.ExpertBlob.quantize(sgu, sdn, cfg.wtype, cfg.wscale)
        del sgu, sdn
    wr = torch.from_numpy(case.router_w()).to(dev)
    b = case.bias()
    bias = torch.from_numpy(b).to(dev) if b is not None else None
    lay = M.Layer(T, blob, shared, rcfg, wr, bias)
    xs = [torch.from_numpy(S.Case.make(cfg, T, seed=80_000_000 + 1_000_000 * rank + s).x()).to(dev)
          for s in range(2)]
    y = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    steps = max(1, args.prefill_steps)
    nst = len(M.MOE_STAGES)
    ev = M.moe_stage_events()
    pairs = []
    with torch.cuda.stream(stream):
        for i in range(nst):
            b_ev = torch.cuda.Event(enable_timing=True, external=True)
            e_ev = torch.cuda.Event(enable_timing=True, external=True)
            b_ev.record(stream)
            e_ev.record(stream)
            ev.begin[i], ev.end[i] = b_ev.cuda_event, e_ev.cuda_event
            pairs.append((b_ev, e_ev))
        for s in range(3):
            lay(xs[s % 2], y, stream)
    stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for s in range(steps):
            lay(xs[s % 2], y, stream)
        e1.record(stream)
    stream.synchronize()
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item()) / steps
    # stage times of one more step: gate/up stage = tile plan + gather + gate/up GEMM (+ the
    # streaming kernel, idle here), down stage = the down GEMM
    with torch.cuda.stream(stream):
        lay(xs[0], y, stream, events=ev)
    stream.synchronize()
    stage = {n: pairs[i][0].elapsed_time(pairs[i][1]) * 1e3 for i, n in enumerate(M.MOE_STAGES)}
    peaks, _ = load_peaks()
    # the GEMMs run on fp16 tensor cores (kind::f16; the integer codes are exact in fp16):
    # their peak is the dense fp16 = bf16 rate, measured as a burst (the GEMMs of this short
    # timed loop run at full clocks)
    f16_peak = peaks["bf16_tflops"]
    ops = layer_int_ops(cfg, T)
    gemm_us = stage["gate_up"] + stage["down"]
    ach = ops / (gemm_us * 1e-6) / 1e12
    return {
        "workload": workload_desc(cfg, T), "T": T, "value": round(world * T / (ms / 1e3), 1),
        "unit": "tok/s", "ms_per_step": round(ms, 4), "steps": steps,
        "stage_us": {k: round(v, 1) for k, v in stage.items()},
        "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": round(f16_peak, 1),
                     "unit": "TFLOP/s", "frac": round(ach / f16_peak, 4),
                     "kernel": "k_expert_mma gate/up + down (tcgen05.mma kind::f16 on the integer codes, exact fp32 "
                               "group dots, per-group fp32 epilogue)",
                     "ops_per_step": int(ops),
                     "peak_source": "measured bf16 TFLOP/s burst (MEASURED_PEAKS.json); dense fp16 runs at the bf16 rate"},
        "note": "the per-group fp32 epilogue (2 fp32 operations per element per quantization group) bounds the "
                "tensor-core path",
    }


def gpu_arm(args, cfg, T):
    import torch
    import torch.distributed as dist
    import quantized_expert_ffn_logits_b200 as M

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    R = args.replicas
    G = step_plan(args.steps, args.period, args.event_steps)[0]
    rep_seeds, x_seeds = rank_seeds(rank, R, G)
    rcfg = M.RouteCfg(score=cfg.score, top_k=cfg.top_k, renormalize=cfg.renormalize,
                      routed_scaling_factor=cfg.rsf, act=cfg.act, top_p=args.top_p)
    layers, n_active_of, kept_of = [], [], []
    for r in range(R):
        case = S.Case.make(cfg, T, replica=rep_seeds[r])
        gu = torch.empty((cfg.E, 2 * cfg.I, cfg.H), dtype=torch.float32, device=dev)
        case.gate_up_gpu(gu)
        dn = torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.float32, device=dev)
        case.down_gpu(dn)
        blob = M.ExpertBlob.quantize(gu, dn, cfg.wtype, cfg.wscale)
        del gu, dn
        shared = None
        if cfg.shared_I:
            sgu = torch.empty((1, 2 * cfg.shared_I, cfg.H), dtype=torch.float32, device=dev)
            sdn = torch.empty((1, cfg.H, cfg.shared_I), dtype=torch.float32, device=dev)
            case.shared_gate_up_gpu(sgu)
            case.shared_down_gpu(sdn)
            shared = M.ExpertBlob.quantize(sgu, sdn, cfg.wtype, cfg.wscale)
            del sgu, sdn
        wr = torch.from_numpy(case.router_w()).to(dev)
        b = case.bias()
        bias = torch.from_numpy(b).to(dev) if b is not None else None
        layers.append(M.Layer(T, blob, shared, rcfg, wr, bias))
    torch.cuda.synchronize()
    # distinct token batches (one per step of a graph), resident in HBM before timing
    xs = []
    for s in range(G):
        xc = S.Case.make(cfg, T, seed=x_seeds[s])
        xs.append(torch.from_numpy(xc.x()).to(dev))
    y = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    # distinct experts per step (for the algorithmic byte counts)
    for s in range(G):
        lay = layers[s % R]
        idx, _ = M.moe_route_topk(M.moe_router_logits(xs[s], lay.router_w), lay.router_bias, rcfg)
        n_active_of.append(int(torch.unique(idx[idx >= 0]).numel()))   # -1: dropped by top-p
        kept_of.append(int((idx >= 0).sum()))
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    # warm-up (eager)
    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            layers[s % R](xs[s % G], y, stream)
    stream.synchronize()

    # Graphs (step_plan): `graph` = G steps and `graph_rem` = the remainder, neither with event
    # nodes, are the timed region; `graph_ev` = Ge steps with every stage bracketed by CUDA
    # events (external event nodes, which cut the programmatic edges around them) is replayed
    # once after the timed region for the per-stage durations.
    G, n_main, rem, Ge = step_plan(args.steps, args.period, args.event_steps)
    nst = len(M.MOE_STAGES)
    evs = []
    with torch.cuda.stream(stream):
        for s in range(Ge):
            e = M.moe_stage_events()
            pair = []
            for i in range(nst):
                b_ev = torch.cuda.Event(enable_timing=True, external=True)
                e_ev = torch.cuda.Event(enable_timing=True, external=True)
                b_ev.record(stream)
                e_ev.record(stream)
                e.begin[i] = b_ev.cuda_event
                e.end[i] = e_ev.cuda_event
                pair.append((b_ev, e_ev))
            evs.append((e, pair))
    stream.synchronize()
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        for s in range(Ge):
            layers[s % R](xs[s], y, stream, events=evs[s][0])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for s in range(G):
            layers[s % R](xs[s], y, stream)
    graph_rem = None
    if rem:
        graph_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_rem, stream=stream):
            for s in range(rem):
                layers[s % R](xs[s], y, stream)
    # one untimed replay of each
    with torch.cuda.stream(stream):
        graph.replay()
        graph_ev.replay()
        if graph_rem is not None:
            graph_rem.replay()
    stream.synchronize()

    # ------------------------------------------------------------ timed region
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(gpu_id)
    time.sleep(0.1)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    w0 = time.perf_counter()
    graphs = {"graph": graph, "graph_rem": graph_rem}
    with torch.cuda.stream(stream):
        # a ~50 us spin ahead of the start event keeps the GPU busy while the host submits
        # the graph replays, so the timed region holds device time only (no submission
        # latency between the start event and the first step)
        torch.cuda._sleep(100_000)
        start.record(stream)
        for name, _, _ in timed_replays(args.steps, args.period, args.event_steps):
            graphs[name].replay()
        end.record(stream)
    stream.synchronize()
    w1 = time.perf_counter()
    torch.cuda.nvtx.range_pop()
    barrier()
    clocks.mark(w0, w1)
    clk = clocks.stop()
    ms_max = max_over_ranks(start.elapsed_time(end), world, dev)

    # per-stage device times: the instrumented graph, replayed after the timed region
    with torch.cuda.stream(stream):
        graph_ev.replay()
    stream.synchronize()
    stage_ms = {n: [] for n in M.MOE_STAGES}
    for s in range(Ge):
        for i, n in enumerate(M.MOE_STAGES):
            b_ev, e_ev = evs[s][1][i]
            stage_ms[n].append(b_ev.elapsed_time(e_ev))
    stage_us = {n: (1e3 * statistics.mean(v) if v else None) for n, v in stage_ms.items()}

    value = whole_job_rate(T, world, args.steps, ms_max)
    peaks, peak_src = load_peaks()
    n_act = float(np.mean(n_active_of))
    # dominant kernel: the expert kernel (weight streaming, HBM-bound); with group-32
    # activations one launch runs gate/up, SwiGLU, h quantization, down and the combine, and
    # the gate/up stage events bracket it
    fused = cfg.act == "g32_f16"
    gu_us = stage_us["gate_up"]
    gu_bytes = float(np.mean([(expert_bytes if fused else gateup_bytes)(cfg, T, a) for a in n_active_of]))
    one_launch = layers[0].kernels == 1
    how = (f"gate/up stage events of {Ge} instrumented steps replayed after the timed region "
           f"(event nodes around the expert kernel: the duration includes its launch latency)")
    if one_launch:
        # one kernel per step (single-token routing inside it): it also reads the router weight
        # and x and writes y, and its average launch duration is the event-free timed region
        # over its launches
        gu_bytes = float(np.mean([layer_bytes(cfg, T, a) for a in n_active_of]))
        gu_us = ms_max * 1e3 / args.steps
        how = f"one launch per step: CUDA events around the {args.steps} event-free timed steps / launches"
    roof = None
    if gu_us:
        ach = gu_bytes / (gu_us * 1e-6) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": traffic_from_profiles(cfg, T),
                "kernel": (("k_expert_ring (single token: routing, gate/up, SwiGLU, h quantization, down, "
                            "weighted combine)" if one_launch else
                            "k_expert_ring (gate/up, SwiGLU, h quantization, down, weighted combine)")
                           if fused else "k_expert_ring (gate/up pass)"),
                "bytes_per_launch": int(gu_bytes), "us_per_launch": round(gu_us, 3), "timing": how,
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback 6.65 TB/s"}
    lb = float(np.mean([layer_bytes(cfg, T, a) for a in n_active_of]))
    step_s = ms_max / 1e3 / args.steps
    layer = {"bytes_per_step": int(lb), "gbs": round(lb / step_s / 1e9, 1),
             "frac_hbm": round(lb / step_s / 1e9 / peaks["hbm_gbs"], 4),
             "int8_tops": round(layer_int_ops(cfg, T, float(np.mean(kept_of))) / step_s / 1e12, 2),
             "routed_pairs_per_step": round(float(np.mean(kept_of)), 2),
             "distinct_experts_per_step": round(n_act, 2),
             "stage_us": {k: (round(v, 3) if v is not None else None) for k, v in stage_us.items()}}

    # ---------------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        ne = min(args.steps, args.e2e_steps)
        xh = [torch.from_numpy(S.Case.make(cfg, T, seed=95_000_000 + s).x()).pin_memory() for s in range(min(ne, 64))]
        yh = torch.empty((T, cfg.H), dtype=torch.float32).pin_memory()
        with torch.cuda.stream(stream):
            for s in range(3):
                layers[s % R].forward_host(xh[s % len(xh)], yh, stream)
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for s in range(ne):
                layers[s % R].forward_host(xh[s % len(xh)], yh, stream)
            e1.record(stream)
        stream.synchronize()
        barrier()
        te = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e = {"value": world * T * ne / (float(te.item()) / 1e3), "unit": "tok/s",
               "h2d_bytes_per_step": T * cfg.H * 4, "d2h_bytes_per_step": T * cfg.H * 4,
               "steps": ne, "path": "Layer.forward_host -> moe_layer_forward_host (C ABI, one call per step: "
                       "pinned host x copied in, the layer, y copied out), eager"}

    prefill = None
    if not args.no_prefill:
        prefill = prefill_arm(args, dev, world, M, torch, dist)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle(cfg, T, args.top_p)

    launches = layers[0].kernels * args.steps
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": line_config(cfg, T, args, world),
        "roofline": roof,
        "layer": layer,
        "prefill": prefill,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    del graph, graph_rem, graph_ev
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def traffic_from_profiles(cfg, T):
    """DRAM bytes (read + write) per launch of the expert kernel from the committed ncu
    summary, if it was taken on this workload with the current kernel source; else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "k_expert_ring_traffic.json")
    src = os.path.join(ROOT, "quantized_expert_ffn_logits_b200", "csrc", "expert_stream.cu")
    try:
        with open(path) as f:
            d = json.load(f)
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if d.get("source_sha256_16") != h or d.get("workload") != f"{cfg.name}:{T}":
            return None
        return d.get("dram_bytes_per_launch")
    except Exception:
        return None


def fp8_convert_arm(args):
    """The FP8 checkpoint converter (GLM page, FP8 -> int4): moe_quantize_experts_fp8 on the
    OLMoE-shaped expert set (E4M3 codes with 128 x 128 block scales -> packed int4, group-32
    fp16 scales), device-resident input, CUDA events over K conversions. Bound: HBM (read the
    codes and scales once, write the blob once)."""
    import torch
    import quantized_expert_ffn_logits_b200 as M
    cfg = S.CONFIGS["olmoe_int4"]
    E, H, I = cfg.E, cfg.H, cfg.I
    cdiv = lambda a: (a + 127) // 128
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(8)
    def codes(shape):
        c = torch.randint(0, 256, shape, dtype=torch.uint8, device=dev, generator=g)
        return torch.where((c & 0x7F) == 0x7F, torch.full_like(c, 0x3A), c)   # no NaN codes
    gu8, dn8 = codes((E, 2 * I, H)), codes((E, H, I))
    sgu = torch.rand((E, cdiv(2 * I), cdiv(H)), device=dev, generator=g) * 2 ** -8 + 2 ** -9
    sdn = torch.rand((E, cdiv(H), cdiv(I)), device=dev, generator=g) * 2 ** -8 + 2 ** -9
    blob = M.ExpertBlob(cfg.wtype, cfg.wscale, E, H, I, device=dev)
    for _ in range(args.warmup):
        M.moe_quantize_experts_fp8(gu8, sgu, dn8, sdn, blob)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        M.moe_quantize_experts_fp8(gu8, sgu, dn8, sdn, blob)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    nbytes = gu8.numel() + dn8.numel() + 4 * (sgu.numel() + sdn.numel()) + blob.nbytes
    peaks, src = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {"metric": "FP8 checkpoint -> int4 blob conversion (moe_quantize_experts_fp8)",
            "value": round(gbs, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8->int4", "data": "synthetic",
            "config": {"workload": f"OLMoE-shaped experts E{E} H{H} I{I}: E4M3 codes + 128x128 block "
                                   f"scales -> {cfg.wtype} {cfg.wscale} blob",
                       "bytes_per_step": int(nbytes), "experts_per_s": round(E / (ms * 1e-3), 1)},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None,
                         "peak_source": src},
            "gpu_launches": 2 * args.steps}     # a blob memset and the conversion kernel per step
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="config[:T], config one of " + ", ".join(S.CONFIG_ORDER))
    ap.add_argument("--replicas", type=int, default=8, help="layer replicas rotated per step")
    ap.add_argument("--period", type=int, default=256, help="steps per captured graph")
    ap.add_argument("--event-steps", type=int, default=32,
                    help="steps with per-stage event records, replayed after the timed region")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill (4k tokens) measurement")
    ap.add_argument("--prefill-workload", default=PREFILL_WORKLOAD)
    ap.add_argument("--prefill-steps", type=int, default=20)
    ap.add_argument("--fp8-convert", action="store_true",
                    help="time the FP8 checkpoint converter instead of the layer (one JSON line)")
    ap.add_argument("--top-p", type=float, default=0.0,
                    help="adaptive expert top-p of the main workload (0 = off; the prefill half "
                         "is measured without it)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    cfg, T = parse_workload(args.workload)
    if args.fp8_convert:
        return fp8_convert_arm(args)
    if args.impl == "reference":
        return reference_arm(args, cfg, T)
    return gpu_arm(args, cfg, T)


if __name__ == "__main__":
    sys.exit(main())
