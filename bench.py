#!/usr/bin/env python
"""Benchmark: one MoE layer forward (hidden 1280, 64 routed experts, top-6, fused
shared expert) on a B200, through libfocr_moe.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward of the layer over one batch of synthetic tokens (router,
softmax/top-6, dispatch, routed + shared experts, combine).  The default workload
is the largest single-GPU layer workload: prefill of 289 tokens (273 visual rows +
16 prompt rows) through an int4 (group 64) layer with bf16 router and shared
expert, where every expert is hit.  Steps rotate over packed copies of the layer
(far above the 126 MB L2) and over a pool of distinct token batches, so the weights
come from HBM.  Under torchrun every rank runs an independent replica (no data
exchange: the path does not shard), and `value` sums all ranks' tokens over the
slowest rank's time.  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and achieved HBM GB/s (% of B200 peak) vs CPU oracle"
UNIT = "tokens/s"
N_COPIES = 16
DEFAULT_WORKLOAD = "prefill289_int4_g64"
PEAK_FALLBACK_GBS = 6650.0           # profiling recipe's fallback copy bandwidth
PEAK_FALLBACK_TFLOPS = 1590.0        # ... and cuBLAS bf16 burst throughput
PEAK_FALLBACK_TFLOPS_SUSTAINED = 1400.0
GRAPH_STEPS = 160                    # forwards per captured CUDA graph


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=N_COPIES, help="packed layer copies to rotate over")
    ap.add_argument("--eager", action="store_true", help="launch every step from Python (no CUDA graph)")
    return ap.parse_args()


TNAME = {0: "bf16", 1: "int8", 2: "int4"}


def describe(name: str, world: int) -> dict:
    """The workload's config (the same dict in both arms)."""
    from weight_quantized_expert_b200 import synth
    if name in synth.STEP_WORKLOADS:
        w = synth.STEP_WORKLOADS[name]
        d = {"workload": name, "tokens_per_step": w["T"], "kind": w["kind"], "seed": w["seed"],
             "parallelism": f"replicas x{world}"}
        if w["kind"] == "rswa":
            d.update(sequences=w["T"], reference_rows=w["R"], generated=w["n_gen"], heads=10, head_dim=128,
                     ring=128, kv="fp32")
        if w["kind"] == "w8a8":
            d.update(matrix="129280 x 1280 int8, one fp32 scale per row (the lm_head's shape)",
                     activations="int8, one fp32 scale per token", accumulate="exact integer (i32)")
        if w["kind"] == "stack":
            d.update(wiring="h <- RMSNorm(h + FFN(h)) per layer (eps 1e-6, gamma 1); lm_head on the last norm",
                     moe_layers=w["moe_layers"], moe="int4 g64, bf16 router and shared expert",
                     dense="int8 g128", lm_head="int8 per-row")
        return d
    w = synth.WORKLOADS[name]
    return {"workload": name, "tokens_per_step": w["T"], "routed": f"{TNAME[w['routed']]} g{w['group']}",
            "shared": TNAME[w["shared"]] if w["shared"] == 0 else f"{TNAME[w['shared']]} g{w['group']}",
            "router": "bf16", "seed": w["seed"], "hidden": 1280, "experts": "64 routed top-6 + shared 1792",
            "parallelism": f"replicas x{world}"}


def precision(T: int):
    """(dtype, description) of the arithmetic the path runs for a batch of T tokens."""
    if T > 8:
        return "f16+bf16", ("tcgen05 MMAs: gate/up with f16 operands (x rounded to f16, weights dequantised to "
                            "f16 q*s), down with bf16 operands (SwiGLU output and weights q*s rounded to bf16), "
                            "fp32 accumulation in TMEM; router fp64")
    return "f16", ("mma.sync with f16 operands (int4/int8 codes exact, activations rounded to f16; bf16 "
                   "weights exact with bf16 hi+lo activations), fp32 accumulation; router fp64")


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, 'measured'|'fallback')."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        tf = float(d.get("bf16_tflops", PEAK_FALLBACK_TFLOPS))
        return float(d["hbm_gbs"]), tf, float(d.get("bf16_tflops_sustained", tf)), "measured"
    return PEAK_FALLBACK_GBS, PEAK_FALLBACK_TFLOPS, PEAK_FALLBACK_TFLOPS_SUSTAINED, "fallback"


def sources_hash(files=None) -> str:
    """Identity of the kernel code a profile was taken on: the listed CUDA/C++ sources (all of csrc/
    when none are listed) with comments and blank space removed (the sources hold no comment markers
    inside string literals), so a comment edit keeps a profile valid and any code change in those
    files invalidates it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_quantized_expert_b200", "csrc")
    paths = sorted(glob.glob(os.path.join(csrc, "*"))) if not files else sorted(os.path.join(csrc, f) for f in files)
    for f in paths:
        src = open(f, encoding="utf-8").read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(os.path.basename(f).encode())
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per step from the committed ncu summary, if it matches these sources."""
    for f in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        txt = open(f).read()
        m_w = re.search(r"^workload:\s*(\S+)", txt, re.M)
        m_t = re.search(r"^traffic_bytes_per_step:\s*(\d+)", txt, re.M)
        m_h = re.search(r"^sources_sha256:\s*(\S+)", txt, re.M)
        m_s = re.search(r"^sources:\s*(.+)$", txt, re.M)
        files = m_s.group(1).split() if m_s else None
        if m_w and m_t and m_h and m_w.group(1) == workload and m_h.group(1) == sources_hash(files):
            return int(m_t.group(1))
    return None


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"focr_clocks_{os.getpid()}_gpu{index}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ ranks (one replica per GPU)

def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank runs an independent replica, the job is done when the
    last one is.  Collective over the default process group (NCCL on GPUs, gloo in the CPU tests)."""
    if world == 1:
        return ms
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(tokens_per_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job tokens/s: the tokens all ranks processed over the slowest rank's time."""
    return tokens_per_step * steps * world / (ms / 1e3)


# ------------------------------------------------------------------ CPU oracle timing

def _oracle_layer(name: str):
    import oracle
    from weight_quantized_expert_b200 import synth
    w = synth.WORKLOADS[name]
    _, layer = synth.workload(name)
    om = oracle.OracleMoE(layer)
    del layer
    pool = synth.hidden(w["seed"] + 1000, 4096, skew=w.get("skew", False))
    return om, pool


def _timed_tokens(run, pool, batch: int, budget_s: float, threads: int):
    """Run batches of `batch` tokens until about `budget_s` have passed; returns (tokens, seconds)."""
    done, total = 0, 0.0
    while total < budget_s and done + batch <= pool.shape[0]:
        t0 = time.perf_counter()
        run(pool[done:done + batch], threads)
        total += time.perf_counter() - t0
        done += batch
    return done, total


def oracle_baseline(name: str, budget_s: float = 18.0) -> dict:
    """The CPU oracle on bounded samples of the workload's tokens: single-threaded, and with its
    OpenMP loop over tokens on every host core (batches of the workload's own size, so a batch of
    T tokens keeps min(T, cores) threads busy)."""
    import oracle
    from weight_quantized_expert_b200 import synth
    om, pool = _oracle_layer(name)
    T = synth.WORKLOADS[name]["T"]
    cores = oracle.max_threads()

    def run(x, th):
        om.forward(x, nthreads=th)

    n1, t1 = _timed_tokens(run, pool, 1, budget_s * 0.3, 1)
    batch = max(T, cores)                       # enough tokens for every core
    nall, tall = _timed_tokens(run, pool, batch, budget_s * 0.7, cores)
    used = min(cores, batch)
    return {"value": nall / tall, "unit": UNIT, "cores": used, "kind": "oracle",
            "single_thread_value": n1 / t1,
            "sample": f"{nall} tokens of workload {name} in batches of {batch} through the CPU oracle (plain C, "
                      f"fp64, OpenMP over tokens, {used} threads) in {tall:.1f} s; single-threaded: {n1} tokens "
                      f"in {t1:.1f} s; layer quantisation excluded"}


def step_oracle_baseline(w: dict, budget_s: float = 12.0) -> dict:
    """tokens/s of the CPU oracle on a bounded sample of a companion / stack workload."""
    import oracle
    from weight_quantized_expert_b200 import synth
    cores = oracle.max_threads()
    kind = w["kind"]
    lm = oracle.OracleLMHead(synth.lm_head(w["seed"])) if kind in ("lm_head", "stack") else None
    w8 = oracle.OracleW8A8(synth.lm_head(w["seed"])) if kind == "w8a8" else None
    dn = None
    if kind in ("dense", "stack"):
        d = synth.dense_mlp(w["seed"])
        dn = oracle.OracleDense(d.gate, d.up, d.down, oracle.W_INT8, 128)
        del d
    om = oracle.OracleMoE(synth.moe_layer(w["seed"], synth.W_INT4, synth.W_BF16, 64)) if kind == "stack" else None

    def run(x, th):
        if kind == "lm_head":
            lm.forward(x, nthreads=th)
        elif kind == "w8a8":
            w8.forward(x)
        elif kind == "dense":
            dn.forward(x, nthreads=th)
        else:
            h = oracle.rmsnorm(x + dn.forward(x, nthreads=th), eps=1e-6)
            for _ in range(w["moe_layers"]):
                h = oracle.rmsnorm(h + om.forward(h, nthreads=th)["out"], eps=1e-6)
            lm.forward(h, nthreads=th)

    pool = synth.hidden(w["seed"] + 5000, 512)
    if kind == "w8a8":   # the oracle's W8A8 GEMV is single-threaded
        cores = 1
    batch = max(1, min(cores, 8)) if kind == "stack" else cores
    nall, tall = _timed_tokens(run, pool, batch, budget_s, cores)
    if nall == 0:   # one batch did not fit the budget: time one anyway
        t0 = time.perf_counter()
        run(pool[:batch], cores)
        nall, tall = batch, time.perf_counter() - t0
    used = min(cores, batch)
    what = {"stack": "dense layer 0, 11 MoE layers, RMSNorm, lm_head",
            "w8a8": "W8A8 GEMV (129280 x 1280)"}.get(kind, kind)
    return {"value": nall / tall, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{nall} tokens through the CPU oracle's {what} in batches of {batch} ({used} threads, "
                      f"{'plain C, int64 dot' if kind == 'w8a8' else 'plain C, fp64, OpenMP'}) in {tall:.1f} s"}


# ------------------------------------------------------------------ reference arm

def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step is the oracle forward of one batch of the
    workload's tokens on the host cores, steps capped so the run stays within a few minutes."""
    if rank != 0:
        return
    import oracle
    from weight_quantized_expert_b200 import synth
    cores = oracle.max_threads()
    if args.workload in synth.STEP_WORKLOADS:
        w = synth.STEP_WORKLOADS[args.workload]
        cpu = rswa_oracle_baseline(w, budget_s=60.0) if w["kind"] == "rswa" else step_oracle_baseline(w, budget_s=60.0)
        v = cpu["value"]
        dtype = "int64" if w["kind"] == "w8a8" else "f64"
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": w["T"] / v * 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
                          "data": "synthetic", "config": describe(args.workload, world), "cpu_baseline": cpu,
                          "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return
    T = synth.WORKLOADS[args.workload]["T"]
    om, pool = _oracle_layer(args.workload)
    used = min(cores, T)
    t0 = time.perf_counter()
    om.forward(pool[:T], nthreads=cores)
    per_step = time.perf_counter() - t0
    budget = 150.0
    steps, warm = args.steps, args.warmup
    if (steps + warm) * per_step > budget:
        warm = min(warm, 1)
        steps = max(1, int(budget / per_step) - warm)
    span = pool.shape[0] - T
    for i in range(warm):
        s = (i * T) % span
        om.forward(pool[s:s + T], nthreads=cores)
    t0 = time.perf_counter()
    for i in range(steps):
        s = (i * T) % span
        om.forward(pool[s:s + T], nthreads=cores)
    dt = time.perf_counter() - t0
    value = steps * T / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": dt / steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": describe(args.workload, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                             "sample": f"{steps} steps x {T} token(s) of the workload through the CPU oracle "
                                       f"(plain C, fp64, OpenMP over the step's tokens: {used} threads)"
                                       + ("" if steps == args.steps else
                                          f"; steps capped from {args.steps} to bound the CPU run")},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ timing helpers

def capture_graphs(step, K: int, stream):
    """CUDA graphs covering exactly K steps: `full` replays of a graph of G = min(K, GRAPH_STEPS)
    steps, then a tail graph of K mod G steps.  Every graph is replayed once here, so no graph
    upload or first-launch work falls inside the timed region."""
    import torch
    G = min(K, GRAPH_STEPS)
    graphs = []
    g_main = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_main, stream=stream):
        for i in range(G):
            step(i, torch.cuda.current_stream())
    graphs.append((g_main, K // G))
    tail = K % G
    if tail:
        g_tail = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_tail, stream=stream):
            for i in range(tail):
                step(i, torch.cuda.current_stream())
        graphs.append((g_tail, 1))
    with torch.cuda.stream(stream):
        for g, _ in graphs:
            g.replay()
    stream.synchronize()
    order = [i for i in range(G)] * (K // G) + [i for i in range(tail)]
    return graphs, order


def timed_replay(graphs, stream, world, dev, local_rank):
    import torch
    clocks = Clocks(local_rank)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for g, n in graphs:
            for _ in range(n):
                g.replay()
        ev1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    return max_over_ranks(ev0.elapsed_time(ev1), world, dev), clk


# ------------------------------------------------------------------ decode-step companions

def step_bytes_companion(w: dict, moe_hits=None) -> int:
    """Algorithmic bytes of one step of a companion / stack workload."""
    from weight_quantized_expert_b200 import roofline
    T = w["T"]
    lm = roofline.VOCAB * roofline.H * 1 + roofline.VOCAB * 4 + T * roofline.H * 4 + T * 4
    dense = roofline.swiglu_bytes(roofline.DENSE_I, roofline.W_INT8, 128) + T * roofline.H * 4 * 2
    if w["kind"] == "lm_head":
        return lm
    if w["kind"] == "w8a8":   # codes, row scales, x in, y out
        return roofline.VOCAB * roofline.H + roofline.VOCAB * 4 + T * roofline.H * 4 + T * roofline.VOCAB * 4
    if w["kind"] == "dense":
        return dense
    moe = sum(roofline.moe_layer_bytes(T, roofline.W_INT4, roofline.W_BF16, 64, h) for h in moe_hits)
    norms = (1 + len(moe_hits)) * T * roofline.H * 4 * 2
    return dense + moe + norms + lm


def run_step_workload(args, rank, world, local_rank):
    """lm_head GEMV + argmax, the dense layer 0, or a whole decode step (dense layer 0, 11 MoE layers with
    residual adds, RMSNorm, lm_head + argmax) through the C ABI; same JSON contract as the layer bench."""
    import torch
    from weight_quantized_expert_b200 import api, synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.STEP_WORKLOADS[args.workload]
    T, kind = w["T"], w["kind"]
    head = mlp = None
    layers = []
    w8 = None
    if kind in ("lm_head", "stack"):
        head = api.focr_lm_head_pack(synth.lm_head(w["seed"]))
    if kind == "w8a8":
        w8 = api.focr_w8a8_pack(synth.lm_head(w["seed"]))
        w8_ws = torch.zeros(api.focr_w8a8_workspace_bytes(w8, T), dtype=torch.uint8, device=dev)
        w8_y = torch.empty(T, w8.N, device=dev)
    if kind in ("dense", "stack"):
        d = synth.dense_mlp(w["seed"])
        mlp = api.focr_dense_mlp_pack(d.gate, d.up, d.down, synth.W_INT8, 128)
        del d
    if kind == "stack":
        base = api.focr_moe_pack_weights(synth.moe_layer(w["seed"], synth.W_INT4, synth.W_BF16, 64))
        layers = [base] + [api.focr_moe_layer_clone(base) for _ in range(w["moe_layers"] - 1)]
    pool_n = 16
    xs = torch.from_numpy(synth.hidden(w["seed"] + 3000 + rank, pool_n * T).reshape(pool_n, T, 1280)).to(dev)
    ws = api.new_workspace(T, dev)
    lm_ws = torch.zeros(api.focr_lm_head_workspace_bytes(T), dtype=torch.uint8, device=dev)
    hb = [torch.empty(T, 1280, device=dev) for _ in range(2)]
    am = torch.empty(T, dtype=torch.int32, device=dev)
    model = api.DecodeModel(mlp, layers, head, eps=1e-6) if kind == "stack" else None
    step_ws = api.new_decode_step_workspace(T, dev) if kind == "stack" else None
    stream = torch.cuda.Stream(device=dev)
    per_dense = 2 if T <= 8 else 2            # (memset or x-rows) + expert kernel(s)
    per_moe = 3 if T <= 8 else 2
    launches = {"lm_head": 1, "dense": per_dense, "w8a8": 2}.get(kind, 0)
    if kind == "stack":
        launches = per_dense + 1 + (per_moe + 1) * len(layers) + 1

    def run(x, st, debug_counts=None):
        if kind == "lm_head":
            api.focr_lm_head_gemv(head, x, argmax=am, workspace=lm_ws, stream=st)
            return
        if kind == "w8a8":
            api.focr_w8a8_gemv(w8, x, y=w8_y, workspace=w8_ws, stream=st)
            return
        if kind == "dense":
            api.focr_dense_mlp_forward(mlp, x, out=hb[0], workspace=ws, stream=st)
            return
        if debug_counts is None:   # the timed path: one C-ABI call for the whole decode step
            api.focr_decode_step(model, x, argmax=am, workspace=step_ws, stream=st)
            return
        # h <- RMSNorm(h + FFN(h)) for the dense layer and every MoE layer; the last norm feeds lm_head
        # (layer by layer here only to read each layer's routing counts for the byte count)
        api.focr_dense_mlp_forward(mlp, x, out=hb[0], workspace=ws, flags=api.FWD_RESIDUAL, stream=st)
        api.focr_rmsnorm(hb[0], eps=1e-6, out=hb[1], stream=st)
        for li, L in enumerate(layers):
            dbg = {"counts": debug_counts[li]} if debug_counts is not None else None
            api.focr_moe_layer_forward(L, hb[1], out=hb[0], workspace=ws, debug=dbg, stream=st,
                                       flags=api.FWD_RESIDUAL)
            api.focr_rmsnorm(hb[0], eps=1e-6, out=hb[1], stream=st)
        api.focr_lm_head_gemv(head, hb[1], argmax=am, workspace=lm_ws, stream=st)

    hits = None
    if kind == "stack":   # experts hit per layer, for the algorithmic bytes
        counts = [torch.empty(64, dtype=torch.int32, device=dev) for _ in layers]
        per = []
        with torch.cuda.stream(stream):
            for j in range(pool_n):
                run(xs[j], stream, counts)
                per.append([int((c > 0).sum().item()) for c in counts])
        stream.synchronize()
        hits = [sum(p[li] for p in per) / pool_n for li in range(len(layers))]
    bytes_step = step_bytes_companion(w, hits)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            run(xs[i % pool_n], stream)
    stream.synchronize()
    if kind == "stack":   # a device error in the warm-up ends the run before the timed steps
        api.focr_moe_check(step_ws[256:], stream)
    elif kind == "dense":
        api.focr_moe_check(ws, stream)
    elif kind == "w8a8":
        api.focr_w8a8_check(w8_ws, stream)
    elif kind == "lm_head":
        api.focr_lm_head_check(lm_ws, stream)
    K = args.steps
    graphs, _ = capture_graphs(lambda i, st: run(xs[i % pool_n], st), K, stream)
    ms, clk = timed_replay(graphs, stream, world, dev, local_rank)
    ms_step = ms / K
    value = job_rate(T, K, world, ms)
    peak, _, _, peak_kind = peaks()
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    # end to end: pinned host x in, the step, the step's result (argmax, or the dense output) out
    out_t = hb[0] if kind == "dense" else (w8_y if kind == "w8a8" else am)
    hx = torch.from_numpy(synth.hidden(w["seed"] + 4000, T)).pin_memory()
    hy = torch.empty(out_t.shape, dtype=out_t.dtype).pin_memory()
    dx = torch.empty(T, 1280, device=dev)
    K_e2e = min(K, 200)
    with torch.cuda.stream(stream):
        for _ in range(5):
            dx.copy_(hx, non_blocking=True)
            run(dx, stream)
            hy.copy_(out_t, non_blocking=True)
        stream.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(K_e2e):
            dx.copy_(hx, non_blocking=True)
            run(dx, stream)
            hy.copy_(out_t, non_blocking=True)
        f1.record(stream)
        stream.synchronize()
    e2e = job_rate(T, K_e2e, world, max_over_ranks(f0.elapsed_time(f1), world, dev))
    api.focr_moe_check(ws, stream)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = step_oracle_baseline(w)
    if rank == 0:
        dtype, prec = precision(T)
        if kind == "w8a8":
            dtype, prec = "s8", ("int8 weights and per-token int8 activations, mma.sync m16n8k32 s8 with exact "
                                 "s32 accumulation; scales applied in fp64, one rounding to fp32")
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": dtype, "precision": prec, "data": "synthetic", "config": describe(args.workload, world),
                "timing": {"graph": f"CUDA graph replay ({min(K, GRAPH_STEPS)} steps per graph, every graph "
                                    "replayed once before the timed region)",
                           "l2": "one step streams every layer once (> 1.5 GB)" if kind == "stack" else
                                 "inputs re-read every step"},
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "traffic": profiled_traffic(args.workload),
                             "peak_kind": peak_kind,
                             "kernel": "one step of the workload (all its launches, timed together)",
                             "algorithmic_bytes_per_step": bytes_step},
                "cpu_baseline": cpu,
                "e2e": {"value": e2e, "unit": UNIT, "h2d_bytes_per_step": T * 1280 * 4,
                        "d2h_bytes_per_step": int(out_t.numel() * out_t.element_size()), "steps": K_e2e},
                "gpu_launches": launches * K, "clocks": clk}
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ R-SWA decode attention

def rswa_step_bytes(w: dict) -> int:
    """Algorithmic bytes of one R-SWA decode step: every attended key and value row read once
    (reference rows and the 128-slot window), q / k_new / v_new read, out written, the ring slot written."""
    B, R, n = w["T"], w["R"], w["n_gen"]
    row = 10 * 128 * 4
    return B * ((R + min(n, 128)) * 2 * row + 4 * row + 2 * row)


def rswa_oracle_baseline(w: dict, budget_s: float = 12.0) -> dict:
    """sequences/s of the CPU oracle's R-SWA step (single-threaded) on the workload's shapes."""
    import oracle
    from weight_quantized_expert_b200 import synth
    B, R = w["T"], w["R"]
    a = synth.rswa_inputs(w["seed"], B, R)
    done, t = 0, 0.0
    while t < budget_s and done < 4096:
        t0 = time.perf_counter()
        oracle.rswa_decode(a["q"], a["k_new"], a["v_new"], a["k_ref"], a["v_ref"], [R] * B, a["k_ring"],
                           a["v_ring"], [w["n_gen"]] * B)
        t += time.perf_counter() - t0
        done += B
    return {"value": done / t, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} sequence-steps of workload rswa (B = {B}, {R} reference rows, 128-slot window) "
                      f"through the CPU oracle (plain C, fp64, 1 thread) in {t:.1f} s"}


def run_rswa_workload(args, rank, world, local_rank):
    """One R-SWA decode attention step (focr_rswa_decode) for T sequences; same JSON contract."""
    import torch
    from weight_quantized_expert_b200 import api, synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.STEP_WORKLOADS[args.workload]
    B, R, n = w["T"], w["R"], w["n_gen"]
    per_copy = (R + 128) * 2 * 10 * 128 * 4 * B
    ncopy = max(2, -(-160 * 2 ** 20 // per_copy))   # copies of the KV cache, together above L2
    a = synth.rswa_inputs(w["seed"], B, R)
    copies = []
    for c in range(ncopy):
        t = {k: torch.from_numpy(v).to(dev) for k, v in a.items()} if c == 0 else \
            {k: v.clone() for k, v in copies[0].items()}
        copies.append(t)
    rl = torch.full((B,), R, dtype=torch.int32, device=dev)
    ng = torch.full((B,), n, dtype=torch.int32, device=dev)
    out = torch.empty(B, 10, 128, device=dev)
    ws = torch.empty(api.focr_rswa_workspace_bytes(B, R), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def run(i, st, q=None):
        c = copies[i % ncopy]
        api.focr_rswa_decode(c["q"] if q is None else q, c["k_new"], c["v_new"], c["k_ref"], c["v_ref"], rl,
                             c["k_ring"], c["v_ring"], ng, out=out, workspace=ws, stream=st)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            run(i, stream)
    stream.synchronize()
    K = args.steps
    graphs, _ = capture_graphs(lambda i, st: run(i, st), K, stream)
    ms, clk = timed_replay(graphs, stream, world, dev, local_rank)
    ms_step = ms / K
    value = job_rate(B, K, world, ms)
    bytes_step = rswa_step_bytes(w)
    peak, _, _, peak_kind = peaks()
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    # end to end: the step's q in from pinned host memory, its output read back
    hq = torch.from_numpy(a["q"]).pin_memory()
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq = torch.empty_like(copies[0]["q"])
    K_e2e = min(K, 200)
    with torch.cuda.stream(stream):
        for i in range(5):
            dq.copy_(hq, non_blocking=True)
            run(i, stream, dq)
            ho.copy_(out, non_blocking=True)
        stream.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(K_e2e):
            dq.copy_(hq, non_blocking=True)
            run(i, stream, dq)
            ho.copy_(out, non_blocking=True)
        f1.record(stream)
        stream.synchronize()
    e2e = job_rate(B, K_e2e, world, max_over_ranks(f0.elapsed_time(f1), world, dev))
    cpu = rswa_oracle_baseline(w) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "precision": "fp32 dot products and online softmax, split keys merged in fp32",
                "data": "synthetic", "config": describe(args.workload, world),
                "timing": {"graph": f"CUDA graph replay ({min(K, GRAPH_STEPS)} steps per graph, every graph "
                                    "replayed once before the timed region)",
                           "l2": f"steps rotate over {ncopy} copies of the KV cache ({ncopy * per_copy / 2**20:.0f} MB, "
                                 "above L2)"},
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "traffic": profiled_traffic(args.workload),
                             "peak_kind": peak_kind, "kernel": "one step (rswa_partial_kernel + rswa_combine_kernel)",
                             "algorithmic_bytes_per_step": bytes_step},
                "cpu_baseline": cpu,
                "e2e": {"value": e2e, "unit": UNIT, "h2d_bytes_per_step": int(hq.numel() * 4),
                        "d2h_bytes_per_step": int(ho.numel() * 4), "steps": K_e2e},
                "gpu_launches": 2 * K, "clocks": clk}
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def run_ours(args, rank, world, local_rank):
    import torch
    from weight_quantized_expert_b200 import api, roofline, synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.WORKLOADS[args.workload]
    T = w["T"]
    _, layer = synth.workload(args.workload)
    base = api.focr_moe_pack_weights(layer)
    del layer
    n_copies = max(1, args.copies)
    copies = [base] + [api.focr_moe_layer_clone(base) for _ in range(n_copies - 1)]
    pool_n = 64 if T <= 64 else 16
    if w.get("prefill"):
        # prefill batches: the workload's own 289 rows first, then other seeded 289-row batches
        xs_np = np.stack([synth.prefill_hidden(w["seed"] + 100 * j + rank) for j in range(pool_n)])
    else:
        xs_np = synth.hidden(w["seed"] + 2000 + rank, pool_n * T, skew=w.get("skew", False)).reshape(pool_n, T, 1280)
    xs = torch.from_numpy(xs_np).to(dev)
    outs = torch.empty(pool_n, T, 1280, device=dev)
    ws = api.new_workspace(T, dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i, st=None):
        api.focr_moe_layer_forward(copies[i % n_copies], xs[i % pool_n], outs[i % pool_n], ws, stream=st)

    # experts hit per batch (for the algorithmic bytes): route each pool entry once
    hits = []
    counts = torch.empty(64, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        for j in range(pool_n):
            api.focr_moe_layer_forward(copies[0], xs[j], outs[j], ws, debug={"counts": counts}, stream=stream)
            hits.append(int((counts > 0).sum().item()))
    stream.synchronize()
    step_bytes = [roofline.moe_layer_bytes(T, w["routed"], w["shared"], w["group"], h) for h in hits]

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    stream.synchronize()
    api.focr_moe_check(ws, stream)   # a device error in the warm-up ends the run before the timed steps
    K = args.steps
    if args.eager:
        clocks = Clocks(local_rank)
        clocks.start()
        torch.cuda.synchronize(dev)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for i in range(K):
                step(i, stream)
            ev1.record(stream)
        torch.cuda.synchronize(dev)
        clk = clocks.stop()
        ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
        order = list(range(K))
        graph_note = "eager launches"
    else:
        graphs, order = capture_graphs(step, K, stream)
        ms, clk = timed_replay(graphs, stream, world, dev, local_rank)
        graph_note = (f"CUDA graph replay ({min(K, GRAPH_STEPS)} forwards per graph, every graph replayed once "
                      "before the timed region)")
    avg_bytes = sum(step_bytes[i % pool_n] for i in order) / len(order)
    ms_per_step = ms / K
    value = job_rate(T, K, world, ms)
    peak, tf_burst, tf_sus, peak_kind = peaks()
    achieved = avg_bytes / (ms_per_step / 1e3) / 1e9
    traffic = profiled_traffic(args.workload)
    flops = roofline.moe_layer_flops(T)
    tflops = flops / (ms_per_step / 1e3) / 1e12

    # end to end through the C ABI with host buffers: H2D of x, forward, D2H of out
    K_e2e = min(K, 2000)
    hx = torch.from_numpy(xs_np[:8].copy()).pin_memory()
    hy = torch.empty(8, T, 1280).pin_memory()
    dx = torch.empty(T, 1280, device=dev)
    dy = torch.empty(T, 1280, device=dev)
    with torch.cuda.stream(stream):
        for i in range(20):
            dx.copy_(hx[i % 8], non_blocking=True)
            api.focr_moe_layer_forward(copies[i % n_copies], dx, dy, ws, stream=stream)
            hy[i % 8].copy_(dy, non_blocking=True)
        stream.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K_e2e):
            dx.copy_(hx[i % 8], non_blocking=True)
            api.focr_moe_layer_forward(copies[i % n_copies], dx, dy, ws, stream=stream)
            hy[i % 8].copy_(dy, non_blocking=True)
        e1.record(stream)
        stream.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_rate(T, K_e2e, world, ms_e2e)
    api.focr_moe_check(ws, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(args.workload)
    if rank == 0:
        dtype, prec = precision(T)
        kernel = ("one layer forward: router -> gate/up -> down kernels, chained by programmatic dependent "
                  "launch (timed together)" if T <= 8 else
                  "one layer forward: router -> tensor-core grouped expert kernel (tcgen05, TMEM), chained by "
                  "programmatic dependent launch (timed together)")
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic, "peak_kind": peak_kind, "kernel": kernel,
                "algorithmic_bytes_per_step": avg_bytes,
                "nominal_peak_gbs": 7700.0, "frac_of_nominal": achieved / 7700.0,
                "tensor": {"achieved_tflops": tflops, "algorithmic_flops_per_step": flops,
                           "peak_tflops": tf_sus, "frac": tflops / tf_sus,
                           "peak_note": f"bf16 dense, sustained ({peak_kind}); burst {tf_burst}"}}
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": dtype, "precision": prec, "data": "synthetic",
                "config": describe(args.workload, world),
                "timing": {"graph": graph_note,
                           "l2": f"rotated over {n_copies} packed layer copies "
                                 f"(~{n_copies * base.device_bytes // 2**20} MB; L2 is 126 MB) and {pool_n} "
                                 "distinct token batches"},
                "roofline": roof,
                "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * 1280 * 4,
                        "d2h_bytes_per_step": T * 1280 * 4, "steps": K_e2e},
                "gpu_launches": (3 if T <= 8 else 2) * K,
                "clocks": clk}
        print(json.dumps(line), flush=True)
    del copies


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        from weight_quantized_expert_b200 import synth
        if args.workload in synth.STEP_WORKLOADS and synth.STEP_WORKLOADS[args.workload]["kind"] == "rswa":
            run_rswa_workload(args, rank, world, local_rank)
        elif args.workload in synth.STEP_WORKLOADS:
            run_step_workload(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
