#!/usr/bin/env python
"""Benchmark of the DECO MoE FFN layer forward pass on B200; prints ONE JSON line.

Workload ("edge_decode"): the edge-scale DECO layer -- d_model 2048, 64 routed
non-gated experts of width 256 with NormSiLU, a shared expert of width 1024,
bf16 storage, fp32 accumulation, ~20 % mean activation -- at the decode batch
sizes T = 1, 4 and 16.  One step = one forward pass for each of the three
batches (21 tokens).  Inputs are synthetic and seeded (synth.make_layer).  L2 is
defeated by rotating over enough independent weight copies that every step
reads weights that are not L2 resident.

The step is captured in a CUDA graph per weight copy and replayed.  Timing:
CUDA events on the launching stream around K replays, barrier +
synchronize on both sides, max over ranks.  Several GPUs run independent
replicas (the layer shards by token with no exchange): value = all ranks'
tokens / max time ("weak" scaling).

Extra keys: roofline of the dominant kernel (live CUDA-event kernel times
from an instrumented replay of the same graphs), e2e through the public API
with pinned host buffers, clocks sampled during the run, the CPU oracle as
the baseline, and (rank 0, one GPU) prefill and dense-FFN comparisons.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DECODE_TS = (1, 4, 16)
DECODE_KERNELS = ("route", "up", "down", "combine")   # the decode path's launches per forward
# DRAM bytes (read + write) per launch from an ncu capture of the current decode
# kernels on the edge layer (profiles/decode_kernels_edge_decode_t16.md); a kernel
# changed since its capture has no entry
NCU_DRAM_BYTES = {("route", 16): 5_638_144, ("up", 16): 65_105_152 + 562_432,
                  ("down", 16): 70_251_520 + 1_234_944}
METRIC = "MoE-layer tokens/s (decode)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--profile-tokens", type=int, default=0,
                    help="profiling mode: only run eager forward passes of the edge layer at this "
                         "batch size (warmup + steps), print nothing; for ncu captures")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# --------------------------------------------------------------------------
# ranks: one process per GPU, independent replicas (tokens never interact in
# an FFN layer); the only cross-rank traffic is the barrier and the max of the
# timed durations

def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's duration (every rank calls this, in the same order)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank processed `steps` steps in at most `ms`."""
    return world * tokens_per_step * steps / (ms / 1000.0)


# --------------------------------------------------------------------------
# CPU oracle timing (the baseline arm and cpu_baseline)

def oracle_tokens_per_s(budget_s: float, max_steps: int | None = None):
    """Time the fp64 oracle on whole steps of the decode workload (21 tokens),
    single-threaded, until `budget_s` of CPU work (or max_steps) is done."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle as O
    from synth import CONFIGS, make_layer

    cfg = CONFIGS["edge_decode_t16"]
    L = make_layer(cfg["shape"], cfg["seed"])
    L64 = {k: O.to_f64(v) for k, v in L.items()}
    L64["W_bar_up"] = O.mean_up(L64["W_up"], "bf16")
    x = L64.pop("x")
    steps = tokens = 0
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        while True:
            for T in DECODE_TS:
                O.layer_forward_tokens(x[:T], L64, cfg["shape"].eps)
                tokens += T
            steps += 1
            el = time.perf_counter() - t0
            if el >= budget_s or (max_steps and steps >= max_steps):
                break
    return tokens / el, steps, tokens, el


def run_reference(args, rank, world):
    if rank != 0:
        return
    # each step is one full 21-token step, capped so the run stays within minutes
    per_step = 0.5
    steps = max(1, min(args.steps, int(150 / per_step)))
    for _ in range(min(args.warmup, 1)):
        oracle_tokens_per_s(0.0, max_steps=1)
    v, st, tok, el = oracle_tokens_per_s(1e9, max_steps=steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": st, "warmup": args.warmup, "ms_per_step": 1000 * el / st, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "edge_decode", "T": list(DECODE_TS), "d_model": 2048, "E": 64,
                   "d_e": 256, "d_s": 1024, "storage": "bf16", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{st} steps x 21 tokens of the edge_decode workload, "
                                   "numpy fp64, one thread"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is busy."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return None
        busy = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in busy:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in busy), "sm_max_mhz": busy[0]["smax"],
                "reasons": sorted(reasons), "samples": len(busy)}


def layer_bytes(shape, union_experts: int):
    """Algorithmic HBM bytes per kernel for one decode forward: the weights
    each kernel must read (only the union of active experts) plus x in / out."""
    D, E, d_e, d_s, T = shape.D, shape.E, shape.d_e, shape.d_s, shape.T
    es = 2 if shape.dtype == "bf16" else 4
    return {
        "route": ((E + d_e + d_s) * D + T * D) * es,
        "count": 0,
        "scatter": 0,
        "up": (union_experts * d_e * D + T * D) * es,
        "down": (union_experts * D * d_e + D * d_s) * es,
        "combine": 2 * T * D * es,
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.profile_tokens:
        profile_only(args)
        return

    import numpy as np
    import torch

    import sparse_moe_ffn_relu_b200 as deco
    from synth import CONFIGS, LayerShape, make_layer

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    P = peaks()
    cfg = CONFIGS["edge_decode_t16"]
    base = cfg["shape"]
    Lc = make_layer(base, cfg["seed"])
    x_full = Lc.pop("x")
    G0 = {k: v.to(dev) for k, v in Lc.items()}
    G0["W_bar_up"] = deco.mean_up(G0["W_up"])
    wbytes = sum(t.numel() * t.element_size() for t in G0.values())
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    n_copies = max(2, math.ceil(3 * l2 / wbytes) + 1)
    copies = [G0] + [{k: v.clone() for k, v in G0.items()} for _ in range(n_copies - 1)]

    xs = {T: x_full[:T].to(dev) for T in DECODE_TS}
    outs = {T: torch.empty_like(xs[T]) for T in DECODE_TS}
    shapes = {T: deco.layer_shape(xs[T], G0, base.eps) for T in DECODE_TS}
    wss = {T: deco.alloc_workspace(shapes[T], dev) for T in DECODE_TS}

    def step(G):
        for T in DECODE_TS:
            deco.forward(xs[T], G, out=outs[T], workspace=wss[T], eps=base.eps)

    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for G in copies:
            step(G)
    torch.cuda.synchronize()

    graphs = []
    for G in copies:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(G)
        graphs.append(g)

    # events around every kernel of every forward (eager calls: the library
    # records them with cudaEventRecord between its launches; PDL is off then)
    nk = len(deco.PREFILL_KERNELS)
    ev = {T: [torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)] for T in DECODE_TS}
    for es in ev.values():          # torch creates CUDA events lazily, on first record
        for e in es:
            e.record(stream)
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            graphs[i % n_copies].replay()
        stream.synchronize()
        sampler.start()
        # keep the GPU busy ~1 s before the timed region so clocks settle and are sampled
        t_end = time.perf_counter() + 1.0
        i = 0
        while time.perf_counter() < t_end:
            for _ in range(50):
                graphs[i % n_copies].replay()
                i += 1
            stream.synchronize()
        barrier()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            graphs[i % n_copies].replay()
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
        clocks = sampler.stop()
    ms = max_over_ranks(start.elapsed_time(end), dist, dev)
    tokens_per_step = sum(DECODE_TS)
    value = job_tokens_per_s(world, tokens_per_step, args.steps, ms)

    # live kernel durations: eager forwards on the rotating weight copies
    kt = {T: {k: [] for k in deco.PREFILL_KERNELS} for T in DECODE_TS}
    with torch.cuda.stream(stream):
        for i in range(min(args.steps, 60) + 3):
            G = copies[i % n_copies]
            for T in DECODE_TS:
                deco.set_profiling(ev[T])
                deco.forward(xs[T], G, out=outs[T], workspace=wss[T], eps=base.eps)
                deco.set_profiling(None)
            stream.synchronize()
            if i < 3:
                continue
            for T in DECODE_TS:
                for j, k in enumerate(deco.PREFILL_KERNELS):
                    kt[T][k].append(ev[T][2 * j].elapsed_time(ev[T][2 * j + 1]))
    # routing statistics -> union of active experts per batch
    union, ratio = {}, []
    for T in DECODE_TS:
        rt = deco.routing(xs[T], G0)
        act = rt["active"].bool()
        union[T] = int(act.any(dim=0).sum().item())
        ratio.append(float(act.float().mean().item()))
    bytes_k = {T: layer_bytes(LayerShape(T, base.D, base.E, base.d_e, base.d_s, base.dtype), union[T])
               for T in DECODE_TS}
    mean_ms = {T: {k: statistics.mean(v) for k, v in kt[T].items()} for T in DECODE_TS}
    tot_k = {k: sum(mean_ms[T][k] for T in DECODE_TS) for k in DECODE_KERNELS}
    # the dominant kernel (most time per step), at the largest decode batch
    dom = max(tot_k, key=tot_k.get)
    T_r = max(DECODE_TS)
    dom_bytes = bytes_k[T_r][dom]
    dom_ms = mean_ms[T_r][dom]
    achieved = dom_bytes / (dom_ms / 1000.0) / 1e9
    step_bytes = sum(sum(b.values()) for b in bytes_k.values())
    layer_gbs = step_bytes / (ms / args.steps / 1000.0) / 1e9

    # end to end through the public API: pinned host x -> device -> layer -> host
    xh = {T: xs[T].cpu().pin_memory() for T in DECODE_TS}
    oh = {T: torch.empty_like(xh[T]).pin_memory() for T in DECODE_TS}
    xd = {T: torch.empty_like(xs[T]) for T in DECODE_TS}
    e2e_steps = min(args.steps, 500)
    with torch.cuda.stream(stream):
        def e2e_step(G):
            for T in DECODE_TS:
                xd[T].copy_(xh[T], non_blocking=True)
                deco.forward(xd[T], G, out=outs[T], workspace=wss[T], eps=base.eps)
                oh[T].copy_(outs[T], non_blocking=True)
        for i in range(max(3, args.warmup)):
            e2e_step(copies[i % n_copies])
        barrier()
        torch.cuda.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for i in range(e2e_steps):
            e2e_step(copies[i % n_copies])
        e2.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms2 = max_over_ranks(s2.elapsed_time(e2), dist, dev)
    e2e_value = job_tokens_per_s(world, tokens_per_step, e2e_steps, ms2)
    io_bytes = sum(T * base.D * 2 for T in DECODE_TS)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "edge_decode", "T": list(DECODE_TS), "d_model": base.D, "E": base.E,
                   "d_e": base.d_e, "d_s": base.d_s, "storage": "bf16", "accumulate": "fp32",
                   "mean_activation": round(statistics.mean(ratio), 4),
                   "union_experts": {str(T): union[T] for T in DECODE_TS},
                   "l2": f"rotating {n_copies} weight copies ({wbytes / 1e6:.0f} MB each) > 3x L2",
                   "cuda_graph": True, "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": dom, "T": T_r, "achieved": achieved, "peak": P["hbm"],
                     "unit": "GB/s", "frac": achieved / P["hbm"], "traffic": NCU_DRAM_BYTES.get((dom, T_r)),
                     "algorithmic_bytes": dom_bytes,
                     "peak_source": P["src"], "layer_achieved_gbs": layer_gbs,
                     "layer_frac": layer_gbs / P["hbm"],
                     "kernel_ms_by_T": {str(T): {k: round(mean_ms[T][k], 4) for k in DECODE_KERNELS}
                                        for T in DECODE_TS}},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
                "d2h_bytes_per_step": io_bytes},
        "gpu_launches": args.steps * len(DECODE_TS) * len(DECODE_KERNELS),
        "clocks": clocks,
    }
    if rank == 0 and world == 1:
        v, st, tok, el = oracle_tokens_per_s(12.0)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{st} steps ({tok} tokens) of the edge_decode workload, "
                                          f"{el:.1f} s, numpy fp64, one thread"}
        if not args.no_extras:
            line["extras"] = extras(deco, dev, stream, P)
    if rank == 0:
        print(json.dumps(line), flush=True)
    for g in graphs:
        del g
    if dist is not None:
        dist.destroy_process_group()


def profile_only(args):
    """Eager forward passes of the edge layer at one batch size, for ncu:
    warmup forwards first, then `steps` more.  Kernels in launch order:
    kd_route, kd_up, kd_down, kd_combine (T <= 16); k_router, k_router_exact,
    k_tab_count, k_tab_scatter, kp_gemm<0..3>, k_combine (T > 16)."""
    import torch

    import sparse_moe_ffn_relu_b200 as deco
    from synth import CONFIGS, LayerShape, make_layer
    base = CONFIGS["edge_decode_t16"]["shape"]
    shape = LayerShape(args.profile_tokens, base.D, base.E, base.d_e, base.d_s, base.dtype)
    L = make_layer(shape, CONFIGS["edge_decode_t16"]["seed"])
    G = {k: v.cuda() for k, v in L.items()}
    G["W_bar_up"] = deco.mean_up(G["W_up"])
    ws = deco.alloc_workspace(deco.layer_shape(G["x"], G))
    out = torch.empty_like(G["x"])
    for _ in range(args.warmup + args.steps):
        deco.forward(G["x"], G, out=out, workspace=ws)
    torch.cuda.synchronize()


def extras(deco, dev, stream, P):
    """Prefill (T=4096) and dense-FFN comparisons on one GPU."""
    import torch

    from synth import CONFIGS, make_dense, make_layer
    out = {}
    cfg = CONFIGS["edge_prefill_t4096"]
    shape = cfg["shape"]
    L = make_layer(shape, cfg["seed"], jitter=cfg["jitter"], zero_every=cfg["zero_every"])
    G = {k: v.to(dev) for k, v in L.items()}
    G["W_bar_up"] = deco.mean_up(G["W_up"])
    ws = deco.alloc_workspace(deco.layer_shape(G["x"], G), dev)
    o = torch.empty_like(G["x"])

    def timeit(fn, n=10):
        with torch.cuda.stream(stream):
            for _ in range(2):
                fn()
            torch.cuda.synchronize()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            for _ in range(n):
                fn()
            e.record(stream)
            torch.cuda.synchronize()
        return s.elapsed_time(e) / n

    ms = timeit(lambda: deco.forward(G["x"], G, out=o, workspace=ws))
    act = deco.routing(G["x"], G)["active"].bool()
    n_t = act.sum(dim=1).double()
    D, E, de, ds = shape.D, shape.E, shape.d_e, shape.d_s
    flops = float((2 * D * E + 2 * D * de + n_t * 4 * D * de + 4 * D * ds).sum())
    # per-kernel device time, eager calls with events between the kernels
    names = deco.PREFILL_KERNELS
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
    kt = {k: [] for k in names}
    with torch.cuda.stream(stream):
        for e in ev:
            e.record(stream)
        deco.set_profiling(ev)
        for _ in range(6):
            deco.forward(G["x"], G, out=o, workspace=ws)
            stream.synchronize()
            for j, k in enumerate(names):
                kt[k].append(ev[2 * j].elapsed_time(ev[2 * j + 1]))
        deco.set_profiling(None)
    kms = {k: statistics.mean(v[1:]) for k, v in kt.items()}
    pairs = float(n_t.sum())
    kflops = {"route": 2.0 * shape.T * D * E, "proj": 2.0 * shape.T * D * (de + ds), "up": 2.0 * pairs * D * de,
              "down": 2.0 * pairs * de * D, "shared": 2.0 * shape.T * ds * D}
    dom = max(kflops, key=lambda k: kms[k])
    dom_tf = kflops[dom] / (kms[dom] / 1e3) / 1e12
    out["prefill_t4096"] = {"ms": ms, "tokens_per_s": shape.T / (ms / 1e3),
                            "roofline": {"bound": "tensor", "kernel": dom, "achieved": round(dom_tf, 1),
                                         "peak": P["bf16"], "unit": "TFLOP/s",
                                         "frac": round(dom_tf / P["bf16"], 4), "peak_source": P["src"]},
                            "tflops": flops / (ms / 1e3) / 1e12,
                            "frac_bf16_peak": flops / (ms / 1e3) / 1e12 / P["bf16"],
                            "mean_activation": float(act.float().mean()),
                            "kernel_ms": {k: round(v, 4) for k, v in kms.items()},
                            "kernel_tflops": {k: round(f / (kms[k] / 1e3) / 1e12, 1)
                                              for k, f in kflops.items()}}
    d_ff = ds + E * de
    for T in (16, 4096):
        Dn = make_dense(T, D, d_ff, "bf16", 7)
        x, W1, W2 = Dn["x"].to(dev), Dn["W1"].to(dev), Dn["W2"].to(dev)
        od = torch.empty_like(x)
        wsd = torch.empty(deco.dense_workspace_size(T, D, d_ff, x.dtype), dtype=torch.uint8, device=dev)
        dms = timeit(lambda: deco.dense_ffn(x, W1, W2, out=od, workspace=wsd))
        xs_ = G["x"][:T]
        os_ = torch.empty_like(xs_)
        ws_ = deco.alloc_workspace(deco.layer_shape(xs_, G), dev)
        sms = timeit(lambda: deco.forward(xs_, G, out=os_, workspace=ws_))
        out[f"dense_vs_sparse_t{T}"] = {"dense_ms": dms, "sparse_ms": sms, "speedup": dms / sms}
        del W1, W2
    return out


if __name__ == "__main__":
    main()
