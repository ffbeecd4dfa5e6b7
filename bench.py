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
from eager forwards on the rotating copies), e2e through the public API with
pinned host buffers, clocks sampled during the run, the CPU oracle as the
baseline (one thread, and all host cores), and (rank 0, one GPU) prefill,
the activation-ratio sweep against the equal-parameter dense FFN, TopK vs
ReLU routing, and the 8-layer d_model-4096 stack.

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
METRIC = "MoE-layer tokens/s (decode)"
# DRAM bytes (read + write) per launch of the decode kernel at T = 16 from an
# ncu capture of the current kernel (None until one is taken; a kernel changed
# since its capture has no entry): kd_layer, edge layer, T = 16, 139.93 MB read
# + 7.39 MB written, from `ncu --set full` of `bench.py --profile-tokens 16`
NCU_DRAM_BYTES = {("layer", 16): 147_320_576}


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
    ap.add_argument("--profile-dense", action="store_true",
                    help="with --profile-tokens: the equal-parameter dense FFN instead")
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

def _oracle_layer():
    import oracle as O
    from synth import CONFIGS, make_layer
    cfg = CONFIGS["edge_decode_t16"]
    L = make_layer(cfg["shape"], cfg["seed"])
    L64 = {k: O.to_f64(v) for k, v in L.items()}
    L64["W_bar_up"] = O.mean_up(L64["W_up"], "bf16")
    x = L64.pop("x")
    return x, L64, cfg["shape"].eps


def oracle_tokens_per_s(budget_s: float, max_steps: int | None = None):
    """Time the fp64 oracle on whole steps of the decode workload (21 tokens),
    single-threaded, until `budget_s` of CPU work (or max_steps) is done."""
    from threadpoolctl import threadpool_limits

    import oracle as O
    x, L64, eps = _oracle_layer()
    steps = tokens = 0
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        while True:
            for T in DECODE_TS:
                O.layer_forward_tokens(x[:T], L64, eps)
                tokens += T
            steps += 1
            el = time.perf_counter() - t0
            if el >= budget_s or (max_steps and steps >= max_steps):
                break
    return tokens / el, steps, tokens, el


_POOL_LAYER = None


def _pool_init():
    from threadpoolctl import threadpool_limits
    threadpool_limits(limits=1)


def _pool_tokens(args):
    import oracle as O
    x, L64, eps = _POOL_LAYER
    toks, reps = args
    for _ in range(reps):
        O.layer_forward_tokens(x, L64, eps, toks)
    return len(toks) * reps


def oracle_all_cores(budget_s: float = 10.0):
    """The same oracle on every host core: worker processes (forked before any
    CUDA call, sharing the fp64 layer copy-on-write) each evaluate tokens of
    the T = 16 batch, one thread each.  Returns tokens/s, workers, sample."""
    import multiprocessing as mp
    global _POOL_LAYER
    _POOL_LAYER = _oracle_layer()
    n = max(1, min(os.cpu_count() or 1, 64))
    # calibrate: one token's cost on one core
    import oracle as O
    x, L64, eps = _POOL_LAYER
    t0 = time.perf_counter()
    O.layer_forward_tokens(x, L64, eps, [0])
    per_tok = max(time.perf_counter() - t0, 1e-3)
    reps = max(1, int(budget_s / per_tok / 16))
    work = [([i % 16 for i in range(w, w + 16)], reps) for w in range(n)]
    ctx = mp.get_context("fork")
    with ctx.Pool(n, initializer=_pool_init) as pool:
        pool.map(_pool_tokens, [([0], 1)] * n)          # warm the workers
        t0 = time.perf_counter()
        done = sum(pool.map(_pool_tokens, work))
        el = time.perf_counter() - t0
    _POOL_LAYER = None
    return done / el, n, f"{n} processes x {reps} x 16 tokens of the edge_decode layer, {el:.1f} s"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


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


def layer_bytes(T, D, E, d_e, d_s, union_experts: int, es: int = 2) -> int:
    """Algorithmic HBM bytes of one decode forward: every weight it must read
    (W_r, W_bar_up, W_s_up, W_s_down, and W_up / W_down of the union of the
    batch's active experts only), x in and out, b_r and s."""
    return (((E + d_e + d_s) * D + union_experts * 2 * d_e * D + D * d_s + 2 * T * D) * es
            + 8 * E)


def dense_bytes(T, D, d_ff, es: int = 2) -> int:
    return (2 * d_ff * D + 2 * T * D) * es


def layer_flops(n_t, D, E, d_e, d_s) -> float:
    """Algorithmic FLOPs of a prefill forward: router, mean and shared
    up-projections for every token, routed up and down per active pair, the
    shared down-projection (no padding counted)."""
    T = len(n_t)
    return float(T * (2 * D * E + 2 * D * d_e + 4 * D * d_s) + 4 * D * d_e * sum(n_t))


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
    # the all-core oracle timing forks worker processes: before any CUDA call
    cpu_all = None
    if rank == 0 and world == 1 and not args.no_extras:
        cpu_all = oracle_all_cores()

    import torch

    import sparse_moe_ffn_relu_b200 as deco
    from synth import CONFIGS, make_layer

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

    # live kernel durations: eager forwards on the rotating weight copies; the
    # decode path is one kernel (timing slot "layer")
    names = deco.ALL_SLOTS
    ev = {T: [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))] for T in DECODE_TS}
    with torch.cuda.stream(stream):
        for es in ev.values():          # torch creates CUDA events lazily, on first record
            for e in es:
                e.record(stream)
    torch.cuda.synchronize()
    kt = {T: [] for T in DECODE_TS}
    slot = names.index("layer")
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
                kt[T].append(ev[T][2 * slot].elapsed_time(ev[T][2 * slot + 1]))
    # routing statistics -> union of active experts per batch
    union, ratio, per_tok = {}, [], []
    for T in DECODE_TS:
        rt = deco.routing(xs[T], G0)
        act = rt["active"].bool()
        union[T] = int(act.any(dim=0).sum().item())
        ratio.append(float(act.float().mean().item()))
        per_tok += act.float().mean(dim=1).tolist()
    D, E, d_e, d_s = base.D, base.E, base.d_e, base.d_s
    bytes_T = {T: layer_bytes(T, D, E, d_e, d_s, union[T]) for T in DECODE_TS}
    kms = {T: statistics.mean(kt[T]) for T in DECODE_TS}
    T_r = max(DECODE_TS)
    achieved = bytes_T[T_r] / (kms[T_r] / 1000.0) / 1e9
    step_bytes = sum(bytes_T.values())
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
        "config": {"workload": "edge_decode", "T": list(DECODE_TS), "d_model": D, "E": E,
                   "d_e": d_e, "d_s": d_s, "storage": "bf16", "accumulate": "fp32",
                   "mean_activation": round(statistics.mean(ratio), 4),
                   "min_token_activation": round(min(per_tok), 4),
                   "max_token_activation": round(max(per_tok), 4),
                   "zero_expert_tokens": int(sum(1 for v in per_tok if v == 0.0)),
                   "union_experts": {str(T): union[T] for T in DECODE_TS},
                   "l2": f"rotating {n_copies} weight copies ({wbytes / 1e6:.0f} MB each) > 3x L2",
                   "cuda_graph": True, "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": "kd_layer", "T": T_r, "achieved": achieved, "peak": P["hbm"],
                     "unit": "GB/s", "frac": achieved / P["hbm"], "traffic": NCU_DRAM_BYTES.get(("layer", T_r)),
                     "traffic_source": "ncu capture of this kernel (dram__bytes_read.sum + dram__bytes_write.sum), "
                                       "not measured in this run",
                     "algorithmic_bytes": bytes_T[T_r],
                     "peak_source": P["src"], "layer_achieved_gbs": layer_gbs,
                     "layer_frac": layer_gbs / P["hbm"],
                     "kernel_us_by_T": {str(T): round(1000 * kms[T], 2) for T in DECODE_TS},
                     "frac_by_T": {str(T): round(bytes_T[T] / (kms[T] / 1e3) / 1e9 / P["hbm"], 4)
                                   for T in DECODE_TS}},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
                "d2h_bytes_per_step": io_bytes},
        "gpu_launches": args.steps * len(DECODE_TS),
        "clocks": clocks,
    }
    if rank == 0 and world == 1:
        v, st, tok, el = oracle_tokens_per_s(12.0)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{st} steps ({tok} tokens) of the edge_decode workload, "
                                          f"{el:.1f} s, numpy fp64, one thread"}
        if cpu_all is not None:
            line["cpu_baseline_all_cores"] = {"value": cpu_all[0], "unit": "tokens/s", "cores": cpu_all[1],
                                              "kind": "oracle", "cpu": cpu_model(), "sample": cpu_all[2]}
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
    kd_layer (T <= 16); k_router, k_router_exact, k_tab_count, k_tab_scan,
    k_tab_scatter, kp_gemm<0..3>, k_combine (T > 16).  --profile-dense: the
    dense FFN."""
    import torch

    import sparse_moe_ffn_relu_b200 as deco
    from synth import CONFIGS, LayerShape, make_dense, make_layer
    base = CONFIGS["edge_decode_t16"]["shape"]
    if args.profile_dense:
        Dn = make_dense(args.profile_tokens, base.D, base.d_s + base.E * base.d_e, "bf16", 7)
        x, W1, W2 = Dn["x"].cuda(), Dn["W1"].cuda(), Dn["W2"].cuda()
        out = torch.empty_like(x)
        for _ in range(args.warmup + args.steps):
            deco.dense_ffn(x, W1, W2, out=out)
        torch.cuda.synchronize()
        return
    shape = LayerShape(args.profile_tokens, base.D, base.E, base.d_e, base.d_s, base.dtype)
    L = make_layer(shape, CONFIGS["edge_decode_t16"]["seed"])
    G = {k: v.cuda() for k, v in L.items()}
    G["W_bar_up"] = deco.mean_up(G["W_up"])
    ws = deco.alloc_workspace(deco.layer_shape(G["x"], G))
    out = torch.empty_like(G["x"])
    for _ in range(args.warmup + args.steps):
        deco.forward(G["x"], G, out=out, workspace=ws)
    torch.cuda.synchronize()


# --------------------------------------------------------------------------
# extras (rank 0, one GPU)

def _time_graphs(torch, stream, fns, reps=100):
    """Mean ms of one call of each fn in `fns` (one per weight copy), captured
    in CUDA graphs and replayed in rotation, so consecutive calls read
    different copies."""
    graphs = []
    with torch.cuda.stream(stream):
        for fn in fns:
            fn()
        torch.cuda.synchronize()
        for fn in fns:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            graphs.append(g)
        for i in range(3 * len(graphs)):
            graphs[i % len(graphs)].replay()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for i in range(reps):
            graphs[i % len(graphs)].replay()
        e.record(stream)
        torch.cuda.synchronize()
    for g in graphs:
        del g
    return s.elapsed_time(e) / reps


def _time_eager(torch, stream, fn, n=10):
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


def _copies(torch, G, n):
    return [G] + [{k: v.clone() for k, v in G.items()} for _ in range(n - 1)]


def extras(deco, dev, stream, P):
    import torch
    out = {}
    for name, fn in (("prefill_t4096", extra_prefill), ("ratio_sweep", extra_sweep),
                     ("topk_vs_relu", extra_topk), ("stack_8_layers_d4096", extra_stack),
                     ("experts_on_host", extra_host_experts), ("backward", extra_backward)):
        try:   # one failing extra is reported in its own entry, not in place of the bench line
            out[name] = fn(deco, dev, stream, P, torch)
        except Exception as exc:   # noqa: BLE001
            out[name] = {"error": f"{type(exc).__name__}: {exc}"}
            try:
                torch.cuda.synchronize()
                torch.cuda.empty_cache()
            except Exception:   # noqa: BLE001
                pass
    out["context"] = ("the pages report model-level decode speedups of DECO's kernel over dense "
                      "inference of 3.00x (Jetson AGX Orin) and 2.58x (RTX 4090), through FR-Spec on "
                      "Spec-Bench; other hardware and a whole model, not this layer")
    return out


def extra_prefill(deco, dev, stream, P, torch):
    """Config 3: the edge layer at T = 4096 with per-token activation jitter."""
    from synth import CONFIGS, make_layer
    cfg = CONFIGS["edge_prefill_t4096"]
    shape = cfg["shape"]
    L = make_layer(shape, cfg["seed"], jitter=cfg["jitter"], zero_every=cfg["zero_every"])
    G = {k: v.to(dev) for k, v in L.items()}
    G["W_bar_up"] = deco.mean_up(G["W_up"])
    ws = deco.alloc_workspace(deco.layer_shape(G["x"], G), dev)
    o = torch.empty_like(G["x"])
    ms = _time_eager(torch, stream, lambda: deco.forward(G["x"], G, out=o, workspace=ws))
    act = deco.routing(G["x"], G)["active"].bool()
    n_t = act.sum(dim=1).tolist()
    D, E, de, ds = shape.D, shape.E, shape.d_e, shape.d_s
    flops = layer_flops(n_t, D, E, de, ds)
    # per-kernel device time, eager calls with events between the kernels
    names = deco.ALL_SLOTS
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
    kt = {k: [] for k in deco.PREFILL_KERNELS}
    with torch.cuda.stream(stream):
        for e in ev:
            e.record(stream)
        deco.set_profiling(ev)
        for _ in range(6):
            deco.forward(G["x"], G, out=o, workspace=ws)
            stream.synchronize()
            for j, k in enumerate(deco.PREFILL_KERNELS):
                kt[k].append(ev[2 * j].elapsed_time(ev[2 * j + 1]))
        deco.set_profiling(None)
    kms = {k: statistics.mean(v[1:]) for k, v in kt.items()}
    pairs = float(sum(n_t))
    kflops = {"route": 2.0 * shape.T * D * E, "proj": 2.0 * shape.T * D * (de + ds), "up": 2.0 * pairs * D * de,
              "down": 2.0 * pairs * de * D, "shared": 2.0 * shape.T * ds * D}
    dom = max(kflops, key=lambda k: kms[k])
    dom_tf = kflops[dom] / (kms[dom] / 1e3) / 1e12
    per_tok = act.float().mean(dim=1)
    return {"ms": ms, "tokens_per_s": shape.T / (ms / 1e3),
            "roofline": {"bound": "tensor", "kernel": dom, "achieved": round(dom_tf, 1),
                         "peak": P["bf16"], "unit": "TFLOP/s",
                         "frac": round(dom_tf / P["bf16"], 4), "peak_source": P["src"]},
            "tflops": flops / (ms / 1e3) / 1e12,
            "frac_bf16_peak": flops / (ms / 1e3) / 1e12 / P["bf16"],
            "mean_activation": float(per_tok.mean()), "min_token_activation": float(per_tok.min()),
            "max_token_activation": float(per_tok.max()),
            "zero_expert_tokens": int((per_tok == 0).sum()),
            "kernel_ms": {k: round(v, 4) for k, v in kms.items()},
            "kernel_tflops": {k: round(f / (kms[k] / 1e3) / 1e12, 1) for k, f in kflops.items()}}


def extra_sweep(deco, dev, stream, P, torch):
    """Config 5: the edge layer at 5/10/20/40/100 % mean activation, T = 1, 4,
    16 (CUDA graphs over rotating weight copies, L2 defeated) and T = 4096
    (eager), each next to the equal-parameter dense FFN (d_ff = d_s + E d_e)."""
    from synth import CONFIGS, LayerShape, make_dense, make_layer
    base = CONFIGS["edge_decode_t16"]["shape"]
    D, E, de, ds = base.D, base.E, base.d_e, base.d_s
    d_ff = ds + E * de
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    res = {"d_ff": d_ff, "dense": {}, "sparse": {}}
    # dense FFN
    Dn = make_dense(4096, D, d_ff, "bf16", 7)
    W = {"W1": Dn["W1"].to(dev), "W2": Dn["W2"].to(dev)}
    nd = max(2, math.ceil(3 * l2 / (2 * d_ff * D * 2)) + 1)
    Wc = _copies(torch, W, nd)
    xd_all = Dn["x"].to(dev)
    for T in (1, 4, 16, 4096):
        x = xd_all[:T]
        o = torch.empty_like(x)
        wsd = torch.empty(deco.dense_workspace_size(T, D, d_ff, x.dtype), dtype=torch.uint8, device=dev)
        if T <= 16:
            ms = _time_graphs(torch, stream, [lambda c=c: deco.dense_ffn(x, c["W1"], c["W2"], out=o, workspace=wsd)
                                              for c in Wc])
            res["dense"][str(T)] = {"us": round(1000 * ms, 2),
                                    "hbm_frac": round(dense_bytes(T, D, d_ff) / (ms / 1e3) / 1e9 / P["hbm"], 4)}
        else:
            ms = _time_eager(torch, stream, lambda: deco.dense_ffn(x, W["W1"], W["W2"], out=o, workspace=wsd))
            tf = 4.0 * T * D * d_ff / (ms / 1e3) / 1e12
            res["dense"][str(T)] = {"us": round(1000 * ms, 2), "tflops": round(tf, 1),
                                    "tensor_frac": round(tf / P["bf16"], 4)}
    del Wc, W
    torch.cuda.empty_cache()
    for ratio in (0.05, 0.1, 0.2, 0.4, 1.0):
        shape = LayerShape(4096, D, E, de, ds, "bf16")
        L = make_layer(shape, 1, ratio=ratio)
        x_all = L.pop("x").to(dev)
        G = {k: v.to(dev) for k, v in L.items()}
        G["W_bar_up"] = deco.mean_up(G["W_up"])
        wb = sum(t.numel() * t.element_size() for t in G.values())
        Gc = _copies(torch, G, max(2, math.ceil(3 * l2 / wb) + 1))
        row = {}
        for T in (1, 4, 16, 4096):
            x = x_all[:T]
            o = torch.empty_like(x)
            ws = deco.alloc_workspace(deco.layer_shape(x, G), dev)
            act = deco.routing(x, G)["active"].bool()
            if T <= 16:
                ms = _time_graphs(torch, stream, [lambda c=c: deco.forward(x, c, out=o, workspace=ws) for c in Gc])
                nb = layer_bytes(T, D, E, de, ds, int(act.any(dim=0).sum()))
                row[str(T)] = {"us": round(1000 * ms, 2), "hbm_frac": round(nb / (ms / 1e3) / 1e9 / P["hbm"], 4),
                               "activation": round(float(act.float().mean()), 4),
                               "speedup_vs_dense": round(res["dense"][str(T)]["us"] / (1000 * ms), 3)}
            else:
                ms = _time_eager(torch, stream, lambda: deco.forward(x, G, out=o, workspace=ws))
                tf = layer_flops(act.sum(dim=1).tolist(), D, E, de, ds) / (ms / 1e3) / 1e12
                row[str(T)] = {"us": round(1000 * ms, 2), "tflops": round(tf, 1),
                               "tensor_frac": round(tf / P["bf16"], 4),
                               "activation": round(float(act.float().mean()), 4),
                               "speedup_vs_dense": round(res["dense"][str(T)]["us"] / (1000 * ms), 3)}
            del ws
        res["sparse"][f"{int(round(100 * ratio))}%"] = row
        del Gc, G
        torch.cuda.empty_cache()
    return res


def extra_topk(deco, dev, stream, P, torch):
    """TopK routing at k = round(0.2 E) against DECO's ReLU routing at ~20 %
    on the edge layer (the paper's §5 comparison), T = 1, 16 (graphs over
    rotating copies) and 4096 (eager)."""
    from synth import CONFIGS, LayerShape, make_layer
    base = CONFIGS["edge_decode_t16"]["shape"]
    D, E, de, ds = base.D, base.E, base.d_e, base.d_s
    k = int(round(0.2 * E))
    shape = LayerShape(4096, D, E, de, ds, "bf16")
    L = make_layer(shape, 1)
    x_all = L.pop("x").to(dev)
    G = {kk: v.to(dev) for kk, v in L.items()}
    G["W_bar_up"] = deco.mean_up(G["W_up"])
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    wb = sum(t.numel() * t.element_size() for t in G.values())
    Gc = _copies(torch, G, max(2, math.ceil(3 * l2 / wb) + 1))
    res = {"k": k}
    for T in (1, 16, 4096):
        x = x_all[:T]
        o = torch.empty_like(x)
        row = {}
        for name, tk in (("relu", 0), ("topk", k)):
            ws = deco.alloc_workspace(deco.layer_shape(x, G, topk=tk), dev)
            if T <= 16:
                ms = _time_graphs(torch, stream,
                                  [lambda c=c: deco.forward(x, c, out=o, workspace=ws, topk=tk) for c in Gc])
            else:
                ms = _time_eager(torch, stream, lambda: deco.forward(x, G, out=o, workspace=ws, topk=tk))
            act = deco.routing(x, G, topk=tk)["active"].bool()
            row[name] = {"us": round(1000 * ms, 2), "activation": round(float(act.float().mean()), 4),
                         "union_experts": int(act.any(dim=0).sum())}
        res[str(T)] = row
    del Gc, G
    torch.cuda.empty_cache()
    return res


def extra_host_experts(deco, dev, stream, P, torch):
    """The edge layer with its routed experts' W_up and W_down in pinned host
    memory (the offloaded-parameter setting of the paper's §1): only the
    activated experts' rows cross the host link.  T = 1, 4, 16 at ~20 %
    activation and T = 1 with every expert active, eager; the rate is the
    activated experts' bytes over the time."""
    from synth import CONFIGS, make_layer
    base = CONFIGS["edge_decode_t16"]["shape"]
    per_expert = 2 * base.d_e * base.D * 2   # W_up[e] and W_down[e], bf16
    res = {"note": "general kernels; x, router, mean and shared expert in HBM"}
    for label, ratio, Ts in (("20%", 0.2, (1, 4, 16)), ("100%", 1.0, (1,))):
        L = make_layer(base, CONFIGS["edge_decode_t16"]["seed"], ratio=ratio)
        x_all = L.pop("x").to(dev)
        G = {k: v.to(dev) for k, v in L.items()}
        G["W_bar_up"] = deco.mean_up(G["W_up"])
        H = dict(G)
        H["W_up"], H["W_down"] = G["W_up"].cpu().pin_memory(), G["W_down"].cpu().pin_memory()
        row = {}
        for T in Ts:
            x = x_all[:T]
            o = torch.empty_like(x)
            ws = deco.alloc_workspace(deco.layer_shape(x, H), dev)
            ms = _time_eager(torch, stream, lambda: deco.forward(x, H, out=o, workspace=ws), n=5)
            union = int(deco.routing(x, G)["active"].bool().any(dim=0).sum())
            row[str(T)] = {"us": round(1000 * ms, 1), "union_experts": union,
                           "host_link_gbs": round(union * per_expert / (ms / 1e3) / 1e9, 1)}
        res[label] = row
        del H, G
    torch.cuda.empty_cache()
    return res


def extra_backward(deco, dev, stream, P, torch):
    """The layer's backward pass (CUDA-core kernels, fixed-order sums) on the
    edge layer at T = 1, 16 and 256, eager.  Bytes: the weights it reads once
    (router, mean, shared, the union's W_up and W_down) plus the fp32
    gradients it writes (every weight's); the rate is against HBM."""
    from synth import CONFIGS, LayerShape, make_layer
    base = CONFIGS["edge_decode_t16"]["shape"]
    D, E, de, ds = base.D, base.E, base.d_e, base.d_s
    res = {"note": "first version: CUDA cores, fixed-order sums"}
    shape = LayerShape(256, D, E, de, ds, "bf16")
    L = make_layer(shape, CONFIGS["edge_decode_t16"]["seed"])
    x_all = L.pop("x").to(dev)
    G = {k: v.to(dev) for k, v in L.items()}
    G["W_bar_up"] = deco.mean_up(G["W_up"])
    grad_bytes = 4 * sum(t.numel() for k, t in G.items() if k != "W_bar_up")
    for T in (1, 16, 256):
        x = x_all[:T]
        dy = torch.randn(T, D, device=dev).to(torch.bfloat16)
        union = int(deco.routing(x, G)["active"].bool().any(dim=0).sum())
        wbytes = 2 * (D * (E + de + ds) + D * ds + union * 2 * de * D)
        ms = _time_eager(torch, stream, lambda: deco.backward(x, G, dy), n=5)
        gbs = (wbytes + grad_bytes + T * D * 4) / (ms / 1e3) / 1e9
        res[str(T)] = {"ms": round(ms, 3), "union_experts": union, "gbs": round(gbs, 1),
                       "hbm_frac": round(gbs / P["hbm"], 4) if "hbm" in P else None}
    del G
    torch.cuda.empty_cache()
    return res


def extra_stack(deco, dev, stream, P, torch):
    """Config 4: 8 stacked layers (d_model 4096, 128 routed experts of width
    256, shared width 2048, bf16, ~20 %), residual adds, T = 16 (decode
    kernel; the 4.6 GB of weights exceed L2) and T = 16384 (tensor-core
    kernels); tokens/s of the stack and per layer."""
    from synth import CONFIGS, make_layer
    base = CONFIGS["large_t16384"]["shape"]
    D, E, de, ds = base.D, base.E, base.d_e, base.d_s
    layers = []
    for l in range(8):
        L = make_layer(base, 3, layer=l, with_x=(l == 0))
        x0 = L.pop("x") if l == 0 else None
        G = {k: v.to(dev) for k, v in L.items()}
        G["W_bar_up"] = deco.mean_up(G["W_up"])
        layers.append(G)
        if l == 0:
            x_all = x0.to(dev)
        del L
    res = {}
    for T in (16, 16384):
        x = x_all[:T].contiguous()
        bufs = [torch.empty_like(x), torch.empty_like(x)]
        ws = deco.alloc_workspace(deco.layer_shape(x, layers[0], residual=True), dev)

        def stack():
            cur = x
            for i, G in enumerate(layers):
                nxt = bufs[i & 1]
                deco.forward(cur, G, out=nxt, workspace=ws, eps=base.eps, residual=True)
                cur = nxt
        if T <= 16:
            ms = _time_graphs(torch, stream, [stack], reps=50)
            acts = []
            cur = x
            for i, G in enumerate(layers):
                acts.append(deco.routing(cur, G)["active"].bool())
                nxt = torch.empty_like(x)
                deco.forward(cur, G, out=nxt, eps=base.eps, residual=True)
                cur = nxt
            nb = sum(layer_bytes(T, D, E, de, ds, int(a.any(dim=0).sum())) for a in acts)
            res[str(T)] = {"ms": round(ms, 4), "tokens_per_s": T / (ms / 1e3),
                           "hbm_frac": round(nb / (ms / 1e3) / 1e9 / P["hbm"], 4),
                           "mean_activation": round(float(torch.stack(acts).float().mean()), 4)}
        else:
            ms = _time_eager(torch, stream, stack, n=3)
            flops = 0.0
            cur = x
            acts = []
            for G in layers:
                a = deco.routing(cur, G)["active"].bool()
                acts.append(float(a.float().mean()))
                flops += layer_flops(a.sum(dim=1).tolist(), D, E, de, ds)
                nxt = torch.empty_like(x)
                deco.forward(cur, G, out=nxt, workspace=ws, eps=base.eps, residual=True)
                cur = nxt
                del a
            tf = flops / (ms / 1e3) / 1e12
            res[str(T)] = {"ms": round(ms, 3), "tokens_per_s": T / (ms / 1e3), "tflops": round(tf, 1),
                           "tensor_frac": round(tf / P["bf16"], 4),
                           "mean_activation": round(statistics.mean(acts), 4)}
        del ws
        torch.cuda.empty_cache()
    del layers
    torch.cuda.empty_cache()
    return res


if __name__ == "__main__":
    main()
