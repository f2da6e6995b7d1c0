#!/usr/bin/env python
"""Throughput of the NVFP4 W4A16 MoE FFN layer forward (libtfmoe) on B200.

Default workload (N=1): the decode layer shape -- H=2048, I=768, E=128, top-8,
T=8 tokens per forward -- three seeded layers (seeds 1, 2, 3) rotated so that
consecutive forwards read different weights (each forward touches ~137 MB; a
layer is re-read only after two other layers' ~274 MB, which exceeds the
126 MB L2). A step is one forward of the whole layer (router, top-k, permute,
gate/up + SwiGLU, down, combine) over one batch; eight distinct seeded
activation batches rotate per layer. Forwards are replayed from CUDA graphs of
up to 100 consecutive forwards.

Printed JSON line (rank 0): value = tokens/s over all ranks, e2e = the same
metric through tfmoe_forward_host with pinned host buffers (copies inside the
timed region), roofline of the dominant kernel measured live with CUDA events,
cpu_baseline = the fp64 oracle on a bounded sample on this host's cores.

--impl reference times the fp64 CPU oracle (the only reference this layer has)
on the same workload, one token per step.

Multi-GPU (torchrun): replicas only -- every rank runs its own layers on its
own GPU with no data-path collective (weak scaling); the timed region is
bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "NVFP4 MoE layer tok/s; decode HBM GB/s, prefill TFLOP/s vs B200 peak"
NVFP4_BYTES_PER_WEIGHT = 0.5625        # 4-bit code + one E4M3 byte per 16 weights
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

WORKLOADS = {
    # name: (layer shape index, tokens per forward, seeds)
    "decode": (1, 8, (1, 2, 3)),
    "decode_t1": (1, 1, (1, 2, 3)),
    "tiny": (0, 4, (0,)),
    "zipf": (2, 256, (4,)),
    "prefill": (3, 8192, (5,)),
    "sweep_t1": (4, 1, (6,)),
    "sweep_t32": (4, 32, (6,)),
    "sweep_t256": (4, 256, (6,)),
    "sweep_t2048": (4, 2048, (6,)),
    "sweep_t7234": (4, 7234, (6,)),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 10):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms={interval_ms}", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def code_only(text: str) -> str:
    """C/CUDA source with comments, trailing blanks and empty lines removed (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':                                   # string literal, escapes included
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "\n".join(l.rstrip() for l in "".join(out).splitlines() if l.strip())


def kernel_source_hash(stage: str = "gemv_gate_up"):
    """Hash of the code (not the comments) of the stage's kernel file + common.cuh + internal.h."""
    h = hashlib.sha256()
    files = ("mma.cu",) if stage.startswith("mma") else ("gemv.cu",)
    for f in files + ("common.cuh", "internal.h"):
        src = open(os.path.join(ROOT, "nvfp4_weight_only_route_b200", "csrc", f), encoding="utf-8").read()
        h.update(code_only(src).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, stage: str):
    """DRAM bytes per launch from a committed ncu capture of this workload, if it matches the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    ent = json.load(open(p)).get(workload, {}).get(stage)
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash(stage):
        return None
    return ent.get("dram_bytes_per_launch")


def workload_label(name: str, H: int, I: int, E: int, k: int, T: int, seeds) -> str:
    """config.workload of both arms: the workload named by what it is, with its sizes."""
    return f"{name}: H={H} I={I} E={E} top-{k} T={T} tokens/forward, seeds {list(seeds)} rotated"


def work_per_forward(mean_active: float, T: int, H: int, I: int, E: int, k: int):
    """Algorithmic bytes and FLOPs of one forward: the active experts' NVFP4 weights read
    once (3 H I weights each), the bf16 router weights, x in and out; expert and router FLOPs.
    The intermediates and the routing state are implementation traffic, not counted."""
    nbytes = mean_active * 3 * H * I * NVFP4_BYTES_PER_WEIGHT + E * H * 2 + T * H * 2 * 2
    flops = 2.0 * T * k * 3 * H * I + 2.0 * T * H * E
    return nbytes, flops


def roofline_for(kernel: str, us: float, H: int, I: int, gemv_experts: float, mma_pairs: float, mma_experts: float,
                 hbm_peak: float, bf16_peak: float, measured: bool, traffic, how: str) -> dict:
    """The roofline object of the dominant kernel from its average launch time `us`.
    GEMV launches read gemv_experts x rows x K weights (HBM bound). A tensor-core launch
    does 2 x pairs x rows x K FLOPs on mma_experts x rows x K weights; its bound follows
    its arithmetic intensity against the ratio of the measured peaks."""
    hbm_src = "measured (MEASURED_PEAKS.json hbm_gbs)" if measured else "fallback"
    if kernel in ("gemv_gate_up", "gemv_down"):
        alg = gemv_experts * (2 * I * H if kernel == "gemv_gate_up" else H * I) * NVFP4_BYTES_PER_WEIGHT
        achieved = alg / (us * 1e-6) / 1e9
        return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic, "algorithmic_bytes_per_launch": alg,
                "avg_launch_us": us, "peak_source": hbm_src, "how": how}
    if kernel in ("mma_gate_up", "mma_down"):
        rows = 2 * I if kernel == "mma_gate_up" else H
        kdim = H if kernel == "mma_gate_up" else I
        flops = 2.0 * mma_pairs * rows * kdim
        wbytes = mma_experts * rows * kdim * NVFP4_BYTES_PER_WEIGHT
        t_s = us * 1e-6
        if wbytes > 0 and flops / wbytes < (bf16_peak * 1e12) / (hbm_peak * 1e9):
            achieved = wbytes / t_s / 1e9
            return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak, "traffic": traffic, "algorithmic_bytes_per_launch": wbytes,
                    "algorithmic_flops_per_launch": flops, "avg_launch_us": us, "peak_source": hbm_src,
                    "how": how}
        achieved = flops / t_s / 1e12
        return {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": achieved / bf16_peak, "traffic": traffic, "algorithmic_flops_per_launch": flops,
                "algorithmic_bytes_per_launch": wbytes, "avg_launch_us": us,
                "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops, burst)" if measured else "fallback",
                "how": how}
    return {"bound": "hbm", "kernel": kernel, "achieved": None, "peak": hbm_peak, "unit": "GB/s", "frac": None,
            "traffic": traffic, "avg_launch_us": us}


def oracle_cpu_sample(shape, layers, xs, seconds: float):
    """Time the fp64 oracle on whole decode batches (or single tokens for big shapes)."""
    from oracle import oracle
    oracle.build()
    tokens, n, t0 = 0, 0, time.perf_counter()
    while True:
        L = layers[n % len(layers)]
        x = xs[n % len(xs)]
        if shape.H * shape.I * shape.k * x.shape[0] > 2 ** 27:
            x = x[n % x.shape[0]: n % x.shape[0] + 1]
        oracle.forward(L, x, top_k=shape.k)
        tokens += x.shape[0]
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return tokens / el, oracle.max_threads(), f"{n} oracle forwards, {tokens} tokens, {el:.1f} s"


def dist_setup(n_gpus, backend: str = "nccl"):
    """Rank, world size, local rank and the process group (None for one process). Replicas only:
    the group carries the timing barrier and the max over ranks, never the data path."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return rank, world, local, pg


def barrier(pg, torch, cuda: bool = True):
    if pg is not None:
        pg.barrier()
    if cuda:
        torch.cuda.synchronize()


def max_over_ranks(pg, torch, v: float, device: str = "cuda") -> float:
    if pg is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def replica_seed(seed: int, rank: int) -> int:
    """Each replica runs its own seeded layers (rank 0 the listed seeds)."""
    return seed + 1000 * rank


def weak_value(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_step * steps / (ms / 1e3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from nvfp4_weight_only_route_b200 import synth
    from oracle import oracle
    oracle.build()
    shape_idx, T, seeds = WORKLOADS[args.workload]
    shape = synth.SHAPES[shape_idx]
    layers = [synth.make_layer(shape, s) for s in seeds]
    xs = [synth.make_x(shape, s, T, stream=r) for s in seeds for r in range(2)]

    def step(i):
        x = xs[i % len(xs)]
        j = (i // len(xs)) % x.shape[0]
        oracle.forward(layers[i % len(layers)], x[j:j + 1], top_k=shape.k)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    value = args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(args.workload, shape.H, shape.I, shape.E, shape.k, T, seeds),
                   "global_batch": T, "parallelism": "single GPU",
                   "reference": "fp64 CPU oracle on the host cores, one token of the workload per step"},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": f"{args.steps} steps of one token each"},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["tfmoe", "reference"], default="tfmoe")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--flags", type=int, default=0, help="descriptor flags (1 = force GEMV, 2 = force MMA)")
    ap.add_argument("--gemv-max-tokens", type=int, default=0,
                    help="per-expert token count up to which the GEMV regime is used (0 = library default)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", type=int, default=100, help="forwards per CUDA graph (0 = no graphs)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch

    from nvfp4_weight_only_route_b200 import synth, tfmoe
    rank, world, local, pg = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, bf16_sustained, peak_src = load_peaks()

    shape_idx, T, seeds = WORKLOADS[args.workload]
    shape = synth.SHAPES[shape_idx]
    H, I, E, k = shape.H, shape.I, shape.E, shape.k
    n_x = 8 if T <= 256 else 2
    layers_np, layers, xs = [], [], []
    for s in seeds:
        lnp = synth.make_layer(shape, replica_seed(s, rank))
        layers_np.append(lnp)
        L = tfmoe.MoELayer(H, I, E, k, T, has_router_bias=lnp["router_bias"] is not None, flags=args.flags,
                           gemv_max_tokens=args.gemv_max_tokens)
        L.load_weights(tfmoe.layer_to_device(lnp, dev))
        layers.append(L)
        xs.append([torch.from_numpy(synth.make_x(shape, s, T, stream=r + 100 * rank).view(np.int16)).to(dev)
                   for r in range(n_x)])
    torch.cuda.synchronize()
    out = torch.empty((T, H), dtype=torch.int16, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def fwd(i):
        L = layers[i % len(layers)]
        x = xs[i % len(layers)][(i // len(layers)) % n_x]
        tfmoe.check(L.forward_raw(x.data_ptr(), T, out.data_ptr(), stream.cuda_stream))
        return L

    # ---- parity gate against the oracle (rank 0), sampled tokens for large T
    parity = "skipped"
    if rank == 0:
        from oracle import oracle
        worst = 0.0
        for li, L in enumerate(layers):
            with torch.cuda.stream(stream):
                fwd(li)
            stream.synchronize()
            tfmoe.check(L.sync_status(stream))
            got = out.cpu().numpy().view(np.uint16)
            ids_g = L.buffer_tensor(tfmoe.BUF_TOPK_IDS, torch.int32, (T, k)).cpu().numpy()
            x_np = xs[li][0].cpu().numpy().view(np.uint16)
            idx = np.arange(T) if T <= 64 else np.unique(np.linspace(0, T - 1, 16).astype(int))
            ref = oracle.forward(layers_np[li], x_np[idx], top_k=k, intermediates=True)
            if not np.array_equal(ids_g[idx], ref["ids"]):
                raise SystemExit("parity gate: routing differs from the oracle")
            g64 = (got[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            half_ulp = 0.5 * 2.0 ** (np.floor(np.log2(np.maximum(np.maximum(np.abs(g64), np.abs(ref["out64"])), 2.0 ** -126))) - 7)
            tol = 4e-3 * ref["S"] + 1e-3 + half_ulp
            err = np.abs(g64 - ref["out64"])
            if not np.all(err <= tol):
                raise SystemExit(f"parity gate: output outside tolerance (worst {float(np.max(err / tol)):.3f})")
            worst = max(worst, float(np.max(err / tol)))
        parity = f"ok: ids bit-exact, worst |err|/tol {worst:.3f} on {len(layers)} layer(s)"

    # ---- routing statistics for the algorithmic byte / flop counts
    active, gemv_experts, launches_per_fwd = [], [], 0
    n_inputs = len(layers) * n_x
    for i in range(n_inputs):
        with torch.cuda.stream(stream):
            L = fwd(i)
        stream.synchronize()
        launches_per_fwd = L.last_launch_count()
        cnt = L.buffer_tensor(tfmoe.BUF_EXPERT_COUNTS, torch.int32, (E,)).cpu().numpy()
        reg = L.buffer_tensor(tfmoe.BUF_REGIME, torch.int32, (E,)).cpu().numpy()
        active.append(int(np.sum(cnt > 0)))
        gemv_experts.append(int(np.sum(reg == 1)))
    mean_active = float(np.mean(active))
    mean_gemv = float(np.mean(gemv_experts))
    bytes_per_fwd, flops_per_fwd = work_per_forward(mean_active, T, H, I, E, k)

    # ---- CUDA graphs of consecutive forwards, all captured before timing. Each graph
    # starts at input index 0 and holds a whole number of input cycles when it can.
    cycle = len(layers) * n_x
    G = 0
    if args.graph > 0:
        G = max(cycle, (args.graph // cycle) * cycle) if args.steps >= cycle else args.steps
        G = min(G, args.steps)
    graphs = {}

    def make_graph(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for j in range(n):
                fwd(j)
        return g

    def run_steps(n, start):
        if G == 0:
            with torch.cuda.stream(stream):
                for j in range(n):
                    fwd(start + j)
            return
        done = 0
        while done < n:
            m = min(G, n - done)
            graphs[m].replay()
            done += m

    if G:
        sizes = {G} if args.steps >= G else set()
        if args.steps % G:
            sizes.add(args.steps % G)
        w_full, w_rem = divmod(args.warmup, G)
        if w_rem:
            sizes.add(w_rem)
        for m in sorted(sizes):
            graphs[m] = make_graph(m)
            graphs[m].replay()          # first replay of every graph happens before timing
        stream.synchronize()
    run_steps(args.warmup, 0)
    stream.synchronize()

    # ---- timed region
    sampler = ClockSampler(local) if rank == 0 else None
    barrier(pg, torch)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        run_steps(args.steps, args.warmup)
        ev1.record(stream)
    stream.synchronize()
    barrier(pg, torch)
    clocks = sampler.stop() if sampler else None
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(pg, torch, ms_local)
    value = weak_value(world, T, args.steps, ms)

    # ---- per-kernel timing for the roofline: one forward per layer on a known batch, then
    # a CUDA graph that re-enqueues one stage of those forwards, rotating over the layers
    # (so consecutive launches read different weights), timed with events on its stream.
    gemv_units, mma_pairs, mma_units = [], [], []
    for li, L in enumerate(layers):
        with torch.cuda.stream(stream):
            tfmoe.check(L.forward_raw(xs[li][0].data_ptr(), T, out.data_ptr(), stream.cuda_stream))
        stream.synchronize()
        reg = L.buffer_tensor(tfmoe.BUF_REGIME, torch.int32, (E,)).cpu().numpy()
        cnt = L.buffer_tensor(tfmoe.BUF_EXPERT_COUNTS, torch.int32, (E,)).cpu().numpy()
        gemv_units.append(int(np.sum(reg == 1)))
        mma_pairs.append(int(np.sum(cnt[reg == 2])))
        mma_units.append(int(np.sum(reg == 2)))
    kernel_us = {}
    for stage in ("gemv_gate_up", "gemv_down", "gather", "mma_gate_up", "mma_down", "combine"):
        sid = tfmoe.STAGE_ID[stage]
        # one launch per layer, timed once, sizes the graph to ~5 ms of work
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        launched = 0
        with torch.cuda.stream(stream):
            e0.record(stream)
            for li, L in enumerate(layers):
                tfmoe.check(L.forward_stage_raw(sid, xs[li][0].data_ptr(), T, out.data_ptr(), stream.cuda_stream))
                launched += L.last_launch_count()
            e1.record(stream)
        stream.synchronize()
        if launched == 0:
            continue
        est_us = max(1.0, e0.elapsed_time(e1) * 1e3 / len(layers))
        reps = int(max(2, min(50, 5000.0 / est_us / len(layers))))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(reps):
                for li, L in enumerate(layers):
                    tfmoe.check(L.forward_stage_raw(sid, xs[li][0].data_ptr(), T, out.data_ptr(), stream.cuda_stream))
        for _ in range(3):      # the first replays of a new graph run slow; keep them out of the timing
            g.replay()
        stream.synchronize()
        samples = []
        for _ in range(5):
            with torch.cuda.stream(stream):
                e0.record(stream)
                g.replay()
                e1.record(stream)
            stream.synchronize()
            samples.append(e0.elapsed_time(e1) * 1e3 / (reps * len(layers)))
        kernel_us[stage] = float(np.median(samples))
        del g
    dominant = max(kernel_us, key=kernel_us.get)
    how = (f"median of 5 replays of a graph of back-to-back launches rotating {len(layers)} layer(s), "
           "CUDA events on the launch stream")
    roofline = roofline_for(dominant, kernel_us[dominant], H, I, float(np.mean(gemv_units)),
                            float(np.mean(mma_pairs)), float(np.mean(mma_units)), hbm_peak, bf16_peak,
                            peak_src == "measured", ncu_traffic(args.workload, dominant), how)

    # ---- per-stage times of ordinary (profiled, host-synchronised) forwards; these include
    # host launch gaps and are reported for orientation only
    prof_steps = min(args.steps, 100)
    for L in layers:
        L.profile(True)
        L.profile_read(reset=True)
    for i in range(prof_steps):
        with torch.cuda.stream(stream):
            fwd(i)
    stage_ms = {}
    for L in layers:
        for name, (ms_tot, calls) in L.profile_read(reset=True).items():
            a_, c_ = stage_ms.get(name, (0.0, 0))
            stage_ms[name] = (a_ + ms_tot, c_ + calls)
        L.profile(False)
    stage_avg_us = {n: (v[0] / v[1] * 1e3 if v[1] else 0.0) for n, v in stage_ms.items()}
    layer_gbs = bytes_per_fwd / (ms / args.steps * 1e-3) / 1e9
    layer_tflops = flops_per_fwd / (ms / args.steps * 1e-3) / 1e12

    # ---- end to end through the host-buffer entry point (pinned memory)
    x_host = [xs[li][r].cpu().pin_memory() for li in range(len(layers)) for r in range(min(n_x, 2))]
    out_host = torch.empty((T, H), dtype=torch.int16).pin_memory()
    e2e_steps = min(args.steps, 500)
    barrier(pg, torch)
    t0 = time.perf_counter()
    for i in range(e2e_steps):
        L = layers[i % len(layers)]
        L.forward_host(x_host[i % len(x_host)], out_host, T=T, stream=stream)
    el = time.perf_counter() - t0
    el = max_over_ranks(pg, torch, el)
    e2e = {"value": world * T * e2e_steps / el, "unit": "tok/s", "h2d_bytes_per_step": T * H * 2,
           "d2h_bytes_per_step": T * H * 2, "steps": e2e_steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = oracle_cpu_sample(shape, layers_np, [x.cpu().numpy().view(np.uint16) for x in xs[0]],
                                             args.cpu_seconds)
        cpu = {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 activations, nvfp4 weights, fp32 accumulate", "data": "synthetic",
            "config": {"workload": workload_label(args.workload, H, I, E, k, T, seeds), "global_batch": T * world,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2: rotating seeded layers / full weight sets exceed 126 MB",
                       "flags": args.flags, "gemv_max_tokens": args.gemv_max_tokens or "default",
                       "graph_forwards": G},
            "roofline": roofline,
            "layer": {"algorithmic_bytes_per_forward": bytes_per_fwd, "hbm_gbs": layer_gbs,
                      "hbm_frac": layer_gbs / hbm_peak, "hbm_frac_of_8tbs": layer_gbs / 8000.0,
                      "flops_per_forward": flops_per_fwd, "tflops": layer_tflops,
                      "tensor_frac": layer_tflops / bf16_peak, "active_experts_mean": mean_active,
                      "mma_pairs_mean": float(np.mean(mma_pairs)), "gemv_experts_mean": float(np.mean(gemv_units)),
                      "kernel_us_graph": kernel_us, "stage_avg_us_profiled": stage_avg_us},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_fwd * args.steps,
            "clocks": clocks,
            "parity": parity,
        }
        print(json.dumps(line), flush=True)
    for g in graphs.values():
        del g
    graphs.clear()
    for L in layers:
        L.close()
    if pg is not None:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
