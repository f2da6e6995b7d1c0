#!/usr/bin/env python
"""Throughput of the NVFP4 W4A16 MoE FFN layer forward (libtfmoe) on B200.

Headline workload (N=1, the default): the large sparse-MoE layer -- H=4096,
I=2688, E=256, top-8 (4.76 GB of NVFP4 expert weights per layer) -- at T=7234
tokens per forward (the length of the 7,234-token prompt in the numbers table
of the DGX Spark GB10 bandwidth-budget page). Five seeded layers (seeds 6..10)
rotate, one forward each in turn; `value` is the median over the seeds of each
seed's tokens/s. A step is one forward of the whole layer (router, top-k,
permute, gate/up + SwiGLU, down, combine) over one batch. Every forward reads
4.76 GB of weights, far more than the 126 MB L2.

The same JSON line carries `per_config`: tokens/s, the layer's fraction of the
HBM roofline (8 TB/s and the measured copy bandwidth) or of the bf16 tensor
peak, the dominant kernel's roofline and the parity result for the tiny layer,
decode T=1 and T=8, batched decode with Zipf load (T=256), prefill (T=8192) and
the large sweep at T = 1, 32, 256, 2048 (N=1 only).

Printed JSON line (rank 0): value = tokens/s over all ranks, e2e = the same
metric through tfmoe_forward_host with pinned host buffers (copies inside the
timed region), roofline of the dominant kernel measured live with CUDA events,
cpu_baseline = the fp64 oracle on a bounded token sample of the same workload
on this host's cores.

--impl reference times the fp64 CPU oracle (the only reference this layer has)
on the same workload and the same kind of sample as cpu_baseline: each step is
one oracle call on a fixed number of the workload's tokens.

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
NOMINAL_HBM_GBS = 8000.0               # the ~8 TB/s the decode target is stated against

SWEEP_SEEDS = (6, 7, 8, 9, 10)
WORKLOADS = {
    # name: (layer shape index, tokens per forward, seeds)
    "tiny": (0, 4, (0,)),
    "decode_t1": (1, 1, (1, 2, 3)),
    "decode": (1, 8, (1, 2, 3)),
    "zipf": (2, 256, (4,)),
    "prefill": (3, 8192, (5,)),
    "sweep_t1": (4, 1, SWEEP_SEEDS),
    "sweep_t32": (4, 32, SWEEP_SEEDS),
    "sweep_t256": (4, 256, SWEEP_SEEDS),
    "sweep_t2048": (4, 2048, SWEEP_SEEDS),
    "sweep_t7234": (4, 7234, SWEEP_SEEDS),
    "decode_shared_norm": (1, 8, (1, 2, 3)),
}
# Workloads whose layer has a shared expert of m slots (width m * I) and that run through
# tfmoe_forward_add_norm (shared expert + residual add + RMS norm: the add_moe_norm step).
SHARED_NORM = {"decode_shared_norm": 1}
NORM_EPS = 1e-6
HEADLINE = "sweep_t7234"
PER_CONFIG = ["tiny", "decode_t1", "decode", "zipf", "prefill", "sweep_t1", "sweep_t32", "sweep_t256",
              "sweep_t2048", "decode_shared_norm"]
# Tokens of the workload per oracle call, for the CPU baseline and the reference arm.
ORACLE_SAMPLE_TOKENS = {"tiny": 4, "decode_t1": 1, "decode": 8, "zipf": 16, "prefill": 8}


def oracle_tokens_per_call(name: str) -> int:
    return ORACLE_SAMPLE_TOKENS.get(name, 8)


def regime_of(name: str) -> str:
    """Which roofline a workload is held to: decode-shaped layers stream their active
    weights (HBM), prefill-shaped ones are one large contraction (tensor); the
    large sweep at T=2048 sits at the crossover and is reported against both."""
    T = WORKLOADS[name][1]
    if name == "prefill" or (name.startswith("sweep") and T >= 7234):
        return "tensor"
    if name.startswith("sweep") and T == 2048:
        return "both"
    return "hbm"


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
    extra = ""
    if name in SHARED_NORM:
        extra = f", shared expert Is={SHARED_NORM[name] * I}, residual add and RMS norm (tfmoe_forward_add_norm)"
    return f"{name}: H={H} I={I} E={E} top-{k} T={T} tokens/forward{extra}, seeds {list(seeds)} rotated"


class AddNormLayer:
    """A layer with a shared expert whose forward_raw runs tfmoe_forward_add_norm with this
    object's device residual, norm weights and out_norm buffers, so that every measurement
    below drives the whole add_moe_norm step; everything else goes to the layer."""

    def __init__(self, layer, residual, norm_w, out_norm):
        self.layer, self.residual, self.norm_w, self.out_norm = layer, residual, norm_w, out_norm

    def forward_raw(self, x_ptr: int, T: int, out_ptr: int, stream_handle: int) -> int:
        return self.layer.lib.tfmoe_forward_add_norm(self.layer.handle, x_ptr, T, self.residual.data_ptr(),
                                                     self.norm_w.data_ptr(), out_ptr, self.out_norm.data_ptr(),
                                                     stream_handle)

    def __getattr__(self, name):
        return getattr(self.layer, name)


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


def oracle_rate(layer_np, x_np, k: int, tokens_per_call: int, *, seconds: float = 0.0, calls: int = 0,
                nthreads: int = 0, start: int = 0):
    """Time the fp64 oracle on consecutive `tokens_per_call`-token slices of x_np (wrapping),
    for at least `seconds` or exactly `calls` calls. Returns (tokens/s, calls, tokens, seconds)."""
    from oracle import oracle
    oracle.build()
    T = x_np.shape[0]
    n = min(tokens_per_call, T)
    done, tokens = 0, 0
    t0 = time.perf_counter()
    while True:
        j = ((start + done) * n) % T
        sl = x_np[j:j + n] if j + n <= T else np.concatenate([x_np[j:], x_np[:j + n - T]])
        oracle.forward(layer_np, sl, top_k=k, nthreads=nthreads)
        done += 1
        tokens += n
        el = time.perf_counter() - t0
        if (calls and done >= calls) or (not calls and el >= seconds):
            break
    return tokens / el, done, tokens, el


def log(msg: str):
    print(f"[bench {time.strftime('%H:%M:%S')}] {msg}", file=sys.stderr, flush=True)


def cpu_description() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


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
    """The reference arm: the fp64 CPU oracle on the same workload, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from nvfp4_weight_only_route_b200 import synth
    from oracle import oracle
    oracle.build()
    name = args.workload or HEADLINE
    shape_idx, T, seeds = WORKLOADS[name]
    shape = synth.SHAPES[shape_idx]
    n = oracle_tokens_per_call(name)
    layers = [synth.make_layer(shape, s) for s in seeds]
    xs = [synth.make_x(shape, s, T) for s in seeds]

    def step(i):
        li = i % len(layers)
        oracle_rate(layers[li], xs[li], shape.k, n, calls=1, start=i // len(layers))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    value = args.steps * min(n, T) / el
    sample = (f"{args.steps} steps, each one oracle call on {min(n, T)} consecutive tokens of a T={T} batch, "
              f"layers of seeds {list(seeds)} in turn")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(name, shape.H, shape.I, shape.E, shape.k, T, seeds),
                   "global_batch": T, "parallelism": "single GPU",
                   "reference": "fp64 CPU oracle on the host cores"},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": sample, "cpu": cpu_description()},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class Bench:
    """Seeded layers on one GPU and the measurements made on them."""

    def __init__(self, args, rank, world, local, pg):
        import torch
        from nvfp4_weight_only_route_b200 import synth, tfmoe
        self.torch, self.synth, self.tfmoe = torch, synth, tfmoe
        self.args, self.rank, self.world, self.pg = args, rank, world, pg
        self.dev = torch.device("cuda", local)
        self.stream = torch.cuda.Stream(device=self.dev)
        self.hbm_peak, self.bf16_peak, self.bf16_sustained, self.peak_src = load_peaks()
        self.layers = {}        # (shape index, seed) -> [host layer or None, MoELayer]
        self.max_tokens = {}    # shape index -> the largest T any workload of this run uses
        self.gen_s = 0.0

    def plan(self, names):
        for n in names:
            si, T, _ = WORKLOADS[n]
            self.max_tokens[si] = max(self.max_tokens.get(si, 0), T)

    def layer(self, si, seed, m=0):
        key = (si, seed, m)
        if key not in self.layers:
            torch = self.torch
            shape = self.synth.SHAPES[si]
            t0 = time.perf_counter()
            rs = replica_seed(seed, self.rank)
            lnp = self.synth.make_layer(shape, rs)
            if m:
                lnp.update(self.synth.make_shared(shape, rs, m * shape.I))
            L = self.tfmoe.MoELayer(shape.H, shape.I, shape.E, shape.k, self.max_tokens[si],
                                    has_router_bias=lnp["router_bias"] is not None, flags=self.args.flags,
                                    gemv_max_tokens=self.args.gemv_max_tokens, shared_intermediate=m * shape.I,
                                    norm_eps=NORM_EPS)
            L.load_weights(self.tfmoe.layer_to_device(lnp, self.dev))
            if m:
                T = self.max_tokens[si]
                res = self.synth.make_residual(shape, rs, T)
                gam = self.synth.make_norm_weight(shape, rs)
                dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(self.dev)
                L = AddNormLayer(L, dev(res), dev(gam), torch.empty((T, shape.H), dtype=torch.int16, device=self.dev))
                lnp["_residual"], lnp["_norm_w"] = res, gam
            torch.cuda.synchronize()
            self.gen_s += time.perf_counter() - t0
            self.layers[key] = [lnp, L]
        return self.layers[key]

    def slim(self, si, seed, m=0):
        """Keep only the router of a host layer whose expert weights no check reads again."""
        lnp = self.layers[(si, seed, m)][0]
        for k in list(lnp):
            if k not in ("router_w", "router_bias"):
                lnp[k] = None

    def inputs(self, name, n_x):
        si, T, seeds = WORKLOADS[name]
        shape = self.synth.SHAPES[si]
        return [[self.torch.from_numpy(self.synth.make_x(shape, s, T, stream=r + 100 * self.rank).view(np.int16))
                 .to(self.dev) for r in range(n_x)] for s in seeds]

    def parity(self, name, Ls, lnps, xs, n_sample, sample_layers):
        """Routing of every token against the oracle's routing step (bit-exact ids and
        selected logits; every other logit exact or within the library's stated bound of the
        tensor-core approximation), the output on sampled tokens within the tolerance."""
        from oracle import oracle
        torch, tfmoe = self.torch, self.tfmoe
        si, T, _ = WORKLOADS[name]
        k, E = self.synth.SHAPES[si].k, self.synth.SHAPES[si].E
        m = SHARED_NORM.get(name, 0)
        out = torch.empty((T, self.synth.SHAPES[si].H), dtype=torch.int16, device=self.dev)
        worst = 0.0
        norm_note = ""
        for li, L in enumerate(Ls):
            with torch.cuda.stream(self.stream):
                tfmoe.check(L.forward_raw(xs[li][0].data_ptr(), T, out.data_ptr(), self.stream.cuda_stream))
            self.stream.synchronize()
            tfmoe.check(L.sync_status(self.stream))
            x_np = xs[li][0].cpu().numpy().view(np.uint16)
            ids_all = L.buffer_tensor(tfmoe.BUF_TOPK_IDS, torch.int32, (T, k + m)).cpu().numpy()
            if m and not np.array_equal(ids_all[:, k:], np.tile(E + np.arange(m), (T, 1))):
                raise SystemExit(f"parity gate ({name}): shared-expert slots missing from the routing")
            ids_g = ids_all[:, :k]
            log_g = L.buffer_tensor(tfmoe.BUF_LOGITS, torch.float32, (T, E)).cpu().numpy()
            r = oracle.route(lnps[li], x_np, top_k=k)
            if not (np.array_equal(ids_g, r["ids"]) and
                    np.array_equal(np.take_along_axis(log_g, r["ids"], 1), np.take_along_axis(r["logits"], r["ids"], 1))):
                raise SystemExit(f"parity gate ({name}): routing differs from the oracle")
            xf = (x_np.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            wf = (lnps[li]["router_w"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            bound = (xf.shape[1] + 34) * 2.0 ** -22 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1))
            if lnps[li].get("router_bias") is not None:
                bound = bound + 2.0 ** -21 * np.abs(lnps[li]["router_bias"].astype(np.float64))[None, :]
            if not np.all(np.abs(log_g.astype(np.float64) - r["logits"]) <= bound * 1.01 + 1e-6):
                raise SystemExit(f"parity gate ({name}): router logits outside the stated bound")
            if li >= sample_layers:
                continue
            got = out.cpu().numpy().view(np.uint16)
            idx = np.arange(T) if T <= n_sample else np.unique(np.linspace(0, T - 1, n_sample).astype(int))
            if m:
                res_np, gam_np = lnps[li]["_residual"][:T], lnps[li]["_norm_w"]
                ref = oracle.forward(lnps[li], x_np[idx], top_k=k, intermediates=False, residual=res_np[idx],
                                     norm_w=gam_np, eps=NORM_EPS)
                got_n = L.out_norm[:T].cpu().numpy().view(np.uint16)[idx]
                want_n = oracle.rms_norm(got[idx], gam_np, NORM_EPS)
                gv = (got_n.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                wv = (want_n.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                if not np.all(np.abs(gv - wv) <= 2.0 ** -7 * np.abs(wv)):
                    raise SystemExit(f"parity gate ({name}): RMS norm differs from the oracle's norm of the same row")
                norm_note = (f"; RMS norm of the output equal to the oracle's norm of the same rows on "
                             f"{int(np.sum(got_n == want_n))}/{got_n.size} elements, the rest within one ulp")
            else:
                ref = oracle.forward(lnps[li], x_np[idx], top_k=k, intermediates=False)
            g64 = (got[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            half_ulp = 0.5 * 2.0 ** (np.floor(np.log2(np.maximum(np.maximum(np.abs(g64), np.abs(ref["out64"])),
                                                                 2.0 ** -126))) - 7)
            tol = 4e-3 * ref["S"] + 1e-3 + half_ulp
            err = np.abs(g64 - ref["out64"])
            if not np.all(err <= tol):
                raise SystemExit(f"parity gate ({name}): output outside tolerance (worst {float(np.max(err / tol)):.3f})")
            worst = max(worst, float(np.max(err / tol)))
        return (f"ok: ids and selected logits bit-exact (others within the stated bound) for all {T} tokens x {len(Ls)} layer(s); output within "
                f"4e-3*S+1e-3 on {min(T, n_sample)} sampled tokens x {min(len(Ls), sample_layers)} layer(s), "
                f"worst |err|/tol {worst:.3f}{norm_note}")

    def routing_stats(self, name, Ls, xs):
        torch, tfmoe = self.torch, self.tfmoe
        si, T, _ = WORKLOADS[name]
        E = self.synth.SHAPES[si].E + SHARED_NORM.get(name, 0)      # expert slots
        out = torch.empty((T, self.synth.SHAPES[si].H), dtype=torch.int16, device=self.dev)
        st = {"active": [], "gemv": [], "mma_pairs": [], "mma": []}
        launches = 0
        for li, L in enumerate(Ls):
            for xb in xs[li]:
                with torch.cuda.stream(self.stream):
                    tfmoe.check(L.forward_raw(xb.data_ptr(), T, out.data_ptr(), self.stream.cuda_stream))
                self.stream.synchronize()
                launches = L.last_launch_count()
                cnt = L.buffer_tensor(tfmoe.BUF_EXPERT_COUNTS, torch.int32, (E,)).cpu().numpy()
                reg = L.buffer_tensor(tfmoe.BUF_REGIME, torch.int32, (E,)).cpu().numpy()
                st["active"].append(int(np.sum(cnt > 0)))
                st["gemv"].append(int(np.sum(reg == 1)))
                st["mma_pairs"].append(int(np.sum(cnt[reg == 2])))
                st["mma"].append(int(np.sum(reg == 2)))
        return {k: float(np.mean(v)) for k, v in st.items()}, launches

    def kernel_times(self, name, Ls, xs):
        """Average launch time of each expert-path kernel: a CUDA graph of back-to-back
        single-stage replays (tfmoe_forward_stage) rotating the layers, median of 5 replays."""
        torch, tfmoe = self.torch, self.tfmoe
        si, T, _ = WORKLOADS[name]
        out = torch.empty((T, self.synth.SHAPES[si].H), dtype=torch.int16, device=self.dev)
        s = self.stream
        for li, L in enumerate(Ls):       # leave every layer's workspace holding input 0's routing
            with torch.cuda.stream(s):
                tfmoe.check(L.forward_raw(xs[li][0].data_ptr(), T, out.data_ptr(), s.cuda_stream))
        s.synchronize()
        kernel_us = {}
        for stage in ("gemv_gate_up", "gemv_down", "gather", "mma_gate_up", "mma_down", "combine"):
            sid = tfmoe.STAGE_ID[stage]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            launched = 0
            with torch.cuda.stream(s):
                e0.record(s)
                for li, L in enumerate(Ls):
                    tfmoe.check(L.forward_stage_raw(sid, xs[li][0].data_ptr(), T, out.data_ptr(), s.cuda_stream))
                    launched += L.last_launch_count()
                e1.record(s)
            s.synchronize()
            if launched == 0:
                continue
            est_us = max(1.0, e0.elapsed_time(e1) * 1e3 / len(Ls))
            reps = int(max(2, min(50, 5000.0 / est_us / len(Ls))))
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for _ in range(reps):
                    for li, L in enumerate(Ls):
                        tfmoe.check(L.forward_stage_raw(sid, xs[li][0].data_ptr(), T, out.data_ptr(), s.cuda_stream))
            for _ in range(3):      # the first replays of a new graph run slow; keep them out of the timing
                g.replay()
            s.synchronize()
            samples = []
            for _ in range(5):
                with torch.cuda.stream(s):
                    e0.record(s)
                    g.replay()
                    e1.record(s)
                s.synchronize()
                samples.append(e0.elapsed_time(e1) * 1e3 / (reps * len(Ls)))
            kernel_us[stage] = float(np.median(samples))
            del g
        return kernel_us

    def timed(self, name, Ls, xs, steps, warmup, graph, per_forward, clocks=False):
        """Device time of `steps` forwards rotating layers (then inputs). With per_forward,
        an event pair brackets every forward (large batches only) and per-layer mean times
        come back too. Bracketed by barriers; the max over ranks is taken."""
        torch, tfmoe = self.torch, self.tfmoe
        si, T, _ = WORKLOADS[name]
        s = self.stream
        out = torch.empty((T, self.synth.SHAPES[si].H), dtype=torch.int16, device=self.dev)
        n_x = len(xs[0])

        def fwd(i):
            L = Ls[i % len(Ls)]
            x = xs[i % len(Ls)][(i // len(Ls)) % n_x]
            tfmoe.check(L.forward_raw(x.data_ptr(), T, out.data_ptr(), s.cuda_stream))

        cycle = len(Ls) * n_x
        G = 0
        if graph > 0 and not per_forward:
            G = max(cycle, (graph // cycle) * cycle) if steps >= cycle else steps
            G = min(G, steps)
        graphs = {}

        def make_graph(n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for j in range(n):
                    fwd(j)
            return g

        def run(n, start, evs=None):
            if G == 0:
                with torch.cuda.stream(s):
                    for j in range(n):
                        if evs is not None:
                            evs[j].record(s)
                        fwd(start + j)
                    if evs is not None:
                        evs[n].record(s)
                return
            done = 0
            while done < n:
                m = min(G, n - done)
                graphs[m].replay()
                done += m

        if G:
            sizes = {G} if steps >= G else set()
            if steps % G:
                sizes.add(steps % G)
            if warmup % G:
                sizes.add(warmup % G)
            for m in sorted(sizes):
                graphs[m] = make_graph(m)
                graphs[m].replay()          # the first replay of every graph happens before timing
            s.synchronize()
        run(warmup, 0)
        s.synchronize()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)] if per_forward else None
        sampler = ClockSampler(self.dev.index) if (clocks and self.rank == 0) else None
        barrier(self.pg, torch)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            ev0.record(s)
            run(steps, warmup, evs)
            ev1.record(s)
        s.synchronize()
        barrier(self.pg, torch)
        clk = sampler.stop() if sampler else None
        ms = max_over_ranks(self.pg, torch, ev0.elapsed_time(ev1))
        per_layer = None
        if per_forward:
            per_layer = []
            for li in range(len(Ls)):
                ts = [evs[j].elapsed_time(evs[j + 1]) for j in range(steps) if (warmup + j) % len(Ls) == li]
                per_layer.append(max_over_ranks(self.pg, torch, float(np.mean(ts))) if ts else None)
        for g in graphs.values():
            del g
        graphs.clear()
        return ms, per_layer, clk, G

    def fractions(self, name, ms_per_fwd, stats):
        si, T, _ = WORKLOADS[name]
        sh = self.synth.SHAPES[si]
        nbytes, flops = work_per_forward(stats["active"], T, sh.H, sh.I, sh.E, sh.k)
        m = SHARED_NORM.get(name, 0)
        if m:   # the shared slots count in "active"; add the residual read and the normed output written
            nbytes += T * sh.H * 2 * 2
            flops += 2.0 * T * m * 3 * sh.H * sh.I
        t = ms_per_fwd * 1e-3
        gbs, tfl = nbytes / t / 1e9, flops / t / 1e12
        d = {"algorithmic_bytes_per_forward": nbytes, "hbm_gbs": gbs, "hbm_frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
             "hbm_frac_of_measured": gbs / self.hbm_peak, "flops_per_forward": flops, "tflops": tfl,
             "tensor_frac_of_measured": tfl / self.bf16_peak, "active_experts_mean": stats["active"],
             "regime": regime_of(name)}
        reg = regime_of(name)
        if reg == "hbm":
            d["target"], d["target_frac"] = "HBM roofline (8 TB/s) >= 0.70", d["hbm_frac_of_8tbs"]
        elif reg == "tensor":
            d["target"], d["target_frac"] = "bf16 tensor peak (measured) >= 0.50", d["tensor_frac_of_measured"]
        else:
            bind = max(d["hbm_frac_of_8tbs"], d["tensor_frac_of_measured"])
            d["target"], d["target_frac"] = "the higher of the two (crossover)", bind
        return d

    def roofline(self, name, kernel_us, stats):
        si, T, _ = WORKLOADS[name]
        sh = self.synth.SHAPES[si]
        dominant = max(kernel_us, key=kernel_us.get)
        how = ("median of 5 replays of a CUDA graph of back-to-back single-stage launches rotating the workload's "
               "layers, CUDA events on the launch stream")
        return roofline_for(dominant, kernel_us[dominant], sh.H, sh.I, stats["gemv"], stats["mma_pairs"],
                            stats["mma"], self.hbm_peak, self.bf16_peak, self.peak_src == "measured",
                            ncu_traffic(name, dominant), how)

    def measure(self, name, steps, warmup, graph, n_sample, sample_layers, clocks=False, target_s=None):
        si, T, seeds = WORKLOADS[name]
        m = SHARED_NORM.get(name, 0)
        entries = [self.layer(si, sd, m) for sd in seeds]
        lnps, Ls = [e[0] for e in entries], [e[1] for e in entries]
        n_x = 8 if T <= 256 else 2
        xs = self.inputs(name, n_x)
        parity = self.parity(name, Ls, lnps, xs, n_sample, sample_layers) if self.rank == 0 else "rank 0 only"
        for sd in seeds[max(1, sample_layers):]:
            self.slim(si, sd, m)
        log(f"{name}: parity {parity}")
        stats, launches = self.routing_stats(name, Ls, xs)
        per_forward = T >= 1024
        if target_s:        # size the timed run to about target_s of device time
            ms1, _, _, _ = self.timed(name, Ls, xs, len(Ls) * n_x, 1, 0, False)
            est = ms1 / (len(Ls) * n_x)
            steps = int(max(len(Ls), min(4000, target_s * 1e3 / max(est, 1e-3))))
        ms, per_layer, clk, G = self.timed(name, Ls, xs, steps, warmup, graph, per_forward, clocks)
        if per_layer:
            t_med = float(np.median([v for v in per_layer if v is not None]))
            value = self.world * T / (t_med * 1e-3)
        else:
            t_med = ms / steps
            value = weak_value(self.world, T, steps, ms)
        kernel_us = self.kernel_times(name, Ls, xs)
        res = {"workload": workload_label(name, self.synth.SHAPES[si].H, self.synth.SHAPES[si].I,
                                          self.synth.SHAPES[si].E, self.synth.SHAPES[si].k, T, seeds),
               "tok_s": value, "ms_per_forward": t_med, "forwards_timed": steps, "graph_forwards": G,
               "layer": self.fractions(name, t_med, stats), "roofline": self.roofline(name, kernel_us, stats),
               "kernel_us": kernel_us, "parity": parity, "launches_per_forward": launches,
               "mma_pairs_mean": stats["mma_pairs"], "gemv_experts_mean": stats["gemv"]}
        if per_layer:
            res["per_seed_ms_per_forward"] = dict(zip([str(x) for x in seeds], per_layer))
            res["value_is"] = "median over seeds of each seed's tokens/s"
        return res, ms, clk, Ls, xs

    def e2e(self, name, Ls, xs, steps):
        torch = self.torch
        si, T, _ = WORKLOADS[name]
        H = self.synth.SHAPES[si].H
        x_host = [xs[li][r].cpu().pin_memory() for li in range(len(Ls)) for r in range(min(len(xs[li]), 2))]
        out_host = torch.empty((T, H), dtype=torch.int16).pin_memory()
        barrier(self.pg, torch)
        t0 = time.perf_counter()
        for i in range(steps):
            Ls[i % len(Ls)].forward_host(x_host[i % len(x_host)], out_host, T=T, stream=self.stream)
        el = max_over_ranks(self.pg, torch, time.perf_counter() - t0)
        return {"value": self.world * T * steps / el, "unit": "tok/s", "h2d_bytes_per_step": T * H * 2,
                "d2h_bytes_per_step": T * H * 2, "steps": steps,
                "how": "tfmoe_forward_host: pinned host x in, pinned host out, returns after the copy out"}

    def cpu_baseline(self, name, seconds, one_thread: bool = False):
        si, T, _ = WORKLOADS[name]
        lnp = self.layers[(si, WORKLOADS[name][2][0], SHARED_NORM.get(name, 0))][0]
        x_np = self.synth.make_x(self.synth.SHAPES[si], WORKLOADS[name][2][0], T)
        n = oracle_tokens_per_call(name)
        from oracle import oracle
        v, calls, tokens, el = oracle_rate(lnp, x_np, self.synth.SHAPES[si].k, n, seconds=seconds)
        d = {"value": v, "unit": "tok/s", "cores": oracle.max_threads(), "kind": "oracle", "cpu": cpu_description(),
             "sample": f"{calls} oracle calls of {min(n, T)} consecutive tokens of the T={T} batch ({tokens} tokens, "
                       f"{el:.1f} s)" + ("; tokens/s extrapolates to the full batch" if n < T else "")}
        if one_thread:
            v1, c1, t1, e1 = oracle_rate(lnp, x_np, self.synth.SHAPES[si].k, min(n, T), calls=1, nthreads=1)
            d["one_thread"] = {"value": v1, "unit": "tok/s", "cores": 1,
                               "sample": f"one oracle call of {min(n, T)} tokens ({e1:.1f} s)"}
        return d


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tfmoe", "reference"], default="tfmoe")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=None,
                    help=f"the timed workload (default {HEADLINE})")
    ap.add_argument("--flags", type=int, default=0, help="descriptor flags (1 = force GEMV, 2 = force MMA)")
    ap.add_argument("--gemv-max-tokens", type=int, default=0,
                    help="per-expert token count up to which the GEMV regime is used (0 = library default)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--graph", type=int, default=100, help="forwards per CUDA graph for small batches (0 = none)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    rank, world, local, pg = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    b = Bench(args, rank, world, local, pg)
    name = args.workload or HEADLINE
    per_config = (not args.no_per_config) and world == 1 and args.workload is None
    b.plan([name] + (PER_CONFIG if per_config else []))

    log(f"headline {name}")
    head, ms, clocks, Ls, xs = b.measure(name, args.steps, args.warmup, args.graph, n_sample=12, sample_layers=len(
        WORKLOADS[name][2]), clocks=True)
    e2e = b.e2e(name, Ls, xs, min(args.steps, 20 if WORKLOADS[name][1] > 256 else 500))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = b.cpu_baseline(name, args.cpu_seconds)

    pcs = None
    if per_config and rank == 0:
        pcs = {}
        for pc in PER_CONFIG:
            big = WORKLOADS[pc][1] > 256
            try:
                r, _, _, _, _ = b.measure(pc, 0, 3, args.graph, n_sample=8 if big else 64, sample_layers=1,
                                          target_s=0.3)
                log(f"{pc}: {r['tok_s']:.0f} tok/s, {r['ms_per_forward'] * 1e3:.1f} us per forward")
                if not args.no_cpu_baseline:
                    r["cpu_baseline"] = b.cpu_baseline(pc, 2.0,
                                                       one_thread=pc in ("tiny", "decode_t1", "decode", "zipf"))
            except (Exception, SystemExit) as exc:     # a per-config line fails alone, visibly
                log(f"{pc}: failed: {exc!r}")
                r = {"error": repr(exc)}
            pcs[pc] = r

    if rank == 0:
        si, T, seeds = WORKLOADS[name]
        line = {
            "metric": METRIC, "value": head["tok_s"], "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 activations, nvfp4 weights, fp32 accumulate", "data": "synthetic",
            "config": {"workload": head["workload"], "global_batch": T * world,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2: every forward reads its layer's active weights "
                             "(4.76 GB for the headline), and seeded layers rotate",
                       "value": head.get("value_is", "tokens over the timed device time"),
                       "flags": args.flags, "gemv_max_tokens": args.gemv_max_tokens or "default"},
            "roofline": head["roofline"],
            "layer": dict(head["layer"], kernel_us_graph=head["kernel_us"],
                          per_seed_ms_per_forward=head.get("per_seed_ms_per_forward")),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": head["launches_per_forward"] * args.steps,
            "clocks": clocks,
            "parity": head["parity"],
            "per_config": pcs,
            "setup_s": {"layers_generated_and_loaded": b.gen_s},
        }
        print(json.dumps(line), flush=True)
    for _, L in b.layers.values():
        L.close()
    if pg is not None:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
