#!/usr/bin/env python
"""Throughput of the ASP (deflated form) NVFP4 W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5]
                    [--impl qwam|reference] [--no-per-config]

Default workload (c5): one denoising step of the two-expert model, all of its
600 distinct linears in model order from one CUDA graph ("FastWAM UR3 3-task
— 4-bit quantisations", the paragraph under the top table: 2 experts x 30
blocks x {self q/k/v/o, cross q/k/v/o, ffn.0, ffn.2}):
  video expert   d 3072, ffn 14336, 4096 tokens, r = 0 (plain smoothed +
                 rotated NVFP4 path), Hadamard block 128
  action expert  d 1024, ffn 4096, 32 tokens, r = 32, block 128; its cross
                 k/v projections read the 4096-token context
One step = the whole set: every layer's activation prologue (smoothing, block
FWHT, rank-r projection and deflation, NVFP4 quantisation) and its tcgen05
block-scaled FP4 GEMM with the low-rank branch, global scales and bias in the
epilogue.  Weights are prepared offline, outside the timed region; their 3.1 GB
of FP4 codes and scales and the layers' 20 GB of activations are far above the
126 MB L2, so every step streams its operands from HBM.  The headline is
TFLOP/s of the step (GB/s beside it); the roofline object is that of the
dominant kernel group.

With the default workload on one GPU the line also carries per_config: the
single layers (c2 action attention 32 x 1024 -> 1024, c3 video attention
4096 x 3072 -> 3072 at r = 32 and r = 0, c4 video FFN up and down), the
action-expert half of the step (c5action), and the boundary's other arms on
the same layers (c3r0fp8 / c2fp8: the FP8 W8A8 arm, against the FP8 peak;
c2shared: the shared-weight arm; c3int4 / c2int4: the SVDQuant INT4 arm,
whose products run on the FP8 tensor-core kind), each with its own roofline,
cpu_baseline and e2e.  --workload <name> runs one of those alone.

Timing: CUDA events around K steps replayed from a CUDA graph (one untimed
replay first), barrier + synchronize on both sides, max over ranks.  Multi-GPU
runs are independent replicas (the layer needs no exchange between GPUs):
weak scaling.

--impl reference times the float64 CPU oracle (oracle/) on the same workload
and metric, on this host's cores: a deliberately slow correctness reference.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
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

from bit_w4a4_quantised_b200 import workloads  # noqa: E402

METRIC = "ASP-NVFP4 linear TFLOP/s and GB/s per layer, % of FP4/HBM roofline"
L2_BYTES = 126 * 10 ** 6
DTYPE = "nvfp4 (e2m1 x e4m3 block-16) GEMM, fp32 accumulate; bf16 in/out; bf16 rank-r branch"
DTYPE_FP8 = "fp8 e4m3 (per-tensor scales) GEMM, fp32 accumulate; bf16 in/out; bf16 rank-r branch"
DTYPE_INT4 = ("int4 group-64 (fp16 scales) levels as e4m3 on f8f6f4 tensor cores, exact group sums, fp32 "
              "rescale per group; bf16 in/out; bf16 rank-r branch")
DTYPES = {"nvfp4": DTYPE, "fp8": DTYPE_FP8, "int4": DTYPE_INT4}

STEP = dict(desc="one denoising step of the 2-expert model: 600 linears (video d 3072, ffn 14336, 4096 tokens, "
                 "r=0; action d 1024, ffn 4096, 32 tokens, cross k/v over the 4096-token context, r=32), b=128",
            unit="TFLOP/s", steps=20, warmup=3)

# seconds of timed oracle work in the reference arm of the whole step
REFERENCE_BUDGET_S = 90.0

SETS = {
    "c5action": dict(desc="one denoising step of the action expert: 300 linears (d 1024, ffn 4096, "
                          "32 tokens; cross k/v over the 4096-token context), r=32, b=128",
                     unit="GB/s", steps=20, warmup=3, cross_kv_context=True),
    "c5action32": dict(desc="one denoising step of the action expert: 300 linears (d 1024, ffn 4096, "
                            "every one at 32 tokens, cross k/v included), r=32, b=128",
                       unit="GB/s", steps=20, warmup=3, cross_kv_context=False),
}

WORKLOADS = {
    "c2": dict(make=lambda i, seed: workloads.c2_action_attn(seed=seed, layer=i),
               desc="action-expert attention projection, 32 tokens, 1024->1024, r=32, b=128",
               unit="GB/s", steps=200000, warmup=50),
    "c1": dict(make=lambda i, seed: workloads.draw_layer(
        "c1_tiny_64x256x256_r32_b16", 64, 256, 256, 32, 16, seed=seed, config_id=1, layer=i,
        n_outliers=4, outlier_scale=20.0),
        desc="tiny ASP layer, 64 tokens, 256->256, r=32, b=16", unit="GB/s", steps=200000, warmup=50),
    "c3": dict(make=lambda i, seed: workloads.c3_video_attn(32, seed=seed, layer=i),
               desc="video-expert attention projection, 4096 tokens, 3072->3072, r=32, b=128",
               unit="TFLOP/s", steps=2000, warmup=10),
    "c3r0": dict(make=lambda i, seed: workloads.c3_video_attn(0, seed=seed, layer=i),
                 desc="video-expert attention projection, 4096 tokens, 3072->3072, r=0, b=128",
                 unit="TFLOP/s", steps=2000, warmup=10),
    "c4up": dict(make=lambda i, seed: workloads.c4_video_ffn_up(seed=seed + i),
                 desc="video-expert FFN up, 4096 tokens, 3072->14336, r=32, b=128",
                 unit="TFLOP/s", steps=500, warmup=5),
    "c4down": dict(make=lambda i, seed: workloads.c4_video_ffn_down(seed=seed + i),
                   desc="video-expert FFN down, 4096 tokens, 14336->3072, r=32, b=128",
                   unit="TFLOP/s", steps=500, warmup=5),
    # the video FFN layers as the denoising step holds them (r = 0): --workload only, for
    # per-shape evidence on the step's video GEMM group
    "c5ffn0": dict(make=lambda i, seed: workloads.c5_layer(8, seed=seed + i),
                   desc="video-expert FFN up as in the denoising step, 4096 tokens, 3072->14336, r=0, b=128",
                   unit="TFLOP/s", steps=500, warmup=5),
    "c5ffn2": dict(make=lambda i, seed: workloads.c5_layer(9, seed=seed + i),
                   desc="video-expert FFN down as in the denoising step, 4096 tokens, 14336->3072, r=0, b=128",
                   unit="TFLOP/s", steps=500, warmup=5),
    # the other arms of the boundary on the same layers
    "c3r0fp8": dict(make=lambda i, seed: workloads.c3_video_attn(0, seed=seed, layer=i), fmt="fp8",
                    desc="FP8 W8A8 arm: video-expert attention projection, 4096 tokens, 3072->3072, r=0, b=128",
                    unit="TFLOP/s", steps=2000, warmup=10),
    "c2fp8": dict(make=lambda i, seed: workloads.c2_action_attn(seed=seed, layer=i), fmt="fp8",
                  desc="FP8 W8A8 arm: action-expert attention projection, 32 tokens, 1024->1024, r=32, b=128",
                  unit="GB/s", steps=200000, warmup=50),
    "c2shared": dict(make=lambda i, seed: workloads.c2_action_attn(seed=seed, layer=i), variant="shared",
                     desc="shared-weight arm: action-expert attention projection, 32 tokens, 1024->1024, r=32, "
                          "b=128", unit="GB/s", steps=200000, warmup=50),
    "c3int4": dict(make=lambda i, seed: workloads.c3_video_attn_int4(seed=seed, layer=i), fmt="int4",
                   variant="svdquant",
                   desc="SVDQuant INT4 arm: video-expert attention projection, 4096 tokens, 3072->3072, r=32, "
                        "no rotation", unit="TFLOP/s", steps=2000, warmup=10),
    "c2int4": dict(make=lambda i, seed: workloads.c2_action_attn_int4(seed=seed, layer=i), fmt="int4",
                   variant="svdquant",
                   desc="SVDQuant INT4 arm: action-expert attention projection, 32 tokens, 1024->1024, r=32, "
                        "no rotation", unit="GB/s", steps=200000, warmup=50),
}

# per_config entries of the default run: (steps, warm-up, seconds of oracle work)
PER_CONFIG = {"c2": (20000, 50, 8.0), "c3": (400, 10, 8.0), "c3r0": (400, 10, 8.0), "c4up": (100, 5, 8.0),
              "c4down": (100, 5, 8.0), "c5action": (10, 3, 8.0), "c3r0fp8": (400, 10, 6.0),
              "c2fp8": (20000, 50, 6.0), "c2shared": (20000, 50, 6.0), "c3int4": (400, 10, 6.0),
              "c2int4": (20000, 50, 6.0)}


def set_layers(wl):
    """The set's layer specs and their indices into the step's 600 linears."""
    specs = workloads.c5_layer_specs(cross_kv_context=wl["cross_kv_context"])
    idx = [i for i, sp in enumerate(specs) if sp.name.startswith("action.")]
    return specs, idx


def step_kinds(specs):
    """The distinct layer kinds of a step: {(expert, M, K, N, r): [indices]}."""
    kinds = {}
    for i, sp in enumerate(specs):
        kinds.setdefault((sp.name.split(".")[0], sp.M, sp.K, sp.N, sp.r), []).append(i)
    return kinds


# ---------------------------------------------------------------------------
# Algorithmic work per layer (minimal bytes / flops of the method itself).
# ---------------------------------------------------------------------------
def elem_bytes(fmt):
    """Bytes of one quantised element with its share of the scales, as the
    format stores it: NVFP4 0.5 + 1/16 (E4M3 per 16), FP8 1, INT4 0.5 + 2/64
    (fp16 per 64; the device holds the levels as bytes, which the algorithmic
    count does not credit)."""
    return {"nvfp4": 0.5625, "fp8": 1.0, "int4": 0.53125}[fmt]


def layer_bytes(M, K, N, r, fmt="nvfp4"):
    """x (bf16) + the quantised weight with its scales (elem_bytes) + L (bf16)
    + V (fp32) + s (fp32) + bias (bf16) + y (bf16)."""
    wb = elem_bytes(fmt)
    return 2 * M * K + wb * N * K + 2 * N * r + 4 * K * r + 4 * K + 2 * N + 2 * M * N


def layer_flops(M, K, N, r):
    return 2 * M * N * K + 2 * M * N * r + 4 * M * K * r


def prologue_bytes(M, K, N, r, fmt="nvfp4"):
    """Reads x, V, s; writes the quantised activation (elem_bytes) and u'."""
    eb = elem_bytes(fmt)
    return 2 * M * K + 4 * K * r + 4 * K + eb * M * K + 2 * M * r


def gemm_bytes(M, K, N, r, fmt="nvfp4"):
    """Reads the quantised activations and weights (elem_bytes), L, u', bias;
    writes y."""
    eb = elem_bytes(fmt)
    return eb * M * K + eb * N * K + 2 * N * r + 2 * M * r + 2 * N + 2 * M * N


def gemm_flops(M, K, N, r):
    return 2 * M * N * K + 2 * M * N * r


def prologue_flops(M, K, N, r):
    return 4 * M * K * r


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def fp8_peak(peaks, timed_alone):
    """Dense FP8 peak = 2 x the bf16 peak (nominal 4.5 / 2.25 PFLOP/s)."""
    burst, sust = 2.0 * peaks["bf16_tflops"], 2.0 * peaks["bf16_tflops_sustained"]
    which = "burst" if timed_alone else "sustained"
    note = (f"dense FP8 = 2 x {peaks['source']} {which} cuBLAS bf16 (nominal ratio 4.5/2.25 PFLOP/s); "
            f"the other fraction against 2 x the {'sustained' if timed_alone else 'burst'} figure")
    return (burst, sust, note) if timed_alone else (sust, burst, note)


def fp4_peak(peaks, timed_alone):
    """Dense NVFP4 peak = 4 x the bf16 peak (nominal 9 / 2.25 PFLOP/s): the
    burst figure for a kernel timed alone, the sustained one for a kernel
    timed inside a long step.  Returns (peak, other, note)."""
    burst, sust = 4.0 * peaks["bf16_tflops"], 4.0 * peaks["bf16_tflops_sustained"]
    if timed_alone:
        return burst, sust, (f"dense FP4 = 4 x {peaks['source']} burst cuBLAS bf16 ({peaks['bf16_tflops']} TFLOP/s; "
                             f"nominal ratio 9/2.25 PFLOP/s); frac_sustained against 4 x the sustained figure")
    return sust, burst, (f"dense FP4 = 4 x {peaks['source']} sustained cuBLAS bf16 ({peaks['bf16_tflops_sustained']} "
                         f"TFLOP/s, kernels timed inside a long step; nominal ratio 9/2.25 PFLOP/s); frac_burst "
                         f"against 4 x the burst figure")


# Sources every kernel's traffic depends on (launch planning included), and the
# file that builds each kernel family.
SHARED_SOURCES = ("common.cuh", "quant.cuh", "kernels.h", "api.cu")
KERNEL_SOURCES = {"fp4_gemm": ("gemm.cu",), "prologue": ("prologue.cu",), "onepass": ("prologue_wide.cu",),
                  "wide_prologue": ("prologue_wide.cu",), "group_gemm": ("group_gemm.cu",)}


def sources_digest(names):
    """sha256 over the named files of csrc/ (name and bytes, in sorted order)."""
    h = hashlib.sha256()
    for name in sorted(names):
        with open(os.path.join(ROOT, "bit_w4a4_quantised_b200", "csrc", name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()


def traffic_sources(family):
    return sorted(set(SHARED_SOURCES) | set(KERNEL_SOURCES[family]))


def recorded_traffic(workload, kernel):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    sources of the captured kernel (its .cu file, the shared headers and the
    launch planning) changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{workload}:{kernel}")
    if not e or not e.get("sources"):
        return None
    try:
        if e.get("sources_sha256") != sources_digest(e["sources"]):
            return None
    except OSError:
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.gpu_id = gpu_id

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id:
            cmd[1:1] = ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        time.sleep(0.15)
        self.out = ""
        if self.proc:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            p = [t.strip() for t in line.split(",")]
            if len(p) < 7:
                continue
            try:
                rows.append((float(p[0]), float(p[1]), float(p[2]) if p[2] not in ("[N/A]", "N/A") else 0.0, p[3:7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------------------
# Oracle timing (CPU).
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        import threadpoolctl
        n = [i["num_threads"] for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:
        return None


def oracle_call(prep, case, fmt="nvfp4"):
    """The per-call work of the layer in the float64 oracle: activation side,
    FP4 (FP8) product on dequantised operands, low-rank branch, bias."""
    from oracle import asp
    act = asp.activation_prologue(case.x, case.s, case.V, case.b, fmt=fmt, deflated=fmt != "int4")
    y = asp.nvfp4_gemm(act["deq"], prep["deq"]) + act["u"] @ prep["L"].T + case.bias.astype("float64")[None, :]
    return y


def oracle_prepare(c, fmt="nvfp4", variant="deflated"):
    from oracle import asp
    if variant == "shared":
        return asp.prepare_weight_shared(c.W, c.s, c.V, c.b)
    return asp.prepare_weight(c.W, c.s, c.V, c.b, fmt=fmt)


def time_oracle(cases, budget_s, fmt="nvfp4", variant="deflated"):
    """Run oracle calls over the given cases (weights prepared outside the
    clock) until budget_s of CPU work has elapsed; returns (calls, seconds)."""
    preps = [oracle_prepare(c, fmt, variant) for c in cases]
    n, t = 0, 0.0
    while True:
        c, p = cases[n % len(cases)], preps[n % len(cases)]
        t0 = time.perf_counter()
        oracle_call(p, c, fmt)
        t += time.perf_counter() - t0
        n += 1
        if t >= budget_s:
            return n, t


def oracle_step_sampler(specs, seed, cross_kv_context=True):
    """One layer of every distinct kind of a step, its weights prepared here
    (outside any clock).  Returns (run, kinds): run() makes one oracle call of
    each kind and returns (the step's seconds extrapolated by the kinds'
    counts, the oracle seconds actually spent)."""
    from oracle import asp
    prepared = []
    for _, members in sorted(step_kinds(specs).items()):
        c = workloads.c5_layer(members[0], seed, cross_kv_context=cross_kv_context)
        prepared.append((asp.prepare_weight(c.W, c.s, c.V, c.b), c, len(members)))

    def run():
        step_s, spent = 0.0, 0.0
        for prep, c, count in prepared:
            t0 = time.perf_counter()
            oracle_call(prep, c)
            dt = time.perf_counter() - t0
            spent += dt
            step_s += dt * count
        return step_s, spent

    return run, len(prepared)


def time_oracle_step(specs, seed, cross_kv_context=True):
    """One sample of oracle_step_sampler: (step seconds, seconds spent, kinds)."""
    run, kinds = oracle_step_sampler(specs, seed, cross_kv_context)
    step_s, spent = run()
    return step_s, spent, kinds


def cores_used():
    return {"affinity": len(os.sched_getaffinity(0)), "blas_threads": blas_threads()}


# ---------------------------------------------------------------------------
def per_unit(value_units, seconds, unit):
    if unit == "GB/s":
        return value_units / seconds / 1e9
    return value_units / seconds / 1e12


def replica_instance_seed(rank, i):
    """Layer-instance index of instance i on a replica rank: every rank draws
    its own weights and activations (no two ranks share an instance)."""
    return rank * 100003 + i


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank timings (the slowest rank sets the job's
    time).  dist is torch.distributed when the job has more than one rank."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


class Ctx:
    """The GPU run's plumbing: device, stream, ranks, the binding."""

    def __init__(self, args):
        import torch
        import torch.distributed as dist
        from bit_w4a4_quantised_b200 import binding as qw
        self.torch, self.dist, self.qw = torch, dist, qw
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torch.distributed.run (one process per GPU)")
        torch.cuda.set_device(local)
        self.dev = torch.device("cuda", local)
        if self.world > 1:
            import datetime
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=self.dev)
        self.stream = torch.cuda.Stream(device=self.dev)
        self.uuid = None
        try:
            u = str(torch.cuda.get_device_properties(self.dev).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_ranks(self, vals):
        return max_over_ranks(vals, self.dist if self.world > 1 else None, self.dev)

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def timed_graphs(ctx, plan):
    """Replay [(graph, reps), ...] between CUDA events on the bench stream,
    after one untimed replay of each graph (graph upload and first-launch
    cost stay outside), with the clock sampler running.  Returns (ms, clocks)."""
    torch = ctx.torch
    with torch.cuda.stream(ctx.stream):
        for g, reps in plan:
            if reps:
                g.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx.barrier()
    torch.cuda.synchronize()
    with ClockSampler(ctx.uuid) as clk:
        with torch.cuda.stream(ctx.stream):
            t0.record()
            for g, reps in plan:
                for _ in range(reps):
                    g.replay()
            t1.record()
        torch.cuda.synchronize()
    ctx.barrier()
    return t0.elapsed_time(t1), clk.summary()


def hbm_roof(kernel, nbytes, dur_ms, peaks):
    achieved = nbytes / (dur_ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "peak_note": f"{peaks['source']} HBM copy bandwidth", "frac": achieved / peaks["hbm_gbs"],
            "kernel": kernel}


def tensor_roof(kernel, flops, dur_ms, peaks, timed_alone, fmt="nvfp4"):
    achieved = flops / (dur_ms / 1e3) / 1e12
    # the INT4 arm's products run on kind::f8f6f4: the FP8 peak
    peak, other, note = (fp4_peak if fmt == "nvfp4" else fp8_peak)(peaks, timed_alone)
    r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "peak_note": note,
         "frac": achieved / peak, "kernel": kernel}
    r["frac_sustained" if timed_alone else "frac_burst"] = achieved / other
    return r


# ---------------------------------------------------------------------------
# One layer, rotating over enough instances to exceed L2.
# ---------------------------------------------------------------------------
def bench_layer(ctx, args, name, steps, warmup, cpu_budget):
    torch, qw = ctx.torch, ctx.qw
    wl = WORKLOADS[name]
    fmt, variant = wl.get("fmt", "nvfp4"), wl.get("variant", "deflated")
    probe = wl["make"](0, args.seed)
    M, K, N, r, hb = probe.M, probe.K, probe.N, probe.r, probe.b
    warmup = max(3, warmup)
    wdev = {"nvfp4": 0.5625, "fp8": 1.0, "int4": 1.0625}[fmt]  # device bytes per weight
    per_inst = (wdev * N * K + 2 * N * max(r, 1) + 8 * K * max(r, 1) + 4 * K + 2 * N
                + 2 * M * K + 2 * M * N)
    P = args.instances or max(1, min(256, math.ceil(1.5 * L2_BYTES / per_inst)))
    handles, xs, ys = [], [], []
    for i in range(P):
        c = probe if i == 0 and ctx.rank == 0 else wl["make"](replica_instance_seed(ctx.rank, i), args.seed)
        W = torch.from_numpy(c.W).to(ctx.dev).to(torch.bfloat16)
        s = torch.from_numpy(c.s).to(ctx.dev)
        V = torch.from_numpy(c.V).to(ctx.dev) if c.r else None
        bias = torch.from_numpy(c.bias).to(ctx.dev).to(torch.bfloat16)
        handles.append(qw.prepare_weight(W, s, V, bias, c.b, variant=variant, fmt=fmt))
        xs.append(torch.from_numpy(c.x).to(ctx.dev).to(torch.bfloat16))
        ys.append(torch.empty((M, N), dtype=torch.bfloat16, device=ctx.dev))
        del W, s, V, bias
    plan = qw.plan_info(M, handles[0])
    working_set = P * per_inst
    torch.cuda.synchronize()

    def step(j, evs=None):
        k = j % P
        if evs is not None:
            evs[0].record()
        qw.prologue(xs[k], handles[k])
        if evs is not None:
            evs[1].record()
        qw.gemm(M, handles[k], ys[k])
        if evs is not None:
            evs[2].record()

    with torch.cuda.stream(ctx.stream):
        for j in range(warmup):
            step(j)
    torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during warm-up")

    # the timed graph has no event nodes (they would sit between the two
    # kernels and stop the GEMM from starting early); per-kernel durations come
    # from a copy of it with events, replayed right after
    G = min(steps, P)
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(G)]
    g_main, g_prof = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_main, stream=ctx.stream):
        for j in range(G):
            step(j)
    with torch.cuda.graph(g_prof, stream=ctx.stream):
        for j in range(G):
            step(j, ev[j])
    graphs = [(g_main, steps // G)]
    if steps % G:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=ctx.stream):
            for j in range(steps % G):
                step(j)
        graphs.append((g_rem, 1))
    torch.cuda.synchronize()
    ms, clocks = timed_graphs(ctx, graphs)
    with torch.cuda.stream(ctx.stream):
        for _ in range(max(1, min(steps // G, 20))):
            g_prof.replay()
    torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during the timed region")
    pro_ms = [ev[j][0].elapsed_time(ev[j][1]) for j in range(G)]
    gem_ms = [ev[j][1].elapsed_time(ev[j][2]) for j in range(G)]

    # end to end through the public API with host buffers
    E = min(steps, 2000 if M <= 128 else 50)
    hx = [xs[k].cpu().pin_memory() for k in range(min(P, 16))]
    hy = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(min(P, 16))]
    dx = [torch.empty_like(xs[0]) for _ in range(2)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e(j):
        dx[j % 2].copy_(hx[j % len(hx)], non_blocking=True)
        qw.linear(dx[j % 2], handles[j % P], ys[j % P])
        hy[j % len(hy)].copy_(ys[j % P], non_blocking=True)

    with torch.cuda.stream(ctx.stream):
        for j in range(3):
            e2e(j)
    torch.cuda.synchronize()
    ctx.barrier()
    with torch.cuda.stream(ctx.stream):
        e0.record()
        for j in range(E):
            e2e(j)
        e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    ms, e2e_ms = ctx.max_ranks([ms, e2e_ms])

    unit = wl["unit"]
    lb, lf = layer_bytes(M, K, N, r, fmt), layer_flops(M, K, N, r)
    units = lb if unit == "GB/s" else lf
    value = per_unit(units * steps * ctx.world, ms / 1e3, unit)
    peaks = measured_peaks()
    pro_avg, gem_avg = sum(pro_ms) / G, sum(gem_ms) / G
    dominant = "gemm" if gem_avg >= pro_avg else "prologue"
    gemm_kernel = "group_gemm_kernel" if fmt == "int4" else "fp4_gemm_kernel"
    if dominant == "gemm" and unit == "TFLOP/s":
        roof = tensor_roof(gemm_kernel, gemm_flops(M, K, N, r), gem_avg, peaks, timed_alone=True, fmt=fmt)
    elif dominant == "gemm":
        roof = hbm_roof(gemm_kernel, gemm_bytes(M, K, N, r, fmt), gem_avg, peaks)
    else:
        roof = hbm_roof("prologue_kernel", prologue_bytes(M, K, N, r, fmt), pro_avg, peaks)
    roof["traffic"] = recorded_traffic(name, roof["kernel"])
    roof["avg_launch_us"] = (gem_avg if dominant == "gemm" else pro_avg) * 1e3
    roof["duration_note"] = ("CUDA events around each kernel in replays of the timed graph with event nodes "
                             "added, right after the timed region")
    roof["kernel_share"] = {"prologue": pro_avg / (pro_avg + gem_avg), "gemm": gem_avg / (pro_avg + gem_avg)}
    roof["kernel_us"] = {"prologue": pro_avg * 1e3, "gemm": gem_avg * 1e3}

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": ctx.world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPES[fmt],
        "data": "synthetic (seeded; shapes of the Fast-WAM experts, random-init weights)",
        "config": {"workload": f"{name}: {wl['desc']}", "M": M, "K": K, "N": N, "r": r, "hadamard_block": hb,
                   "parallelism": f"replicas x{ctx.world}",
                   "l2": f"rotating {P} distinct layer instances, {working_set / 1e6:.0f} MB > 126 MB L2; "
                         f"CUDA graph"},
        "per_layer": {"us": ms / steps * 1e3, "GB/s": lb * steps / (ms / 1e3) / 1e9,
                      "TFLOP/s": lf * steps / (ms / 1e3) / 1e12, "alg_bytes": lb, "alg_flops": lf},
        "roofline": roof,
        "e2e": {"value": per_unit(units * E * ctx.world, e2e_ms / 1e3, unit), "unit": unit,
                "h2d_bytes_per_step": 2 * M * K, "d2h_bytes_per_step": 2 * M * N, "steps": E,
                "note": "qwam_linear per step with that step's x copied in from pinned host memory and y read back"},
        "gpu_launches": plan["kernels"] * steps,
        "plan": plan,
        "clocks": clocks,
    }
    if ctx.rank == 0 and ctx.world == 1:
        cases = [probe] + [wl["make"](i, args.seed) for i in range(1, 3 if M <= 128 else 1)]
        n, t = time_oracle(cases, cpu_budget, fmt, variant)
        cores = cores_used()
        line["cpu_baseline"] = {"value": per_unit(units * n, t, unit), "unit": unit,
                                "cores": cores["blas_threads"] or cores["affinity"], "kind": "oracle",
                                "sample": f"{n} float64 oracle layer calls ({t:.1f} s) on {len(cases)} instance(s); "
                                          f"weights prepared outside the clock"}
    else:
        line["cpu_baseline"] = None
    for h in handles:
        h.destroy()
    del xs, ys, g_main, g_prof
    torch.cuda.empty_cache()
    return line


# ---------------------------------------------------------------------------
# A set of distinct layers run in model order from one CUDA graph: the whole
# denoising step (both experts) or the action expert's half of it.
# ---------------------------------------------------------------------------
def _run_layers(ctx, layers, steps, warmup):
    """Time `steps` replays of one graph holding every layer's two launches in
    order; returns (ms, clocks, prologue ms per layer, GEMM ms per layer)."""
    torch, qw = ctx.torch, ctx.qw

    def run_all(evs=None):
        for k, L in enumerate(layers):
            if evs is not None:
                evs[k][0].record()
            qw.prologue(L["x"], L["h"])
            if evs is not None:
                evs[k][1].record()
            qw.gemm(L["M"], L["h"], L["y"])
            if evs is not None:
                evs[k][2].record()

    with torch.cuda.stream(ctx.stream):
        for _ in range(max(3, warmup)):
            run_all()
    torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in layers]
    g_main, g_prof = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_main, stream=ctx.stream):
        run_all()
    with torch.cuda.graph(g_prof, stream=ctx.stream):
        run_all(ev)
    torch.cuda.synchronize()
    ms, clocks = timed_graphs(ctx, [(g_main, steps)])
    with torch.cuda.stream(ctx.stream):
        g_prof.replay()
    torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during the timed region")
    pro = [e[0].elapsed_time(e[1]) for e in ev]
    gem = [e[1].elapsed_time(e[2]) for e in ev]
    del g_main, g_prof
    return ms, clocks, pro, gem


def _prepare(ctx, d):
    """Prepare one device-drawn layer; keeps x, a y buffer and the handle."""
    qw = ctx.qw
    h = qw.prepare_weight(d["W"], d["s"], d["V"], d["bias"], d["b"])
    y = ctx.torch.empty((d["M"], d["N"]), dtype=ctx.torch.bfloat16, device=ctx.dev)
    return {"name": d.get("name", ""), "M": d["M"], "K": d["K"], "N": d["N"], "r": d["r"], "x": d["x"], "y": y,
            "h": h}


def _group_roofs(layers, pro, gem, peaks, timed_alone):
    """Per (expert, kernel) group: its share of the step and its roofline
    (GEMM groups of 4096-token layers against the FP4 peak, the rest HBM)."""
    groups = {}
    for L, p, g in zip(layers, pro, gem):
        ex = L["name"].split(".")[0] or "layer"
        sh = (L["M"], L["K"], L["N"], L["r"])
        for kern, dur in (("prologue", p), ("gemm", g)):
            e = groups.setdefault((ex, kern), {"ms": 0.0, "bytes": 0.0, "flops": 0.0, "launches": 0})
            e["ms"] += dur
            e["launches"] += 1
            e["bytes"] += (prologue_bytes if kern == "prologue" else gemm_bytes)(*sh)
            e["flops"] += (prologue_flops if kern == "prologue" else gemm_flops)(*sh)
    total = sum(e["ms"] for e in groups.values())
    out = {}
    for (ex, kern), e in groups.items():
        kname = "fp4_gemm_kernel" if kern == "gemm" else "prologue_kernel"
        big_m = all(L["M"] > 128 for L in layers if (L["name"].split(".")[0] or "layer") == ex)
        if kern == "gemm" and big_m:
            roof = tensor_roof(kname, e["flops"], e["ms"], peaks, timed_alone)
        else:
            roof = hbm_roof(kname, e["bytes"], e["ms"], peaks)
        roof.update(share=e["ms"] / total, launches=e["launches"], total_us=e["ms"] * 1e3,
                    avg_launch_us=e["ms"] / e["launches"] * 1e3)
        out[f"{ex}.{kern}"] = roof
    return out


def bench_set(ctx, args, name, steps, warmup, cpu_budget):
    """The action-expert half of the step (c5action / c5action32)."""
    torch, qw = ctx.torch, ctx.qw
    wl = SETS[name]
    specs, idx = set_layers(wl)
    ctxkv = wl["cross_kv_context"]
    shapes = [(specs[i].M, specs[i].K, specs[i].N, specs[i].r) for i in idx]
    set_bytes = sum(layer_bytes(*sh) for sh in shapes)
    set_flops = sum(layer_flops(*sh) for sh in shapes)
    layers = []
    for i in idx:
        c = workloads.c5_layer(i, args.seed + ctx.rank * 100003, cross_kv_context=ctxkv)
        d = {"name": c.name, "M": c.M, "K": c.K, "N": c.N, "r": c.r, "b": c.b,
             "x": torch.from_numpy(c.x).to(ctx.dev).to(torch.bfloat16),
             "W": torch.from_numpy(c.W).to(ctx.dev).to(torch.bfloat16), "s": torch.from_numpy(c.s).to(ctx.dev),
             "V": torch.from_numpy(c.V).to(ctx.dev) if c.r else None,
             "bias": torch.from_numpy(c.bias).to(ctx.dev).to(torch.bfloat16)}
        layers.append(_prepare(ctx, d))
    plans = [qw.plan_info(L["M"], L["h"]) for L in layers]
    torch.cuda.synchronize()
    ms, clocks, pro, gem = _run_layers(ctx, layers, steps, warmup)
    e2e_ms, E, h2d, d2h = _set_e2e(ctx, layers, steps, every_layer_io=True)
    ms, e2e_ms = ctx.max_ranks([ms, e2e_ms])
    peaks = measured_peaks()
    unit = wl["unit"]
    value = per_unit(set_bytes * steps * ctx.world, ms / 1e3, unit)
    groups = _group_roofs(layers, pro, gem, peaks, timed_alone=False)
    dom = max(groups, key=lambda k: groups[k]["share"])
    roof = dict(groups[dom], group=dom, traffic=recorded_traffic(name, dom),
                duration_note="CUDA events around each kernel of every layer, one replay of the set's graph with "
                              "event nodes added, right after the timed region",
                set_frac=value / ctx.world / peaks["hbm_gbs"])
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": ctx.world, "steps": steps,
        "warmup": max(3, warmup), "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE,
        "data": "synthetic (seeded; shapes of the Fast-WAM action expert, random-init weights)",
        "config": {"workload": f"{name}: {wl['desc']}", "layers": len(idx),
                   "tokens": {"action": 32, "cross_kv": 4096 if ctxkv else 32}, "d": 1024, "ffn": 4096, "r": 32,
                   "hadamard_block": 128, "parallelism": f"replicas x{ctx.world}",
                   "l2": f"{len(idx)} distinct layers, {sum(0.5625 * s[1] * s[2] for s in shapes) / 1e9:.2f} GB of "
                         f"FP4 weights > 126 MB L2; CUDA graph"},
        "per_step": {"us": ms / steps * 1e3, "alg_bytes": set_bytes, "alg_flops": set_flops,
                     "layers_us_median": statistics.median(p + g for p, g in zip(pro, gem)) * 1e3},
        "roofline": roof,
        "kernel_groups": groups,
        "e2e": {"value": per_unit(set_bytes * E * ctx.world, e2e_ms / 1e3, unit), "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": E,
                "note": "qwam_linear for every layer with its x copied in from pinned host memory and its y read "
                        "back, every step"},
        "gpu_launches": sum(pl["kernels"] for pl in plans) * steps,
        "clocks": clocks,
    }
    if ctx.rank == 0 and ctx.world == 1:
        sample = [workloads.c5_layer(idx[k], args.seed, cross_kv_context=ctxkv) for k in (0, 8)]
        n, t = time_oracle(sample, cpu_budget)
        sb = sum(layer_bytes(c.M, c.K, c.N, c.r) for c in sample)
        cores = cores_used()
        line["cpu_baseline"] = {"value": per_unit(sb / len(sample) * n, t, unit), "unit": unit,
                                "cores": cores["blas_threads"] or cores["affinity"], "kind": "oracle",
                                "sample": f"{n} float64 oracle calls ({t:.1f} s) alternating the set's first "
                                          f"self-attention projection and first ffn.0 (32 tokens); weights "
                                          f"prepared outside the clock"}
    else:
        line["cpu_baseline"] = None
    for L in layers:
        L["h"].destroy()
    del layers
    torch.cuda.empty_cache()
    return line


def _set_e2e(ctx, layers, steps, every_layer_io):
    """The set through the public call (qwam_linear per layer, eager).  With
    every_layer_io each layer's x comes from pinned host memory and its y goes
    back every step; otherwise only the first layer of each expert takes its x
    from the host and the last layer of each expert returns its y (the other
    layers' inputs stay on the device, as activations do in a forward pass).
    Returns (ms for E steps, E, h2d bytes per step, d2h bytes per step)."""
    torch, qw = ctx.torch, ctx.qw
    if every_layer_io:
        ins, outs = list(range(len(layers))), list(range(len(layers)))
    else:
        experts = {}
        for k, L in enumerate(layers):
            experts.setdefault(L["name"].split(".")[0], []).append(k)
        ins = [ks[0] for ks in experts.values()]
        outs = [ks[-1] for ks in experts.values()]
    hx = {k: layers[k]["x"].cpu().pin_memory() for k in ins}
    hy = {k: torch.empty(layers[k]["y"].shape, dtype=torch.bfloat16).pin_memory() for k in outs}
    E = max(1, min(steps, 5))

    def e2e_step():
        for k, L in enumerate(layers):
            if k in hx:
                L["x"].copy_(hx[k], non_blocking=True)
            qw.linear(L["x"], L["h"], L["y"])
            if k in hy:
                hy[k].copy_(L["y"], non_blocking=True)

    with torch.cuda.stream(ctx.stream):
        e2e_step()
    torch.cuda.synchronize()
    ctx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(ctx.stream):
        e0.record()
        for _ in range(E):
            e2e_step()
        e1.record()
    torch.cuda.synchronize()
    h2d = sum(2 * layers[k]["M"] * layers[k]["K"] for k in ins)
    d2h = sum(2 * layers[k]["M"] * layers[k]["N"] for k in outs)
    return e0.elapsed_time(e1), E, h2d, d2h


def bench_step(ctx, args, steps, warmup, cpu_budget):
    """The whole denoising step: 600 linears, both experts, one CUDA graph."""
    torch, qw = ctx.torch, ctx.qw
    specs = workloads.c5_layer_specs(cross_kv_context=True)
    shapes = [(sp.M, sp.K, sp.N, sp.r) for sp in specs]
    step_bytes = sum(layer_bytes(*sh) for sh in shapes)
    step_flops = sum(layer_flops(*sh) for sh in shapes)
    layers = []
    t_prep = time.perf_counter()
    for i in range(len(specs)):
        d = workloads.c5_layer_device(i, ctx.dev, seed=args.seed + ctx.rank * 100003, cross_kv_context=True)
        layers.append(_prepare(ctx, d))
        del d
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    t_prep = time.perf_counter() - t_prep
    plans = [qw.plan_info(L["M"], L["h"]) for L in layers]
    ms, clocks, pro, gem = _run_layers(ctx, layers, steps, warmup)
    e2e_ms, E, h2d, d2h = _set_e2e(ctx, layers, steps, every_layer_io=False)
    ms, e2e_ms = ctx.max_ranks([ms, e2e_ms])
    peaks = measured_peaks()
    value = per_unit(step_flops * steps * ctx.world, ms / 1e3, "TFLOP/s")
    groups = _group_roofs(layers, pro, gem, peaks, timed_alone=False)
    dom = max(groups, key=lambda k: groups[k]["share"])
    roof = dict(groups[dom], group=dom, traffic=recorded_traffic("c5", dom),
                duration_note="CUDA events around each kernel of every layer, one replay of the step's graph with "
                              "event nodes added, right after the timed region; achieved = the group's algorithmic "
                              "flops (or bytes) over its summed durations")
    weights = sum(0.5625 * s[1] * s[2] + 2 * s[2] * s[3] for s in shapes)
    act = sum(2 * s[0] * s[1] + 2 * s[0] * s[2] for s in shapes)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ctx.world, "steps": steps,
        "warmup": max(3, warmup), "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE,
        "data": "synthetic (seeded on the device with the input recipe; shapes of the Fast-WAM experts, "
                "random-init weights)",
        "config": {"workload": f"c5: {STEP['desc']}", "layers": len(specs),
                   "video": {"layers": 300, "tokens": 4096, "d": 3072, "ffn": 14336, "r": 0},
                   "action": {"layers": 300, "tokens": 32, "cross_kv_tokens": 4096, "d": 1024, "ffn": 4096, "r": 32},
                   "hadamard_block": 128, "parallelism": f"replicas x{ctx.world}",
                   "l2": f"{len(specs)} distinct layers: {weights / 1e9:.2f} GB of FP4 weights + L, "
                         f"{act / 1e9:.1f} GB of activations > 126 MB L2; one CUDA graph"},
        "per_step": {"us": ms / steps * 1e3, "TFLOP/s": step_flops * steps / (ms / 1e3) / 1e12,
                     "GB/s": step_bytes * steps / (ms / 1e3) / 1e9, "alg_bytes": step_bytes,
                     "alg_flops": step_flops, "prepare_s": t_prep},
        "roofline": roof,
        "kernel_groups": groups,
        "e2e": {"value": per_unit(step_flops * E * ctx.world, e2e_ms / 1e3, "TFLOP/s"), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": E,
                "note": "qwam_linear for all 600 layers in order (eager, no graph); each expert's first input "
                        "copied in from pinned host memory and its last output read back every step, the other "
                        "inputs resident on the device as a forward pass keeps its activations"},
        "gpu_launches": sum(pl["kernels"] for pl in plans) * steps,
        "clocks": clocks,
    }
    if ctx.rank == 0 and ctx.world == 1:
        step_s, spent, nk = time_oracle_step(specs, args.seed)
        cores = cores_used()
        line["cpu_baseline"] = {"value": step_flops / step_s / 1e12, "unit": "TFLOP/s",
                                "cores": cores["blas_threads"] or cores["affinity"], "kind": "oracle",
                                "sample": f"one float64 oracle call of each of the step's {nk} distinct layer kinds "
                                          f"({spent:.1f} s), extrapolated to the 600 layers by the kinds' counts "
                                          f"({step_s:.0f} s per step); weights prepared outside the clock"}
    else:
        line["cpu_baseline"] = None
    for L in layers:
        L["h"].destroy()
    del layers
    torch.cuda.empty_cache()
    return line


# ---------------------------------------------------------------------------
# The reference arm: the float64 oracle on this host's cores.
# ---------------------------------------------------------------------------
def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    cores = cores_used()
    ncores = cores["blas_threads"] or cores["affinity"]
    line = {"impl": "reference", "metric": METRIC, "n_gpus": args.gpus, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64"}
    if args.workload == "c5":
        specs = workloads.c5_layer_specs(cross_kv_context=True)
        step_flops = sum(layer_flops(sp.M, sp.K, sp.N, sp.r) for sp in specs)
        run, nk = oracle_step_sampler(specs, args.seed)
        K_req = args.steps if args.steps is not None else STEP["steps"]
        W_req = args.warmup if args.warmup is not None else STEP["warmup"]
        for _ in range(W_req):
            run()
        samples, walls = [], []
        t_start = time.perf_counter()
        while len(samples) < K_req and (not samples or time.perf_counter() - t_start < REFERENCE_BUDGET_S):
            step_s, spent = run()
            samples.append(step_s)
            walls.append(spent)
        step_s = statistics.fmean(samples)
        value = step_flops / step_s / 1e12
        line.update(value=value, unit="TFLOP/s", steps=len(samples), warmup=W_req,
                    ms_per_step=statistics.fmean(walls) * 1e3,
                    data="synthetic (seeded; shapes of the Fast-WAM experts)",
                    config={"workload": f"c5: {STEP['desc']}", "layers": len(specs),
                            "parallelism": f"replicas x{args.gpus}"},
                    cpu_baseline={"value": value, "unit": "TFLOP/s", "cores": ncores, "kind": "oracle",
                                  "sample": f"each step one oracle call of each of the step's {nk} distinct layer "
                                            f"kinds (ms_per_step is that wall time), extrapolated to the 600 layers "
                                            f"by the kinds' counts ({step_s:.0f} s per denoising step); "
                                            f"{len(samples)} timed steps of {K_req} requested (bounded to "
                                            f"~{REFERENCE_BUDGET_S:.0f} s) after {W_req} warm-up steps; weights "
                                            f"prepared outside the clock"})
    elif args.workload in SETS:
        from oracle import asp
        wl = SETS[args.workload]
        specs, idx = set_layers(wl)
        set_bytes = sum(layer_bytes(specs[i].M, specs[i].K, specs[i].N, specs[i].r) for i in idx)
        n, t, nbytes = 0, 0.0, 0.0
        while t < 60.0 and n < len(idx):
            c = workloads.c5_layer(idx[n], args.seed, cross_kv_context=wl["cross_kv_context"])
            prep = asp.prepare_weight(c.W, c.s, c.V, c.b)
            t0 = time.perf_counter()
            oracle_call(prep, c)
            t += time.perf_counter() - t0
            nbytes += layer_bytes(c.M, c.K, c.N, c.r)
            n += 1
        value = per_unit(nbytes, t, wl["unit"])
        line.update(value=value, unit=wl["unit"], steps=1, warmup=0, ms_per_step=set_bytes / value / 1e6,
                    data="synthetic (seeded; shapes of the Fast-WAM action expert)",
                    config={"workload": f"{args.workload}: {wl['desc']}", "layers": len(idx),
                            "parallelism": f"replicas x{args.gpus}"},
                    cpu_baseline={"value": value, "unit": wl["unit"], "cores": ncores, "kind": "oracle",
                                  "sample": f"the first {n} of the set's {len(idx)} layers in model order "
                                            f"({t:.1f} s of oracle work, bounded to ~60 s), weights prepared outside "
                                            f"the clock"})
    else:
        from oracle import asp
        wl = WORKLOADS[args.workload]
        unit = wl["unit"]
        fmt, variant = wl.get("fmt", "nvfp4"), wl.get("variant", "deflated")
        cases = [wl["make"](i, args.seed) for i in range(2)]
        c0 = cases[0]
        units_per_step = (layer_bytes(c0.M, c0.K, c0.N, c0.r, fmt) if unit == "GB/s"
                          else layer_flops(c0.M, c0.K, c0.N, c0.r))
        preps = [oracle_prepare(c, fmt, variant) for c in cases]
        W_req = args.warmup if args.warmup is not None else wl["warmup"]
        warm, t_w = 0, time.perf_counter()
        while warm < max(1, W_req) and (warm == 0 or time.perf_counter() - t_w < 30.0):
            oracle_call(preps[warm % 2], cases[warm % 2], fmt)
            warm += 1
        t0 = time.perf_counter()
        oracle_call(preps[0], cases[0], fmt)
        first = time.perf_counter() - t0
        K_req = args.steps if args.steps is not None else wl["steps"]
        steps = max(1, min(K_req, int(60.0 / max(first, 1e-6))))
        t0 = time.perf_counter()
        for i in range(steps):
            oracle_call(preps[i % 2], cases[i % 2], fmt)
        dt = time.perf_counter() - t0
        value = per_unit(units_per_step * steps, dt, unit)
        line.update(value=value, unit=unit, steps=steps, warmup=warm, ms_per_step=dt / steps * 1e3,
                    data="synthetic (seeded; shapes of the Fast-WAM experts)",
                    config={"workload": f"{args.workload}: {wl['desc']}", "M": c0.M, "K": c0.K, "N": c0.N,
                            "r": c0.r, "hadamard_block": c0.b, "parallelism": f"replicas x{args.gpus}"},
                    cpu_baseline={"value": value, "unit": unit, "cores": ncores, "kind": "oracle",
                                  "sample": f"{steps} oracle layer calls of {K_req} requested (bounded to ~60 s) "
                                            f"after {warm} warm-up calls of {W_req} requested (bounded to ~30 s), "
                                            f"weights prepared outside the clock"})
    line["e2e"] = {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="c5", choices=["c5"] + sorted(WORKLOADS) + sorted(SETS))
    ap.add_argument("--impl", default="qwam", choices=["qwam", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--instances", type=int, default=0,
                    help="distinct layer instances to rotate over (default: enough to exceed L2)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-per-config", action="store_true", help="with c5: skip the per_config entries")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    ctx = Ctx(args)
    if args.workload == "c5":
        line = bench_step(ctx, args, args.steps if args.steps is not None else STEP["steps"],
                          args.warmup if args.warmup is not None else STEP["warmup"], args.cpu_budget)
        if ctx.world == 1 and not args.no_per_config:
            per = {}
            for name, (st, wu, cb) in PER_CONFIG.items():
                if name in SETS:
                    per[name] = bench_set(ctx, args, name, st, wu, cb)
                else:
                    per[name] = bench_layer(ctx, args, name, st, wu, cb)
            line["per_config"] = per
            line["gpu_launches_per_config"] = sum(v["gpu_launches"] for v in per.values())
    elif args.workload in SETS:
        wl = SETS[args.workload]
        line = bench_set(ctx, args, args.workload, args.steps if args.steps is not None else wl["steps"],
                         args.warmup if args.warmup is not None else wl["warmup"], args.cpu_budget)
    else:
        wl = WORKLOADS[args.workload]
        line = bench_layer(ctx, args, args.workload, args.steps if args.steps is not None else wl["steps"],
                           args.warmup if args.warmup is not None else wl["warmup"], args.cpu_budget)
    if ctx.rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
