#!/usr/bin/env python
"""Throughput of the ASP (deflated form) NVFP4 W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2]
                    [--impl qwam|reference]

One step = one layer call on one batch of synthetic input: the activation
prologue (smoothing, block FWHT, rank-r projection and deflation, NVFP4
quantisation) and the tcgen05 block-scaled FP4 GEMM with the low-rank branch,
global scales and bias in its epilogue.  Weights are prepared offline, outside
the timed region.  Steps rotate over enough distinct layer instances (weights
and activations) that the working set exceeds the 126 MB L2, so every step
streams its operands from HBM.  Timing: CUDA events around K steps replayed
from a CUDA graph, barrier + synchronize on both sides, max over ranks.

The default workload is the action-expert attention projection
(32 tokens, 1024 -> 1024, rank 32, Hadamard block 128).  Multi-GPU runs are
independent replicas (the layer needs no exchange between GPUs): weak scaling.

--workload c5action runs one denoising step of the action expert as a set:
its 300 distinct linears (30 blocks x self q/k/v/o, cross q/k/v/o, ffn.0,
ffn.2; d 1024, ffn 4096, 32 tokens, cross k/v over the 4096-token context,
r 32) back to back in one CUDA graph, programmatic dependent launch between
kernels; one step = the whole set, reported as aggregate GB/s against HBM
(0.28 GB of distinct FP4 weights per step, above L2); --workload c5action32 is the
same set with the cross k/v projections at 32 tokens (the other reading of the
config).

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


def _c5_like(i, seed):
    return workloads.c5_layer(i, seed)


SETS = {
    "c5action": dict(desc="one denoising step of the action expert: 300 linears (d 1024, ffn 4096, "
                          "32 tokens; cross k/v over the 4096-token context), r=32, b=128",
                     unit="GB/s", steps=20, warmup=3, cross_kv_context=True),
    "c5action32": dict(desc="one denoising step of the action expert: 300 linears (d 1024, ffn 4096, "
                            "every one at 32 tokens, cross k/v included), r=32, b=128",
                       unit="GB/s", steps=20, warmup=3, cross_kv_context=False),
}


def set_layers(wl):
    """The set's layer specs and their indices into the step's 600 linears."""
    specs = workloads.c5_layer_specs(cross_kv_context=wl["cross_kv_context"])
    idx = [i for i, sp in enumerate(specs) if sp.name.startswith("action.")]
    return specs, idx


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
}


# ---------------------------------------------------------------------------
# Algorithmic work per layer (minimal bytes / flops of the method itself).
# ---------------------------------------------------------------------------
def layer_bytes(M, K, N, r):
    """x (bf16) + packed W_d with E4M3 scales (0.5625 B/weight) + L (bf16) +
    V (fp32) + s (fp32) + bias (bf16) + y (bf16)."""
    return 2 * M * K + 0.5625 * N * K + 2 * N * r + 4 * K * r + 4 * K + 2 * N + 2 * M * N


def layer_flops(M, K, N, r):
    return 2 * M * N * K + 2 * M * N * r + 4 * M * K * r


def prologue_bytes(M, K, N, r):
    """Reads x, V, s; writes FP4 codes + scales (0.5625 B/element) and u'."""
    return 2 * M * K + 4 * K * r + 4 * K + 0.5625 * M * K + 2 * M * r


def gemm_bytes(M, K, N, r):
    """Reads FP4 activations + scales, W_d + scales, L, u', bias; writes y."""
    return 0.5625 * M * K + 0.5625 * N * K + 2 * N * r + 2 * M * r + 2 * N + 2 * M * N


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


def csrc_digest():
    files = sorted(glob.glob(os.path.join(ROOT, "bit_w4a4_quantised_b200", "csrc", "*")))
    h = hashlib.sha256()
    for p in files:
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload, kernel):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel sources changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{workload}:{kernel}")
    if not e or e.get("csrc_sha256") != csrc_digest():
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


def oracle_call(prep, case):
    """The per-call work of the layer in the float64 oracle: activation side,
    FP4 product on dequantised operands, low-rank branch, bias."""
    from oracle import asp
    act = asp.activation_prologue(case.x, case.s, case.V, case.b)
    y = asp.nvfp4_gemm(act["deq"], prep["deq"]) + act["u"] @ prep["L"].T + case.bias.astype("float64")[None, :]
    return y


def time_oracle(cases, budget_s):
    """Run oracle calls over the given cases (weights prepared outside the
    clock) until budget_s of CPU work has elapsed; returns (calls, seconds)."""
    from oracle import asp
    preps = [asp.prepare_weight(c.W, c.s, c.V, c.b) for c in cases]
    n, t = 0, 0.0
    while True:
        c, p = cases[n % len(cases)], preps[n % len(cases)]
        t0 = time.perf_counter()
        oracle_call(p, c)
        t += time.perf_counter() - t0
        n += 1
        if t >= budget_s:
            return n, t


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


def run_reference(args, wl, shape):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    M, K, N, r, _ = shape
    unit = wl["unit"]
    units_per_step = layer_bytes(M, K, N, r) if unit == "GB/s" else layer_flops(M, K, N, r)
    cases = [wl["make"](i, args.seed) for i in range(2)]
    from oracle import asp
    preps = [asp.prepare_weight(c.W, c.s, c.V, c.b) for c in cases]
    for i in range(args.warmup if args.warmup is not None else 1):
        oracle_call(preps[i % 2], cases[i % 2])
        if unit != "GB/s":
            break  # large layers: one warm-up call is plenty on a CPU
    t0 = time.perf_counter()
    oracle_call(preps[0], cases[0])
    first = time.perf_counter() - t0
    K_req = args.steps if args.steps is not None else wl["steps"]
    steps = max(1, min(K_req, int(60.0 / max(first, 1e-6))))
    t0 = time.perf_counter()
    for i in range(steps):
        oracle_call(preps[i % 2], cases[i % 2])
    dt = time.perf_counter() - t0
    value = per_unit(units_per_step * steps, dt, unit)
    cores = cores_used()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": steps, "warmup": args.warmup, "ms_per_step": dt / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the Fast-WAM experts)",
        "config": config_of(args, wl, shape, None),
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores["blas_threads"] or cores["affinity"],
                         "kind": "oracle",
                         "sample": f"{steps} oracle layer calls of {K_req} requested (bounded to ~60 s), "
                                   f"weights prepared outside the clock"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(args, wl, shape, instances):
    M, K, N, r, b = shape
    cfg = {"workload": f"{args.workload}: {wl['desc']}", "M": M, "K": K, "N": N, "r": r,
           "hadamard_block": b, "parallelism": f"replicas x{args.gpus}"}
    if instances is not None:
        cfg["l2"] = instances
    return cfg


def run_set(args, wl):
    """A layer set (one denoising step of the action expert): every step runs
    all of its distinct layers once, in model order, from one CUDA graph."""
    specs, idx = set_layers(wl)
    unit = wl["unit"]
    ctx = wl["cross_kv_context"]
    shapes = [(specs[i].M, specs[i].K, specs[i].N, specs[i].r) for i in idx]
    set_bytes = sum(layer_bytes(*sh) for sh in shapes)
    set_flops = sum(layer_flops(*sh) for sh in shapes)
    cfg = {"workload": f"{args.workload}: {wl['desc']}", "layers": len(idx),
           "tokens": {"action": 32, "cross_kv": 4096 if ctx else 32}, "d": 1024, "ffn": 4096, "r": 32,
           "hadamard_block": 128, "parallelism": f"replicas x{args.gpus}"}
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_set_reference(args, wl, idx, set_bytes, cfg)

    import torch
    import torch.distributed as dist
    from bit_w4a4_quantised_b200 import binding as qw

    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
    steps = args.steps if args.steps is not None else wl["steps"]
    warmup = max(3, args.warmup if args.warmup is not None else wl["warmup"])

    handles, xs, ys = [], [], []
    for i in idx:
        c = workloads.c5_layer(i, args.seed + rank * 100003, cross_kv_context=ctx)
        handles.append(qw.prepare_weight(torch.from_numpy(c.W).to(dev).to(torch.bfloat16),
                                         torch.from_numpy(c.s).to(dev),
                                         torch.from_numpy(c.V).to(dev) if c.r else None,
                                         torch.from_numpy(c.bias).to(dev).to(torch.bfloat16), c.b))
        xs.append(torch.from_numpy(c.x).to(dev).to(torch.bfloat16))
        ys.append(torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev))
    plans = [qw.plan_info(sh[0], h) for sh, h in zip(shapes, handles)]
    n_layers = len(idx)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def run_all(evs=None):
        for k in range(n_layers):
            if evs is not None:
                evs[k][0].record()
            qw.prologue(xs[k], handles[k])
            if evs is not None:
                evs[k][1].record()
            qw.gemm(shapes[k][0], handles[k], ys[k])
            if evs is not None:
                evs[k][2].record()

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            run_all()
    torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during warm-up")
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(n_layers)]
    g_main, g_prof = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_main, stream=stream):
        run_all()
    with torch.cuda.graph(g_prof, stream=stream):
        run_all(ev)
    torch.cuda.synchronize()

    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        pass
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_uuid) as clk:
        with torch.cuda.stream(stream):
            t_start.record()
            for _ in range(steps):
                g_main.replay()
            t_end.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    with torch.cuda.stream(stream):
        g_prof.replay()
    torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during the timed region")
    pro_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(n_layers)]
    gem_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(n_layers)]

    # end to end through the public API: each layer's x in from pinned host
    # memory, its y back out, every step
    hx = [x.cpu().pin_memory() for x in xs]
    hy = [torch.empty(y.shape, dtype=torch.bfloat16).pin_memory() for y in ys]
    dx = [torch.empty_like(x) for x in xs]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    E = max(1, min(steps, 5))

    def e2e_step():
        for k in range(n_layers):
            dx[k].copy_(hx[k], non_blocking=True)
            qw.linear(dx[k], handles[k], ys[k])
            hy[k].copy_(ys[k], non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with torch.cuda.stream(stream):
        e0.record()
        for _ in range(E):
            e2e_step()
        e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], dist if world > 1 else None, dev)

    peaks = measured_peaks()
    value = per_unit(set_bytes * steps * world, ms / 1e3, unit)
    # dominant kernel over the set: the one with more total device time;
    # achieved = its algorithmic bytes over the set / its summed durations
    pro_t, gem_t = sum(pro_ms), sum(gem_ms)
    dominant = "gemm" if gem_t >= pro_t else "prologue"
    kb = sum((gemm_bytes if dominant == "gemm" else prologue_bytes)(*sh) for sh in shapes)
    dur = gem_t if dominant == "gemm" else pro_t
    achieved = kb / (dur / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "peak_note": f"{peaks['source']} HBM copy bandwidth", "frac": achieved / peaks["hbm_gbs"],
            "kernel": "fp4_gemm_kernel" if dominant == "gemm" else "prologue_kernel", "traffic": None,
            "avg_launch_us": dur / n_layers * 1e3,
            "duration_note": "CUDA events around each kernel of every layer, one replay of the set's graph "
                             "with event nodes added, right after the timed region",
            "kernel_share": {"prologue": pro_t / (pro_t + gem_t), "gemm": gem_t / (pro_t + gem_t)},
            "set_frac": value / world / peaks["hbm_gbs"]}
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 block-16) GEMM, fp32 accumulate; bf16 in/out; bf16 rank-r branch",
        "data": "synthetic (seeded; shapes of the Fast-WAM action expert, random-init weights)",
        "config": dict(cfg, l2=f"{n_layers} distinct layers, "
                              f"{sum(0.5625 * sh[1] * sh[2] for sh in shapes) / 1e9:.2f} GB of FP4 weights "
                              f"> 126 MB L2; CUDA graph"),
        "per_step": {"us": ms / steps * 1e3, "alg_bytes": set_bytes, "alg_flops": set_flops,
                     "layers_us_median": statistics.median(p + g for p, g in zip(pro_ms, gem_ms)) * 1e3},
        "roofline": roof,
        "e2e": {"value": per_unit(set_bytes * E * world, e2e_ms / 1e3, unit), "unit": unit,
                "h2d_bytes_per_step": sum(2 * sh[0] * sh[1] for sh in shapes),
                "d2h_bytes_per_step": sum(2 * sh[0] * sh[2] for sh in shapes), "steps": E},
        "gpu_launches": sum(pl["kernels"] for pl in plans) * steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1:
        sample = [workloads.c5_layer(idx[k], args.seed, cross_kv_context=ctx) for k in (0, 8)]
        n, t = time_oracle(sample, args.cpu_budget)
        sb = sum(layer_bytes(c.M, c.K, c.N, c.r) for c in sample)
        cores = cores_used()
        line["cpu_baseline"] = {"value": per_unit(sb / len(sample) * n, t, unit), "unit": unit,
                                "cores": cores["blas_threads"] or cores["affinity"], "kind": "oracle",
                                "sample": f"{n} float64 oracle calls ({t:.1f} s) alternating the set's first "
                                          f"self-attention projection and first ffn.0 (32 tokens); weights "
                                          f"prepared outside the clock"}
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        del g_main, g_prof
        dist.destroy_process_group()
    return 0


def run_set_reference(args, wl, idx, set_bytes, cfg):
    """The oracle on a bounded sample of the set: its layers in order, as many
    as fit in ~60 s of CPU work, reported in the set's unit."""
    from oracle import asp
    unit = wl["unit"]
    t_budget = 60.0
    n, t, nbytes = 0, 0.0, 0.0
    while t < t_budget and n < len(idx):
        c = workloads.c5_layer(idx[n], args.seed, cross_kv_context=wl["cross_kv_context"])
        prep = asp.prepare_weight(c.W, c.s, c.V, c.b)
        t0 = time.perf_counter()
        oracle_call(prep, c)
        t += time.perf_counter() - t0
        nbytes += layer_bytes(c.M, c.K, c.N, c.r)
        n += 1
    value = per_unit(nbytes, t, unit)
    cores = cores_used()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": 1, "warmup": 0, "ms_per_step": t / n * len(idx) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes of the Fast-WAM action expert)", "config": cfg,
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores["blas_threads"] or cores["affinity"],
                         "kind": "oracle",
                         "sample": f"the first {n} of the set's {len(idx)} layers in model order "
                                   f"({t:.1f} s of oracle work, bounded to ~60 s), weights prepared outside the "
                                   f"clock; ms_per_step extrapolates to the whole set"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="c2", choices=sorted(WORKLOADS) + sorted(SETS))
    ap.add_argument("--impl", default="qwam", choices=["qwam", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a CUDA graph")
    ap.add_argument("--instances", type=int, default=0,
                    help="distinct layer instances to rotate over (default: enough to exceed L2)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args()
    if args.workload in SETS:
        return run_set(args, SETS[args.workload])
    wl = WORKLOADS[args.workload]
    probe = wl["make"](0, args.seed)
    shape = (probe.M, probe.K, probe.N, probe.r, probe.b)
    if args.impl == "reference":
        return run_reference(args, wl, shape)

    import torch
    import torch.distributed as dist
    from bit_w4a4_quantised_b200 import binding as qw

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torch.distributed.run (one process per GPU)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    M, K, N, r, hb = shape
    steps = args.steps if args.steps is not None else wl["steps"]
    warmup = args.warmup if args.warmup is not None else wl["warmup"]
    warmup = max(3, warmup)

    # ---- instances: enough distinct layers that the rotation exceeds L2 ----
    per_inst = (N * K / 2 + N * K / 16 + 2 * N * max(r, 1) + 8 * K * max(r, 1) + 4 * K + 2 * N
                + 2 * M * K + 2 * M * N)
    P = args.instances or max(1, min(256, math.ceil(1.5 * L2_BYTES / per_inst)))
    handles, xs, ys = [], [], []
    for i in range(P):
        c = probe if i == 0 and rank == 0 else wl["make"](replica_instance_seed(rank, i), args.seed)
        x = torch.from_numpy(c.x).to(dev).to(torch.bfloat16)
        W = torch.from_numpy(c.W).to(dev).to(torch.bfloat16)
        s = torch.from_numpy(c.s).to(dev)
        V = torch.from_numpy(c.V).to(dev) if c.r else None
        bias = torch.from_numpy(c.bias).to(dev).to(torch.bfloat16)
        handles.append(qw.prepare_weight(W, s, V, bias, c.b))
        xs.append(x)
        ys.append(torch.empty((M, N), dtype=torch.bfloat16, device=dev))
        del W, s, V, bias
    plan = qw.plan_info(M, handles[0])
    working_set = P * per_inst

    stream = torch.cuda.Stream(device=dev)
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

    with torch.cuda.stream(stream):
        for j in range(warmup):
            step(j)
    torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during warm-up")

    G = min(steps, P)
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(G)]
    use_graph = not args.no_graph
    graphs = []
    if use_graph:
        # the timed graph has no event nodes (they would sit between the two
        # kernels and stop the GEMM from starting early); per-kernel durations
        # come from a copy of it with events, replayed right after
        g_main = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_main, stream=stream):
            for j in range(G):
                step(j)
        graphs.append(g_main)
        g_prof = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_prof, stream=stream):
            for j in range(G):
                step(j, ev[j])
        graphs.append(g_prof)
        rem = steps % G
        if rem:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem, stream=stream):
                for j in range(rem):
                    step(j)
        reps = steps // G
        torch.cuda.synchronize()

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        pass
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_uuid) as clk:
        with torch.cuda.stream(stream):
            t_start.record()
            if use_graph:
                for _ in range(reps):
                    g_main.replay()
                if steps % G:
                    g_rem.replay()
            else:
                for j in range(steps):
                    step(j, ev[j % G] if j >= steps - G else None)
            t_end.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    if use_graph:
        with torch.cuda.stream(stream):
            for _ in range(max(1, min(reps, 20))):
                g_prof.replay()
        torch.cuda.synchronize()
    if qw.device_error():
        raise RuntimeError("device wait expired during the timed region")
    pro_ms = [ev[j][0].elapsed_time(ev[j][1]) for j in range(G)]
    gem_ms = [ev[j][1].elapsed_time(ev[j][2]) for j in range(G)]

    # ---- end to end through the public API with host buffers ----
    E = min(steps, 2000 if M <= 128 else 50)
    hx = [xs[k].cpu().pin_memory() for k in range(min(P, 16))]
    hy = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(min(P, 16))]
    dx = [torch.empty_like(xs[0]) for _ in range(2)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for j in range(3):
            dx[j % 2].copy_(hx[j % len(hx)], non_blocking=True)
            qw.linear(dx[j % 2], handles[j % P], ys[j % P])
            hy[j % len(hy)].copy_(ys[j % P], non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with torch.cuda.stream(stream):
        e0.record()
        for j in range(E):
            dx[j % 2].copy_(hx[j % len(hx)], non_blocking=True)
            qw.linear(dx[j % 2], handles[j % P], ys[j % P])
            hy[j % len(hy)].copy_(ys[j % P], non_blocking=True)
        e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], dist if world > 1 else None, dev)

    unit = wl["unit"]
    lb, lf = layer_bytes(M, K, N, r), layer_flops(M, K, N, r)
    units = lb if unit == "GB/s" else lf
    value = per_unit(units * steps * world, ms / 1e3, unit)
    e2e_value = per_unit(units * E * world, e2e_ms / 1e3, unit)

    # ---- roofline of the dominant kernel ----
    peaks = measured_peaks()
    pro_avg, gem_avg = sum(pro_ms) / G, sum(gem_ms) / G
    dominant = "gemm" if gem_avg >= pro_avg else "prologue"
    dur_ms = gem_avg if dominant == "gemm" else pro_avg
    if dominant == "gemm" and unit == "TFLOP/s":
        achieved = gemm_flops(M, K, N, r) / (dur_ms / 1e3) / 1e12
        peak = 4.0 * peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "peak_note": f"dense FP4 = 4 x {peaks['source']} sustained cuBLAS bf16 "
                             f"({peaks['bf16_tflops_sustained']} TFLOP/s; nominal ratio 9/2.25 PFLOP/s)"}
    else:
        kb = gemm_bytes(M, K, N, r) if dominant == "gemm" else prologue_bytes(M, K, N, r)
        achieved = kb / (dur_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "peak_note": f"{peaks['source']} HBM copy bandwidth"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = "fp4_gemm_kernel" if dominant == "gemm" else "prologue_kernel"
    roof["traffic"] = recorded_traffic(args.workload, roof["kernel"])
    roof["avg_launch_us"] = dur_ms * 1e3
    roof["duration_note"] = ("CUDA events around each kernel in replays of the timed graph with event nodes "
                             "added, right after the timed region" if use_graph else
                             "CUDA events around each kernel in the last steps of the timed region")
    roof["kernel_share"] = {"prologue": pro_avg / (pro_avg + gem_avg), "gemm": gem_avg / (pro_avg + gem_avg)}

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 block-16) GEMM, fp32 accumulate; bf16 in/out; bf16 rank-r branch",
        "data": "synthetic (seeded; shapes of the Fast-WAM experts, random-init weights)",
        "config": config_of(args, wl, shape, f"rotating {P} distinct layer instances, "
                                              f"{working_set / 1e6:.0f} MB > 126 MB L2; "
                                              f"{'CUDA graph' if use_graph else 'eager'}"),
        "per_layer": {"us": ms / steps * 1e3, "GB/s": lb * steps / (ms / 1e3) / 1e9,
                      "TFLOP/s": lf * steps / (ms / 1e3) / 1e12, "alg_bytes": lb, "alg_flops": lf},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": 2 * M * K,
                "d2h_bytes_per_step": 2 * M * N, "steps": E},
        "gpu_launches": plan["kernels"] * steps,
        "plan": plan,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1:
        cases = [probe] + [wl["make"](i, args.seed) for i in range(1, 3 if M <= 128 else 1)]
        n, t = time_oracle(cases, args.cpu_budget)
        cores = cores_used()
        line["cpu_baseline"] = {"value": per_unit(units * n, t, unit), "unit": unit,
                                "cores": cores["blas_threads"] or cores["affinity"], "kind": "oracle",
                                "sample": f"{n} float64 oracle layer calls ({t:.1f} s) on {len(cases)} instance(s); "
                                          f"weights prepared outside the clock"}
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        del graphs
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
