"""Benchmark of the SVDQuant W4A4 + rank-32 linear layer on B200.

One step = one pass of the whole hot path over one batch: the fused
down-projection + quantize kernel (K1) and the NVFP4 GEMM with the fused
up-projection + bias epilogue (K2), on the FLUX.1-shaped attention output
projection (M = 4608 tokens, K = N = 3072, rank 32, NVFP4 g16/E4M3), inputs
resident in HBM, L2 flushed between steps outside the timed events (a 256 MiB
write, then a read of the same buffer so that no dirty lines of the flush are
left for the timed kernels to write back).  The value is whole-job TFLOP/s of the layer's algorithmic work
2MNK + 2M*32*(K+N), device-timed with CUDA events on the launch stream, max
over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: replicas only (each rank runs its own tokens; the layer has no
exchange step), launched by torchrun; scaling is weak.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fused W4A4+rank-32 linear TFLOPS, % NVFP4 peak; µs/layer vs unfused"
WORKLOAD = "attn_out"
RANK = 32
NOMINAL_FP4_DENSE_TFLOPS = 9000.0
FP4_OVER_BF16 = 4.0          # nominal dense ratio (9 PF / 2.25 PF)


def layer_flops(M, K, N, r=RANK):
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def k2_flops(M, K, N, r=RANK):
    return 2.0 * M * N * K + 2.0 * M * r * N


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def profile_traffic():
    """DRAM bytes (read + write) per K2 launch from the committed ncu summary,
    or None when the summary is missing or was taken on different K2 source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "k2_gemm_attn_out.md")
    src = os.path.join(ROOT, "w4a4_diffusion_transformer_b200", "csrc", "k2_gemm.cu")
    try:
        text = open(path).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if f"k2_gemm.cu: {sha}" not in text:
            return None
        for line in text.splitlines():
            if line.startswith("dram_bytes_per_launch:"):
                return int(line.split(":")[1])
    except Exception:
        return None
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._idx = device_index
        self._period = period_s
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self._idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            names = {
                "hw_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwSlowdown", 0x8),
                "hw_thermal_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                "sw_thermal_slowdown": getattr(pynvml, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                "sw_power_cap": getattr(pynvml, "nvmlClocksEventReasonSwPowerCap", 0x4),
                "hw_power_brake_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
            }

            def run():
                while not self._stop.is_set():
                    try:
                        self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
                        mask = fn(h)
                        for n, bit in names.items():
                            if mask & bit:
                                self.reasons.add(n)
                    except Exception as e:       # keep sampling best-effort
                        self.error = str(e)
                    time.sleep(self._period)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
        except Exception as e:
            self.error = str(e)
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "nvml", **({"error": self.error} if self.error and not self.samples else {})}


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_baseline(d, M, K, N, target_s=10.0):
    """The CPU oracle (NumPy float64) as it stands, on a bounded sample."""
    from oracle import svdq_oracle as o
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    p = o.prepare(d["W"], d["bias"], d["Xc"])           # offline step, not timed
    X = d["X"]
    reps, rows, t0 = 0, 0, time.perf_counter()
    while True:
        o.forward(p, X)
        reps += 1
        rows += M
        if time.perf_counter() - t0 >= target_s:
            break
    dt = time.perf_counter() - t0
    return {"value": layer_flops(rows, K, N) / dt / 1e12, "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{reps} x full {M}-token forward of {WORKLOAD} (oracle quantize + float64 matmul), "
                      f"{dt:.1f} s on the host"}


def run_reference(args):
    """Reference arm: the CPU oracle timed on the host, on bounded samples."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synthetic as syn
    from oracle import svdq_oracle as o
    d = syn.layer(WORKLOAD)
    shp = d["shape"]
    M, K, N = shp.M, shp.K, shp.N
    p = o.prepare(d["W"], d["bias"], d["Xc"])
    rows = 256                                             # bounded sample per step
    X = d["X"][:rows]
    for _ in range(args.warmup):
        o.forward(p, X)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.forward(p, X)
    dt = time.perf_counter() - t0
    val = layer_flops(rows, K, N) * args.steps / dt / 1e12
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    out = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic",
           "config": {"workload": f"{WORKLOAD} {M}x{K}->{N} NVFP4 g16 E4M3 r{RANK}", "M": M, "K": K, "N": N,
                      "rank": RANK, "parallelism": "replicas"},
           "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                            "sample": f"{rows} of {M} tokens per step, oracle forward (NumPy float64)"},
           "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch

    import synthetic as syn
    import w4a4_diffusion_transformer_b200 as pkg
    from w4a4_diffusion_transformer_b200 import build as pkg_build

    world, rank, local = dist_setup(args.gpus)
    if rank == 0:
        pkg_build.build()
    barrier(world)
    pkg.load()
    dev = torch.cuda.current_device()

    d = syn.layer(WORKLOAD)
    shp = d["shape"]
    M, K, N = shp.M, shp.K, shp.N
    L = pkg.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]),
                          fmt="nvfp4", rank=RANK, device=dev)
    stream = torch.cuda.current_stream()
    x = torch.from_numpy(d["X"]).to(torch.bfloat16).cuda()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    wsb = L.workspace_bytes(M)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    # the two kernels' intermediate buffers for the split (per-kernel timed) calls
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(L.act_scale_bytes(M), dtype=torch.uint8, device="cuda")
    xl = torch.empty((M, RANK), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_sink = torch.empty(1, dtype=torch.int64, device="cuda")

    def flush_l2(i):
        flush.fill_(i & 0xFF)                                     # evict: write > L2
        torch.sum(flush.view(torch.int64), dim=0, keepdim=True, out=flush_sink)   # clean the lines

    def step_fused():
        L.quantize_act(x, M, codes, scales, xl, stream, 0)
        L.gemm(codes, scales, xl, M, y, stream, 0)

    def time_variant(fn, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            flush_l2(i)
            evs[i][0].record(stream)
            fn()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / n

    # ---- warm-up
    for _ in range(args.warmup):
        step_fused()
    L.forward(x, M, y, ws, wsb, stream, pkg.FWD_CHECK)
    torch.cuda.synchronize()

    # ---- timed region: exactly `steps` fused steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        for i in range(args.steps):
            flush_l2(i)
            ev[i][0].record(stream)
            L.quantize_act(x, M, codes, scales, xl, stream, 0)
            ev[i][1].record(stream)
            L.gemm(codes, scales, xl, M, y, stream, 0)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    k1_ms = [a.elapsed_time(b) for a, b, _ in ev]
    k2_ms = [b.elapsed_time(c) for _, b, c in ev]
    step_ms = sum(k1_ms) / args.steps + sum(k2_ms) / args.steps
    step_ms_max = allreduce_max(step_ms, world)
    k2_avg = sum(k2_ms) / args.steps
    k1_avg = sum(k1_ms) / args.steps
    value = layer_flops(M, K, N) * world / (step_ms_max * 1e-3) / 1e12

    # ---- measurement variants (outside the timed region): bare GEMM and unfused layer
    n_var = max(50, min(500, args.steps))

    def bare():
        L.quantize_act(x, M, codes, scales, xl, stream, 1)
        L.gemm(codes, scales, xl, M, y, stream, pkg.FWD_NO_BRANCH)

    def unfused():
        L.forward(x, M, y, ws, wsb, stream, pkg.FWD_UNFUSED)

    def bare_gemm():
        L.gemm(codes, scales, xl, M, y, stream, pkg.FWD_NO_BRANCH)

    bare_ms = time_variant(bare, n_var)
    unfused_ms = time_variant(unfused, n_var)
    L.quantize_act(x, M, codes, scales, xl, stream, 0)
    bare_k2_ms = time_variant(bare_gemm, n_var)
    L.check(stream)

    # ---- end to end through the public API with host buffers
    xh = torch.from_numpy(d["X"]).to(torch.bfloat16).pin_memory()
    yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    n_e2e = max(20, min(200, args.steps))
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
    for i in range(n_e2e):
        flush_l2(i)
        e2e_ev[i][0].record(stream)
        x.copy_(xh, non_blocking=True)
        L.forward(x, M, y, ws, wsb, stream, 0)
        yh.copy_(y, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(sum(a.elapsed_time(b) for a, b in e2e_ev) / n_e2e, world)

    peaks, peak_src = measured_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    k2_achieved = k2_flops(M, K, N) / (k2_avg * 1e-3) / 1e12
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD} {M}x{K}->{N} NVFP4 g16 E4M3 r{RANK}", "M": M, "K": K, "N": N,
                   "rank": RANK, "parallelism": "replicas" if world > 1 else "single",
                   "l2": "flushed between steps outside the timed events (256 MiB write + read)"},
        "us_per_layer": step_ms_max * 1e3, "k1_us": k1_avg * 1e3, "k2_us": k2_avg * 1e3,
        "pct_nvfp4_peak": {"of_measured": value / world / fp4_peak, "of_nominal": value / world /
                           NOMINAL_FP4_DENSE_TFLOPS, "measured_peak_tflops": fp4_peak,
                           "peak_source": f"{peak_src} bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/BF16 ratio)"},
        "bare_us": bare_ms * 1e3, "bare_k2_us": bare_k2_ms * 1e3, "unfused_us": unfused_ms * 1e3,
        "lowrank_overhead": step_ms / bare_ms - 1.0, "lowrank_overhead_k2": k2_avg / bare_k2_ms - 1.0,
        "unfused_overhead": unfused_ms / step_ms - 1.0,
        "roofline": {"bound": "tensor", "kernel": "k2_gemm (NVFP4 block-scaled tcgen05 + fused up-proj)",
                     "achieved": k2_achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": k2_achieved / fp4_peak,
                     "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} x {FP4_OVER_BF16:g}",
                     "traffic": profile_traffic()},
        "e2e": {"value": layer_flops(M, K, N) * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                "path": "svdq_linear_forward with pinned host X/Y, copies inside the timed events"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(d, M, K, N)
    L.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
