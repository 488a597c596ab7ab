"""Benchmark of the SVDQuant W4A4 + rank-32 linear layer on B200.

One step = one pass of the whole hot path over one batch: the fused
down-projection + quantize kernel (K1) and the NVFP4 GEMM with the fused
up-projection + bias epilogue (K2), on the FLUX.1-shaped attention output
projection (M = 4608 tokens, K = N = 3072, rank 32, NVFP4 g16/E4M3), inputs
resident in HBM.  Steps run back to back, as the layers of a transformer do,
and cycle through six independent sets of inputs, outputs, workspaces and
prepared weights of about 70 MB each: 420 MB, more than the 126 MB L2, so
every step reads its data from HBM, not from a cache warmed by the step before.
The value is whole-job TFLOP/s of the layer's algorithmic work
2MNK + 2M*32*(K+N), device-timed with one pair of CUDA events around the timed
steps on the launch stream (K1 and K2 back to back per step, as a caller runs
them), max over ranks.  The per-kernel durations behind the roofline fractions
are timed the same way after the steps, each kernel alone over the rotating
sets.  "isolated" repeats the layer and kernel timings one launch at a time
between its own events after an L2 flush (a 256 MiB write, then a read of the
same buffer), which adds the launch latency of every launch.  The JSON line
also carries the other rows of the hot path on their FLUX.1-shaped layers
(INT4 QKV, the fc1 -> GELU -> fc2 pair, the W4A16 adaptive-norm GEMV) under
"other_layers", timed one launch at a time after an L2 flush.

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
N_SETS = 6                   # rotating input sets, 6 x ~70 MB > L2
FP4_OVER_BF16 = 4.0          # nominal dense ratio (9 PF / 2.25 PF)
INT8_OVER_BF16 = 2.0         # nominal dense ratio (4.5 POPS / 2.25 PF)
W8A8_RANK = 16


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

    def _sample(self):
        import pynvml
        try:
            self.samples.append(pynvml.nvmlDeviceGetClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            mask = fn(self._h)
            for n, bit in self._names.items():
                if mask & bit:
                    self.reasons.add(n)
        except Exception as e:       # keep sampling best-effort
            self.error = str(e)

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self._idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._names = {
                "hw_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwSlowdown", 0x8),
                "hw_thermal_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                "sw_thermal_slowdown": getattr(pynvml, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                "sw_power_cap": getattr(pynvml, "nvmlClocksEventReasonSwPowerCap", 0x4),
                "hw_power_brake_slowdown": getattr(pynvml, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
            }

            def run():
                while not self._stop.is_set():
                    self._sample()
                    time.sleep(self._period)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
        except Exception as e:
            self.error = str(e)
        return self

    def __exit__(self, *a):
        # one more sample at the end of the region (a region shorter than the
        # sampling period still gets a sample from each end)
        if self._thread:
            self._sample()
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
    """Max of x over the ranks (the slowest rank's time sets the job's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def guarded(errors, name, fn):
    """Run one secondary section.  Its failure is recorded under `name` in
    `errors` (so it shows in the JSON line) instead of ending the run: the
    headline numbers are measured before any secondary section starts."""
    try:
        return fn()
    except Exception as e:          # noqa: BLE001 - recorded, not hidden
        errors[name] = f"{type(e).__name__}: {e}"[:400]
        return None


def whole_job_tflops(flops_per_step, world, step_ms_max):
    """Whole-job throughput: every rank runs its own replica of the step, and
    the job takes as long as its slowest rank."""
    return flops_per_step * world / (step_ms_max * 1e-3) / 1e12


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


def time_events(stream, n, flush_l2, fn):
    """Mean device time (ms) of fn() over n calls, each bracketed by CUDA events
    on `stream` after an L2 flush."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        flush_l2(i)
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / n


def time_rotating(stream, n, fn):
    """Mean device time (ms) per call of fn(i), i = 0..n-1, run back to back
    between one pair of CUDA events on `stream`."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(n):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def library_nvfp4_gemm_us(M, K, N, n, n_sets=N_SETS):
    """Context only: cuBLASLt's bare NVFP4 GEMM (no low-rank branch, no bias) at
    the same shape through torch._scaled_mm, back to back over rotating operand
    sets like the timed steps; None where this PyTorch build has no FP4 path."""
    import torch
    try:
        dev = "cuda"
        rup = lambda x, m: (x + m - 1) // m * m
        g = torch.Generator(device=dev).manual_seed(7)
        As = [torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
              .view(torch.float4_e2m1fn_x2) for _ in range(n_sets)]
        Bs = [torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
              .view(torch.float4_e2m1fn_x2) for _ in range(n_sets)]
        sa = torch.ones(rup(M, 128) * rup(K // 16, 4), device=dev).to(torch.float8_e4m3fn)
        sb = torch.ones(rup(N, 128) * rup(K // 16, 4), device=dev).to(torch.float8_e4m3fn)
        stream = torch.cuda.current_stream()
        f = lambda i: torch._scaled_mm(As[i % n_sets], Bs[i % n_sets].t(), scale_a=sa, scale_b=sb,
                                       out_dtype=torch.bfloat16)
        for i in range(2 * n_sets):
            f(i)
        return time_rotating(stream, n, f) * 1e3
    except Exception:
        return None


def nvfp4_peak_probe(dev, n=200):
    """The dense NVFP4 ceiling measured on this GPU: cuBLASLt's block-scaled
    NVFP4 GEMM at 8192^3 (torch._scaled_mm, a library probe off the hot path),
    back to back over three operand sets (192 MB, more than L2), with the SM
    clock sampled while it runs."""
    M = K = N = 8192
    with ClockSampler(dev) as clk:
        us = library_nvfp4_gemm_us(M, K, N, n, n_sets=3)
    if us is None:
        return None
    return {"tflops": 2.0 * M * N * K / (us * 1e-6) / 1e12, "us": us, "shape": "8192x8192x8192",
            "clocks": clk.summary(),
            "how": "cuBLASLt block-scaled NVFP4 (E2M1, E4M3 scales per 16) GEMM through torch._scaled_mm, "
                   f"{n} launches back to back over 3 operand sets, one pair of CUDA events"}


def block_b4(pkg, syn, stream, n, peaks, fp4_peak):
    """The FLUX.1-dev double-stream block linears at batch 4 (M = 18432 tokens):
    QKV, attention output, fc1 (GELU epilogue) and fc2 on fc1's output, all
    NVFP4 r = 32, each timed as layers run (K1 + K2 back to back) and K2 alone;
    plus the adaptive-norm W4A16 GEMV on 4 rows.  Each layer's input and output
    exceed L2 (113 MB or more), so one set per layer reads from HBM."""
    import torch
    dev = torch.cuda.current_device()
    out = {}
    total_us = 0.0
    total_flops = 0.0
    h = None
    p1_calib = None
    for name in ("qkv", "out", "fc1", "fc2"):
        d = syn.layer("block_b4", name)
        if name == "fc2":
            d["Xc"] = p1_calib
        L = pkg.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]),
                              fmt="nvfp4", rank=RANK, device=dev)
        K, N = d["W"].shape
        x = h if name == "fc2" else torch.from_numpy(d.pop("X")).to(torch.bfloat16).cuda()
        M = x.shape[0]
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        codes = torch.empty(L.act_code_bytes(M), dtype=torch.uint8, device="cuda")
        scales = torch.empty(L.act_scale_bytes(M), dtype=torch.uint8, device="cuda")
        xl = torch.empty((M, RANK), dtype=torch.bfloat16, device="cuda")
        flags = pkg.FWD_GELU if name == "fc1" else 0

        def k1(i):
            L.quantize_act(x, M, codes, scales, xl, stream, 0)

        def k2(i):
            L.gemm(codes, scales, xl, M, y, stream, flags)

        def layer(i):
            k1(i)
            k2(i)

        for i in range(3):
            layer(i)
        L.check(stream)
        lay = time_rotating(stream, n, layer)
        k2_ms = time_rotating(stream, n, k2)
        L.check(stream)
        k2t = k2_flops(M, K, N) / (k2_ms * 1e-3) / 1e12
        out[name] = {"shape": f"{M}x{K}->{N}", "us_per_layer": lay * 1e3, "k2_us": k2_ms * 1e3,
                     "layer_tflops": layer_flops(M, K, N) / (lay * 1e-3) / 1e12, "k2_tflops": k2t,
                     "k2_frac": k2t / fp4_peak}
        total_us += lay * 1e3
        total_flops += layer_flops(M, K, N)
        if name == "fc1":
            h = y
            # fc2 calibrates on fc1's output for fc1's calibration batch (this library, offline)
            xc = torch.from_numpy(d["Xc"]).to(torch.bfloat16).cuda()
            hc = torch.empty((xc.shape[0], N), dtype=torch.bfloat16, device="cuda")
            wsc = torch.empty(L.workspace_bytes(xc.shape[0]), dtype=torch.uint8, device="cuda")
            L.forward(xc, xc.shape[0], hc, wsc, wsc.numel(), stream, pkg.FWD_GELU | pkg.FWD_CHECK)
            p1_calib = hc.float().cpu().numpy()
        else:
            del y
        L.close()
        del x
    # adaptive-norm modulation, W4A16 on the 4 conditioning rows
    da = syn.layer("block_b4", "adaln", with_run=False)
    Ka, Na = da["W"].shape
    La = pkg.Layer.prepare(syn.bf16_bits(da["W"]), syn.bf16_bits(da["bias"]), None, fmt="w4a16", rank=0,
                           device=dev)
    xa = torch.from_numpy(syn.activations(4, 4, 4, Ka, syn.ROLE_X_RUN, outliers=False)).to(torch.bfloat16).cuda()
    ya = torch.empty((4, Na), dtype=torch.bfloat16, device="cuda")
    La.forward(xa, 4, ya, None, 0, stream, pkg.FWD_CHECK)
    ta = time_rotating(stream, n, lambda i: La.forward(xa, 4, ya, None, 0, stream, 0))
    La.check(stream)
    La.close()
    wbytes = Na * Ka // 2 + Na * (Ka // 64) * 2 + 4 * Ka * 2 + 4 * Na * 2 + Na * 4
    out["adaln_w4a16"] = {"shape": f"4x{Ka}->{Na}", "us": ta * 1e3,
                          "hbm_frac": wbytes / (ta * 1e-3) / 1e9 / peaks["hbm_gbs"],
                          "note": "the same 30 MB of weights every launch (L2-warm after the first)"}
    total_us += ta * 1e3
    out["stack"] = {"us": total_us, "tflops": total_flops / (total_us * 1e-6) / 1e12,
                    "frac": total_flops / (total_us * 1e-6) / 1e12 / fp4_peak,
                    "note": "sum of the per-layer times (QKV, out, fc1+GELU, fc2, adaLN); "
                            "attention itself is not part of this stack"}
    return out


def other_layers(pkg, syn, stream, flush_l2, n, peaks, only=None):
    """The other hot-path rows on their FLUX.1-shaped layers (not the headline):
    the INT4 variant (fused QKV 4608x3072->9216), the MLP pair (fc1 with the GELU
    epilogue, fc2 on fc1's output) and the W4A16 adaptive-norm GEMV (4x3072->18432).
    Each is timed like the headline, back to back over rotating sets of prepared
    weights and buffers whose total exceeds L2, and once more one launch at a
    time after an L2 flush ("isolated")."""
    import torch
    out = {}
    bf16_peak = peaks["bf16_tflops"]
    dev = torch.cuda.current_device()

    def w4a4_layer(d, fmt, X, flags, key, n_sets=2):
        M, K, N = X.shape[0], d["W"].shape[0], d["W"].shape[1]
        r = W8A8_RANK if fmt == "w8a8" else RANK
        sets = []
        for _ in range(n_sets):
            L = pkg.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]),
                                  fmt=fmt, rank=r, device=dev)
            x = X.clone() if isinstance(X, torch.Tensor) else torch.from_numpy(X).to(torch.bfloat16).cuda()
            sets.append((L, x, torch.empty((M, N), dtype=torch.bfloat16, device="cuda"),
                         torch.empty(L.act_code_bytes(M), dtype=torch.uint8, device="cuda"),
                         torch.empty(L.act_scale_bytes(M), dtype=torch.uint8, device="cuda"),
                         torch.empty((M, RANK), dtype=torch.bfloat16, device="cuda")))

        def k1(i):
            L, x, y, codes, scales, xl = sets[i % n_sets]
            L.quantize_act(x, M, codes, scales, xl, stream, 0)

        def k2(i):
            L, x, y, codes, scales, xl = sets[i % n_sets]
            L.gemm(codes, scales, xl, M, y, stream, flags)

        def layer(i):
            k1(i)
            k2(i)

        for i in range(2 * n_sets):
            layer(i)
        for st in sets:
            st[0].check(stream)
        lay = time_rotating(stream, n, layer)
        k2_ms = time_rotating(stream, n, k2)
        iso = time_events(stream, max(10, n // 4), flush_l2, lambda: k2(0))
        for st in sets:
            st[0].check(stream)
        k2t = k2_flops(M, K, N, r) / (k2_ms * 1e-3) / 1e12
        ratio = {"nvfp4": FP4_OVER_BF16, "w8a8": INT8_OVER_BF16}.get(fmt, 1.0)
        peak = bf16_peak * ratio
        note = {"nvfp4": f" x {FP4_OVER_BF16:g}", "w8a8": f" x {INT8_OVER_BF16:g} (INT8 dense rate)"}.get(
            fmt, " (FP16 tensor rate, the INT4 GEMM's dequantized operands)")
        out[key] = {"shape": f"{M}x{K}->{N}", "format": fmt, "rank": r, "us_per_layer": lay * 1e3,
                    "k2_us": k2_ms * 1e3, "layer_tflops": layer_flops(M, K, N, r) / (lay * 1e-3) / 1e12,
                    "k2_tflops": k2t, "k2_frac": k2t / peak, "isolated_k2_us": iso * 1e3, "rotating_sets": n_sets,
                    "k2_peak": f"{peak:g} TFLOP/s = measured bf16 burst" + note}
        y0 = sets[0][2]
        for st in sets:
            st[0].close()
        return y0

    def want(name):
        return only is None or name in only

    errors = {}
    # INT4 variant
    if want("int4"):
        def int4():
            d = syn.layer("qkv_int4")
            w4a4_layer(d, "int4", d["X"], 0, "int4_qkv")
        guarded(errors, "int4", int4)
    # W8A8 variant (rank 16 at 8 bits) on the attention-output shape
    if want("w8a8"):
        def w8a8():
            d = syn.layer("attn_out")
            w4a4_layer(d, "w8a8", d["X"], 0, "w8a8_attn_out")
        guarded(errors, "w8a8", w8a8)
    if want("mlp"):
        guarded(errors, "mlp", lambda: mlp_pair(pkg, syn, stream, n, w4a4_layer, dev, out))
    if want("lora"):
        guarded(errors, "lora", lambda: lora_layer(pkg, syn, stream, n, dev, out))
    if want("w4a16"):
        guarded(errors, "w4a16", lambda: w4a16_adaln(pkg, syn, stream, flush_l2, n, peaks, dev, out))
    if errors:
        out["section_errors"] = errors
    return out


def mlp_pair(pkg, syn, stream, n, w4a4_layer, dev, out):
    """The MLP pair: fc1 (GELU), then fc2 on fc1's output (fc2 calibrates on
    fc1's output for fc1's calibration batch), then the same pair through the
    chain and as two separate layers."""
    import torch
    d1 = syn.layer("mlp", "fc1")
    h = w4a4_layer(d1, "nvfp4", d1["X"], pkg.FWD_GELU, "fc1_gelu")
    L1 = pkg.Layer.prepare(syn.bf16_bits(d1["W"]), syn.bf16_bits(d1["bias"]), syn.bf16_bits(d1["Xc"]),
                           fmt="nvfp4", rank=RANK, device=dev)
    xc = torch.from_numpy(d1["Xc"]).to(torch.bfloat16).cuda()
    hc = torch.empty((xc.shape[0], d1["W"].shape[1]), dtype=torch.bfloat16, device="cuda")
    wsc = torch.empty(L1.workspace_bytes(xc.shape[0]), dtype=torch.uint8, device="cuda")
    L1.forward(xc, xc.shape[0], hc, wsc, wsc.numel(), stream, pkg.FWD_GELU | pkg.FWD_CHECK)
    L1.close()
    d2 = syn.layer("mlp", "fc2")
    d2["Xc"] = hc.float().cpu().numpy()
    w4a4_layer(d2, "nvfp4", h, 0, "fc2")
    del h
    # the same pair through the chain: fc1's epilogue writes fc2's quantized
    # input (codes, scales, down-projection partials), against the two layers
    # one after the other with fc1's BF16 output through HBM
    M1, K1, N1 = d1["X"].shape[0], d1["W"].shape[0], d1["W"].shape[1]
    N2 = d2["W"].shape[1]
    csets = []
    for _ in range(2):
        L1c = pkg.Layer.prepare(syn.bf16_bits(d1["W"]), syn.bf16_bits(d1["bias"]), syn.bf16_bits(d1["Xc"]),
                                fmt="nvfp4", rank=RANK, device=dev)
        L2c = pkg.Layer.prepare(syn.bf16_bits(d2["W"]), syn.bf16_bits(d2["bias"]), syn.bf16_bits(d2["Xc"]),
                                fmt="nvfp4", rank=RANK, device=dev)
        wsb = max(pkg.mlp_workspace_bytes(L1c, L2c, M1, pkg.FWD_GELU),
                  pkg.mlp_workspace_bytes(L1c, L2c, M1, pkg.FWD_GELU | pkg.FWD_UNFUSED))
        csets.append((L1c, L2c, torch.from_numpy(d1["X"]).to(torch.bfloat16).cuda(),
                      torch.empty((M1, N2), dtype=torch.bfloat16, device="cuda"),
                      torch.empty(wsb, dtype=torch.uint8, device="cuda"), wsb))

    def chain(flags):
        def f(i):
            L1c, L2c, x, y, ws, wsb = csets[i % len(csets)]
            pkg.mlp_forward(L1c, L2c, x, M1, y, ws, wsb, stream, flags)
        return f

    for fl in (pkg.FWD_GELU, pkg.FWD_GELU | pkg.FWD_UNFUSED):
        for i in range(4):
            chain(fl)(i)
    for st in csets:
        st[0].check(stream)
        st[1].check(stream)
    t_chain = time_rotating(stream, n, chain(pkg.FWD_GELU))
    t_sep = time_rotating(stream, n, chain(pkg.FWD_GELU | pkg.FWD_UNFUSED))
    for st in csets:
        st[0].check(stream)
        st[1].check(stream)
    fl2 = layer_flops(M1, K1, N1) + layer_flops(M1, N1, N2)
    out["mlp_chain"] = {"shape": f"{M1}x{K1}->{N1}->{N2}", "format": "nvfp4", "us_chain": t_chain * 1e3,
                        "us_separate": t_sep * 1e3, "tflops_chain": fl2 / (t_chain * 1e-3) / 1e12,
                        "tflops_separate": fl2 / (t_sep * 1e-3) / 1e12, "speedup": t_sep / t_chain,
                        "note": "fc1 (GELU) -> fc2; chain: fc2's input quantized in fc1's epilogue "
                                "(svdq_mlp_forward), separate: the two layers' forwards with fc1's BF16 "
                                "output through HBM (SVDQ_FWD_UNFUSED)"}
    for st in csets:
        st[0].close()
        st[1].close()
    del csets


def lora_layer(pkg, syn, stream, n, dev, out):
    """The attention-output layer with a rank-32 LoRA adapter in its branch
    (svdq_set_lora) against the same layer without one, back to back over
    rotating sets; fused and unfused."""
    import numpy as np
    import torch
    d = syn.layer("attn_out")
    M, K = d["X"].shape
    N = d["W"].shape[1]
    g = np.random.default_rng([5, K, N])
    A = syn.to_bf16(g.standard_normal((K, 32)) / np.sqrt(K))
    B = syn.to_bf16(g.standard_normal((32, N)) * 0.1)
    sets = []
    for _ in range(3):
        L = pkg.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]),
                              fmt="nvfp4", rank=RANK, device=dev)
        sets.append([L, torch.from_numpy(d["X"]).to(torch.bfloat16).cuda(),
                     torch.empty((M, N), dtype=torch.bfloat16, device="cuda"), None])

    def alloc():
        for st in sets:
            st[3] = torch.empty(st[0].workspace_bytes(M), dtype=torch.uint8, device="cuda")

    def fwd(flags):
        def f(i):
            L, x, y, ws = sets[i % len(sets)]
            L.forward(x, M, y, ws, ws.numel(), stream, flags)
        return f

    alloc()
    t0 = time_rotating(stream, n, fwd(0))
    for st in sets:
        st[0].set_lora(syn.bf16_bits(A), syn.bf16_bits(B), 0.5)
    alloc()
    for i in range(len(sets)):
        fwd(pkg.FWD_CHECK)(i)
    t1 = time_rotating(stream, n, fwd(0))
    t2 = time_rotating(stream, n, fwd(pkg.FWD_UNFUSED))
    for st in sets:
        st[0].check(stream)
        st[0].close()
    out["lora_attn_out"] = {"shape": f"{M}x{K}->{N}", "format": "nvfp4", "rank": RANK, "lora_rank": 32,
                            "us_without": t0 * 1e3, "us_with": t1 * 1e3, "us_with_unfused": t2 * 1e3,
                            "note": "adapter appended to the 16-bit branch: one more down-projection pass "
                                    "of the first kernel and one more ring stage per output tile"}


def w4a16_adaln(pkg, syn, stream, flush_l2, n, peaks, dev, out):
    """The W4A16 adaptive-norm GEMV (30 MB of weights per set)."""
    import torch
    da = syn.layer("block_b4", "adaln", with_run=False)
    Ma, Ka, Na = 4, da["W"].shape[0], da["W"].shape[1]
    n_sets = N_SETS
    La = [pkg.Layer.prepare(syn.bf16_bits(da["W"]), syn.bf16_bits(da["bias"]), None, fmt="w4a16", rank=0,
                            device=dev) for _ in range(n_sets)]
    xa = torch.from_numpy(syn.activations(4, 4, Ma, Ka, syn.ROLE_X_RUN, outliers=False)).to(torch.bfloat16).cuda()
    ya = [torch.empty((Ma, Na), dtype=torch.bfloat16, device="cuda") for _ in range(n_sets)]
    for i in range(n_sets):
        La[i].forward(xa, Ma, ya[i], None, 0, stream, pkg.FWD_CHECK)
    t = time_rotating(stream, n, lambda i: La[i % n_sets].forward(xa, Ma, ya[i % n_sets], None, 0, stream, 0))
    t_iso = time_events(stream, max(10, n // 4), flush_l2, lambda: La[0].forward(xa, Ma, ya[0], None, 0, stream, 0))
    for L in La:
        L.check(stream)
    wbytes = Na * Ka // 2 + Na * (Ka // 64) * 2 + Ma * Ka * 2 + Ma * Na * 2 + Na * 4
    gbs = wbytes / (t * 1e-3) / 1e9
    out["w4a16_adaln"] = {"shape": f"{Ma}x{Ka}->{Na}", "format": "w4a16 int4 g64", "us": t * 1e3,
                          "algorithmic_bytes": wbytes, "GBs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                          "isolated_us": t_iso * 1e3, "rotating_sets": n_sets}
    for L in La:
        L.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-layers", action="store_true")
    ap.add_argument("--only", default=None,
                    help="comma-separated other-layer sections to run (int4, w8a8, mlp, lora, w4a16, block); "
                         "the library probes run only with all sections (the default)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

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
    stream = torch.cuda.current_stream()

    class Set:
        """One independent copy of the layer's data: prepared weights, X, Y,
        the workspace of the one-call forward and the two kernels' buffers."""

        def __init__(self):
            self.L = pkg.Layer.prepare(syn.bf16_bits(d["W"]), syn.bf16_bits(d["bias"]), syn.bf16_bits(d["Xc"]),
                                       fmt="nvfp4", rank=RANK, device=dev)
            self.x = torch.from_numpy(d["X"]).to(torch.bfloat16).cuda()
            self.y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            self.wsb = self.L.workspace_bytes(M)
            self.ws = torch.empty(self.wsb, dtype=torch.uint8, device="cuda")
            self.codes = torch.empty(self.L.act_code_bytes(M), dtype=torch.uint8, device="cuda")
            self.scales = torch.empty(self.L.act_scale_bytes(M), dtype=torch.uint8, device="cuda")
            self.xl = torch.empty((M, RANK), dtype=torch.bfloat16, device="cuda")

        def k1(self, mode=0):
            self.L.quantize_act(self.x, M, self.codes, self.scales, self.xl, stream, mode)

        def k2(self, flags=0):
            self.L.gemm(self.codes, self.scales, self.xl, M, self.y, stream, flags)

    sets = [Set() for _ in range(N_SETS)]
    L, x, y, ws, wsb = sets[0].L, sets[0].x, sets[0].y, sets[0].ws, sets[0].wsb
    set_bytes = (M * K * 2 + M * N * 2 + wsb + sets[0].codes.numel() + sets[0].scales.numel() +
                 M * RANK * 2 + N * K // 2 + N * K // 16 + (K + N) * RANK * 2 + (K + N) * 4)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_sink = torch.empty(1, dtype=torch.int64, device="cuda")

    def flush_l2(i):
        flush.fill_(i & 0xFF)                                     # evict: write > L2
        torch.sum(flush.view(torch.int64), dim=0, keepdim=True, out=flush_sink)   # clean the lines

    def step(i):
        # the layer as a caller runs it: K1 then K2 back to back on one stream (K2
        # is a programmatic dependent launch of K1: its prologue overlaps K1's tail)
        st = sets[i % N_SETS]
        st.k1()
        st.k2()

    # ---- warm-up
    for i in range(max(args.warmup, N_SETS)):
        step(i)
    for st in sets:
        st.L.forward(st.x, M, st.y, st.ws, st.wsb, stream, pkg.FWD_CHECK)
    torch.cuda.synchronize()

    # ---- timed region: exactly `steps` steps back to back, one event pair around them
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        step_ms = time_rotating(stream, args.steps, step)
    barrier(world)
    step_ms_max = allreduce_max(step_ms, world)
    value = whole_job_tflops(layer_flops(M, K, N), world, step_ms_max)
    for st in sets:
        st.L.check(stream)

    # ---- per-kernel durations, each kernel alone over the rotating sets
    n_k = max(100, min(1000, args.steps))
    k2_ms = time_rotating(stream, n_k, lambda i: sets[i % N_SETS].k2())
    k1_ms = time_rotating(stream, n_k, lambda i: sets[i % N_SETS].k1())

    # ---- measurement variants: bare GEMM and unfused layer
    n_var = max(50, min(500, args.steps))

    def bare(i):
        sets[i % N_SETS].k1(1)
        sets[i % N_SETS].k2(pkg.FWD_NO_BRANCH)

    def unfused(i):
        st = sets[i % N_SETS]
        st.L.forward(st.x, M, st.y, st.ws, st.wsb, stream, pkg.FWD_UNFUSED)

    bare_ms = time_rotating(stream, n_var, bare)
    unfused_ms = time_rotating(stream, n_var, unfused)
    for st in sets:
        st.k1()
    bare_k2_ms = time_rotating(stream, n_var, lambda i: sets[i % N_SETS].k2(pkg.FWD_NO_BRANCH))
    for st in sets:
        st.L.check(stream)

    # ---- isolated launches: one event pair per launch after an L2 flush
    n_iso = max(50, min(300, args.steps))
    iso_layer_ms = time_events(stream, n_iso, flush_l2, lambda: step(0))
    iso_k2_ms = time_events(stream, n_iso, flush_l2, lambda: sets[0].k2())
    iso_k1_ms = time_events(stream, n_iso, flush_l2, lambda: sets[0].k1())
    L.check(stream)

    # ---- end to end through the public API with host buffers
    xh = torch.from_numpy(d["X"]).to(torch.bfloat16).pin_memory()
    yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()

    def e2e():
        x.copy_(xh, non_blocking=True)
        L.forward(x, M, y, ws, wsb, stream, 0)
        yh.copy_(y, non_blocking=True)

    e2e_ms = allreduce_max(time_events(stream, max(20, min(200, args.steps)), flush_l2, e2e), world)

    peaks, peak_src = measured_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    k2_achieved = k2_flops(M, K, N) / (k2_ms * 1e-3) / 1e12
    k1_bytes = M * K * 2 + M * K // 2 + M * K // 16 + M * RANK * 2 + K * 4
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD} {M}x{K}->{N} NVFP4 g16 E4M3 r{RANK}", "M": M, "K": K, "N": N,
                   "rank": RANK, "parallelism": "replicas" if world > 1 else "single",
                   "l2": f"inputs larger than L2: steps back to back over {N_SETS} rotating sets of inputs, "
                         f"outputs, workspaces and prepared weights ({N_SETS} x {set_bytes / 1e6:.0f} MB)"},
        "us_per_layer": step_ms_max * 1e3, "k1_us": k1_ms * 1e3, "k2_us": k2_ms * 1e3,
        "pct_nvfp4_peak": {"of_measured": value / world / fp4_peak, "of_nominal": value / world /
                           NOMINAL_FP4_DENSE_TFLOPS, "measured_peak_tflops": fp4_peak,
                           "peak_source": f"{peak_src} bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/BF16 ratio)"},
        "bare_us": bare_ms * 1e3, "bare_k2_us": bare_k2_ms * 1e3, "unfused_us": unfused_ms * 1e3,
        "lowrank_overhead": step_ms / bare_ms - 1.0, "lowrank_overhead_k2": k2_ms / bare_k2_ms - 1.0,
        "unfused_overhead": unfused_ms / step_ms - 1.0,
        "roofline": {"bound": "tensor", "kernel": "k2_gemm (NVFP4 block-scaled tcgen05 + fused up-proj)",
                     "achieved": k2_achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": k2_achieved / fp4_peak,
                     "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} x {FP4_OVER_BF16:g}",
                     "timing": f"K2 alone, {n_k} launches back to back over the {N_SETS} rotating sets "
                               "between one pair of CUDA events on the launch stream, after the timed steps",
                     "traffic": profile_traffic()},
        "k1_roofline": {"bound": "hbm", "achieved": k1_bytes / (k1_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": k1_bytes / (k1_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "algorithmic_bytes": k1_bytes},
        "e2e": {"value": layer_flops(M, K, N) * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                "path": "svdq_linear_forward with pinned host X/Y, copies inside the timed events"},
        "isolated": {"layer_us": iso_layer_ms * 1e3, "k1_us": iso_k1_ms * 1e3, "k2_us": iso_k2_ms * 1e3,
                     "timing": "one launch (or one K1+K2 step) between its own CUDA events after an L2 flush"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    only = None if args.only is None else set(args.only.split(","))
    errors = {}
    if rank == 0 and world == 1 and not args.no_other_layers:
        others = guarded(errors, "other_layers", lambda: other_layers(pkg, syn, stream, flush_l2,
                                                                       max(30, min(200, args.steps)), peaks, only))
        out["other_layers"] = others if others is not None else {}
        if only is None or "block" in only:
            blk = guarded(errors, "block_b4", lambda: block_b4(pkg, syn, stream, max(20, min(100, args.steps)),
                                                                peaks, fp4_peak))
            if blk is not None:
                out["other_layers"]["block_b4"] = blk
    if rank == 0 and world == 1 and not args.no_other_layers and only is None:
        def library_probes():
            lib_us = library_nvfp4_gemm_us(M, K, N, n_k)
            out["library_context"] = {
                "cublaslt_nvfp4_gemm_us": lib_us, "k2_us": k2_ms * 1e3, "bare_k2_us": bare_k2_ms * 1e3,
                "note": "bare NVFP4 GEMM of the same shape through torch._scaled_mm (no low-rank branch, no bias), "
                        "back to back over rotating operand sets; context, not a baseline"}
            probe = nvfp4_peak_probe(dev)
            if probe is not None:
                out["nvfp4_peak_measured"] = probe
                out["pct_nvfp4_peak"]["of_cublaslt_8192"] = value / world / probe["tflops"]
                out["roofline"]["frac_of_cublaslt_8192"] = k2_achieved / probe["tflops"]
        guarded(errors, "library_probes", library_probes)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = guarded(errors, "cpu_baseline", lambda: cpu_baseline(d, M, K, N))
        if cpu is not None:
            out["cpu_baseline"] = cpu
    if errors:
        out["section_errors"] = errors
    for st in sets:
        st.L.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
