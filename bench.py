"""Benchmark of the SVDQuant W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the FLUX-like fused QKV projection, NVFP4, M = 4608 tokens (4096
image + 512 text), K = 3072, N = 9216, rank 32, synthetic seeded inputs with
the outlier recipe of workloads.py.  A step is one pass of the whole layer
(kernel 1: quantize + low-rank down; kernel 2: block-scaled FP4 GEMM + fused
low-rank up + bias) over the batch.  Metric: effective TFLOP/s = 2 M N K per
step time (low-rank flops not counted), also reported as us/layer and as the
fraction of the FP4 tensor peak.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and
a device synchronize on both sides, timed with CUDA events on the launching
stream; the slowest rank's time counts.  Each step uses the next of three
rotating X / Y buffer sets (together larger than the 126 MB L2), so
activations and outputs come from HBM.  Under torchrun every rank runs its
own batch (weak scaling; no collective on the data path).  Kernel 2 is
launched so that it may start while kernel 1 finishes (programmatic
dependent launch), and the next step's kernel 1 while kernel 2 finishes, so
the timed region holds no events between kernels; the per-kernel times of
the roofline objects come from an instrumented pass of the same steps right
after it (events around each kernel on the launching stream).

--impl reference times the CPU oracle (float64 numpy) on the host cores on a
bounded sample of the same workload, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(name="nvfp4_qkv_M4608_K3072_N9216_r32", fmt="nvfp4", M=4608, K=3072, N=9216, rank=32)
# --workload: the QKV projection is the bench line; the others are the
# remaining parity configurations, timed the same way for their profiles.
WORKLOADS = ("qkv", "int4_qkv", "mlp_fc1", "mlp_fc2", "lora", "awq_adaln", "mlp_pair", "small", "lora_sweep", "awq_qkv", "library_fp4")
INT8_PER_BF16 = 2.0         # nominal dense INT8 : BF16 tensor throughput (4.5 : 2.25)
METRIC = "SVDQuant W4A4 linear effective TFLOPS & % of FP4 tensor peak; µs/layer"
UNIT = "TFLOP/s"
FP4_PER_BF16 = 4.0          # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PFLOP/s)
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ helpers
def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return dict(bf16=float(d["bf16_tflops"]), bf16_sustained=float(d.get("bf16_tflops_sustained", 0)) or None,
                    hbm=float(d["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=None, hbm=FALLBACK_HBM_GBS, source="fallback")


def file_sha(paths):
    """First 16 hex digits of the sha256 of the files' contents, in order."""
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def kernel_sources(name):
    d = os.path.join(ROOT, "rank_gemm_b200", "csrc")
    return [os.path.join(d, name), os.path.join(d, "common.cuh"), os.path.join(d, "kernels.h")]


def profiled_traffic(profile_name, kernel_src):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source (the kernel file, common.cuh, kernels.h) as it is now;
    else None."""
    path = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line and line.strip().startswith(("dram_bytes_per_launch", "kernel_sha256", "units_scale")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_sha256") != file_sha(kernel_src):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index, period_s=0.002):
        self.ok = False
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass
        self._stop = threading.Event()

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of x over all ranks (plumbing only: one float)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput in TFLOP/s: every rank did `steps` steps."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------------ the CPU oracle (baseline / reference arm)
def oracle_setup():
    import workloads
    from oracle import svdquant as S
    L = workloads.qkv()
    pw = S.calibrate_and_prepare("nvfp4", L.X, L.W, L.bias, L.rank)
    return L, pw


def oracle_step(L, pw, rows, cols):
    """Oracle forward on rows [0, rows) and output columns [0, cols) of the
    workload: a slice of the prepared weights, no change to the oracle."""
    import dataclasses
    from oracle import svdquant as S
    sub = dataclasses.replace(pw, N=cols, qR=pw.qR[:cols], sR=pw.sR[:cols], L2=pw.L2[:, :cols], bias=pw.bias[:cols])
    return S.forward(sub, L.X[:rows])


def oracle_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max(int(i.get("num_threads", 1)) for i in info) if info else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(L, pw, rows=1152, reps=3):
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        oracle_step(L, pw, rows, L.N)
        ts.append(time.perf_counter() - t0)
    t = statistics.median(ts)
    return {"value": round(2.0 * rows * L.N * L.K / t / 1e12, 6), "unit": UNIT, "cores": oracle_threads(),
            "kind": "oracle",
            "sample": "float64 numpy oracle forward (activation quantize, dequantized FP4 GEMM, low-rank "
                      "down/up, bias) on rows 0..%d of the M=4608 QKV workload, all 9216 outputs; median of %d"
                      % (rows - 1, reps),
            "seconds_per_sample": round(t, 3)}


def run_reference(args, world, rank):
    if rank != 0:
        return
    L, pw = oracle_setup()
    # size the per-step sample so that warm-up + steps take about two minutes
    rows, cols = 64, 512
    t0 = time.perf_counter()
    oracle_step(L, pw, rows, cols)
    t1 = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    scale = max(budget / max(t1, 1e-6), 1e-3)
    cols = int(min(L.N, max(16, cols * scale)) // 16 * 16)
    for _ in range(args.warmup):
        oracle_step(L, pw, rows, cols)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(L, pw, rows, cols)
    el = time.perf_counter() - t0
    value = 2.0 * rows * cols * L.K * args.steps / el / 1e12
    out = {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "impl": "reference", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded, FLUX-shaped, outlier channels)",
           "config": {"workload": WORKLOAD["name"], "M": L.M, "K": L.K, "N": L.N, "rank": L.rank,
                      "format": "nvfp4", "sample_rows": rows, "sample_cols": cols},
           "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "kind": "oracle", "cores": oracle_threads(),
                            "sample": "oracle forward on rows 0..%d x output columns 0..%d per step"
                                      % (rows - 1, cols - 1)},
           "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ our arm
def gpu_factors(B, Wt, X, rank, torch):
    """Offline quantizer step on the GPU, all in the library: smoothing
    factors and activation scale from the calibration kernel, then the
    low-rank split of W^ (svdq_lowrank_factors: randomized subspace
    iteration in float64)."""
    M, K = X.shape
    N = Wt.shape[0]
    lam = torch.empty(K, dtype=torch.float32, device="cuda")
    act = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(B.svdq_calibrate_workspace_bytes(K), dtype=torch.uint8, device="cuda")
    B.svdq_calibrate(M, K, N, X, Wt, 0.5, lam, act, ws)
    L1f = torch.empty(K, rank, dtype=torch.bfloat16, device="cuda")
    L2 = torch.empty(rank, N, dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    B.svdq_lowrank_factors(K, N, rank, Wt, lam, L1f, L2)
    SPLIT_SECONDS.append(time.perf_counter() - t0)
    torch.cuda.synchronize()
    return lam, float(act.item()), L1f, L2


SPLIT_SECONDS = []


def build_layer(name, B, torch, dev):
    """Device tensors of one workload plus its prepared weights handle."""
    import numpy as np
    import workloads

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(dev)

    def prepare(fmt, X0, W, bias, rank, lora=None):
        Wt = dev_bf16(W.T)
        lam, act, L1f, L2 = gpu_factors(B, Wt, X0, rank, torch)
        la, lb, lr = (dev_bf16(lora[0]), dev_bf16(lora[1]), lora[0].shape[1]) if lora else (None, None, 0)
        return B.svdq_prepare_weights(fmt, W.shape[0], W.shape[1], rank, Wt, lam, L1f, L2, dev_bf16(bias),
                                      la, lb, lr, act)

    epi = B.SVDQ_EPI_NONE
    if name in ("qkv", "int4_qkv"):
        L = workloads.qkv() if name == "qkv" else workloads.int4_qkv()
        X0 = dev_bf16(L.X)
        h = prepare(L.fmt, X0, L.W, L.bias, L.rank)
        return dict(name=L.name, fmt=L.fmt, X0=X0, h=h, M=L.M, K=L.K, N=L.N, rank=L.rank, lora=0, epi=epi)
    if name in ("mlp_fc1", "mlp_fc2"):
        fc1, (W2, b2, _) = workloads.mlp_pair()
        X1 = dev_bf16(fc1.X)
        h1 = prepare("nvfp4", X1, fc1.W, fc1.bias, fc1.rank)
        if name == "mlp_fc1":
            return dict(name=fc1.name, fmt="nvfp4", X0=X1, h=h1, M=fc1.M, K=fc1.K, N=fc1.N, rank=fc1.rank, lora=0,
                        epi=B.SVDQ_EPI_GELU_TANH)
        # fc2's activation: this library's fc1 output (GELU), computed once
        Y1 = torch.empty(fc1.M, fc1.N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(B.svdq_linear_workspace_bytes(h1, fc1.M), dtype=torch.uint8, device=dev)
        B.svdq_linear(h1, fc1.M, X1, B.SVDQ_EPI_GELU_TANH, Y1, ws)
        torch.cuda.synchronize()
        B.svdq_free_weights(h1)
        del ws
        h2 = prepare("nvfp4", Y1, W2, b2, 32)
        return dict(name="nvfp4_mlp_fc2_M%d_K12288_N3072_r32" % fc1.M, fmt="nvfp4", X0=Y1, h=h2, M=fc1.M,
                    K=12288, N=3072, rank=32, lora=0, epi=epi)
    if name == "lora":
        base = workloads.lora_sweep_base()
        M = 4096
        X0 = dev_bf16(base.X[:M])
        h = prepare("nvfp4", X0, base.W, base.bias, 32, (base.lora_A, base.lora_B))
        return dict(name="nvfp4_lora_M4096_K3072_N3072_r32_lora%d" % base.lora_A.shape[1], fmt="nvfp4", X0=X0,
                    h=h, M=M, K=3072, N=3072, rank=32, lora=base.lora_A.shape[1], epi=epi)
    raise ValueError(name)


def run_ours(args, world, rank, local):
    import numpy as np
    import torch
    import workloads
    from rank_gemm_b200 import build as _b
    if rank == 0:
        _b.build()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", init_method="env://", world_size=world, rank=rank,
                                timeout=__import__("datetime").timedelta(seconds=120))
        dist.barrier()
    from rank_gemm_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    lay = build_layer(args.workload, B, torch, dev)
    M, K, N, r, h, X0, fmt, epi = (lay[k] for k in ("M", "K", "N", "rank", "h", "X0", "fmt", "epi"))
    r_tot = r + lay["lora"]
    nv = fmt == "nvfp4"

    sets = 3
    Xs = [X0] + [X0.clone() for _ in range(sets - 1)]
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(sets)]
    qb, sb, lb = B.svdq_act_buffer_sizes(h, M)
    acts = [(torch.empty(qb, dtype=torch.uint8, device=dev), torch.empty(sb, dtype=torch.uint8, device=dev),
             torch.empty(lb, dtype=torch.uint8, device=dev)) for _ in range(sets)]
    stream = torch.cuda.current_stream(dev)

    def step(i, ev=None):
        qX, sX, LR = acts[i % sets]
        if ev:
            ev[0].record(stream)
        B.svdq_quantize_act_lowrank_down(h, M, Xs[i % sets], qX, sX, LR, stream)
        if ev:
            ev[1].record(stream)
        B.svdq_w4a4_gemm_lowrank_up(h, M, qX, sX, LR, epi, Ys[i % sets], stream)
        if ev:
            ev[2].record(stream)

    K_steps, W_steps = args.steps, args.warmup
    for i in range(W_steps):
        step(i)
    torch.cuda.synchronize()
    assert B.svdq_poll_device_error(stream) == 0

    # The timed region holds only the steps: an event between kernel 1 and
    # kernel 2 would serialise their programmatic launch overlap.
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for i in range(K_steps):
            step(i)
        t_stop.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_stop)
    status = B.svdq_poll_device_error(stream)
    max_ms = max_over_ranks(total_ms, world, dev)
    # Per-kernel durations: an instrumented pass of the same steps right after
    # the timed region, with events around each kernel on the launching stream.
    n_split = min(K_steps, 500)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_split)]
    torch.cuda.synchronize()
    for i in range(n_split):
        step(i, evs[i])
    torch.cuda.synchronize()
    k1_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    k2_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    flops = 2.0 * M * N * K
    value = weak_scaling_value(flops, K_steps, world, max_ms)
    peaks = measured_peaks()
    # the contraction's own peak: FP4 (NVFP4) or INT8 (INT4 codes run on the
    # int8 tensor core), each the measured bf16 peak times the nominal ratio
    ratio = FP4_PER_BF16 if nv else INT8_PER_BF16
    # a long back-to-back run that met the power cap is held to the measured
    # sustained peak (the bf16 GEMM looped for seconds under the same cap);
    # a run that did not is held to the burst figure
    capped = "sw_power_cap" in clocks.summary().get("reasons", []) and peaks["bf16_sustained"]
    tc_peak = (peaks["bf16_sustained"] if capped else peaks["bf16"]) * ratio
    peak_kind = "sustained" if capped else "burst"
    k2_tflops = flops / (k2_ms * 1e-3) / 1e12
    # algorithmic bytes: each operand once, scales counted once (the four
    # replicas kernel 2 reads are an implementation cost and show in traffic)
    g = 16 if nv else 64
    sbytes = 1 if nv else 2
    sx_once = -(-M // 128) * 128 * (K // g) * sbytes
    r_pad = -(-r_tot // 64) * 64
    bytes_k1 = M * K * 2 + K * 4 + r_tot * K * 2 + M * K // 2 + sx_once + M * r_pad * 2
    bytes_k2 = (M * K // 2 + sx_once + M * r_pad * 2 + (N * K // 2) + N * (K // g) * sbytes + N * r_pad * 2 + N * 4
                + M * N * 2)
    k2_src = "gemm_nvfp4.cu" if nv else "gemm_int4.cu"
    traffic = profiled_traffic("%s_%s.md" % (k2_src[:-3], args.workload), kernel_sources(k2_src))
    traffic_k1 = profiled_traffic("quant_down_%s.md" % args.workload, kernel_sources("quant_down.cu"))

    # low-rank overhead (the "Nunchaku engine design" figure's comparison):
    # plain W4A4 path (quantize + GEMM, no low-rank branch), the fused layer,
    # and the naive four-launch path, each timed over the same steps
    def timed(fn, n):
        for i in range(3):
            fn(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for i in range(n):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    def plain(i):
        qX, sX, LR = acts[i % sets]
        B.svdq_quantize_act(h, M, Xs[i % sets], qX, sX, stream)
        B.svdq_w4a4_gemm(h, M, qX, sX, Ys[i % sets], stream)   # no GELU: timing only

    def unfused(i):
        qX, sX, LR = acts[i % sets]
        B.svdq_quantize_act(h, M, Xs[i % sets], qX, sX, stream)
        B.svdq_lowrank_down(h, M, Xs[i % sets], LR, stream)
        B.svdq_w4a4_gemm(h, M, qX, sX, Ys[i % sets], stream)
        B.svdq_lowrank_up(h, M, LR, epi, Ys[i % sets], stream)

    n_ov = min(K_steps, 100)
    t_plain = timed(plain, n_ov)
    t_fused = timed(lambda i: (B.svdq_quantize_act_lowrank_down(h, M, Xs[i % sets], *acts[i % sets], stream),
                               B.svdq_w4a4_gemm_lowrank_up(h, M, *acts[i % sets], epi,
                                                           Ys[i % sets], stream)), n_ov)
    t_unfused = timed(unfused, n_ov)
    # the per-call NVFP4 activation tensor scale (svdq_linear_dynamic: one
    # extra pass over X for its amax) against the static-scale public call
    wss = [torch.empty(B.svdq_linear_dynamic_workspace_bytes(h, M), dtype=torch.uint8, device=dev)
           for _ in range(sets)]
    t_linear = timed(lambda i: B.svdq_linear(h, M, Xs[i % sets], epi, Ys[i % sets], wss[i % sets], None, stream),
                     n_ov)
    t_dyn = timed(lambda i: B.svdq_linear_dynamic(h, M, Xs[i % sets], epi, Ys[i % sets], wss[i % sets], None,
                                                  stream), n_ov) if nv else None
    del wss

    # end to end through the public call with host buffers: svdq_linear_host
    # moves X in and Y out (page-locked host memory) in row slabs overlapped
    # with the kernels; the events on the caller's stream cover every copy
    e2e_steps = min(K_steps, 50)
    Xh = torch.empty(M, K, dtype=torch.bfloat16, pin_memory=True)
    Xh.copy_(X0.cpu())
    Yh = torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True)
    ws = torch.empty(B.svdq_linear_host_workspace_bytes(h, M), dtype=torch.uint8, device=dev)
    for _ in range(3):
        B.svdq_linear_host(h, M, Xh, epi, Yh, ws, None, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        B.svdq_linear_host(h, M, Xh, epi, Yh, ws, None, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    e2e_value = flops * world / (e2e_ms * 1e-3) / 1e12

    out = None
    if rank == 0:
        out = {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": K_steps,
               "warmup": W_steps, "ms_per_step": round(max_ms / K_steps, 5), "us_per_layer": round(max_ms / K_steps * 1e3, 2),
               "fp4_peak_frac" if nv else "int8_peak_frac": round(value / world / tc_peak, 4),
               "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": fmt,
               "data": "synthetic (seeded, FLUX-shaped, 0.5% outlier channels x20 / x5), random-init weights",
               "config": {"workload": lay["name"], "M": M, "K": K, "N": N, "rank": r, "lora_rank": lay["lora"],
                          "format": fmt, "group": g, "epilogue": "gelu_tanh" if epi else "none",
                          "parallelism": "replicas x%d (each rank its own batch)" % world,
                          "l2": "3 rotating X/Y/workspace sets (%.0f MB) > 126 MB L2"
                                % (sets * (M * K * 2 + M * N * 2 + qb + sb + lb) / 1e6)},
               "roofline": {"kernel": "%s (kernel 2)" % k2_src[:-3], "bound": "tensor", "achieved": round(k2_tflops, 2),
                            "peak": round(tc_peak, 1), "unit": "TFLOP/s", "frac": round(k2_tflops / tc_peak, 4),
                            "peak_source": "%s %s bf16 %.1f TFLOP/s x %.0f (nominal %s:BF16)%s"
                                           % (peaks["source"], peak_kind, tc_peak / ratio, ratio,
                                              "FP4" if nv else "INT8",
                                              "; the timed region ran under sw_power_cap" if capped else ""),
                            "traffic": traffic, "algorithmic_bytes": bytes_k2, "us": round(k2_ms * 1e3, 2)},
               "roofline_k1": {"kernel": "quant_down (kernel 1)", "bound": "hbm",
                               "achieved": round(bytes_k1 / (k1_ms * 1e-3) / 1e9, 1), "peak": peaks["hbm"],
                               "unit": "GB/s", "frac": round(bytes_k1 / (k1_ms * 1e-3) / 1e9 / peaks["hbm"], 4),
                               "traffic": traffic_k1, "algorithmic_bytes": bytes_k1, "us": round(k1_ms * 1e3, 2)},
               "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": M * K * 2,
                       "d2h_bytes_per_step": M * N * 2, "ms_per_step": round(e2e_ms, 4),
                       "call": "svdq_linear_host (page-locked X and Y, copies overlapped with the kernels)"},
               "lowrank_overhead": {"plain_w4a4_us": round(t_plain * 1e3, 2), "fused_us": round(t_fused * 1e3, 2),
                                    "unfused_us": round(t_unfused * 1e3, 2),
                                    "fused_over_plain": round(t_fused / t_plain - 1, 4),
                                    "unfused_over_plain": round(t_unfused / t_plain - 1, 4)},
               "dynamic_scale": None if t_dyn is None else
               {"linear_us": round(t_linear * 1e3, 2), "linear_dynamic_us": round(t_dyn * 1e3, 2),
                "overhead": round(t_dyn / t_linear - 1, 4)},
               "prepare": {"lowrank_split_s": round(SPLIT_SECONDS[-1], 4) if SPLIT_SECONDS else None,
                           "split": "svdq_lowrank_factors (randomized subspace iteration, float64)"},
               "gpu_launches": 2 * K_steps,
               "device_status": status,
               "clocks": clocks.summary()}
    B.svdq_free_weights(h)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline and args.workload == "qkv":
            L, pw = oracle_setup()
            out["cpu_baseline"] = cpu_baseline(L, pw)
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ fused MLP pair arm
def run_mlp_pair(args, world, rank, local):
    """The FLUX-like MLP pair (fc1 3072 -> 12288 + GELU, fc2 12288 -> 3072,
    M = 4608) as one svdq_mlp call per step (fc1's epilogue writes fc2's
    kernel-1 outputs), against the two layers run separately."""
    import numpy as np
    import torch
    import workloads
    from rank_gemm_b200 import build as _b
    if rank == 0:
        _b.build()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", init_method="env://", world_size=world, rank=rank,
                                timeout=__import__("datetime").timedelta(seconds=120))
        dist.barrier()
    from rank_gemm_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    l1 = build_layer("mlp_fc1", B, torch, dev)
    fc1, (W2, b2, _) = workloads.mlp_pair()
    M, K, N1 = l1["M"], l1["K"], l1["N"]
    # fc2 prepared on this library's fc1 output, as the mlp_fc2 workload does
    Y1 = torch.empty(M, N1, dtype=torch.bfloat16, device=dev)
    ws1 = torch.empty(B.svdq_linear_workspace_bytes(l1["h"], M), dtype=torch.uint8, device=dev)
    B.svdq_linear(l1["h"], M, l1["X0"], B.SVDQ_EPI_GELU_TANH, Y1, ws1)
    Wt2 = torch.from_numpy(np.ascontiguousarray(W2.T)).to(torch.bfloat16).to(dev)
    lam2, act2, L1f2, L22 = gpu_factors(B, Wt2, Y1, 32, torch)
    h2 = B.svdq_prepare_weights("nvfp4", N1, W2.shape[1], 32, Wt2, lam2, L1f2, L22,
                                torch.from_numpy(b2).to(torch.bfloat16).to(dev), act_scale=act2)
    N2 = W2.shape[1]
    sets = 3
    Xs = [l1["X0"]] + [l1["X0"].clone() for _ in range(sets - 1)]
    Ys = [torch.empty(M, N2, dtype=torch.bfloat16, device=dev) for _ in range(sets)]
    wss = [torch.empty(B.svdq_mlp_workspace_bytes(l1["h"], h2, M), dtype=torch.uint8, device=dev)
           for _ in range(sets)]
    stream = torch.cuda.current_stream(dev)
    step = lambda i: B.svdq_mlp(l1["h"], h2, M, Xs[i % sets], B.SVDQ_EPI_GELU_TANH, B.SVDQ_EPI_NONE, Ys[i % sets],
                                wss[i % sets], None, stream)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    max_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    status = B.svdq_poll_device_error(stream)
    # the same pair as two separate layers (fc1's bf16 output through HBM)
    Y1s = [torch.empty(M, N1, dtype=torch.bfloat16, device=dev) for _ in range(sets)]
    wl1 = [torch.empty(B.svdq_linear_workspace_bytes(l1["h"], M), dtype=torch.uint8, device=dev) for _ in range(sets)]
    wl2 = [torch.empty(B.svdq_linear_workspace_bytes(h2, M), dtype=torch.uint8, device=dev) for _ in range(sets)]

    def sep(i):
        B.svdq_linear(l1["h"], M, Xs[i % sets], B.SVDQ_EPI_GELU_TANH, Y1s[i % sets], wl1[i % sets], None, stream)
        B.svdq_linear(h2, M, Y1s[i % sets], B.SVDQ_EPI_NONE, Ys[i % sets], wl2[i % sets], None, stream)
    n_sep = min(args.steps, 300)
    for i in range(3):
        sep(i)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for i in range(n_sep):
        sep(i)
    s1.record(stream)
    torch.cuda.synchronize()
    sep_us = max_over_ranks(s0.elapsed_time(s1), world, dev) / n_sep * 1e3
    # the pair's two calls timed apart: fc1 in emit mode (kernel 1, kernel 2
    # writing fc2's kernel-1 outputs, the LR reduction), then fc2's kernel 2
    qs, ss, ls = B.svdq_act_buffer_sizes(h2, M)
    nb = [[torch.empty(v, dtype=torch.uint8, device=dev) for v in (qs, ss, ls)] for _ in range(sets)]
    wse = [torch.empty(B.svdq_linear_emit_next_workspace_bytes(l1["h"], h2, M), dtype=torch.uint8, device=dev)
           for _ in range(sets)]

    def part_us(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(n_sep):
            fn(i)
        a1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(a0.elapsed_time(a1), world, dev) / n_sep * 1e3
    emit_us = part_us(lambda i: B.svdq_linear_emit_next(l1["h"], h2, M, Xs[i % sets], B.SVDQ_EPI_GELU_TANH,
                                                        *nb[i % sets], wse[i % sets], None, stream))
    fc2_us = part_us(lambda i: B.svdq_w4a4_gemm_lowrank_up(h2, M, *nb[i % sets], B.SVDQ_EPI_NONE, Ys[i % sets],
                                                           stream))
    us = max_ms / args.steps * 1e3
    flops = 2.0 * M * K * N1 + 2.0 * M * N1 * N2
    fc1_flops = 2.0 * M * K * N1
    value = weak_scaling_value(flops, args.steps, world, max_ms)
    peaks = measured_peaks()
    out = None
    if rank == 0:
        out = {"metric": "SVDQuant W4A4 MLP pair (fc1 + GELU -> fc2) effective TFLOPS; µs/pair", "value": round(value, 3),
               "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": round(max_ms / args.steps, 5), "us_per_pair": round(us, 2),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
               "data": "synthetic (seeded, FLUX-shaped MLP), random-init weights",
               "config": {"workload": "nvfp4_mlp_pair_M%d_3072_12288_3072_r32_gelu" % M, "M": M, "K": K, "N1": N1,
                          "N2": N2, "rank": 32, "parallelism": "replicas x%d (each rank its own batch)" % world,
                          "l2": "3 rotating X/Y/workspace sets > 126 MB L2"},
               "fp4_peak_frac": round(value / world / (peaks["bf16"] * FP4_PER_BF16), 4),
               "separate_layers_us": round(sep_us, 2), "fused_saving": round(1 - us / sep_us, 4),
               "split_us": {"fc1_emit": round(emit_us, 2), "fc2_kernel2": round(fc2_us, 2)},
               "roofline": {"bound": "tensor", "kernel": "fc1 in emit mode (kernel 1 + emit kernel 2 + LR reduce)",
                            "achieved": round(fc1_flops / (emit_us * 1e-6) / 1e12, 2),
                            "peak": round(peaks["bf16"] * FP4_PER_BF16, 1), "unit": "TFLOP/s",
                            "frac": round(fc1_flops / (emit_us * 1e-6) / 1e12 / (peaks["bf16"] * FP4_PER_BF16), 4),
                            "traffic": None},
               "gpu_launches": 4 * args.steps, "device_status": status, "clocks": clocks.summary()}
    B.svdq_free_weights(l1["h"])
    B.svdq_free_weights(h2)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ small shapes: config 0 and the LoRA sweep
def layer_bytes(M, K, N, r_tot, fmt):
    """Algorithmic HBM bytes of one whole layer call: X, 1/lambda, the
    factors, the residual codes and scales (once), bias and Y.  The
    intermediates qX, sX and LR pass between the two kernels through L2."""
    g, sb = (16, 1) if fmt == "nvfp4" else (64, 2)
    r_pad = -(-r_tot // 64) * 64
    return (M * K * 2 + K * 4 + r_tot * K * 2 + N * K // 2 + N * (K // g) * sb + N * r_pad * 2 + N * 4
            + M * N * 2)


def run_points(args, world, rank, local, which):
    """Per-point timing for shapes whose working set is smaller than L2: the
    small NVFP4 layer (M=128, K=N=1024, rank 32) or the LoRA sweep (K = N =
    3072, M in {256, 1024, 4096, 16384}, rank in {16, 32, 64, 128}, each with
    a rank-16 LoRA).  Every timed call is preceded by an untimed write of a
    buffer twice the L2 size and a read of another one, so weights and
    activations come from HBM as they do when a model runs the layer once per
    block, and the L2 holds no dirty lines to write back; a call's time is the
    difference of two event-timed loops on its stream (with and without the
    call).  Per point: the layer (kernel 1 + kernel 2),
    kernel 2 alone (after an untimed kernel 1), the plain W4A4 path
    (quantize + GEMM without the low-rank branch) and their ratio."""
    import numpy as np
    import torch
    import workloads
    from rank_gemm_b200 import build as _b
    if rank == 0:
        _b.build()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", init_method="env://", world_size=world, rank=rank,
                                timeout=__import__("datetime").timedelta(seconds=120))
        dist.barrier()
    from rank_gemm_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    evict = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # write twice the L2 size, then read another buffer of that size, so
        # the timed call starts with a cold L2 that holds no dirty lines (a
        # write alone would leave the L2 full of dirty lines whose write-back
        # the timed call would pay for)
        flush.zero_()
        torch.sum(evict, dim=0, out=sink)
    peaks = measured_peaks()
    tc_peak = peaks["bf16"] * FP4_PER_BF16

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(dev)

    def timed(fn, pre=None, n=100):
        """Mean device time of fn with the L2 flushed (and pre run) before
        every call: a loop of n x [flush, pre, fn] between two events minus a
        loop of n x [flush, pre], each loop taken three times (medians).  CUDA
        event timestamps on this part step by about 1 us, too coarse for one
        call of a few microseconds, so no single-call interval is used."""
        def loop(with_fn):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(stream)
            for _ in range(n):
                flush_l2()
                if pre:
                    pre()
                if with_fn:
                    fn()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b)
        for _ in range(3):
            flush_l2()
            if pre:
                pre()
            fn()
        t1, t0 = [], []
        for _ in range(3):
            t1.append(loop(True))
            t0.append(loop(False))
        return (statistics.median(t1) - statistics.median(t0)) / n * 1e3

    if which == "small":
        L = workloads.small()
        X_all = dev_bf16(L.X)
        Wt = dev_bf16(L.W.T)
        lam, act, L1f, L2 = gpu_factors(B, Wt, X_all, L.rank, torch)
        specs = [(L.rank, 0, B.svdq_prepare_weights("nvfp4", L.K, L.N, L.rank, Wt, lam, L1f, L2, dev_bf16(L.bias),
                                                    act_scale=act), [L.M])]
        K, N, name = L.K, L.N, L.name
    else:
        base = workloads.lora_sweep_base()
        X_all = dev_bf16(base.X)
        Wt = dev_bf16(base.W.T)
        rmax = max(workloads.LORA_SWEEP_R)
        lam, act, L1f, L2 = gpu_factors(B, Wt, X_all, rmax, torch)   # one split; smaller ranks take its prefix
        la, lb = dev_bf16(base.lora_A), dev_bf16(base.lora_B)
        lora = base.lora_A.shape[1]
        specs = []
        for r in workloads.LORA_SWEEP_R:
            h = B.svdq_prepare_weights("nvfp4", base.K, base.N, r, Wt, lam, L1f[:, :r].contiguous(),
                                       L2[:r].contiguous(), dev_bf16(base.bias), la, lb, lora, act)
            specs.append((r, lora, h, list(workloads.LORA_SWEEP_M)))
        K, N, name = base.K, base.N, "nvfp4_lora_sweep_K3072_N3072_lora%d" % lora
    n = max(10, min(args.steps, 200))
    points = []
    tot_flops = tot_us = 0.0
    with ClockSampler(local) as clocks:
        for r, lora, h, Ms in specs:
            for M in Ms:
                X = X_all[:M]
                Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
                qb, sb, lb = B.svdq_act_buffer_sizes(h, M)
                qX, sX, LR = (torch.empty(v, dtype=torch.uint8, device=dev) for v in (qb, sb, lb))
                k1 = lambda: B.svdq_quantize_act_lowrank_down(h, M, X, qX, sX, LR, stream)
                k2 = lambda: B.svdq_w4a4_gemm_lowrank_up(h, M, qX, sX, LR, B.SVDQ_EPI_NONE, Y, stream)
                t_layer = timed(lambda: (k1(), k2()), n=n)
                t_k2 = timed(k2, pre=k1, n=n)
                t_plain = timed(lambda: (B.svdq_quantize_act(h, M, X, qX, sX, stream),
                                         B.svdq_w4a4_gemm(h, M, qX, sX, Y, stream)), n=n)
                flops = 2.0 * M * N * K
                nbytes = layer_bytes(M, K, N, r + lora, "nvfp4")
                t_roof = max(flops / (tc_peak * 1e12), nbytes / (peaks["hbm"] * 1e9)) * 1e6
                points.append({"M": M, "rank": r, "lora_rank": lora, "us_per_layer": round(t_layer, 2),
                               "tflops": round(flops / (t_layer * 1e-6) / 1e12, 2),
                               "bound": "tensor" if flops / (tc_peak * 1e12) > nbytes / (peaks["hbm"] * 1e9)
                               else "hbm",
                               "roofline_us": round(t_roof, 2), "roofline_frac": round(t_roof / t_layer, 4),
                               "kernel2_us": round(t_k2, 2), "plain_w4a4_us": round(t_plain, 2),
                               "fused_over_plain": round(t_layer / t_plain - 1, 4)})
                tot_flops += flops
                tot_us += t_layer
    status = B.svdq_poll_device_error(stream)
    for _, _, h, _ in specs:
        B.svdq_free_weights(h)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        one = points[0] if which == "small" else None
        out = {"metric": METRIC, "value": round(tot_flops * world / (tot_us * 1e-6) / 1e12, 3), "unit": UNIT,
               "n_gpus": world, "steps": n, "warmup": 3, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "nvfp4",
               "data": "synthetic (seeded, outlier channels x20 / x5), random-init weights",
               "config": {"workload": name, "K": K, "N": N, "format": "nvfp4", "group": 16,
                          "parallelism": "replicas x%d (each rank its own batch)" % world,
                          "l2": "before every timed call a %d MB buffer is written and another read (2 x L2 each): "
                                "cold L2, no dirty lines" % (2 * l2 // 2 ** 20),
                          "timing": "mean of %d calls per point: a loop of [flush, call] minus a loop of [flush], "
                                    "CUDA events at the loop ends, median of 3 each" % n},
               "points": points, "device_status": status, "clocks": clocks.summary(),
               "gpu_launches": 2 * n * len(points)}
        if one:
            out["us_per_layer"] = one["us_per_layer"]
            out["roofline"] = {"bound": one["bound"], "achieved": one["tflops"], "unit": "TFLOP/s",
                               "frac": one["roofline_frac"], "roofline_us": one["roofline_us"]}
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ AWQ W4A16 arm
AWQ_METRIC = "AWQ W4A16 linear effective TFLOPS & % of HBM bandwidth; µs/layer"


def run_awq(args, world, rank, local):
    """The awq_w4a16 modulation projection (workloads.awq_adaln): one
    svdq_awq_linear call per step.  Five prepared weight sets (32 MB each,
    160 MB together > the 126 MB L2) rotate, so the weights stream from HBM
    on every call, as in a model where the layer runs once per block."""
    import numpy as np
    import torch
    import workloads
    from rank_gemm_b200 import build as _b
    if rank == 0:
        _b.build()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", init_method="env://", world_size=world, rank=rank,
                                timeout=__import__("datetime").timedelta(seconds=120))
        dist.barrier()
    from rank_gemm_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    L = workloads.awq_adaln()
    M, K, N = L.M, L.K, L.N
    sets = 5
    Wt = torch.from_numpy(np.ascontiguousarray(L.W.T)).to(torch.bfloat16).to(dev)
    bias = torch.from_numpy(L.bias).to(torch.bfloat16).to(dev)
    hs = [B.svdq_awq_prepare(K, N, Wt, None, bias) for _ in range(sets)]
    del Wt
    X = torch.from_numpy(L.X).to(torch.bfloat16).to(dev)
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(sets)]
    stream = torch.cuda.current_stream(dev)
    for i in range(args.warmup):
        B.svdq_awq_linear(hs[i % sets], M, X, Ys[i % sets], stream)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            B.svdq_awq_linear(hs[i % sets], M, X, Ys[i % sets], stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    max_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    status = B.svdq_poll_device_error(stream)
    us = max_ms / args.steps * 1e3
    # the kernel's own duration: the same calls captured once in a CUDA graph
    # and replayed (no host launch overhead between them)
    g_stream = torch.cuda.Stream(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=g_stream):
        for i in range(sets):
            B.svdq_awq_linear(hs[i], M, X, Ys[i], g_stream)
    reps = max(1, min(args.steps, 2000) // sets)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(torch.cuda.current_stream(dev))
    for _ in range(reps):
        graph.replay()
    g1.record(torch.cuda.current_stream(dev))
    torch.cuda.synchronize()
    kern_us = max_over_ranks(g0.elapsed_time(g1), world, dev) / (reps * sets) * 1e3
    del graph
    flops = 2.0 * M * N * K
    value = weak_scaling_value(flops, args.steps, world, max_ms)
    peaks = measured_peaks()
    G = K // 64
    # algorithmic bytes: codes, scales and zero points once, X, 1/s, bias, Y
    nbytes = N * K // 2 + G * N * 3 + M * K * 2 + K * 4 + N * 4 + M * N * 2
    gbs = nbytes / (kern_us * 1e-6) / 1e9
    traffic = profiled_traffic("awq_gemv_%s.md" % "adaln", kernel_sources("awq.cu"))
    # end to end through the public call with host buffers
    Xh = torch.empty(M, K, dtype=torch.bfloat16, pin_memory=True)
    Xh.copy_(X.cpu())
    Yh = torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True)
    Xd = torch.empty_like(X)
    e2e_steps = min(args.steps, 200)
    for i in range(3):
        Xd.copy_(Xh, non_blocking=True)
        B.svdq_awq_linear(hs[i % sets], M, Xd, Ys[0], stream)
        Yh.copy_(Ys[0], non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        Xd.copy_(Xh, non_blocking=True)
        B.svdq_awq_linear(hs[i % sets], M, Xd, Ys[0], stream)
        Yh.copy_(Ys[0], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    out = None
    if rank == 0:
        out = {"metric": AWQ_METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 6), "us_per_layer": round(us, 3),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 x int4 -> f32",
               "data": "synthetic (seeded: SiLU(randn) activation, randn*0.02 weight), random-init weights",
               "config": {"workload": L.name, "M": M, "K": K, "N": N, "group": 64, "awq_scale": "none",
                          "parallelism": "replicas x%d (each rank its own batch)" % world,
                          "l2": "%d rotating weight sets (%.0f MB) > 126 MB L2" % (sets, sets * nbytes / 1e6)},
               "roofline": {"kernel": "awq_gemv", "bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm"],
                            "unit": "GB/s", "frac": round(gbs / peaks["hbm"], 4), "traffic": traffic,
                            "algorithmic_bytes": nbytes, "us": round(kern_us, 3),
                            "timing": "CUDA graph of the %d rotating calls, replayed %d times" % (sets, reps),
                            "peak_source": "%s HBM copy bandwidth" % peaks["source"]},
               "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 4), "unit": UNIT,
                       "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                       "ms_per_step": round(e2e_ms, 5)},
               "gpu_launches": args.steps, "device_status": status, "clocks": clocks.summary()}
    for h in hs:
        B.svdq_awq_free(h)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            from oracle import awq as A
            aw = A.prepare(L.W, L.bias)
            ts = []
            for _ in range(3):
                c0 = time.perf_counter()
                A.forward(aw, L.X)
                ts.append(time.perf_counter() - c0)
            t = statistics.median(ts)
            out["cpu_baseline"] = {"value": round(flops / t / 1e12, 6), "unit": UNIT, "cores": oracle_threads(),
                                   "kind": "oracle",
                                   "sample": "float64 numpy oracle forward of the whole layer (dequantize, "
                                             "matmul, bias); median of 3", "seconds_per_sample": round(t, 4)}
        print(json.dumps(out), flush=True)


def run_awq_qkv(args, world, rank, local):
    """The W4A16 side of the "SVDQuant" abstract's comparison on the QKV shape
    (M=4608, K=3072, N=9216): the same activation, weight and bias as the
    NVFP4 QKV line, quantized as an AWQ W4A16 layer (int4, group 64) and run
    by svdq_awq_gemm (16-bit operands on the tensor core); the NVFP4 W4A4
    layer (svdq_linear) is timed the same way in the same process, and the
    line reports their ratio."""
    import numpy as np
    import torch
    import workloads
    from rank_gemm_b200 import build as _b
    if rank == 0:
        _b.build()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", init_method="env://", world_size=world, rank=rank,
                                timeout=__import__("datetime").timedelta(seconds=120))
        dist.barrier()
    from rank_gemm_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    L = workloads.awq_qkv()
    M, K, N = L.M, L.K, L.N
    Wt = torch.from_numpy(np.ascontiguousarray(L.W.T)).to(torch.bfloat16).to(dev)
    bias = torch.from_numpy(L.bias).to(torch.bfloat16).to(dev)
    ha = B.svdq_awq_prepare(K, N, Wt, None, bias)
    lay = build_layer("qkv", B, torch, dev)
    sets = 3
    X0 = lay["X0"]
    Xs = [X0] + [X0.clone() for _ in range(sets - 1)]
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(sets)]
    wss = [torch.empty(B.svdq_linear_workspace_bytes(lay["h"], M), dtype=torch.uint8, device=dev)
           for _ in range(sets)]
    awq = lambda i: B.svdq_awq_gemm(ha, M, Xs[i % sets], Ys[i % sets], stream)
    w4a4 = lambda i: B.svdq_linear(lay["h"], M, Xs[i % sets], B.SVDQ_EPI_NONE, Ys[i % sets], wss[i % sets], None,
                                   stream)
    for i in range(args.warmup):
        awq(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            awq(i)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    max_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    status = B.svdq_poll_device_error(stream)
    n_cmp = min(args.steps, 300)
    for i in range(3):
        w4a4(i)
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for i in range(n_cmp):
        w4a4(i)
    c1.record(stream)
    torch.cuda.synchronize()
    w4a4_us = max_over_ranks(c0.elapsed_time(c1), world, dev) / n_cmp * 1e3
    us = max_ms / args.steps * 1e3
    flops = 2.0 * M * N * K
    value = weak_scaling_value(flops, args.steps, world, max_ms)
    peaks = measured_peaks()
    out = None
    if rank == 0:
        out = {"metric": "AWQ W4A16 linear effective TFLOPS & % of BF16 tensor peak; µs/layer",
               "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 5), "us_per_layer": round(us, 2),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 x int4 -> f32",
               "data": "synthetic (the QKV workload's seeded X, W and bias), random-init weights",
               "config": {"workload": L.name, "M": M, "K": K, "N": N, "group": 64, "awq_scale": "none",
                          "parallelism": "replicas x%d (each rank its own batch)" % world,
                          "l2": "3 rotating X/Y sets (%.0f MB) > 126 MB L2" % (sets * (M * K * 2 + M * N * 2) / 1e6)},
               "roofline": {"kernel": "awq_gemm", "bound": "tensor", "achieved": round(flops / (us * 1e-6) / 1e12, 2),
                            "peak": peaks["bf16"], "unit": "TFLOP/s",
                            "frac": round(flops / (us * 1e-6) / 1e12 / peaks["bf16"], 4), "traffic": None,
                            "peak_source": "%s bf16 (the product runs on bf16 operands)" % peaks["source"]},
               "w4a4_nvfp4_us": round(w4a4_us, 2), "w4a4_over_w4a16_speedup": round(us / w4a4_us, 3),
               "gpu_launches": args.steps, "device_status": status, "clocks": clocks.summary()}
    B.svdq_awq_free(ha)
    B.svdq_free_weights(lay["h"])
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_library_fp4(args, world, rank, local):
    """Context, not a product path: library NVFP4 GEMMs (flashinfer's mm_fp4
    with its cuDNN, CUTLASS and TRT-LLM backends, plain GEMM without the
    low-rank branch) and torch's bf16 matmul on the QKV shape, beside this
    library's kernel 2 (plain and with the fused low-rank branch), CUDA
    events on the same stream, the same box.  Backends that fail to build or
    run are reported as such."""
    import numpy as np
    import torch
    from rank_gemm_b200 import build as _b
    _b.build()
    from rank_gemm_b200 import binding as B
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    M, N, K = WORKLOAD["M"], WORKLOAD["N"], WORKLOAD["K"]
    flops = 2.0 * M * N * K
    n = max(10, min(args.steps, 100))

    def timed(fn):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n * 1e3

    print("library_fp4: timing this library's kernel 2", file=sys.stderr, flush=True)
    out = {"metric": "NVFP4 GEMM on the QKV shape, library kernels beside this library's kernel 2 (context)",
           "unit": "us", "n_gpus": 1, "steps": n, "higher_is_better": False,
           "config": {"workload": WORKLOAD["name"], "M": M, "K": K, "N": N}, "results": {}}
    lay = build_layer("qkv", B, torch, dev)
    h, X0 = lay["h"], lay["X0"]
    qb, sb, lb = B.svdq_act_buffer_sizes(h, M)
    qX, sX, LR = (torch.empty(v, dtype=torch.uint8, device=dev) for v in (qb, sb, lb))
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    B.svdq_quantize_act_lowrank_down(h, M, X0, qX, sX, LR, stream)
    t = timed(lambda: B.svdq_w4a4_gemm(h, M, qX, sX, Y, stream))
    out["results"]["svdq kernel 2, plain W4A4"] = {"us": round(t, 2), "tflops": round(flops / t / 1e6, 1)}
    t = timed(lambda: B.svdq_w4a4_gemm_lowrank_up(h, M, qX, sX, LR, B.SVDQ_EPI_NONE, Y, stream))
    out["results"]["svdq kernel 2, fused low-rank branch"] = {"us": round(t, 2), "tflops": round(flops / t / 1e6, 1)}
    B.svdq_free_weights(h)
    g = torch.Generator(device="cpu").manual_seed(0)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16).to(dev)
    bm = torch.randn(N, K, generator=g).to(torch.bfloat16).to(dev)
    t = timed(lambda: a @ bm.T)
    out["results"]["torch bf16 matmul"] = {"us": round(t, 2), "tflops": round(flops / t / 1e6, 1)}
    try:
        import flashinfer
        from flashinfer import SfLayout, mm_fp4, nvfp4_quantize
        ag = (448 * 6) / a.float().abs().max()
        bg = (448 * 6) / bm.float().abs().max()
        for backend, shuffle in (("cudnn", False), ("cutlass", False), ("trtllm", True)):
            print("library_fp4: flashinfer backend", backend, file=sys.stderr, flush=True)
            try:
                a4, asf = nvfp4_quantize(a, ag, sfLayout=SfLayout.layout_128x4, do_shuffle=False)
                b4, bsf = nvfp4_quantize(bm, bg, sfLayout=SfLayout.layout_128x4, do_shuffle=shuffle)
                y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
                alpha = torch.tensor([1.0 / (ag * bg)], dtype=torch.float32, device=dev)
                t = timed(lambda: mm_fp4(a4, b4.T, asf, bsf.T, alpha, torch.bfloat16, y, backend=backend))
                out["results"]["flashinfer mm_fp4 " + backend] = {"us": round(t, 2), "tflops": round(flops / t / 1e6, 1)}
            except Exception as ex:
                out["results"]["flashinfer mm_fp4 " + backend] = {"unavailable": "%s: %s" % (type(ex).__name__,
                                                                                           str(ex)[:200])}
        out["flashinfer"] = getattr(flashinfer, "__version__", "?")
    except Exception as ex:
        out["results"]["flashinfer"] = {"unavailable": "%s: %s" % (type(ex).__name__, str(ex)[:200])}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=WORKLOADS, default="qkv")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, world, rank)
    elif args.workload == "awq_adaln":
        run_awq(args, world, rank, local)
    elif args.workload == "mlp_pair":
        run_mlp_pair(args, world, rank, local)
    elif args.workload == "awq_qkv":
        run_awq_qkv(args, world, rank, local)
    elif args.workload == "library_fp4":
        if rank == 0:
            run_library_fp4(args, world, rank, local)
    elif args.workload in ("small", "lora_sweep"):
        run_points(args, world, rank, local, args.workload)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
