"""Benchmark of the joint text+image attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {native,reference}]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...

One step is the whole BF16 hot path for one DiT attention call of the
2048x2048-image workload (B=1, H=24, D=128, 512 text + 128x128 image tokens):
rotary table build, the K rotation pass and the attention forward writing bf16
O and the LSE.  Throughput is the dense attention work 4 N^2 D H B per step
over the step time (TFLOP/s).  Each rank runs its own copy of the workload
(weak scaling, no data-path collective); the whole-job value divides the work
of all ranks by the slowest rank's time.

`--impl reference` times the fp64 CPU oracle (the reference arm: there is no
other implementation of this path) on a bounded sample of query rows of the
same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

WORKLOAD = "t2i_2048px"
METRIC = "joint-attention TFLOP/s and % of B200 dense BF16/FP8 tensor peak (1 GPU)"
UNIT = "TFLOP/s"
FALLBACK_PEAK_BF16 = 1590.0
# Datasheet dense (no 2:4 sparsity) tensor peaks of one B200 as the pages quote
# them (bpdata.com "FLUX 3 Image Klein optimalizálása", hardware section):
# BF16 2.25 PFLOP/s, FP8 4.5 PFLOP/s.
NOMINAL_PEAK_BF16 = 2250.0
NOMINAL_PEAK_FP8 = 4500.0
E2E_CHUNK_HEADS = 4          # heads per chunk of the host-buffer pipeline


# ------------------------------------------------------------------ multi-rank
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over all ranks (x itself with one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def whole_job_throughput(flops_per_step_per_rank: float, steps: int, world: int, max_ms: float) -> float:
    """TFLOP/s of the whole job: work of all ranks over the slowest rank's time."""
    return flops_per_step_per_rank * steps * world / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML in a thread."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x1: "gpu_idle", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clocks rather than fail
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((mhz, reasons, util))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        loaded = [s for s in self.samples if s[2] > 0] or self.samples
        reasons = set()
        for _, r, _ in loaded:
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(loaded)}


# ------------------------------------------------------------------ helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    return FALLBACK_PEAK_BF16, "fallback 1.59 PFLOP/s"


def measured_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"])
    return 6650.0


# The translation unit of each profiled kernel; its counters stay valid while
# that file and the shared headers are unchanged.
KERNEL_SOURCES = {"attn_fwd_bf16_kernel": "attn_fwd.cu", "attn_fwd_fp8_kernel": "attn_fwd_fp8.cu",
                  "merge_kernel": "merge.cu", "quantize_kernel": "quant_fp8.cu",
                  "quantize_unrotated_kernel": "quant_fp8.cu", "qkv_proj_pair_kernel": "qkv_proj.cu"}


def profile_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` on the bench workload from the
    committed ncu summary, or None if none was taken of the kernel's current
    source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    entry = d.get("kernels", {}).get(kernel, {})
    if d.get("workload") != WORKLOAD or entry.get("source_sha") != kernel_source_sha(kernel):
        return None
    return entry.get("dram_bytes_per_launch")


def kernel_source_sha(kernel: str) -> str:
    """Hash of the kernel's .cu file and every header in csrc/."""
    import hashlib
    csrc = os.path.join(ROOT, "diffusion_transformer_joint_attn_b200", "csrc")
    names = [KERNEL_SOURCES[kernel]] + sorted(n for n in os.listdir(csrc) if n.endswith((".cuh", ".h")))
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def oracle_sample(w, rows_per_head: int):
    """Rows (b, h, n) of the CPU-baseline sample: the first rows_per_head query
    rows of every head."""
    rows = [(b, h, n) for b in range(w.B) for h in range(w.H) for n in range(rows_per_head)]
    return np.asarray(rows, dtype=np.int64)


def time_oracle(w, q, k, v, rows):
    from oracle import attention as oracle_attention
    from threadpoolctl import threadpool_info
    t0 = time.perf_counter()
    oracle_attention.joint_attention(q, k, v, pos=W.positions(w), rows=rows)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    flops = 4.0 * w.N * w.D * len(rows)
    return flops / dt / 1e12, dt, threads


def time_fp8_variant(args, w, lib, q, k, v, cos, sin, out, lse, stream, dev, world):
    """The FP8 E4M3 variant on the same inputs: per-64-token quantisation of
    the rotated q, k and of v, then the FP8 attention forward.  Timed apart
    from the BF16 step; the kernel's roofline peak mixes the two tensor rates
    (q k^T on E4M3 operands at twice the bf16 rate, P V in fp16)."""
    import torch
    import diffusion_transformer_joint_attn_b200 as dit
    nb = (w.N + 63) // 64
    q8, k8, v8 = (torch.empty(q.shape, dtype=torch.uint8, device=dev) for _ in range(3))
    qs, ks, vs = (torch.empty((w.B, w.H, nb), dtype=torch.float32, device=dev) for _ in range(3))
    s_ptr = stream.cuda_stream

    def step(ev=None):
        if ev is not None:
            ev[2].record(stream)
        assert lib.dit_attn_quantize_fp8(q.data_ptr(), cos.data_ptr(), sin.data_ptr(), q8.data_ptr(), qs.data_ptr(),
                                         w.B, w.H, w.N, w.D, s_ptr) == 0
        if ev is not None:
            ev[3].record(stream)
        assert lib.dit_attn_quantize_fp8(k.data_ptr(), cos.data_ptr(), sin.data_ptr(), k8.data_ptr(), ks.data_ptr(),
                                         w.B, w.H, w.N, w.D, s_ptr) == 0
        if ev is not None:
            ev[4].record(stream)
        assert lib.dit_attn_quantize_fp8(v.data_ptr(), None, None, v8.data_ptr(), vs.data_ptr(),
                                         w.B, w.H, w.N, w.D, s_ptr) == 0
        if ev is not None:
            ev[0].record(stream)
        assert lib.dit_attn_forward_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), qs.data_ptr(), ks.data_ptr(),
                                        vs.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B, w.H, w.n_txt, w.n_img,
                                        w.D, dit.DIT_FP8_E4M3, s_ptr) == 0
        if ev is not None:
            ev[1].record(stream)

    steps = max(1, min(args.steps, 50))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    kern_ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(5)) for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for i in range(steps):
        step(kern_ev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if dit.dit_attn_get_status(stream) != 0:
        raise RuntimeError("device status error in the FP8 timed region")
    max_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    kern_ms = sum(e[0].elapsed_time(e[1]) for e in kern_ev) / steps
    quant_rot_ms = sum(e[2].elapsed_time(e[3]) for e in kern_ev) / steps     # q (rotated)
    quant_v_ms = sum(e[4].elapsed_time(e[0]) for e in kern_ev) / steps       # v (unrotated)
    peak_bf16, src = measured_peaks()
    # the dense FP8 peak: the measured bf16 peak times the nominal FP8 / BF16 ratio (2)
    peak = 2.0 * peak_bf16
    # the kernel's own minimum time with q k^T at the E4M3 rate and P V at the fp16 rate:
    # (F/2) / (2 P) + (F/2) / P = 0.75 F / P
    peak_mixed = peak_bf16 / 0.75
    achieved = w.flops / (kern_ms * 1e-3) / 1e12
    # quantiser: 2 B read + 1 B written per element, 4 B per 64-token block scale, and for q, k the
    # table rows (2 x 64 fp32 per token) once
    elems = w.B * w.H * w.N * w.D
    q_bytes = 3 * elems + 4 * w.B * w.H * nb + 512 * w.N
    v_bytes = 3 * elems + 4 * w.B * w.H * nb
    hbm = measured_hbm()

    def quant_leg(ms, nbytes, kernel):
        return {"kernel_ms": ms, "bytes_per_launch": nbytes,
                "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                             "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "kernel": kernel,
                             "traffic": profile_traffic(kernel) if w.name == WORKLOAD else None,
                             "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)"}}

    quant = {"rotated": quant_leg(quant_rot_ms, q_bytes, "quantize_kernel"),
             "unrotated": quant_leg(quant_v_ms, v_bytes, "quantize_unrotated_kernel")}
    return {"value": whole_job_throughput(w.flops, steps, world, max_ms), "unit": UNIT, "steps": steps,
            "ms_per_step": max_ms / steps, "dtype": "e4m3 (q k^T), fp16 (P V)",
            "step": "quantise rotated q, k and v to E4M3 (per 64 tokens) + FP8 attention forward",
            "gpu_launches": 4 * steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "kernel": "attn_fwd_fp8_kernel",
                         "traffic": profile_traffic("attn_fwd_fp8_kernel")
                         if w.name == WORKLOAD else None,
                         "peak_source": src + " x 2 (dense FP8 = 2x dense BF16, nominal ratio)",
                         "frac_nominal": achieved / NOMINAL_PEAK_FP8,
                         "note_mixed_peak": {"peak": peak_mixed, "frac": achieved / peak_mixed,
                                             "why": "q k^T on E4M3 at 2x, P V on fp16 at 1x the bf16 rate"},
                         "kernel_ms": kern_ms},
            "quantiser": quant}


def time_sparse(args, w, lib, q, k_rot, v_f16, cos, sin, out, lse, stream, dev, dense_ms, density=0.5):
    """dit_attn_forward_sparse on the same prepared operands with a seeded
    random block mask selecting `density` of the (512-row query block,
    128-key tile) pairs.  Throughput counts the selected work only (4 x
    rows x keys x D per selected pair, ragged edges exact)."""
    import torch
    nq, nk = (w.N + 511) // 512, (w.N + 127) // 128
    rng = np.random.default_rng(0)
    mask = (rng.random((w.B, w.H, nq, nk)) < density).astype(np.uint8)
    rows = np.minimum(512, w.N - 512 * np.arange(nq))
    keys = np.minimum(128, w.N - 128 * np.arange(nk))
    flops = 4.0 * w.D * float((mask * rows[None, None, :, None] * keys[None, None, None, :]).sum())
    md = torch.from_numpy(mask).to(dev)
    flags = 0x200 | 0x400          # DIT_K_ROTATED | DIT_V_F16
    s_ptr = stream.cuda_stream

    def launch():
        assert lib.dit_attn_forward_sparse(q.data_ptr(), k_rot.data_ptr(), v_f16.data_ptr(), cos.data_ptr(),
                                           sin.data_ptr(), md.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B, w.H,
                                           w.n_txt, w.n_img, w.D, flags, s_ptr) == 0

    for _ in range(max(3, args.warmup)):
        launch()
    steps = max(1, min(args.steps, 30))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        a.record(stream)
        launch()
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    peak, src = measured_peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    return {"density": float(mask.mean()), "kernel_ms": ms, "time_vs_dense": ms / dense_ms, "launches": steps,
            "selected_tflop": flops / 1e12,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                         "traffic": None, "kernel": "attn_fwd_bf16_kernel (block-sparse)", "peak_source": src}}


def time_launches(launch, stream, dev, n, warmup=3):
    """Per-launch durations (ms) of `n` launches, CUDA events on `stream`."""
    import torch
    for _ in range(warmup):
        launch()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        a.record(stream)
        launch()
        b.record(stream)
    torch.cuda.synchronize(dev)
    return [a.elapsed_time(b) for a, b in ev]


def time_split(args, w, lib, q, k, v, cos, sin, out, lse, stream, dev):
    """The split (compensated q k^T) form on the same inputs: fp16 hi + lo
    operands (dit_attn_prepare_kv_split, timed with the step), three q k^T
    products per tile.  Throughput counts the method's 4 N^2 D H B; the
    kernel's tensor work is twice that (q k^T three times, P V once), which
    its roofline reports."""
    import torch
    import diffusion_transformer_joint_attn_b200 as dit
    k_split = torch.empty((2,) + tuple(k.shape), dtype=torch.float16, device=dev)
    v_f16 = torch.empty(v.shape, dtype=torch.float16, device=dev)
    s_ptr = stream.cuda_stream
    flags = dit.DIT_BF16 | dit.DIT_QK_SPLIT | dit.DIT_V_F16

    def prep():
        assert lib.dit_attn_prepare_kv_split(k.data_ptr(), v.data_ptr(), cos.data_ptr(), sin.data_ptr(),
                                             k_split.data_ptr(), v_f16.data_ptr(), w.B, w.H, w.N, w.D, s_ptr) == 0

    def attn():
        assert lib.dit_attn_forward(q.data_ptr(), k_split.data_ptr(), v_f16.data_ptr(), cos.data_ptr(),
                                    sin.data_ptr(), out.data_ptr(), lse.data_ptr(), w.B, w.H, w.n_txt, w.n_img,
                                    w.D, flags, s_ptr) == 0

    steps = max(1, min(args.steps, 20))
    step_ms = time_launches(lambda: (prep(), attn()), stream, dev, steps)
    kern = time_launches(attn, stream, dev, steps)
    if dit.dit_attn_get_status(stream) != 0:
        raise RuntimeError("device status error in the split-form timing")
    kern_ms = statistics.mean(kern)
    peak, src = measured_peaks()
    tensor_achieved = 2.0 * w.flops / (kern_ms * 1e-3) / 1e12
    return {"value": w.flops / (statistics.mean(step_ms) * 1e-3) / 1e12, "unit": UNIT,
            "ms_per_step": statistics.mean(step_ms),
            "step": "split of rotated K (dit_attn_prepare_kv_split) + split-form attention forward",
            "kernel_ms": kern_ms, "kernel_value": w.flops / (kern_ms * 1e-3) / 1e12,
            "dtype": "fp16 hi + lo (q k^T, 3 products), fp16 (P V)",
            "roofline": {"bound": "tensor", "achieved": tensor_achieved, "peak": peak, "unit": UNIT,
                         "frac": tensor_achieved / peak, "kernel": "attn_fwd_split_kernel", "traffic": None,
                         "peak_source": src,
                         "work": "tensor work 8 N^2 D H B per launch (q k^T x3 + P V), twice the method's count"}}


def time_projection(args, w, lib, cos, sin, stream, dev, C=3072):
    """dit_qkv_project_fp8 on the workload's token count: the QKV projection
    of seeded hidden states x [B, N, 3072] (the FLUX width, 24 heads x 128)
    with a seeded weight [3 H 128, 3072], the rotary embedding of q, k and the
    E4M3 block quantisation of q, k, v in its epilogue.  A GEMM of 2 B N C
    (3 H 128) FLOP; its roofline is the tensor peak."""
    import torch
    g = torch.Generator().manual_seed(5)
    x = torch.randn(w.B, w.N, C, generator=g).to(torch.bfloat16).to(dev)
    wt = (torch.randn(3 * w.H * 128, C, generator=g) / C ** 0.5).to(torch.bfloat16).to(dev)
    bias = (0.1 * torch.randn(3 * w.H * 128, generator=g)).float().to(dev)
    nb = (w.N + 63) // 64
    codes = [torch.empty((w.B, w.H, w.N, 128), dtype=torch.uint8, device=dev) for _ in range(3)]
    scales = [torch.empty((w.B, w.H, nb), dtype=torch.float32, device=dev) for _ in range(3)]
    s_ptr = stream.cuda_stream

    def launch():
        assert lib.dit_qkv_project_fp8(x.data_ptr(), wt.data_ptr(), bias.data_ptr(), cos.data_ptr(), sin.data_ptr(),
                                       *[t.data_ptr() for t in codes], *[t.data_ptr() for t in scales], None, None,
                                       None, w.B, w.N, C, w.H, 128, s_ptr) == 0

    ms = statistics.mean(time_launches(launch, stream, dev, max(1, min(args.steps, 20))))
    import diffusion_transformer_joint_attn_b200 as dit
    if dit.dit_attn_get_status(stream) != 0:
        raise RuntimeError("device status error in the projection timing")
    flops = 2.0 * w.B * w.N * C * 3 * w.H * 128
    peak, src = measured_peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    return {"kernel_ms": ms, "value": achieved, "unit": UNIT, "tflop_per_launch": flops / 1e12,
            "shape": "x [%d, %d, %d] x w [%d, %d]" % (w.B, w.N, C, 3 * w.H * 128, C),
            "step": "QKV projection GEMM with rotary embedding and E4M3 block quantisation in its epilogue",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "kernel": "qkv_proj_pair_kernel" if w.H % 4 == 0 else "qkv_proj_fp8_kernel",
                         "traffic": profile_traffic("qkv_proj_pair_kernel") if w.name == WORKLOAD and w.H % 4 == 0
                         else None,
                         "peak_source": src}}


def time_fused_k(args, w, lib, q, k, v, cos, sin, out, lse, stream, dev):
    """The forward with the rotary embedding of K inside the kernel's tile
    prologue (raw bf16 K and V: each query tile's CTA pair rotates every K
    tile and converts every V tile itself), against the prepared-operand path
    of the main step."""
    import diffusion_transformer_joint_attn_b200 as dit
    s_ptr = stream.cuda_stream

    def attn():
        assert lib.dit_attn_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), cos.data_ptr(), sin.data_ptr(),
                                    out.data_ptr(), lse.data_ptr(), w.B, w.H, w.n_txt, w.n_img, w.D, dit.DIT_BF16,
                                    s_ptr) == 0

    kern = time_launches(attn, stream, dev, max(1, min(args.steps, 10)))
    if dit.dit_attn_get_status(stream) != 0:
        raise RuntimeError("device status error in the fused-K timing")
    kern_ms = statistics.mean(kern)
    peak, src = measured_peaks()
    achieved = w.flops / (kern_ms * 1e-3) / 1e12
    return {"kernel_ms": kern_ms, "value": achieved, "unit": UNIT,
            "step": "attention forward with K rotated and V converted per tile inside the kernel (no operand pass)",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                         "kernel": "attn_fwd_bf16_kernel (in-loop operand instance)", "traffic": None,
                         "peak_source": src}}


def time_flushed(args, w, launch, stream, dev, l2_flush_bytes=256 << 20):
    """Mean duration of `launch` with a 256 MB device write between calls,
    so that each call starts with a cold L2 (the unflushed number relies on
    the inputs being larger than L2 instead)."""
    import torch
    scratch = torch.empty(l2_flush_bytes, dtype=torch.uint8, device=dev)
    steps = max(1, min(args.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    launch()
    for a, b in ev:
        scratch.fill_(1)
        a.record(stream)
        launch()
        b.record(stream)
    torch.cuda.synchronize(dev)
    return sum(a.elapsed_time(b) for a, b in ev) / steps


def time_sdpa_context(args, w, q, k, v, stream, dev):
    """Context only: torch's scaled_dot_product_attention (the backend torch
    picks on this GPU) on the same bf16 [B, H, N, D] shape without rotary
    embedding and without the LSE.  A library call, not this path."""
    import torch
    import torch.nn.functional as F
    try:
        for _ in range(2):
            F.scaled_dot_product_attention(q, k, v)
        torch.cuda.synchronize(dev)
        steps = max(1, min(args.steps, 10))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            F.scaled_dot_product_attention(q, k, v)
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b) / steps
        return {"value": w.flops / (ms * 1e-3) / 1e12, "unit": UNIT, "ms": ms,
                "what": "torch.nn.functional.scaled_dot_product_attention, bf16, no rotary, no LSE (library)"}
    except Exception as e:       # context only: a missing backend is reported, not fatal
        return {"unavailable": str(e)[:200]}


def time_merge(args, w, lib, out, lse, stream, dev):
    """dit_attn_merge of R = 2 bf16 partial results of the workload's shape
    (a 2-way context-parallel split); memory-bound, reported in GB/s of the
    algorithmic bytes (R part rows + lses read, one row + lse written)."""
    import torch
    import diffusion_transformer_joint_attn_b200 as dit
    parts = [out, out.clone()]
    lses = [lse, lse.clone()]
    merged = torch.empty_like(out)
    merged_lse = torch.empty_like(lse)
    R = len(parts)
    optr = (ctypes.c_void_p * R)(*[p.data_ptr() for p in parts])
    lptr = (ctypes.c_void_p * R)(*[p.data_ptr() for p in lses])
    s_ptr = stream.cuda_stream

    def launch():
        assert lib.dit_attn_merge(ctypes.cast(optr, ctypes.c_void_p), ctypes.cast(lptr, ctypes.c_void_p), R,
                                  merged.data_ptr(), merged_lse.data_ptr(), w.B, w.H, w.N, w.D, dit.DIT_BF16,
                                  s_ptr) == 0

    for _ in range(max(3, args.warmup)):
        launch()
    steps = max(1, min(args.steps, 50))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        a.record(stream)
        launch()
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    rows = w.B * w.H * w.N
    nbytes = (R + 1) * rows * (w.D * 2 + 4)
    peak = measured_hbm()
    achieved = nbytes / (ms * 1e-3) / 1e9
    # inputs and output (316 MB at 2048^2) exceed the 126 MB L2; no flush between launches
    return {"R": R, "bytes_per_launch": nbytes, "kernel_ms": ms, "launches": steps,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "kernel": "merge_kernel",
                         "traffic": profile_traffic("merge_kernel") if w.name == WORKLOAD
                         else None,
                         "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)"}}


def workload_config(w, world):
    """The workload keys both arms report."""
    return {"workload": w.name, "B": w.B, "H": w.H, "D": w.D, "n_txt": w.n_txt, "n_img": w.n_img, "N": w.N,
            "inputs": "seeded N(0,1) bf16" + (", channels 3/40/77/110 x16" if w.outliers else ""),
            "parallelism": "replica per GPU" if world > 1 else "single GPU"}


# ------------------------------------------------------------------ native arm
def run_native(args):
    import torch
    import diffusion_transformer_joint_attn_b200 as dit

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = W.WORKLOADS[args.workload]
    dit.load_library()

    q_h, k_h, v_h = W.make_qkv(w, seed=rank)
    pos_h = torch.from_numpy(W.positions(w))
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    pos = pos_h.to(dev)
    cos = torch.empty((w.N, 64), dtype=torch.float32, device=dev)
    sin = torch.empty_like(cos)
    k_rot = torch.empty_like(k)
    v_f16 = torch.empty(v.shape, dtype=torch.float16, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    lib = dit.load_library()
    s_ptr = stream.cuda_stream
    axes = (ctypes.c_int32 * 3)(*W.ROPE_AXES)
    flags = dit.DIT_BF16 | dit.DIT_K_ROTATED | dit.DIT_V_F16

    def step(ev=None):
        # the whole BF16 hot path: rotary table, K / V operand pass, attention forward
        assert lib.dit_rope_table_build(pos.data_ptr(), w.N, w.D, axes, W.ROPE_THETA, cos.data_ptr(),
                                        sin.data_ptr(), s_ptr) == 0
        assert lib.dit_attn_prepare_kv(k.data_ptr(), v.data_ptr(), cos.data_ptr(), sin.data_ptr(), k_rot.data_ptr(),
                                       v_f16.data_ptr(), w.B, w.H, w.N, w.D, s_ptr) == 0
        if ev is not None:
            ev[0].record(stream)
        assert lib.dit_attn_forward(q.data_ptr(), k_rot.data_ptr(), v_f16.data_ptr(), cos.data_ptr(), sin.data_ptr(),
                                    out.data_ptr(), lse.data_ptr(), w.B, w.H, w.n_txt, w.n_img, w.D, flags,
                                    s_ptr) == 0
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = dit.dit_attn_get_status(stream)
    if status != 0:
        raise RuntimeError("device status %d after warm-up" % status)

    kern_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            step(kern_ev[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = t0.elapsed_time(t1)
    kern_ms = sum(a.elapsed_time(b) for a, b in kern_ev) / args.steps
    if dit.dit_attn_get_status(stream) != 0:
        raise RuntimeError("device status error in the timed region")
    max_ms = max_over_ranks(ms, world, dev)
    value = whole_job_throughput(w.flops, args.steps, world, max_ms)

    fp8 = time_fp8_variant(args, w, lib, q, k, v, cos, sin, out, lse, stream, dev, world)
    merge = time_merge(args, w, lib, out, lse, stream, dev)
    sparse = time_sparse(args, w, lib, q, k_rot, v_f16, cos, sin, out, lse, stream, dev, kern_ms)

    def attn_launch():
        assert lib.dit_attn_forward(q.data_ptr(), k_rot.data_ptr(), v_f16.data_ptr(), cos.data_ptr(), sin.data_ptr(),
                                    out.data_ptr(), lse.data_ptr(), w.B, w.H, w.n_txt, w.n_img, w.D, flags,
                                    s_ptr) == 0
    kern_ms_flushed = time_flushed(args, w, attn_launch, stream, dev)
    median50 = statistics.median(time_launches(attn_launch, stream, dev, 50))
    split = time_split(args, w, lib, q, k, v, cos, sin, out, lse, stream, dev)
    fused_k = time_fused_k(args, w, lib, q, k, v, cos, sin, out, lse, stream, dev)
    proj = time_projection(args, w, lib, cos, sin, stream, dev)
    sdpa = time_sdpa_context(args, w, q, k, v, stream, dev)

    # end to end through the public C ABI with host buffers: pinned q, k, v
    # and positions in, O and LSE out; dit_attn_forward_host moves chunks of
    # E2E_CHUNK_HEADS heads through a device workspace, overlapping its copies
    # with the kernels
    q_p, k_p, v_p = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    pos_p = pos_h.pin_memory()
    out_p = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_p = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (q_p, k_p, v_p, pos_p))
    d2h = out_p.numel() * out_p.element_size() + lse_p.numel() * lse_p.element_size()
    ws_bytes = lib.dit_attn_forward_host_workspace(w.B, w.H, w.N, w.D, dit.DIT_BF16, E2E_CHUNK_HEADS)
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def e2e_step():
        pos.copy_(pos_p, non_blocking=True)
        assert lib.dit_rope_table_build(pos.data_ptr(), w.N, w.D, axes, W.ROPE_THETA, cos.data_ptr(),
                                        sin.data_ptr(), s_ptr) == 0
        assert lib.dit_attn_forward_host(q_p.data_ptr(), k_p.data_ptr(), v_p.data_ptr(), cos.data_ptr(),
                                         sin.data_ptr(), out_p.data_ptr(), lse_p.data_ptr(), w.B, w.H, w.n_txt,
                                         w.n_img, w.D, dit.DIT_BF16, workspace.data_ptr(), ws_bytes,
                                         E2E_CHUNK_HEADS, s_ptr) == 0

    for _ in range(min(args.warmup, 3)):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 20))
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = whole_job_throughput(w.flops, e2e_steps, world, e2e_ms)

    peak, peak_src = measured_peaks()
    achieved = w.flops / (kern_ms * 1e-3) / 1e12
    traffic = profile_traffic("attn_fwd_bf16_kernel") if w.name == WORKLOAD else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = oracle_sample(w, args.oracle_rows_per_head)
        val, dt, threads = time_oracle(w, q_h, k_h, v_h, rows)
        cpu = {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": "fp64 numpy oracle on the first %d query rows of each of the %d heads (%d rows of %d, "
                         "%.1f s)" % (args.oracle_rows_per_head, w.H * w.B, len(rows), w.B * w.H * w.N, dt),
               "extrapolated_full_s": dt / len(rows) * w.B * w.H * w.N,
               "extrapolated_note": "extrapolated: per-row time of the sample x all B*H*N rows"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(w, world),
                           step="rope table + K/V operand pass + attention forward (bf16 O, fp32 LSE)",
                           l2="inputs larger than L2 (q, k, v %.0f MB > 126 MB), no flush; flushed kernel time in "
                              "roofline.kernel_ms_l2_flushed" % (6 * w.B * w.H * w.N * w.D / 1e6),
                           pct_of_bf16_peak=100.0 * value / peak,
                           pct_of_nominal_bf16_peak=100.0 * value / NOMINAL_PEAK_BF16),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "attn_fwd_bf16_kernel", "peak_source": peak_src,
                         "kernel_ms": kern_ms, "kernel_ms_l2_flushed": kern_ms_flushed,
                         "achieved_l2_flushed": w.flops / (kern_ms_flushed * 1e-3) / 1e12,
                         "kernel_ms_median_50": median50,
                         "achieved_median_50": w.flops / (median50 * 1e-3) / 1e12,
                         "frac_nominal": achieved / NOMINAL_PEAK_BF16,
                         "peak_nominal": NOMINAL_PEAK_BF16,
                         "frac_note": "frac: of the measured cuBLAS bf16 burst peak; frac_nominal: of the "
                                      "2.25 PFLOP/s datasheet dense BF16 peak"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / e2e_steps,
                    "api": "dit_attn_forward_host, %d heads per chunk, pinned host buffers" % E2E_CHUNK_HEADS},
            "gpu_launches": 3 * args.steps,
            "fp8": fp8,
            "split": split,
            "fused_k": fused_k,
            "qkv_projection": proj,
            "merge": merge,
            "sparse": sparse,
            "context_library_sdpa": sdpa,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    """The fp64 oracle on the host cores: step i evaluates the first
    --reference-rows query rows of head i mod H of the same workload."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = W.WORKLOADS[WORKLOAD]
    q, k, v = W.make_qkv(w, seed=0)
    R = args.reference_rows

    def rows_of(i):
        h = i % w.H
        return np.asarray([(0, h, n) for n in range(R)], dtype=np.int64)

    for i in range(args.warmup):
        time_oracle(w, q, k, v, rows_of(i))
    total = 0.0
    threads = 1
    for i in range(args.steps):
        _, dt, threads = time_oracle(w, q, k, v, rows_of(i))
        total += dt
    flops = 4.0 * w.N * w.D * R
    value = flops * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(w, world),
                       step="fp64 oracle: rotary embedding and exact attention of %d sampled query rows" % R),
        "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": threads,
                         "sample": "fp64 numpy oracle: per step the first %d query rows of one head (heads in turn)"
                                   % R,
                         "extrapolated_full_s": total / args.steps * (w.B * w.H * w.N) / R,
                         "extrapolated_note": "extrapolated: step time x B*H*N / rows per step; an upper bound, "
                                              "since each step also pays the head's table and key rotation once"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=W.ORDER, default=WORKLOAD,
                    help="the bench line is the default workload; others serve profiling")
    ap.add_argument("--oracle-rows-per-head", type=int, default=2048)
    ap.add_argument("--reference-rows", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_native(args)


if __name__ == "__main__":
    main()
