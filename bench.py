#!/usr/bin/env python
"""Benchmark of the B200 SageSLA attention forward (one JSON line on rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]

A step is one whole forward (block statistics, quantization, block scores, Top-K, complement
sums, sparse attention with the linear branch) over the Wan2.1-14B-720P self-attention shape:
B=1, H=40, N=75600 tokens (21x45x80 latent grid), d=128, block 64, Top-K ratio 0.1, with seeded
synthetic bf16 inputs (seed 3) already resident in HBM. The inputs (3 x 774 MB) are larger than
the 126 MB L2, so no flush is needed between steps. Under torchrun every rank runs its own
forward on its own GPU (independent problems, weak scaling, no data-path collective); the
timed region is bracketed by a barrier and a device synchronize and the max over ranks is
reported.

--impl reference times the CPU oracle (test infrastructure, float64) on the host cores, on a
bounded sample of the same workload per step, extrapolated to the whole forward.

--configs (one GPU) prints one JSON line per workload of the benchmark's configuration list
instead: the tiny case (ratio 0.1 and 1.0, with the CPU oracle's full forward timed beside it,
median of 3), Wan2.1-1.3B-480P, 14B-480P and 14B-720P at ratio 0.1, and the locality workload
at ratios 0.05, 0.1 and 0.15, each with tokens/s, executed TOPS and the attention kernel's
fraction of the INT8/FP8 peak (L2 flushed between calls).

--sweep (one GPU) prints one JSON line per point instead: the forward on the 14B-720P random
workload and on the smoothed-field locality workload over Top-K ratios 0.05-0.2 and the dense
mode (ratio 1: every block kept, selection and linear branch skipped), a dense BF16
attention of the same shape through torch's scaled_dot_product_attention for comparison, the
SLA backward (ratio 0.1, bf16 gradients) against torch's dense attention backward, and the
fused-norm and W8A8 kernels on the same token rows.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SageSLA fwd tokens/s and effective TOPS at 14B-720P shape; % of roofline"
UNIT = "tokens/s"
WORKLOAD = "wan21_14b_720p"
RATIO = 0.1
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="another named workload (smaller cases for ncu captures)")
    ap.add_argument("--topk-ratio", type=float, default=None,
                    help="Top-K ratio (default: 0.1; 1.0 is the dense SageAttention mode)")
    ap.add_argument("--configs", action="store_true",
                    help="one JSON line per benchmark workload (tiny, 1.3B-480P, 14B-480P, "
                         "14B-720P, locality at three ratios)")
    ap.add_argument("--sweep", action="store_true",
                    help="Top-K ratio sweep and dense BF16 comparison, one JSON line per point")
    ap.add_argument("--kernel-case", choices=["norm", "w8a8", "bwd", "dense"], default=None,
                    help="run a small case of one next-row kernel a few times (for ncu captures)")
    args = ap.parse_args()
    globals()["WORKLOAD"] = args.workload
    if args.topk_ratio is not None:
        globals()["RATIO"] = args.topk_ratio
    return args


def rank_env():
    """(rank, local rank, world size) from the torchrun environment (1 process if absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(value: float, dist, device) -> float:
    """The maximum of a per-rank time over all ranks (every rank gets it). The tensor lives on
    `device`: the GPU for NCCL, the CPU for gloo."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def kernel_launches(dense: bool) -> int:
    """Kernels of one forward: stats, finalize, quant, scores, top-k, complement GEMM and
    attention; with every block kept only stats, finalize, quant and attention run."""
    return 4 if dense else 7


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The attention output is written in the model's activation dtype (bf16 for the Wan2.1 DiT
# workloads); the f32 output path is covered by the parity tests.
OUT_TORCH = "bfloat16"


def out_dtype_torch(torch):
    return getattr(torch, OUT_TORCH)


def workload_config():
    from sparse_bit_attention_b200 import inputs
    w = inputs.WORKLOADS[WORKLOAD]
    grid = "x".join(str(g) for g in w.grid) if w.grid else "none"
    return w, {"workload": f"{WORKLOAD}: {w.description}, B{w.B} H{w.H} N{w.N} "
                           f"(latent grid {grid}) d128, block 64, topk_ratio {RATIO}, "
                           f"bf16 inputs, seed {w.seed}",
               "B": w.B, "H": w.H, "N": w.N, "head_dim": 128, "block": 64, "topk_ratio": RATIO,
               "out_dtype": OUT_TORCH,
               "l2": f"inputs {3 * w.B * w.H * w.N * 256 / 1e9:.2f} GB > 126 MB L2, no flush"}


def attention_tensor_ops(B, H, nb, k):
    """Useful tensor-core operations of the sparse attention: per kept (query block, key
    block) pair one 64x64x128 Q.K^T and one 64x128x64 P.V, 2 ops per multiply-add."""
    return B * H * nb * k * 2 * (2 * 64 * 64 * 128)


def source_digest():
    h = hashlib.sha256()
    for f in ("attention.cu", "common.cuh"):
        with open(os.path.join(ROOT, "sparse_bit_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def attention_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on the
    current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if (d.get("source_digest") != source_digest() or d.get("workload") != WORKLOAD or
            d.get("out_dtype") != OUT_TORCH):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r.split(", ") for r in self.out.read().strip().splitlines() if r.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_oracle_sample(q, k, v, head: int, n_blocks: int, seed: int):
    """Times the oracle on one head: its whole per-head preparation (statistics, scores, Top-K,
    quantization, key-block states) plus ``n_blocks`` query blocks of both branches.
    Returns (seconds for the sample, extrapolated seconds for the whole head)."""
    import numpy as np
    import oracle as orc
    from sparse_bit_attention_b200 import inputs
    qh, kh, vh = (inputs.as_float64(x[0, head]) for x in (q, k, v))
    t0 = time.perf_counter()
    prep = orc.prepare_head(qh, kh, vh, RATIO)
    hs = orc.key_block_states(kh, vh)
    t1 = time.perf_counter()
    rng = np.random.default_rng(seed)
    rows = rng.choice(prep.nb, size=min(n_blocks, prep.nb), replace=False)
    for i in rows:
        orc.sparse_block_row(prep, int(i), qh, kh, vh)
        orc.linear_block_row(prep, int(i), qh, hs)
    t2 = time.perf_counter()
    return t2 - t0, (t1 - t0) + (t2 - t1) * prep.nb / len(rows)


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def attention_peak(peaks: dict) -> tuple[float, str]:
    """INT8 / FP8 dense tensor peak for the attention kernel: twice the measured bf16 rate
    (the nominal INT8:bf16 ratio on B200), burst figure: one attention launch lasts ~13 ms
    inside a sub-second timed loop, which runs at full clock."""
    return 2.0 * peaks["bf16_tflops"], "2 x bf16_tflops (burst)"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(p.get("num_threads", 1) for p in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    rank, _, _ = rank_env()
    if rank != 0:          # under torchrun, rank 0 alone times the oracle
        return 0
    from sparse_bit_attention_b200 import inputs
    w, cfg = workload_config()
    q, k, v = inputs.make_qkv(WORKLOAD)
    blocks = 8
    times = []
    for s in range(args.warmup + args.steps):
        _, t_head = cpu_oracle_sample(q, k, v, head=s % w.H, n_blocks=blocks, seed=s)
        if s >= args.warmup:
            times.append(t_head)
    t_forward = statistics.mean(times) * w.H        # all heads of one forward
    value = w.B * w.N / t_forward
    cores = blas_threads()
    sample = (f"per step: one head's full preparation over N={w.N} plus {blocks} random query "
              f"blocks of both branches, extrapolated to {w.H} heads x all query blocks; "
              f"CPU: {cpu_model()}")
    cfg["parallelism"] = "1 GPU"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_forward * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, sba, torch, dist, q_cpu, k_cpu, v_cpu, ws, dev, stream, barrier, world):
    """Same forward through the host-buffer C-ABI entry point: the timed region holds the
    host->device copy of Q, K, V from pinned memory, the forward and the device->host copy of
    the output, every step."""
    B, H, N, D = q_cpu.shape
    out_t = out_dtype_torch(torch)
    out_dtype = sba.SAGESLA_F32 if out_t == torch.float32 else sba.SAGESLA_BF16
    need = sba.sagesla_host_workspace_size(B, H, N, D, RATIO, 64, out_dtype)
    del ws
    torch.cuda.empty_cache()
    ws_host = sba.alloc_workspace(need, dev)
    qh, kh, vh = (x.contiguous().pin_memory() for x in (q_cpu, k_cpu, v_cpu))
    oh = torch.empty((B, H, N, D), dtype=out_t).pin_memory()
    sba.sagesla_forward_host(qh, kh, vh, oh, RATIO, workspace=ws_host)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        sba.sagesla_forward_host(qh, kh, vh, oh, RATIO, workspace=ws_host)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dist, dev)
    h2d = 3 * B * H * N * D * 2
    d2h = B * H * N * D * oh.element_size()

    return {"value": B * N * world / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}


def run_cuda(args):
    import torch
    import torch.distributed as dist
    import sparse_bit_attention_b200 as sba
    from sparse_bit_attention_b200 import binding, inputs
    from sparse_bit_attention_b200.build import build

    rank, local, world = rank_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    build()
    sba.load_library()

    w, cfg = workload_config()
    cfg["parallelism"] = f"independent problem per GPU x{world}" if world > 1 else "1 GPU"
    q_cpu, k_cpu, v_cpu = inputs.make_qkv(WORKLOAD)
    q, k, v = (x.to(dev) for x in (q_cpu, k_cpu, v_cpu))
    B, H, N, D = q.shape
    lay = sba.sagesla_get_workspace_layout(B, H, N, D, RATIO)
    ws = sba.alloc_workspace(lay["total_bytes"], dev)
    out = torch.empty((B, H, N, D), dtype=out_dtype_torch(torch), device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        sba.sagesla_forward(q, k, v, RATIO, out=out, workspace=ws)
    st = sba.sagesla_stream_status(stream, ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {sba.sagesla_status_string(st)}")

    n_ev = binding.N_STAGES + 1
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
                for _ in range(args.steps)]
    t_begin, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    t_begin.record(stream)
    for s in range(args.steps):
        sba.sagesla_forward(q, k, v, RATIO, out=out, workspace=ws, stage_events=stage_ev[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    st = sba.sagesla_stream_status(stream, ws)
    if st != 0:
        raise RuntimeError(f"device status after timing: {sba.sagesla_status_string(st)}")
    ms_total = t_begin.elapsed_time(t_end)
    stage_ms = {name: statistics.mean(ev[i].elapsed_time(ev[i + 1]) for ev in stage_ev)
                for i, name in enumerate(binding.STAGE_NAMES)}
    ms_total = max_over_ranks(ms_total, dist, dev)
    ms_step = ms_total / args.steps
    value = B * N * world / (ms_step / 1e3)

    # ---------------- end to end through the host-buffer entry point
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, sba, torch, dist, q_cpu, k_cpu, v_cpu, ws, dev, stream, barrier, world)
        ws = None

    if rank == 0:
        peaks, peak_src = measured_peaks()
        peak_tops, peak_how = attention_peak(peaks)
        ops = attention_tensor_ops(B, H, lay["nb"], lay["k"])
        att_s = stage_ms["attention"] / 1e3
        achieved = ops / att_s / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_tops,
                    "unit": "TFLOP/s", "frac": achieved / peak_tops,
                    "traffic": attention_traffic(),
                    "kernel": "k_attention (INT8 QK^T + FP8 PV, tcgen05)",
                    "peak_source": f"{peak_src}: {peak_how}",
                    "algorithmic_ops_per_launch": ops}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            secs = []
            t_sample = 0.0
            for h in (0, 1):
                ts, th = cpu_oracle_sample(q_cpu, k_cpu, v_cpu, head=h, n_blocks=24, seed=h)
                t_sample += ts
                secs.append(th)
            cpu_value = B * N / (statistics.mean(secs) * H)
            cpu = {"value": cpu_value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                   "cpu_model": cpu_model(),
                   "sample": f"heads 0 and 1: full per-head preparation + 24 random query "
                             f"blocks each ({t_sample:.1f} s of CPU work), extrapolated to "
                             f"{H} heads x {lay['nb']} query blocks"}
        fwd_s = ms_step / 1e3
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "int8+fp8 tensor, f32 softmax", "data": "synthetic", "config": cfg,
                "executed_tops": ops / fwd_s / 1e12,
                "dense_equiv_tops": 4.0 * B * H * N * N * D / fwd_s / 1e12,
                "stage_ms": stage_ms, "roofline": roofline, "cpu_baseline": cpu,
                "e2e": e2e,
                "gpu_launches": kernel_launches(lay["k"] == lay["nb"]) * args.steps,
                "clocks": clock_info}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _time_forward(sba, binding, torch, q, k, v, ratio, steps, warmup, flush=None):
    """Median forward and stage times over `steps` calls (CUDA events on the stream); with
    `flush` (a device buffer larger than L2) the buffer is rewritten before every call."""
    B, H, N, D = q.shape
    lay = sba.sagesla_get_workspace_layout(B, H, N, D, ratio)
    ws = sba.alloc_workspace(lay["total_bytes"], q.device)
    out = torch.empty((B, H, N, D), dtype=out_dtype_torch(torch), device=q.device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        sba.sagesla_forward(q, k, v, ratio, out=out, workspace=ws)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(binding.N_STAGES + 1)]
          for _ in range(steps)]
    for s in range(steps):
        if flush is not None:
            flush.add_(1)
        sba.sagesla_forward(q, k, v, ratio, out=out, workspace=ws, stage_events=ev[s])
    torch.cuda.synchronize()
    st = sba.sagesla_stream_status(stream, ws)
    if st != 0:
        raise RuntimeError(f"device status: {sba.sagesla_status_string(st)}")
    stage = {name: statistics.median(e[i].elapsed_time(e[i + 1]) for e in ev)
             for i, name in enumerate(binding.STAGE_NAMES)}
    total = statistics.median(e[0].elapsed_time(e[-1]) for e in ev)
    del ws, out
    torch.cuda.empty_cache()
    return lay, total, stage


def _time_sdpa(torch, q, k, v, steps, warmup):
    """Dense BF16 attention of the same shape through torch (a library kernel, for context)."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    for backend in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION,
                    SDPBackend.EFFICIENT_ATTENTION):
        try:
            with sdpa_kernel([backend]):
                for _ in range(warmup):
                    F.scaled_dot_product_attention(q, k, v)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(steps):
                    F.scaled_dot_product_attention(q, k, v)
                e1.record()
                torch.cuda.synchronize()
            return backend.name, e0.elapsed_time(e1) / steps
        except RuntimeError:
            continue
    return None, None


def _time_norm(sba, torch, steps, warmup):
    """Fused LayerNorm + AdaLN modulation + per-token INT8 codes on the 14B-720P token rows
    (75600 x 5120 bf16): device time per call and HBM bytes per call."""
    M, K = 75600, 5120
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(M, K, generator=g) * 1.5).to(torch.bfloat16).cuda()
    scale = (torch.randn(1, K, generator=g) * 0.2).to(torch.bfloat16).cuda()
    shift = (torch.randn(1, K, generator=g) * 0.5).to(torch.bfloat16).cuda()
    for _ in range(warmup):
        sba.sagesla_norm_quant(x, sba.SAGESLA_LAYER_NORM, 1e-6, None, None, scale, shift,
                               rows_per_sample=M, want_codes=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        sba.sagesla_norm_quant(x, sba.SAGESLA_LAYER_NORM, 1e-6, None, None, scale, shift,
                               rows_per_sample=M, want_codes=True)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    nbytes = M * K * 2 + M * K * 2 + M * K + M * 4      # x in, bf16 y out, codes out, scales
    return M, K, ms, nbytes


def _time_w8a8(sba, torch, steps, warmup, M=75600, K=5120, N=5120):
    """W8A8 projection of the 14B-720P token rows (M x K int8 codes, N x K block-quantized
    weights, bf16 output with bias) and the same layer in bf16 through torch.matmul."""
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(M, K, generator=g) * 1.5).to(torch.bfloat16).cuda()
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16).cuda()
    _, x8, s_x = sba.sagesla_norm_quant(x, sba.SAGESLA_NO_NORM, 0.0, want_y=False, want_codes=True)
    w8, s_w = sba.sagesla_w8a8_quantize_weight(w)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")

    def timed(fn):
        for _ in range(warmup):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms_w8 = timed(lambda: sba.sagesla_w8a8_gemm(x8, s_x, w8, s_w, bias, out=y))
    ms_bf16 = timed(lambda: torch.addmm(bias, x, w.t()))
    return M, K, N, ms_w8, ms_bf16


def backward_tensor_flops(B, H, nb, k):
    """Tensor-core FLOPs of the SLA backward's sparse branch: per kept (query block, key block)
    pair nine 64x64x128 products (S and dP = dO V^T for the log-sum-exp and D; S, dP and dQ; S^T, dP^T,
    dV and dK), 2 FLOPs per multiply-add; plus the two complement GEMMs (G and dH), each
    2 nb_pad^2 16512 per head."""
    nb_pad = -(-nb // 128) * 128
    return B * H * nb * k * 9 * 2 * (64 * 64 * 128) + B * H * 2 * 2 * nb_pad * nb_pad * 16512


def _time_backward(sba, torch, q, k, v, ratio, steps, warmup):
    """SLA backward (bf16 gradients) on resident inputs and a seeded dO, and torch's dense
    bf16 attention backward of the same shape for context."""
    g = torch.Generator().manual_seed(21)
    d_out = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(q.device)
    B, H, N, D = q.shape
    ws = sba.alloc_workspace(sba.sagesla_sla_backward_workspace_size(B, H, N, D, ratio), q.device)
    grads = [torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) for _ in range(3)]
    run = lambda: sba.sagesla_sla_backward(q, k, v, d_out, ratio, dq=grads[0], dk=grads[1],
                                           dv=grads[2], workspace=ws)
    for _ in range(warmup):
        run()
    st = sba.sagesla_stream_status(None, ws)
    if st != 0:
        raise RuntimeError(f"device status: {sba.sagesla_status_string(st)}")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del ws, grads
    torch.cuda.empty_cache()
    # dense baseline: forward + backward of torch SDPA minus its forward
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    ms_dense, backend = None, None
    for be in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION):
        try:
            with sdpa_kernel([be]):
                qq, kk, vv = (x.detach().requires_grad_(True) for x in (q, k, v))
                out = F.scaled_dot_product_attention(qq, kk, vv)
                out.backward(d_out)
                torch.cuda.synchronize()
                e0.record()
                for _ in range(max(1, steps // 2)):
                    out = F.scaled_dot_product_attention(qq, kk, vv)
                    out.backward(d_out)
                e1.record()
                torch.cuda.synchronize()
                fwd_bwd = e0.elapsed_time(e1) / max(1, steps // 2)
                e0.record()
                for _ in range(max(1, steps // 2)):
                    F.scaled_dot_product_attention(qq, kk, vv)
                e1.record()
                torch.cuda.synchronize()
                ms_dense = fwd_bwd - e0.elapsed_time(e1) / max(1, steps // 2)
                backend = be.name
                del qq, kk, vv, out
            break
        except RuntimeError:
            continue
    torch.cuda.empty_cache()
    return ms, ms_dense, backend


def run_sweep(args):
    import torch
    import sparse_bit_attention_b200 as sba
    from sparse_bit_attention_b200 import binding, inputs
    from sparse_bit_attention_b200.build import build
    build()
    sba.load_library()
    dev = torch.device("cuda", 0)
    steps = max(3, min(args.steps, 10))
    for name, ratios in (("wan21_14b_720p", (0.05, 0.1, 0.15, 0.2, 1.0)),
                         ("locality_14b_720p", (0.05, 0.1, 0.15, 0.2))):
        q, k, v = (x.to(dev) for x in inputs.make_qkv(name))
        B, H, N, D = q.shape
        dense_ops = 4.0 * B * H * N * N * D
        for ratio in ratios:
            lay, ms, stage = _time_forward(sba, binding, torch, q, k, v, ratio, steps, args.warmup)
            ops = attention_tensor_ops(B, H, lay["nb"], lay["k"])
            print(json.dumps({
                "sweep": name, "topk_ratio": ratio, "k": lay["k"], "nb": lay["nb"],
                "ms_per_forward": ms, "tokens_per_s": B * N / (ms / 1e3),
                "attention_ms": stage["attention"],
                "attention_tops": ops / (stage["attention"] / 1e3) / 1e12,
                "dense_equiv_tops": dense_ops / (ms / 1e3) / 1e12,
                "stage_ms": stage}), flush=True)
        if name == "wan21_14b_720p":
            lay = sba.sagesla_get_workspace_layout(B, H, N, D, 0.1)
            ms_b, ms_dense, be = _time_backward(sba, torch, q, k, v, 0.1, max(3, steps // 2),
                                                args.warmup)
            peaks, src = measured_peaks()
            fl = backward_tensor_flops(B, H, lay["nb"], lay["k"])
            print(json.dumps({
                "sweep": "sla_backward", "workload": name, "topk_ratio": 0.1,
                "grad_dtype": "bfloat16", "ms_per_backward": ms_b,
                "tokens_per_s": B * N / (ms_b / 1e3), "tensor_tflop": fl / 1e12,
                "tensor_tflops": fl / (ms_b / 1e3) / 1e12,
                "frac_of_bf16_burst": fl / (ms_b / 1e3) / 1e12 / peaks["bf16_tflops"],
                "peak_source": src, "dense_baseline": f"torch SDPA backward ({be}), bf16",
                "dense_backward_ms": ms_dense}), flush=True)
            backend, ms = _time_sdpa(torch, q, k, v, max(2, steps // 2), 1)
            print(json.dumps({
                "sweep": name, "baseline": "torch scaled_dot_product_attention, bf16 dense",
                "backend": backend, "ms_per_forward": ms,
                "tokens_per_s": B * N / (ms / 1e3) if ms else None,
                "dense_tflops": dense_ops / (ms / 1e3) / 1e12 if ms else None}), flush=True)
        del q, k, v
        torch.cuda.empty_cache()
    M, K, ms, nbytes = _time_norm(sba, torch, steps, args.warmup)
    peaks, src = measured_peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    print(json.dumps({
        "sweep": "fused_norm", "op": "LayerNorm + AdaLN modulation + bf16 out + per-token INT8",
        "M": M, "K": K, "ms_per_call": ms, "hbm_bytes": nbytes, "achieved_gbs": gbs,
        "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"], "peak_source": src}),
        flush=True)
    M, K, N, ms_w8, ms_bf16 = _time_w8a8(sba, torch, steps, args.warmup)
    ops = 2.0 * M * N * K
    peak_int8 = 2.0 * peaks["bf16_tflops"]
    print(json.dumps({
        "sweep": "w8a8_linear", "M": M, "K": K, "N": N, "ms_per_call": ms_w8,
        "tops": ops / (ms_w8 / 1e3) / 1e12, "peak_tops": peak_int8,
        "frac": ops / (ms_w8 / 1e3) / 1e12 / peak_int8,
        "peak_source": f"{src}: 2 x bf16_tflops (burst)",
        "bf16_torch_ms": ms_bf16, "bf16_torch_tflops": ops / (ms_bf16 / 1e3) / 1e12,
        "speedup_vs_bf16": ms_bf16 / ms_w8}), flush=True)
    return 0


def run_configs(args):
    """One line per workload of the benchmark's configuration list (one GPU)."""
    import numpy as np
    import torch
    import sparse_bit_attention_b200 as sba
    from sparse_bit_attention_b200 import binding, inputs
    from sparse_bit_attention_b200.build import build
    build()
    sba.load_library()
    dev = torch.device("cuda", 0)
    peaks, src = measured_peaks()
    peak_tops, peak_how = attention_peak(peaks)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)     # 2 x the 126 MB L2
    steps = max(5, args.steps)
    cases = [("tiny", 0.1), ("tiny", 1.0), ("wan21_1p3b_480p", 0.1), ("wan21_14b_480p", 0.1),
             ("wan21_14b_720p", 0.1), ("locality_14b_720p", 0.05), ("locality_14b_720p", 0.1),
             ("locality_14b_720p", 0.15)]
    loaded = {}
    for name, ratio in cases:
        if name not in loaded:
            loaded.clear()
            torch.cuda.empty_cache()
            loaded[name] = inputs.make_qkv(name)
        q_cpu, k_cpu, v_cpu = loaded[name]
        q, k, v = (x.to(dev) for x in (q_cpu, k_cpu, v_cpu))
        B, H, N, D = q.shape
        lay, ms, stage = _time_forward(sba, binding, torch, q, k, v, ratio, steps, args.warmup,
                                       flush=flush)
        ops = attention_tensor_ops(B, H, lay["nb"], lay["k"])
        att_tops = ops / (stage["attention"] / 1e3) / 1e12
        line = {"config": name, "shape": f"B{B} H{H} N{N} d{D}", "topk_ratio": ratio,
                "k": lay["k"], "nb": lay["nb"], "ms_per_forward": ms,
                "tokens_per_s": B * N / (ms / 1e3), "attention_ms": stage["attention"],
                "executed_tops": att_tops, "frac": att_tops / peak_tops,
                "peak_tops": peak_tops, "peak_source": f"{src}: {peak_how}",
                "dense_equiv_tops": 4.0 * B * H * N * N * D / (ms / 1e3) / 1e12,
                "l2": "flushed before every call", "stage_ms": stage}
        if name == "tiny":
            import oracle as orc
            qa, ka, va = (inputs.as_float64(x) for x in (q_cpu, k_cpu, v_cpu))
            secs = []
            for _ in range(3):
                t0 = time.perf_counter()
                orc.forward(qa, ka, va, ratio)
                secs.append(time.perf_counter() - t0)
            t_cpu = statistics.median(secs)
            line["cpu_baseline"] = {"value": B * N / t_cpu, "unit": UNIT, "cores": blas_threads(),
                                    "kind": "oracle", "cpu_model": cpu_model(),
                                    "sample": "the whole forward (all heads, all query blocks), "
                                              "median of 3 runs, no extrapolation",
                                    "seconds": t_cpu}
        print(json.dumps(line), flush=True)
        del q, k, v
    return 0


def run_kernel_case(args):
    """A few calls of one next-row kernel on a case sized for ncu captures (well above the
    126 MB L2, a few hundred MB on the device)."""
    import torch
    import sparse_bit_attention_b200 as sba
    from sparse_bit_attention_b200.build import build
    build()
    sba.load_library()
    g = torch.Generator().manual_seed(5)
    if args.kernel_case == "norm":
        M, K = 24000, 5120
        x = (torch.randn(M, K, generator=g) * 1.5).to(torch.bfloat16).cuda()
        scale = (torch.randn(1, K, generator=g) * 0.2).to(torch.bfloat16).cuda()
        shift = (torch.randn(1, K, generator=g) * 0.5).to(torch.bfloat16).cuda()
        for _ in range(3):
            sba.sagesla_norm_quant(x, sba.SAGESLA_LAYER_NORM, 1e-6, None, None, scale, shift,
                                   rows_per_sample=M, want_codes=True)
    elif args.kernel_case == "dense":
        # dense mode (Top-K ratio 1: the M=128 dense kernel) on the Wan2.1-1.3B-480P shape
        from sparse_bit_attention_b200 import inputs
        q, k, v = (x.cuda() for x in inputs.make_qkv("wan21_1p3b_480p"))
        B, H, N, D = q.shape
        ws = sba.alloc_workspace(sba.sagesla_workspace_size(B, H, N, D, 1.0))
        out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
        for _ in range(2):
            sba.sagesla_forward(q, k, v, 1.0, out=out, workspace=ws)
        if sba.sagesla_stream_status(None, ws) != 0:
            raise RuntimeError("device status after the dense-mode forward")
    elif args.kernel_case == "bwd":
        # SLA backward on the Wan2.1-1.3B-480P attention shape (B1 H12 N32760, ratio 0.1)
        from sparse_bit_attention_b200 import inputs
        q, k, v = (x.cuda() for x in inputs.make_qkv("wan21_1p3b_480p"))
        d_out = torch.randn(q.shape, generator=g).to(torch.bfloat16).cuda()
        B, H, N, D = q.shape
        ws = sba.alloc_workspace(sba.sagesla_sla_backward_workspace_size(B, H, N, D, 0.1))
        for _ in range(2):
            sba.sagesla_sla_backward(q, k, v, d_out, 0.1, grad_dtype=torch.bfloat16, workspace=ws)
        if sba.sagesla_stream_status(None, ws) != 0:
            raise RuntimeError("device status after the backward")
    else:
        M, K, N = 16384, 5120, 5120
        x = (torch.randn(M, K, generator=g) * 1.5).to(torch.bfloat16).cuda()
        w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
        _, x8, s_x = sba.sagesla_norm_quant(x, sba.SAGESLA_NO_NORM, 0.0, want_y=False,
                                            want_codes=True)
        w8, s_w = sba.sagesla_w8a8_quantize_weight(w)
        for _ in range(3):
            sba.sagesla_w8a8_gemm(x8, s_x, w8, s_w)
    torch.cuda.synchronize()
    print(json.dumps({"kernel_case": args.kernel_case, "ok": True}))
    return 0


def main():
    args = parse_args()
    if args.kernel_case:
        return run_kernel_case(args)
    if args.sweep:
        return run_sweep(args)
    if args.configs:
        return run_configs(args)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
