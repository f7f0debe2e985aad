"""Throughput benchmark of the FP8 (E4M3) P-cast attention forward pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--path fp8|wide|bf16qk|decode|bwd] [--shard replicas|heads]

One step is one forward pass of the 32K causal prefill (B=1, H=32, N=32768,
d=128, Delta=7 sink with k=4, S=256, reverse KV order) through the C ABI.
Rank 0 prints one JSON line: the throughput, the roofline of the dominant
kernel, the oracle's CPU time, the end-to-end figure with host buffers, the
SM clocks sampled during the timed region and the count of kernel launches.
Under torchrun each rank runs its own copy of the workload on its own GPU (no
collective on the data path: weak scaling); the step time is the maximum over
ranks.  --shard heads splits one problem's kv heads across the ranks instead
and all-gathers O and lse (strong scaling).

--impl reference times the CPU oracle (the blockwise E4M3 emulator) on the
host cores instead, on a bounded sample of the same workload per step.

--path wide starts from bfloat16 Q, K, V instead: one step quantises them
(random-sign Hadamard rotation, Q and K per 128-row block, V per head) and
runs the scaled forward pass, which rotates the output back.

--path bf16qk keeps Q and K in bfloat16 (S = Q K^T on the 16-bit tensor-core
path) with E4M3 V: the P-cast summary's kernel-faithful setting.

--path decode times the split-KV decode pass (B=32, H=32, Hkv=8, N=32768,
one query row per head, 32-tile splits) against the HBM roofline.

--path bwd times the backward pass of the 32K prefill (dQ, dK, dV from the
forward's inputs, O, lse and a bfloat16 dO).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import re
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

import numpy as np  # noqa: E402

import synthetic  # noqa: E402

WORKLOAD = synthetic.WORKLOADS["prefill32k"]
P_SCALE = 256.0
KV_ORDER = 1  # reverse
SEED = 3000
METRIC = "FP8 attn fwd TFLOP/s (% of FP8 peak) at N=32K,d=128; output MSE vs FP64"
UNIT = "TFLOP/s"
WORKLOAD_DESC = ("prefill32k: B=1 H=32 N=32768 d=128 causal, E4M3 Q/K/V, Delta=7 sink (k=4), S=256, "
                 "reverse KV order")
KERNEL_NAME = "fwd_v2_kernel"
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "fwd_v2_prefill32k_traffic.txt")
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0  # nominal dense ratio: 4.5 PF FP8 / 2.25 PF BF16
CPU_SAMPLE_ROWS = 2048  # query rows per head the oracle arm evaluates per step


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="fp8", choices=["fp8", "wide", "bf16qk", "decode", "bwd"],
                    help="fp8: E4M3 inputs (the headline); wide: bfloat16 inputs quantised in the step; "
                         "bf16qk: bfloat16 Q and K, E4M3 V; decode: one query row per head, split-KV; "
                         "bwd: the backward pass of the 32K prefill")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="replicas: each rank runs its own copy (weak scaling, the default); heads: the ranks "
                         "split one problem's kv heads and all-gather the output (strong scaling)")
    ap.add_argument("--skip-cpu-baseline", action="store_true",
                    help="omit the oracle timing (used under ncu)")
    ap.add_argument("--head-dim", type=int, default=None, choices=[64, 128],
                    help="run the fp8 path's prefill with this head dimension (64: the 64-key-block kernel; a "
                         "profiling case, not the headline)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="run the fp8 path's prefill at this sequence length instead of 32768 (a smaller case "
                         "for profiling; not the headline workload)")
    return ap.parse_args()


_CODE_TOKENS = re.compile(r'"(?:\\.|[^"\\])*"|\'(?:\\.|[^\'\\])*\'|//[^\n]*|/\*.*?\*/', re.S)


def _strip_comments(src: str) -> str:
    """C/C++ source without comments and with whitespace collapsed (string literals kept)."""
    code = _CODE_TOKENS.sub(lambda m: " " if m.group(0)[0] == "/" else m.group(0), src)
    return " ".join(code.split())


# The device code of the persistent forward kernel (its parameters, PTX
# wrappers and the kernel itself); the other paths' kernels live elsewhere.
KERNEL_SOURCES = ("fwd_v1.cuh", "fwd_v2.cuh", "sm100_ptx.cuh")


def kernel_source_hash() -> str:
    """Hash of the forward kernel's code and its launch configuration.

    Covers the device sources of that kernel and the host function that
    sizes its launch; insensitive to comments and layout.
    """
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "softmax_cast_precision_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as fh:
            h.update(name.encode() + _strip_comments(fh.read()).encode())
    with open(os.path.join(csrc, "api.cu"), encoding="utf-8") as fh:
        api = fh.read()
    for fn in ("launch_v2_on", "launch_v2"):
        m = re.search(r"\nint " + fn + r"\(.*?\n}\n", api, re.S)
        h.update(_strip_comments(m.group(0) if m else api).encode())
    return h.hexdigest()[:16]


def peak_clock_mhz():
    """Median SM clock under load while the measured peaks were taken (None if unknown)."""
    try:
        with open(PEAKS_FILE) as fh:
            return float(json.load(fh)["clocks_under_load"]["sm_mhz_median"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


def fp8_peak():
    """FP8 dense peak: the measured BF16 cuBLAS figure x the nominal FP8/BF16 ratio."""
    try:
        with open(PEAKS_FILE) as fh:
            pk = json.load(fh)
        return pk["bf16_tflops"] * FP8_OVER_BF16, pk["bf16_tflops_sustained"] * FP8_OVER_BF16, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS * FP8_OVER_BF16, 1400.0 * FP8_OVER_BF16, "fallback"


def traffic_per_launch():
    """DRAM bytes per launch from the committed ncu summary, if it is for this kernel source."""
    try:
        with open(PROFILE_SUMMARY) as fh:
            s = json.load(fh)
    except (OSError, ValueError):
        return None
    if s.get("kernel_source_hash") != kernel_source_hash():
        return None
    return s.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            sm.append(clk)
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        loaded = [c for c in sm if c > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def sample_rows(N: int, count: int) -> np.ndarray:
    return synthetic.sampled_rows(N, count)


def visible_pairs(rows: np.ndarray, N: int, causal: bool) -> int:
    return int(np.sum(rows + 1)) if causal else int(len(rows) * N)


def cpu_oracle_run(q, k, v, rows):
    """One bounded step of the oracle arm: the emulator on `rows` of every head."""
    import oracle

    w = WORKLOAD
    t0 = time.perf_counter()
    oracle.emulate(q, k, v, causal=w.causal, block_n=128, p_scale=P_SCALE, reverse=bool(KV_ORDER), rows=rows)
    dt = time.perf_counter() - t0
    flops = 4.0 * w.d * visible_pairs(rows, w.N, w.causal) * w.B * w.H
    return flops, dt


def cpu_baseline(q, k, v):
    import oracle

    rows = sample_rows(WORKLOAD.N, CPU_SAMPLE_ROWS)
    flops, dt = cpu_oracle_run(q, k, v, rows)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"blockwise E4M3 emulator on {len(rows)} evenly spaced query rows of each of the "
                      f"{WORKLOAD.B * WORKLOAD.H} heads ({flops / 1e12:.3f} TFLOP in {dt:.1f} s)"}


def max_over_ranks(x: float, dist, device) -> float:
    """The maximum of a per-rank scalar over all ranks (identity when alone)."""
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(flop_per_rank: float, world: int, ms_per_step_max: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's step time."""
    return flop_per_rank * world / (ms_per_step_max * 1e-3) / 1e12


def rank_seed(rank: int) -> int:
    """Each rank runs its own copy of the workload on its own inputs."""
    return SEED + rank


def mse_vs_fp64(qd, kd, vd, o, rows_np):
    """MSE of the output against exact attention computed in FP64 by PyTorch on
    the same decoded E4M3 inputs, over the given query rows of every head."""
    import torch

    w = WORKLOAD
    rows = torch.from_numpy(rows_np.astype(np.int64)).to(qd.device)
    qf = qd.view(torch.float8_e4m3fn)[:, :, rows].double()
    kf = kd.view(torch.float8_e4m3fn).double()
    vf = vd.view(torch.float8_e4m3fn).double()
    rep = w.H // w.Hkv
    kf, vf = kf.repeat_interleave(rep, 1), vf.repeat_interleave(rep, 1)
    s = qf @ kf.transpose(-1, -2) / math.sqrt(w.d)
    if w.causal:
        keys = torch.arange(w.N, device=qd.device)
        s = s.masked_fill(keys[None, None, None, :] > rows[None, None, :, None], float("-inf"))
    ref = torch.softmax(s, -1) @ vf
    return float(((o[:, :, rows].double() - ref) ** 2).mean().item())


WIDE_WORKLOAD_DESC = ("prefill32k from bfloat16: B=1 H=32 N=32768 d=128 causal, Delta=7 sink (k=4); Q/K/V quantised "
                      "to E4M3 in the step (random-sign Hadamard rotation, Q/K per 128-row block, V per head), "
                      "S=256, reverse KV order, output rotated back")
WIDE_CPU_ROWS = 512


def wide_inputs(seed: int):
    w = WORKLOAD
    q, k, v, _ = synthetic.make_wide_inputs(w.B, w.H, w.Hkv, w.N, w.d, w.delta, seed=seed, n_sink=w.n_sink)
    return q, k, v, synthetic.hadamard_signs(w.d, seed + 7)


def cpu_wide_run(q, k, v, signs, rows):
    """One bounded step of the oracle on the wide path: quantise all of Q, K, V,
    then the emulator on `rows` of every head and the inverse rotation."""
    from oracle import quantize as Qz

    w = WORKLOAD
    t0 = time.perf_counter()
    Qz.quantized_attention(q, k, v, signs, causal=w.causal, p_scale=P_SCALE, reverse=bool(KV_ORDER), rows=rows)
    dt = time.perf_counter() - t0
    return 4.0 * w.d * visible_pairs(rows, w.N, w.causal) * w.B * w.H, dt


def run_wide(args, rank, world, local_rank):
    """The wide path: quantise bfloat16 inputs, then the scaled forward pass."""
    import torch

    from softmax_cast_precision_b200 import fp8attn

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = WORKLOAD
    q, k, v, signs = wide_inputs(rank_seed(rank))
    qb, kb, vb = (torch.from_numpy(x).to(device).to(torch.bfloat16) for x in (q, k, v))
    stream = torch.cuda.current_stream(device)
    ev_q0, ev_q1, ev_f1 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    quant_ms, fwd_ms = [], []

    def step(timed=False):
        if timed:
            ev_q0.record(stream)
        qc, qs = fp8attn.quantize(qb, 128, signs, stream=stream)
        kc, ks = fp8attn.quantize(kb, 128, signs, stream=stream)
        vc, vs = fp8attn.quantize(vb, 0, signs, stream=stream)
        if timed:
            ev_q1.record(stream)
        o, lse = fp8attn.fwd_scaled(qc, kc, vc, qs, ks, vs, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER,
                                    signs=signs, stream=stream)
        if timed:
            ev_f1.record(stream)
            ev_f1.synchronize()
            quant_ms.append(ev_q0.elapsed_time(ev_q1))
            fwd_ms.append(ev_q1.elapsed_time(ev_f1))
        return o, lse

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    fp8attn.check_error(stream=stream, device=device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize(device)
        ev[0].record(stream)
        for i in range(args.steps):
            o, lse = step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(device)
        barrier()
    fp8attn.check_error(stream=stream, device=device)
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, device)
    ms_per_step = total_ms / args.steps
    flops = w.flops()
    # Per-kernel durations, from separately synchronised steps after the timed region.
    for _ in range(5):
        step(timed=True)

    # End to end: bfloat16 inputs from pinned host memory, outputs back.
    qh, kh, vh = (t.cpu().pin_memory() for t in (qb, kb, vb))
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    qd, kd, vd = (torch.empty_like(t) for t in (qb, kb, vb))

    def e2e_step():
        for dst, src in ((qd, qh), (kd, kh), (vd, vh)):
            dst.copy_(src, non_blocking=True)
        oo, ll = fp8attn.fwd_wide(qd, kd, vd, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, signs=signs,
                                  stream=stream)
        oh.copy_(oo, non_blocking=True)
        lh.copy_(ll, non_blocking=True)

    e2e_step()
    e2e_steps = max(3, min(args.steps, 10))
    barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, device)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    mse = None
    if rank == 0:
        rows = sample_rows(w.N, 256)
        mse = wide_mse_vs_fp64(qb, kb, vb, o, rows)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak_burst, peak_sustained, peak_src = fp8_peak()
    fwd_kernel_ms = statistics.mean(fwd_ms)
    quant_kernel_ms = statistics.mean(quant_ms)
    achieved = flops / (fwd_kernel_ms * 1e-3) / 1e12
    hbm = hbm_peak()
    quant_bytes = 3 * (qb.numel() * 3)  # three tensors, 2 B read + 1 B written per element
    line = {
        "metric": METRIC, "value": aggregate_throughput(flops, world, ms_per_step), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3", "data": "synthetic",
        "config": {"workload": WIDE_WORKLOAD_DESC, "flop_per_step_per_gpu": flops,
                   "l2": "inputs exceed L2 (805 MB bfloat16)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "gpu_launches": 6 * args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                     "frac": achieved / peak_burst, "traffic": None,
                     "peak_source": f"{peak_src}: bf16 cuBLAS burst x {FP8_OVER_BF16} (FP8/BF16 nominal)",
                     "kernel": "fwd_v2_kernel<0,1> (scaled)", "kernel_ms": fwd_kernel_ms},
        "roofline_quantize": {"bound": "hbm", "achieved": quant_bytes / (quant_kernel_ms * 1e-3) / 1e9,
                              "peak": hbm, "unit": "GB/s",
                              "frac": quant_bytes / (quant_kernel_ms * 1e-3) / 1e9 / hbm,
                              "algorithmic_bytes": quant_bytes, "ms": quant_kernel_ms,
                              "note": "3 tensors x (2 B read + 1 B written) per element; V's per-head descale "
                                      "reads V twice"},
        "e2e": {"value": aggregate_throughput(flops, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "clocks": clk.summary(),
        "mse_vs_fp64": {"value": mse, "rows": "256 evenly spaced query rows of each head",
                        "reference": "PyTorch float64 softmax(QK^T/sqrt(d))V on the bfloat16 inputs"},
    }
    if not args.skip_cpu_baseline:
        import oracle

        rows = sample_rows(w.N, WIDE_CPU_ROWS)
        f, dt = cpu_wide_run(q, k, v, signs, rows)
        line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"quantisation of all of Q, K, V, then the emulator on {len(rows)} evenly "
                                          f"spaced query rows of each head ({f / 1e12:.3f} TFLOP in {dt:.1f} s)"}
    print(json.dumps(line), flush=True)


BF16QK_WORKLOAD_DESC = ("prefill32k with bfloat16 Q and K: B=1 H=32 N=32768 d=128 causal, Delta=7 sink (k=4), "
                        "E4M3 V, S=256, reverse KV order")


def run_bf16qk(args, rank, world, local_rank):
    """bfloat16 Q and K, E4M3 V: one fp8attn_fwd_bf16qk launch per step."""
    import torch

    from softmax_cast_precision_b200 import fp8attn

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = WORKLOAD
    q, k, v, _ = wide_inputs(rank_seed(rank))
    v8 = torch.from_numpy(np.clip(v, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8)
    qb, kb = (torch.from_numpy(x).to(device).to(torch.bfloat16) for x in (q, k))
    vd = v8.to(device)
    stream = torch.cuda.current_stream(device)

    def step():
        return fp8attn.fwd_bf16qk(qb, kb, vd, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    fp8attn.check_error(stream=stream, device=device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize(device)
        ev[0].record(stream)
        for i in range(args.steps):
            o, lse = step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(device)
        barrier()
    fp8attn.check_error(stream=stream, device=device)
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, device)
    ms_per_step = total_ms / args.steps
    flops = w.flops()
    # End to end from pinned host buffers.
    qh, kh, vh = qb.cpu().pin_memory(), kb.cpu().pin_memory(), v8.pin_memory()
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    qd, kd, vd2 = torch.empty_like(qb), torch.empty_like(kb), torch.empty_like(vd)

    def e2e_step():
        for dst, src in ((qd, qh), (kd, kh), (vd2, vh)):
            dst.copy_(src, non_blocking=True)
        oo, ll = fp8attn.fwd_bf16qk(qd, kd, vd2, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, stream=stream)
        oh.copy_(oo, non_blocking=True)
        lh.copy_(ll, non_blocking=True)

    e2e_step()
    e2e_steps = max(3, min(args.steps, 10))
    barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, device)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    mse = None
    if rank == 0:
        mse = wide_mse_vs_fp64(qb, kb, vd.view(torch.float8_e4m3fn).float(), o, sample_rows(w.N, 256))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak_bf16, _, peak_src = fp8_peak()
    peak_bf16 /= FP8_OVER_BF16
    # Half of the FLOPs (Q K^T) at the 16-bit rate, half (P V) at the FP8 rate.
    peak_mix = 1.0 / (0.5 / peak_bf16 + 0.5 / (peak_bf16 * FP8_OVER_BF16))
    kernel_ms = statistics.mean(per_step)
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": aggregate_throughput(flops, world, ms_per_step), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 QK / e4m3 PV", "data": "synthetic",
        "config": {"workload": BF16QK_WORKLOAD_DESC, "flop_per_step_per_gpu": flops,
                   "l2": "inputs exceed L2 (671 MB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "gpu_launches": args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_mix, "unit": "TFLOP/s",
                     "frac": achieved / peak_mix, "traffic": None,
                     "peak_source": f"{peak_src}: half the FLOPs at the bf16 cuBLAS burst rate, half at x "
                                    f"{FP8_OVER_BF16} (FP8/BF16 nominal)"},
        "e2e": {"value": aggregate_throughput(flops, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "clocks": clk.summary(),
        "mse_vs_fp64": {"value": mse, "rows": "256 evenly spaced query rows of each head",
                        "reference": "PyTorch float64 softmax(QK^T/sqrt(d))V on the bfloat16 Q, K and decoded V"},
    }
    if not args.skip_cpu_baseline:
        import oracle

        rows = sample_rows(w.N, CPU_SAMPLE_ROWS)
        t0 = time.perf_counter()
        oracle.emulate(q, k, v8.numpy(), causal=w.causal, block_n=128, p_scale=P_SCALE, reverse=bool(KV_ORDER),
                       rows=rows)
        dt = time.perf_counter() - t0
        f = 4.0 * w.d * visible_pairs(rows, w.N, w.causal) * w.B * w.H
        line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"blockwise emulator on {len(rows)} evenly spaced query rows of each head "
                                          f"({f / 1e12:.3f} TFLOP in {dt:.1f} s)"}
    print(json.dumps(line), flush=True)


DECODE_SHAPE = dict(B=32, H=32, Hkv=8, N=32768, split_tiles=32)
DECODE_METRIC = "FP8 split-KV decode GB/s of K/V read (HBM roofline)"


def run_decode(args, rank, world, local_rank):
    """One fp8attn_decode call per step (split pass + merge), timed with CUDA events."""
    import torch

    from softmax_cast_precision_b200 import fp8attn

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    sh = DECODE_SHAPE
    B, H, Hkv, N, split = sh["B"], sh["H"], sh["Hkv"], sh["N"], sh["split_tiles"]
    g = torch.Generator(device=device).manual_seed(rank_seed(rank))

    def mk(*shape):
        return torch.randn(shape, device=device, generator=g).clamp(-448, 448).to(torch.float8_e4m3fn).view(
            torch.uint8)

    q, k, v = mk(B, H, 128), mk(B, Hkv, N, 128), mk(B, Hkv, N, 128)
    ws = torch.empty(int(fp8attn.lib().fp8attn_decode_workspace_bytes(B, H, N, split)), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        return fp8attn.decode(q, k, v, p_scale=P_SCALE, kv_order=KV_ORDER, split_tiles=split, workspace=ws,
                              stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    fp8attn.check_error(stream=stream, device=device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize(device)
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(device)
        barrier()
    fp8attn.check_error(stream=stream, device=device)
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, device)
    ms_per_step = total_ms / args.steps
    kv_bytes = 2 * k.numel()
    alg_bytes = kv_bytes + q.numel() + B * H * 128 * 2 + B * H * 4
    # End to end: K/V from pinned host memory (the cache would normally stay resident; this is the
    # worst case the public call can be timed at).
    qh, kh, vh = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    oh = torch.empty((B, H, 128), dtype=torch.bfloat16, pin_memory=True)
    lh = torch.empty((B, H), dtype=torch.float32, pin_memory=True)

    def e2e_step():
        for dst, src in ((qd, qh), (kd, kh), (vd, vh)):
            dst.copy_(src, non_blocking=True)
        o, lse = fp8attn.decode(qd, kd, vd, p_scale=P_SCALE, kv_order=KV_ORDER, split_tiles=split, workspace=ws,
                                stream=stream)
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / 3, dist, device)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    kernel_ms = statistics.mean(ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps))
    hbm = hbm_peak()
    achieved = alg_bytes / (kernel_ms * 1e-3) / 1e9
    line = {
        "metric": DECODE_METRIC, "value": kv_bytes * world / (ms_per_step * 1e-3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": f"decode: B={B} H={H} Hkv={Hkv} N={N} d=128, one query row per head, E4M3 Q/K/V "
                               f"N(0,1), S=256, reverse order inside {split}-tile splits",
                   "l2": f"K/V exceed L2 ({kv_bytes / 1e9:.2f} GB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "gpu_launches": 2 * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": None, "algorithmic_bytes": alg_bytes,
                     "peak_source": "measured copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
        "e2e": {"value": kv_bytes * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": q.numel() + 2 * k.numel(), "d2h_bytes_per_step": B * H * (128 * 2 + 4),
                "ms_per_step": e2e_ms},
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


BWD_WORKLOAD_DESC = ("prefill32k backward: B=1 H=32 N=32768 d=128 causal, E4M3 Q/K/V (Delta=7 sink, k=4), "
                     "O and lse from fp8attn_fwd (S=256, reverse), bfloat16 dO ~ N(0,1); float32 dQ, dK, dV")
BWD_CPU_N = 4096  # the oracle sample: the leading N x N causal block of one head


def run_bwd(args, rank, world, local_rank):
    """The backward pass of the 32K prefill: one fp8attn_bwd call (five launches) per step."""
    import torch

    from softmax_cast_precision_b200 import fp8attn

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = WORKLOAD
    q, k, v, _ = synthetic.workload_inputs(w, seed=rank_seed(rank))
    do = synthetic.make_output_grad((w.B, w.H, w.N, w.d), rank_seed(rank) + 1)
    qd, kd, vd = (torch.from_numpy(x).to(device) for x in (q, k, v))
    dod = torch.from_numpy(do).to(device).to(torch.bfloat16)
    del do
    stream = torch.cuda.current_stream(device)
    o, lse = fp8attn.fwd(qd, kd, vd, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, stream=stream)

    def step():
        return fp8attn.bwd(qd, kd, vd, o, lse, dod, causal=w.causal, p_scale=P_SCALE, stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    fp8attn.check_error(stream=stream, device=device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize(device)
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(device)
        barrier()
    fp8attn.check_error(stream=stream, device=device)
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, device)
    ms_per_step = total_ms / args.steps
    pairs = w.B * w.H * w.N * (w.N + 1) // 2 if w.causal else w.B * w.H * w.N * w.N
    flops = 10.0 * w.d * pairs  # five products of 2 d FLOPs per visible (query, key) pair
    # End to end from pinned host buffers: the forward's inputs and outputs and dO in, the gradients out.
    hosts = [t.cpu().pin_memory() for t in (qd, kd, vd, o, lse, dod)]
    devs = [torch.empty_like(t) for t in (qd, kd, vd, o, lse, dod)]
    outs = [torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, pin_memory=True),
            torch.empty((w.B, w.Hkv, w.N, w.d), dtype=torch.float32, pin_memory=True),
            torch.empty((w.B, w.Hkv, w.N, w.d), dtype=torch.float32, pin_memory=True)]

    def e2e_step():
        for dst, src in zip(devs, hosts):
            dst.copy_(src, non_blocking=True)
        grads = fp8attn.bwd(*devs, causal=w.causal, p_scale=P_SCALE, stream=stream)
        for dst, src in zip(outs, grads[:3]):
            dst.copy_(src, non_blocking=True)

    e2e_step()
    barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / 3, dist, device)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak_bf16, _, peak_src = fp8_peak()
    peak_bf16 /= FP8_OVER_BF16
    # One product (S) at the FP8 rate, four (dP, dV, dK, dQ) at the 16-bit rate.
    peak_mix = 1.0 / (0.8 / peak_bf16 + 0.2 / (peak_bf16 * FP8_OVER_BF16))
    kernel_ms = statistics.mean(ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps))
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    line = {
        "metric": "FP8 P-cast attention backward TFLOP/s at N=32K, d=128", "unit": UNIT,
        "value": aggregate_throughput(flops, world, ms_per_step), "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 S / bf16 dP dV dK dQ", "data": "synthetic",
        "config": {"workload": BWD_WORKLOAD_DESC, "flop_per_step_per_gpu": flops,
                   "l2": "inputs exceed L2 (1.05 GB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "gpu_launches": 5 * args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_mix, "unit": "TFLOP/s",
                     "frac": achieved / peak_mix, "traffic": None,
                     "peak_source": f"{peak_src}: one fifth of the FLOPs at x {FP8_OVER_BF16} (FP8/BF16 nominal) "
                                    "of the bf16 cuBLAS burst rate, four fifths at it"},
        "e2e": {"value": aggregate_throughput(flops, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hosts),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs), "ms_per_step": e2e_ms},
        "clocks": clk.summary(),
    }
    if not args.skip_cpu_baseline:
        import oracle
        from oracle import backward as Bw

        n = BWD_CPU_N
        qs, ks, vs = q[:1, :1, :n], k[:1, :1, :n], v[:1, :1, :n]
        fwd_o = oracle.emulate(qs, ks, vs, causal=w.causal, block_n=128, p_scale=P_SCALE, reverse=bool(KV_ORDER))
        dos = synthetic.make_output_grad((1, 1, n, w.d), 7)
        t0 = time.perf_counter()
        Bw.backward(qs, ks, vs, oracle.bf16_bits_to_float(fwd_o.o_bf16), fwd_o.lse, dos, causal=w.causal,
                    p_scale=P_SCALE)
        dt = time.perf_counter() - t0
        f = 10.0 * w.d * (n * (n + 1) // 2 if w.causal else n * n)
        from threadpoolctl import threadpool_info

        blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": UNIT, "cores": max(blas) if blas else 1,
                                "kind": "oracle",
                                "sample": f"float64 backward oracle on the leading {n} x {n} block of one head "
                                          f"({f / 1e12:.4f} TFLOP in {dt:.1f} s)"}
    print(json.dumps(line), flush=True)


def run_sharded(args, rank, world, local_rank):
    """Strong scaling: one 32K prefill split by kv heads across the ranks; a step
    is every rank's shard plus the all-gather of O and lse (NCCL)."""
    import torch

    from softmax_cast_precision_b200 import fp8attn
    from softmax_cast_precision_b200.parallel import fwd_head_sharded

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = WORKLOAD
    q, k, v, _ = synthetic.workload_inputs(w, seed=SEED)  # the same problem on every rank
    qd, kd, vd = (torch.from_numpy(x).to(device) for x in (q, k, v))
    stream = torch.cuda.current_stream(device)

    def shard_fwd(qs, ks, vs, **kw):
        return fp8attn.fwd(qs, ks, vs, stream=stream, **kw)

    def step():
        if dist is None:
            return fp8attn.fwd(qd, kd, vd, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, stream=stream)
        return fwd_head_sharded(qd, kd, vd, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, compute=shard_fwd)

    for _ in range(args.warmup):
        step()
    fp8attn.check_error(stream=stream, device=device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(device)
        ev[0].record(stream)
        for i in range(args.steps):
            o, lse = step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(device)
        if dist is not None:
            dist.barrier()
    fp8attn.check_error(stream=stream, device=device)
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, device)
    ms_per_step = total_ms / args.steps
    flops = w.flops()
    mse = mse_vs_fp64(qd, kd, vd, o, sample_rows(w.N, 256)) if rank == 0 else None
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": flops / (ms_per_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "flop_per_step": flops, "l2": "inputs exceed L2 (402 MB)",
                   "parallelism": f"kv heads split over {world} ranks, all-gather of O and lse"},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "mse_vs_fp64": {"value": mse, "rows": "256 evenly spaced query rows of each head",
                        "reference": "PyTorch float64 softmax(QK^T/sqrt(d))V on the same E4M3 inputs"},
    }), flush=True)


def hbm_peak() -> float:
    try:
        with open(PEAKS_FILE) as fh:
            return float(json.load(fh)["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        return 6650.0


def wide_mse_vs_fp64(qb, kb, vb, o, rows_np):
    """MSE of the output against FP64 attention on the bfloat16 inputs, over the given rows."""
    import torch

    w = WORKLOAD
    rows = torch.from_numpy(rows_np.astype(np.int64)).to(qb.device)
    qf = qb[:, :, rows].double()
    kf, vf = kb.double(), vb.double()
    rep = w.H // w.Hkv
    kf, vf = kf.repeat_interleave(rep, 1), vf.repeat_interleave(rep, 1)
    s = qf @ kf.transpose(-1, -2) / math.sqrt(w.d)
    if w.causal:
        keys = torch.arange(w.N, device=qb.device)
        s = s.masked_fill(keys[None, None, None, :] > rows[None, None, :, None], float("-inf"))
    ref = torch.softmax(s, -1) @ vf
    return float(((o[:, :, rows].double() - ref) ** 2).mean().item())


def run_reference_wide(args, rank):
    """The oracle arm of the wide path (rank 0 only)."""
    if rank != 0:
        return
    import oracle

    q, k, v, signs = wide_inputs(SEED)
    rows = sample_rows(WORKLOAD.N, 64)
    for _ in range(args.warmup):
        cpu_wide_run(q[:, :, :256], k[:, :, :256], v[:, :, :256], signs, rows[:2] // 128)
    total_flops, total_t = 0.0, 0.0
    for _ in range(args.steps):
        f, dt = cpu_wide_run(q, k, v, signs, rows)
        total_flops += f
        total_t += dt
    value = total_flops / total_t / 1e12
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3/f32",
        "data": "synthetic", "config": {"workload": WIDE_WORKLOAD_DESC, "l2": "inputs exceed L2"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"per step: quantisation of all of Q, K, V and the emulator on {len(rows)} "
                                   "evenly spaced query rows of each head"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_reference(args, rank, world):
    """The oracle arm: emulator steps on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle

    q, k, v, _ = synthetic.workload_inputs(WORKLOAD, seed=SEED)
    rows = sample_rows(WORKLOAD.N, 128)
    for _ in range(args.warmup):
        cpu_oracle_run(q, k, v, rows[:8])
    total_flops, total_t = 0.0, 0.0
    for _ in range(args.steps):
        f, dt = cpu_oracle_run(q, k, v, rows)
        total_flops += f
        total_t += dt
    value = total_flops / total_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3/f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "l2": "inputs exceed L2"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"per step: the emulator on {len(rows)} evenly spaced query rows of each head"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def set_seq_len(args):
    """A smaller case of the same workload for profiling (--seq-len): the
    prefill paths run at sequence length N, the decode path against N keys."""
    global WORKLOAD, WORKLOAD_DESC, WIDE_WORKLOAD_DESC, BF16QK_WORKLOAD_DESC, BWD_WORKLOAD_DESC
    n = args.seq_len
    if args.impl != "ours" or args.shard != "replicas" or n < 1:
        raise SystemExit("--seq-len covers our implementation with replicas")
    if args.path == "decode":
        DECODE_SHAPE["N"] = n
        return
    WORKLOAD = dataclasses.replace(WORKLOAD, name=f"prefill{n}", N=n)
    tag = f"N={n} (profiling case, not the headline)"
    WORKLOAD_DESC = WORKLOAD_DESC.replace("N=32768", tag)
    WIDE_WORKLOAD_DESC = WIDE_WORKLOAD_DESC.replace("N=32768", tag)
    BF16QK_WORKLOAD_DESC = BF16QK_WORKLOAD_DESC.replace("N=32768", tag)
    BWD_WORKLOAD_DESC = BWD_WORKLOAD_DESC.replace("N=32768", tag)


def set_head_dim(args):
    """The fp8 path's prefill at another head dimension (--head-dim; profiling)."""
    global WORKLOAD, WORKLOAD_DESC
    if args.impl != "ours" or args.shard != "replicas" or args.path != "fp8":
        raise SystemExit("--head-dim covers our fp8 path with replicas")
    WORKLOAD = dataclasses.replace(WORKLOAD, d=args.head_dim)
    WORKLOAD_DESC = WORKLOAD_DESC.replace("d=128", f"d={args.head_dim} (profiling case, not the headline)")


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.seq_len is not None:
        set_seq_len(args)
    if args.head_dim is not None:
        set_head_dim(args)
    if args.impl == "reference":
        if args.path in ("bf16qk", "decode", "bwd"):
            raise SystemExit("--impl reference covers --path fp8 and wide")
        return run_reference_wide(args, rank) if args.path == "wide" else run_reference(args, rank, world)
    if args.shard == "heads":
        if args.path != "fp8" or args.impl != "ours":
            raise SystemExit("--shard heads covers the fp8 path")
        return run_sharded(args, rank, world, local_rank)
    if args.path == "bwd":
        return run_bwd(args, rank, world, local_rank)
    if args.path == "wide":
        return run_wide(args, rank, world, local_rank)
    if args.path == "bf16qk":
        return run_bf16qk(args, rank, world, local_rank)
    if args.path == "decode":
        return run_decode(args, rank, world, local_rank)

    import torch

    from softmax_cast_precision_b200 import fp8attn

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    w = WORKLOAD
    q, k, v, _ = synthetic.workload_inputs(w, seed=rank_seed(rank))
    qd, kd, vd = (torch.from_numpy(x).to(device) for x in (q, k, v))
    o = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        fp8attn.fwd(qd, kd, vd, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, out=o, lse_out=lse,
                    stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    fp8attn.check_error(stream=stream, device=device)

    # --- device-timed region: K steps, one kernel launch each --------------
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize(device)
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(device)
        barrier()
    fp8attn.check_error(stream=stream, device=device)
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist, device)
    ms_per_step = total_ms / args.steps
    flops = w.flops()
    value = aggregate_throughput(flops, world, ms_per_step)

    # --- end to end through the public API with host buffers ----------------
    # fwd_host: pinned host inputs and outputs, the copies in and out
    # overlapped with the computation piece by piece; each call returns once
    # the outputs are on the host, and its streams start after and join back
    # into the current stream, so events on that stream span whole calls.
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 10))

    def e2e_step():
        fp8attn.fwd_host(qh, kh, vh, causal=w.causal, p_scale=P_SCALE, kv_order=KV_ORDER, out=oh, lse_out=lh,
                         device=device)

    e2e_step()
    barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, device)
    fp8attn.check_error(stream=stream, device=device)
    h2d = q.nbytes + k.nbytes + v.nbytes
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    mse = mse_vs_fp64(qd, kd, vd, o, sample_rows(w.N, 256)) if rank == 0 else None
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peak_burst, peak_sustained, peak_src = fp8_peak()
    kernel_ms = statistics.mean(per_step)
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    traffic = traffic_per_launch() if args.seq_len is None else None
    clocks = clk.summary()
    # The measured peak was taken at its own (power-capped) clock; the same
    # peak scaled to the clock this kernel ran at gives the fraction per clock.
    p_mhz, k_mhz = peak_clock_mhz(), clocks.get("sm_mhz")
    frac_clock = achieved / (peak_burst * k_mhz / p_mhz) if p_mhz and k_mhz else None
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "flop_per_step_per_gpu": flops,
                   "l2": f"inputs exceed L2 ({(q.nbytes + k.nbytes + v.nbytes) / 1e6:.0f} MB)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "gpu_launches": args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                     "frac": achieved / peak_burst, "traffic": traffic,
                     "peak_source": f"{peak_src}: bf16 cuBLAS burst x {FP8_OVER_BF16} (FP8/BF16 nominal)",
                     "frac_of_sustained": achieved / peak_sustained,
                     "frac_at_kernel_clock": frac_clock,
                     "clock_note": (f"peak measured at a median {p_mhz} MHz, this kernel at {k_mhz} MHz: "
                                    "frac_at_kernel_clock = achieved / (peak x kernel MHz / peak MHz)")},
        "e2e": {"value": aggregate_throughput(flops, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "how": "fp8attn_fwd_host with pinned host buffers: one persistent pass over pieces copied in and out on two copy streams; CUDA events"},
        "clocks": clocks,
        "mse_vs_fp64": {"value": mse, "rows": "256 evenly spaced query rows of each head",
                        "reference": "PyTorch float64 softmax(QK^T/sqrt(d))V on the same E4M3 inputs"},
    }
    if not args.skip_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(q, k, v)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
