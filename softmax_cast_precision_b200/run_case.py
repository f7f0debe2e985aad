"""Run the forward kernel on one synthetic shape and print its device time.

Used to profile a single shape, e.g. under ncu:

    python -m softmax_cast_precision_b200.run_case --H 32 --N 16384 --causal --reps 3
"""
from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=0, help="0 = same as H")
    ap.add_argument("--N", type=int, default=16384)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--delta", type=float, default=7.0)
    ap.add_argument("--scale", type=float, default=256.0)
    ap.add_argument("--order", default="reverse", choices=["forward", "reverse"])
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--reps", type=int, default=1)
    ap.add_argument("--count", action="store_true", help="run the P-collapse count kernel instead")
    a = ap.parse_args()

    import torch

    import synthetic
    from softmax_cast_precision_b200 import fp8attn

    Hkv = a.Hkv or a.H
    q, k, v, _ = synthetic.make_inputs(a.B, a.H, Hkv, a.N, a.d, a.delta, seed=1234)
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))

    def once():
        if a.count:
            fp8attn.pzero_count(qd, kd, vd, causal=a.causal, p_scale=a.scale, kv_order=a.order)
        else:
            fp8attn.fwd(qd, kd, vd, causal=a.causal, p_scale=a.scale, kv_order=a.order)

    for _ in range(a.warmup):
        once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        once()
    e1.record()
    torch.cuda.synchronize()
    fp8attn.check_error()
    ms = e0.elapsed_time(e1) / a.reps
    pairs = a.N * (a.N + 1) // 2 if a.causal else a.N * a.N
    flops = 4.0 * a.d * pairs * a.B * a.H
    print(json.dumps({"shape": vars(a), "ms": ms, "tflops": flops / ms / 1e9}))


if __name__ == "__main__":
    main()
