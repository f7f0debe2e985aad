"""Oracle for the decode / split-KV form of the P-cast attention forward pass.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle``).

One query row per (batch, head) attends to all N keys.  The keys are cut
into splits of ``split_tiles`` consecutive 128-key tiles; each split runs the
blockwise online softmax with the P-cast on its own (its tiles walked forward
or in reverse, so the KV order becomes an order inside each split), and the
splits are merged by their log-sum-exp weights.  This follows the blockwise
recurrence of "Attenzione flash e domanda sulla lunghezza della sequenza"
(sections "L'algoritmo Flash Attention" and "La ricorrenza softmax online":
partial results over disjoint key blocks combine exactly through their
maxima and sums) with the cast of "P-Cast Precision in FP8 Attention",
technical summary, section 1, applied inside every split.  Reading (the
pages do not treat decode): the splits are independent, and the merge is
exact arithmetic on each split's output and log-sum-exp.
"""
from __future__ import annotations

import numpy as np

from . import _values, bf16_bits_to_float, bf16_round_bits, emulate


def split_decode(q, k, v, *, p_scale: float, reverse: bool, split_tiles: int, block_n: int = 128,
                 cast: bool = True, n_sink: int = 4):
    """q [B, H, d], k and v [B, Hkv, N, d] (E4M3 bytes or float values).

    Returns a dict: o (float32 values of the bfloat16 output [B, H, d]),
    o_f64 (the merged output before rounding), lse [B, H] (natural log, in
    logit units), and the per-split outputs and log-sum-exps.
    """
    qf = _values(q)
    kf, vf = _values(k), _values(v)
    if qf.ndim != 3 or kf.ndim != 4 or vf.shape != kf.shape:
        raise ValueError("q must be [B, H, d] and k, v [B, Hkv, N, d]")
    B, H, d = qf.shape
    N = kf.shape[2]
    if N < 1 or split_tiles < 1:
        raise ValueError("N and split_tiles must be positive")
    span = split_tiles * block_n
    outs, lses = [], []
    for lo in range(0, N, span):
        hi = min(N, lo + span)
        qp = np.zeros((B, H, hi - lo, d), dtype=np.float32)
        qp[:, :, 0] = qf
        r = emulate(qp, kf[:, :, lo:hi], vf[:, :, lo:hi], causal=False, block_n=block_n, p_scale=p_scale,
                    reverse=reverse, cast=cast, n_sink=n_sink, rows=[0])
        outs.append(r.o_f32[:, :, 0].astype(np.float64))
        lses.append(r.lse[:, :, 0].astype(np.float64))
    lse_s = np.stack(lses)                     # [splits, B, H]
    o_s = np.stack(outs)                       # [splits, B, H, d]
    top = lse_s.max(axis=0)
    w = np.exp(lse_s - top)
    lse = top + np.log(w.sum(axis=0))
    o64 = (w[..., None] * o_s).sum(axis=0) / w.sum(axis=0)[..., None]
    o = bf16_bits_to_float(bf16_round_bits(o64.astype(np.float32)))
    return {"o": o, "o_f64": o64, "lse": lse, "split_o": o_s, "split_lse": lse_s}
