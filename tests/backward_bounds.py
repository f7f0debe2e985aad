"""Per-element error bounds for a backward-pass result computed the way the
CUDA kernels compute it, compared with the float64 oracle (oracle.backward).
Test helper: no test functions here.

The kernels' arithmetic (fp8attn_bwd):
  * S = Q K^T of E4M3 values accumulated in float32; P = 2^x with the
    float32 argument x = S log2(e)/sqrt(d) - lse log2(e);
  * E4M3(P S) rounded from that float32 P;
  * dP_ij = dO_i . v_j and D_i = dO_i . O_i as float32 sums of exact
    products; dS = P (dP - D) in float32, then rounded to bfloat16;
  * dQ, dK, dV accumulated in float32.

Bounds, element by element, each with its source:
  * dQ_ic (dK likewise, with q for k): the bfloat16 rounding of dS (unit
    roundoff u = 2^-8) contributes at most u sum_j |dS_ij k_jc| / sqrt(d);
    the float32 error of dP_ij - D_i, at most EPS_DOT (A_ij + B_i) with
    A_ij = sum_c |dO_ic v_jc| and B_i = sum_c |dO_ic O_ic|, contributes
    sum_j P_ij EPS_DOT (A_ij + B_i) |k_jc| / sqrt(d).  Both are doubled
    (the float32 error of P and of the accumulation), plus EPS_ACC of the
    magnitude for the accumulation over up to N terms.
  * dV_jc: P from a float32 exponential may round to the other E4M3 value
    where P S lies within a relative AMB of a rounding boundary (AMB covers
    float32 arguments |x| up to 64); the bound is the sum over i of
    |E4M3(P S (1 + AMB)) - E4M3(P S (1 - AMB))| / S |dO_ic|, plus EPS_ACC of
    sum_i E4M3(P_ij S) / S |dO_ic|.
  * delta_i: EPS_DOT sum_c |dO_ic O_ic|.
"""
from __future__ import annotations

import numpy as np

import oracle

U_BF16 = 2.0 ** -8
EPS_DOT = 2.0 ** -16
EPS_ACC = 2.0 ** -12
AMB = 2.0 ** -16


def error_bounds(q, k, v, o, lse, do, *, causal: bool, p_scale: float):
    """Bounds (dq, dk, dv, delta) on |kernel result - oracle result|, same shapes as the results."""
    qf, kf, vf = (oracle.e4m3_decode(x).astype(np.float64) for x in (q, k, v))
    o = np.asarray(o, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    B, H, N, d = qf.shape
    Hkv = kf.shape[1]
    rep = H // Hkv
    bq = np.zeros_like(qf)
    bk = np.zeros_like(kf)
    bv = np.zeros_like(vf)
    mask = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)
    inv = 1.0 / np.sqrt(d)
    S = float(p_scale)

    def cast(x):
        return oracle.e4m3_round(np.minimum(x, 3.0e38).astype(np.float32)).astype(np.float64)

    for b in range(B):
        for h in range(H):
            hk = h // rep
            s = qf[b, h] @ kf[b, hk].T * inv
            p = np.where(mask, np.exp(np.where(mask, s, 0.0) - lse[b, h][:, None]), 0.0)
            dp = do[b, h] @ vf[b, hk].T
            dd = np.sum(do[b, h] * o[b, h], axis=1)
            ds = np.abs(p * (dp - dd[:, None]))
            a = np.abs(do[b, h]) @ np.abs(vf[b, hk]).T
            bb = np.sum(np.abs(do[b, h] * o[b, h]), axis=1)
            w_round = ds
            w_dot = p * EPS_DOT * (a + bb[:, None])
            w = 2.0 * U_BF16 * w_round + 2.0 * w_dot + EPS_ACC * w_round
            bq[b, h] = w @ np.abs(kf[b, hk]) * inv
            bk[b, hk] += w.T @ np.abs(qf[b, h]) * inv
            lo, hi = cast(p * S * (1.0 - AMB)), cast(p * S * (1.0 + AMB))
            mid = cast(p * S)
            bv[b, hk] += (np.abs(hi - lo) / S).T @ np.abs(do[b, h]) + EPS_ACC * (mid / S).T @ np.abs(do[b, h])
    bdelta = EPS_DOT * np.sum(np.abs(do * o), axis=-1)
    tiny = 1e-30
    return bq + tiny, bk + tiny, bv + tiny, bdelta + tiny


def violations(got, ref, bound):
    """(number of elements outside the bound, worst |got - ref| / bound)."""
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    ratio = err / bound
    return int(np.count_nonzero(ratio > 1.0)), float(ratio.max()) if ratio.size else 0.0
