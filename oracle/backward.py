"""Oracle for the backward pass of the P-cast attention (the reference of fp8attn_bwd).

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle``).

The pages describe only the forward pass.  The backward pass here is the
recomputation form of "Attenzione flash e domanda sulla lunghezza della
sequenza" (FlashAttention keeps only O and the log-sum-exp and recomputes P
from them), with the P-cast of "P-Cast Precision in FP8 Attention",
technical summary, section 1, applied where the forward applies it: to the
probabilities that multiply V.  Readings, each stated where it is used:

  * P is recomputed from the saved log-sum-exp: P_ij = exp(s_ij - lse_i),
    s_ij = q_i . k_j / sqrt(d), masked keys 0.
  * dV uses the cast probabilities, as the forward's P V product does:
    dV_j = sum_i E4M3(P_ij S) / S * dO_i.
  * The softmax gradient uses the unquantised P (the cast is taken as the
    identity for differentiation): dP_ij = dO_i . v_j, D_i = dO_i . O_i,
    dS_ij = P_ij (dP_ij - D_i), dQ_i = sum_j dS_ij k_j / sqrt(d),
    dK_j = sum_i dS_ij q_i / sqrt(d).
With cast=False this is the exact gradient of softmax attention, which the
tests check against automatic differentiation.  Everything is float64.
"""
from __future__ import annotations

import numpy as np

from . import _values, e4m3_round


def backward(q, k, v, o, lse, do, *, causal: bool, p_scale: float, cast: bool = True):
    """Gradients (dq, dk, dv) of the P-cast attention for q [B,H,N,d], k, v [B,Hkv,N,d].

    o and lse are the forward outputs ([B,H,N,d], [B,H,N], lse in logit
    units); do is the output gradient [B,H,N,d].  dk and dv sum over the
    query heads sharing a kv head.
    """
    qf = _values(q).astype(np.float64)
    kf = _values(k).astype(np.float64)
    vf = _values(v).astype(np.float64)
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, H, N, d = qf.shape
    Hkv = kf.shape[1]
    rep = H // Hkv
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    scale = 1.0 / np.sqrt(d)
    mask = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)
    for b in range(B):
        for h in range(H):
            hk = h // rep
            s = qf[b, h] @ kf[b, hk].T * scale
            p = np.where(mask, np.exp(np.where(mask, s, 0.0) - lse[b, h][:, None]), 0.0)
            if cast:
                # the cast value of the forward's P V product, rescaled by 1/S
                p_hat = e4m3_round((p * p_scale).astype(np.float32)).astype(np.float64) / p_scale
            else:
                p_hat = p
            dv[b, hk] += p_hat.T @ do[b, h]
            dp = do[b, h] @ vf[b, hk].T
            dd = np.sum(do[b, h] * o[b, h], axis=1)
            ds = p * (dp - dd[:, None])
            dq[b, h] = ds @ kf[b, hk] * scale
            dk[b, hk] += ds.T @ qf[b, h] * scale
    return dq, dk, dv
