"""The backward parity bounds (tests/backward_bounds.py) are attainable and sharp.

A CPU model of the kernels' arithmetic (float32 logits and exponentials,
E4M3(P S) from the float32 P, bfloat16 dS, float32 accumulation) must lie
inside the bounds around the float64 oracle; the same model with one planted
mistake must not:
  * the sign of dS flipped;
  * dV without the division by S;
  * dQ without the 1/sqrt(d) factor;
  * dK missing one query head of its group;
  * dV from the unquantised P (the P-cast dropped), which the dV bound must
    be narrow enough to see.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as Bw
import synthetic
from backward_bounds import error_bounds, violations


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _kernel_model(q, k, v, o, lse, do, *, causal, p_scale, plant=None):
    qf, kf, vf = (oracle.e4m3_decode(x).astype(np.float32) for x in (q, k, v))
    o = np.asarray(o, dtype=np.float32)
    do = np.asarray(do, dtype=np.float32)
    B, H, N, d = qf.shape
    Hkv = kf.shape[1]
    rep = H // Hkv
    c = np.float32(1.4426950408889634 / np.sqrt(d))
    inv = np.float32(1.0 / np.sqrt(d))
    S = np.float32(p_scale)
    mask = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)
    dq, dk, dv = np.zeros_like(qf), np.zeros_like(kf), np.zeros_like(vf)
    delta = np.sum(do * o, axis=-1, dtype=np.float32)
    for b in range(B):
        for h in range(H):
            hk = h // rep
            s = qf[b, h] @ kf[b, hk].T
            x = s * c - (np.asarray(lse[b, h], dtype=np.float32) * np.float32(1.4426950408889634))[:, None]
            p = np.where(mask, np.exp2(x), np.float32(0.0)).astype(np.float32)
            ph = p if plant == "no_cast" else oracle.e4m3_round(p * S).astype(np.float32)
            dp = do[b, h] @ vf[b, hk].T
            ds = _bf16(p * (dp - delta[b, h][:, None]))
            if plant == "ds_sign":
                ds = -ds
            if plant == "no_cast":
                dv[b, hk] += ph.T @ do[b, h]
            else:
                dv[b, hk] += (ph.T @ do[b, h]) / (np.float32(1.0) if plant == "dv_no_div" else S)
            dq[b, h] = (ds @ kf[b, hk]) * (np.float32(1.0) if plant == "dq_no_scale" else inv)
            if not (plant == "dk_drop_head" and h % rep == rep - 1):
                dk[b, hk] += (ds.T @ qf[b, h]) * inv
    return dq, dk, dv, delta


def _setup(B, H, Hkv, N, causal, S, delta, seed):
    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, 128, delta, seed=seed)
    fwd = oracle.emulate(q, k, v, causal=causal, block_n=128, p_scale=S, reverse=True)
    o = oracle.bf16_bits_to_float(fwd.o_bf16)
    do = synthetic.make_output_grad((B, H, N, 128), seed + 1)
    ref = Bw.backward(q, k, v, o, fwd.lse, do, causal=causal, p_scale=S)
    d_ref = np.sum(do.astype(np.float64) * o.astype(np.float64), axis=-1)
    bounds = error_bounds(q, k, v, o, fwd.lse, do, causal=causal, p_scale=S)
    return (q, k, v, o, fwd.lse, do), ref + (d_ref,), bounds


CASES = [
    (1, 4, 2, 300, True, 256.0, 5.0, 61),
    (1, 2, 2, 300, False, 256.0, 5.0, 62),
    (2, 2, 1, 256, True, 448.0, 7.0, 63),
    (1, 2, 1, 200, True, 1.0, 7.0, 64),
    (1, 1, 1, 5, True, 256.0, 5.0, 65),
]


@pytest.mark.parametrize("case", CASES)
def test_kernel_arithmetic_is_inside_the_bounds(case):
    B, H, Hkv, N, causal, S, delta, seed = case
    args, ref, bounds = _setup(B, H, Hkv, N, causal, S, delta, seed)
    got = _kernel_model(*args, causal=causal, p_scale=S)
    for name, g, r, bd in zip(("dq", "dk", "dv", "delta"), got, ref, bounds):
        n, worst = violations(g, r, bd)
        assert n == 0, f"{name}: {n} elements outside the bound (worst ratio {worst:.3g})"


@pytest.mark.parametrize("plant,which", [("ds_sign", 0), ("dv_no_div", 2), ("dq_no_scale", 0),
                                         ("dk_drop_head", 1), ("no_cast", 2)])
def test_planted_mistakes_break_the_bounds(plant, which):
    B, H, Hkv, N, causal, S, delta, seed = CASES[0]
    args, ref, bounds = _setup(B, H, Hkv, N, causal, S, delta, seed)
    got = _kernel_model(*args, causal=causal, p_scale=S, plant=plant)
    n, worst = violations(got[which], ref[which], bounds[which])
    assert n > 0 and worst > 4.0, (plant, n, worst)
