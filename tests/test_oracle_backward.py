"""Pins of the backward-pass oracle (oracle.backward), the reference of the
backward kernels (fp8attn_bwd):

  * without the cast it is the exact gradient of softmax attention: it must
    equal PyTorch's automatic differentiation in float64 (causal and not,
    grouped-query heads);
  * the cast touches only dV (the reading stated in the module), so dQ and dK
    are those of the uncast gradient;
  * with the cast, dV stays within the sum of half E4M3 steps of P S / S times
    |dO| of the exact dV, element by element.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as Bw
import synthetic


def _exact(q, k, v, do, causal):
    """Forward and gradients of exact attention with torch autograd (float64)."""
    B, H, N, d = q.shape
    rep = H // k.shape[1]
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    kr, vr = kt.repeat_interleave(rep, 1), vt.repeat_interleave(rep, 1)
    s = qt @ kr.transpose(-1, -2) / math.sqrt(d)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    lse = torch.logsumexp(s, -1)
    o = torch.softmax(s, -1) @ vr
    (o * torch.tensor(do)).sum().backward()
    return o.detach().numpy(), lse.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def _inputs(B, H, Hkv, N, seed):
    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, 64, 5.0, seed=seed)
    qf, kf, vf = (oracle.e4m3_decode(x).astype(np.float64) for x in (q, k, v))
    do = np.random.default_rng(seed).standard_normal(qf.shape)
    return q, k, v, qf, kf, vf, do


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 2)])
def test_uncast_backward_is_autograd(causal, H, Hkv):
    q, k, v, qf, kf, vf, do = _inputs(1, H, Hkv, 40, seed=7 + H)
    o, lse, gq, gk, gv = _exact(qf, kf, vf, do, causal)
    dq, dk, dv = Bw.backward(q, k, v, o, lse, do, causal=causal, p_scale=256.0, cast=False)
    for got, ref in ((dq, gq), (dk, gk), (dv, gv)):
        assert np.allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_cast_changes_only_dv():
    q, k, v, qf, kf, vf, do = _inputs(1, 2, 1, 50, seed=11)
    o, lse, *_ = _exact(qf, kf, vf, do, True)
    a = Bw.backward(q, k, v, o, lse, do, causal=True, p_scale=256.0, cast=False)
    b = Bw.backward(q, k, v, o, lse, do, causal=True, p_scale=256.0, cast=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[2], b[2])


@pytest.mark.parametrize("S", [1.0, 256.0, 448.0])
def test_cast_dv_within_half_steps(S):
    q, k, v, qf, kf, vf, do = _inputs(1, 2, 2, 64, seed=13)
    o, lse, *_ = _exact(qf, kf, vf, do, False)
    dq, dk, dv = Bw.backward(q, k, v, o, lse, do, causal=False, p_scale=S, cast=True)
    _, _, dv0 = Bw.backward(q, k, v, o, lse, do, causal=False, p_scale=S, cast=False)
    # P from the exact forward; half an E4M3 step of y = P S (subnormal step below 2^-6)
    for h in range(2):
        s = qf[0, h] @ kf[0, h].T / math.sqrt(64)
        p = np.exp(s - lse[0, h][:, None])
        y = p * S
        half = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 1e-300))) - 4), 2.0 ** -10) / S
        bound = half.T @ np.abs(do[0, h])
        assert np.all(np.abs(dv[0, h] - dv0[0, h]) <= bound * (1 + 1e-9) + 1e-12)
