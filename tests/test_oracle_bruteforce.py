"""Brute-force pins of the oracle on tiny inputs.

  * The blockwise emulator (oracle.emulate, C, float32) against a plain
    Python restatement written element by element in float64: for each row,
    the KV blocks in the given order, the running maximum over every block
    so far ("Attenzione flash e domanda sulla lunghezza della sequenza",
    section "L'algoritmo Flash Attention"), P = exp(s - m), the cast
    E4M3(P S) per element ("P-Cast Precision in FP8 Attention", technical
    summary, section 1), the rescale of what was accumulated when the
    maximum grows, and O = acc / (S l) with l the sum of the unquantised P.
    The two differ by float32 rounding, and where float32 rounding moves P S
    across an E4M3 rounding boundary, by one E4M3 step of that element: the
    allowance counts exactly those elements.
  * The plug-in underflow fraction F(Delta, S) (technical summary, section
    2) against a Monte Carlo count of E4M3 zeros among exp(x - m) S with x
    standard normal and m = Delta + delta_k, rounded by the pinned codec.
"""
import math

import numpy as np
import pytest

import oracle


def _e4m3(x: float) -> float:
    return oracle.e4m3_decode_scalar(oracle.e4m3_encode_scalar(x))


def _bruteforce(qf, kf, vf, causal, block, S, reverse, amb=2.0 ** -18):
    """(O, allowance) for every row, float64 loops."""
    B, H, N, d = qf.shape
    rep = H // kf.shape[1]
    o = np.zeros((B, H, N, d))
    allow = np.zeros((B, H, N, d))
    nblocks = -(-N // block)
    for b in range(B):
        for h in range(H):
            hk = h // rep
            for i in range(N):
                last = min(nblocks - 1, i // block) if causal else nblocks - 1
                order = range(last, -1, -1) if reverse else range(0, last + 1)
                m = -math.inf
                l = 0.0
                acc = [0.0] * d
                amb_acc = [0.0] * d
                for t in order:
                    keys = [j for j in range(t * block, min(N, (t + 1) * block)) if not causal or j <= i]
                    s = {}
                    for j in keys:
                        dot = 0.0
                        for c in range(d):
                            dot += qf[b, h, i, c] * kf[b, hk, j, c]
                        s[j] = dot / math.sqrt(d)
                    m_new = max([m] + list(s.values()))
                    alpha = math.exp(m - m_new) if m > -math.inf else 0.0
                    l *= alpha
                    for c in range(d):
                        acc[c] *= alpha
                        amb_acc[c] *= alpha
                    for j in keys:
                        p = math.exp(s[j] - m_new)
                        l += p
                        ph = _e4m3(p * S)
                        lo, hi = _e4m3(p * S * (1 - amb)), _e4m3(p * S * (1 + amb))
                        for c in range(d):
                            acc[c] += ph * vf[b, hk, j, c]
                            amb_acc[c] += abs(hi - lo) * abs(vf[b, hk, j, c])
                    m = m_new
                for c in range(d):
                    o[b, h, i, c] = acc[c] / (S * l)
                    allow[b, h, i, c] = amb_acc[c] / (S * l)
    return o, allow


def _rand_e4m3(rng, shape, scale=1.0):
    return oracle.e4m3_encode((rng.standard_normal(shape) * scale).astype(np.float32))


@pytest.mark.parametrize("N,causal,reverse,S", [
    (16, False, False, 256.0),   # one block: no rescale
    (16, True, True, 1.0),
    (150, True, False, 256.0),   # three blocks of 64, the last ragged
    (150, True, True, 448.0),
    (150, False, True, 1.0),
    (100, False, False, 512.0),  # S above 448: the largest P saturate
])
def test_emulator_equals_bruteforce(N, causal, reverse, S):
    rng = np.random.default_rng(N + int(S) + 2 * causal + reverse)
    d, H, Hkv, block = 64, 2, 1, 64
    q = _rand_e4m3(rng, (1, H, N, d), 0.6)
    k = _rand_e4m3(rng, (1, Hkv, N, d), 0.6)
    v = _rand_e4m3(rng, (1, Hkv, N, d))
    # Sinks: keys 0..3 share a large component with every query (logit +6), so that the
    # maximum grows at the first block in one order and at the last in the other, and the
    # other probabilities fall into E4M3's subnormal range at small S.
    q[..., 0] = oracle.e4m3_encode_scalar(8.0)
    k[..., 0] = 0
    k[:, :, :4, 0] = oracle.e4m3_encode_scalar(6.0)
    qf, kf, vf = (oracle.e4m3_decode(x).astype(np.float64) for x in (q, k, v))
    ref, allow = _bruteforce(qf, kf, vf, causal, block, S, reverse)
    got = oracle.emulate(q, k, v, causal=causal, block_n=block, p_scale=S, reverse=reverse)
    err = np.abs(got.o_f32.astype(np.float64) - ref)
    tol = allow + 1e-5 * np.abs(vf).max()
    assert np.all(err <= tol), float((err - tol).max())


@pytest.mark.parametrize("delta", [4.0, 5.0, 6.0, 7.0, 8.0])
@pytest.mark.parametrize("S", [1.0, 4.0])
def test_plug_in_fraction_by_monte_carlo(delta, S):
    rng = np.random.default_rng(int(10 * delta + S))
    n = 400_000
    x = rng.standard_normal(n)
    m = delta + oracle.delta_k(4)
    codes = oracle.e4m3_encode((np.exp(x - m) * S).astype(np.float32))
    frac = float(np.mean(codes == 0))
    f = float(oracle.f_forward(delta, S))
    assert abs(frac - f) <= 4.0 * math.sqrt(f * (1 - f) / n) + 2e-4, (frac, f)
