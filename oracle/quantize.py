"""Oracle for the quantisation step in front of the attention path.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle``): the test suite, the
smoke check and the benchmark's CPU legs may use it; the product path never
does.

The step: Q, K and V arrive in a wider format (bfloat16 or float32) and are
cast to E4M3 with a descale factor per block, optionally after an
"incoherent processing" rotation by a random orthogonal matrix -- a Hadamard
matrix with random column signs -- that spreads outlier channels over all
head dimensions before the cast ("Attenzione flash e domanda sulla lunghezza
della sequenza", section "FA3: Meccanica della tramoggia", point 3: block
quantisation after a random rotation of the vectors).  Q and K are rotated by the
same matrix R, so Q R (K R)^T = Q K^T; V is rotated too and the output is
rotated back: O = softmax(..) (V R) R^T.

Readings taken where the page is silent (each is stated where it is used):
  * R = diag(signs) H_d / sqrt(d), H_d the Sylvester Hadamard matrix, signs a
    given +-1 vector (an input, drawn by the seeded generator in
    ``synthetic``).
  * A block's descale is the smallest power of two s >= 2^-126 with
    max|x| <= 448 s (448 = largest E4M3 value), so x / s is exact and never
    saturates, and s * E4M3(x / s) is exact in float32.
  * Q and K are scaled per block of 128 rows of one (batch, head) -- the
    query and key tiles of the forward kernel -- and V per (batch, head),
    because a per-tile V scale could not be divided out of the accumulated
    P V products.
  * The rotation is taken from its definition, x R as a float64 matrix
    product (``rotate_fp64``), and the block maxima, descales and casts are
    decided on those float64 values.  An implementation that evaluates R in
    float32 (any fast transform) lands within a bounded distance of them, so
    a comparison with it has to allow the neighbouring code exactly where a
    float64 value lies within that bound of a rounding boundary; the tests
    derive the bound and count those elements.
"""
from __future__ import annotations

import numpy as np

from . import e4m3_decode, e4m3_encode_f64

E4M3_MAX = 448.0


def _check_signs(signs, d: int) -> np.ndarray:
    s = np.asarray(signs, dtype=np.float32).reshape(-1)
    if s.size != d or not np.all(np.abs(s) == 1.0):
        raise ValueError(f"signs must be {d} values of +-1")
    return s


def hadamard_fp64(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_d (d a power of two), entries +-1, in float64."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def rotate_fp64(x, signs) -> np.ndarray:
    """Definition of the rotation: x R with R = diag(signs) H_d / sqrt(d), in float64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    s = _check_signs(signs, d).astype(np.float64)
    return (x * s) @ hadamard_fp64(d) / np.sqrt(d)


def unrotate_fp64(y, signs) -> np.ndarray:
    """Definition of the inverse rotation: y R^T = (y H_d / sqrt(d)) * signs, in float64."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    s = _check_signs(signs, d).astype(np.float64)
    return (y @ hadamard_fp64(d) / np.sqrt(d)) * s


def block_scale(amax) -> np.ndarray:
    """Smallest power of two s >= 2^-126 with amax <= 448 s (1 where amax is 0), as float32.

    Exact rule on the binary exponent: with amax = m 2^E, m in [1, 2), and
    448 = 1.75 2^8, s = 2^(E - 8) when m <= 1.75, else 2^(E - 7).  The floor
    2^-126 (reading: the page gives no range) keeps s and 1/s float32 normals.
    """
    a = np.asarray(amax, dtype=np.float64)
    if np.any(~np.isfinite(a)) or np.any(a < 0):
        raise ValueError("amax must be finite and >= 0")
    m, e = np.frexp(a)             # a = m 2^e, m in [0.5, 1)
    mant, E = 2.0 * m, e - 1       # a = mant 2^E, mant in [1, 2)
    exp = np.maximum(np.where(mant <= 1.75, E - 8, E - 7), -126)
    s = np.where(a > 0, np.ldexp(1.0, exp), 1.0)
    return s.astype(np.float32)


def quantize_blocks(x, block_rows: int, signs=None):
    """Cast [Z, N, d] values to E4M3 codes with one power-of-two scale per block of rows.

    x is taken as float32 values (bfloat16 inputs are exact in float32) and
    carried in float64.  When ``signs`` is given each row is rotated first,
    by the definition (``rotate_fp64``).  Blocks are ``block_rows``
    consecutive rows of one slab z (the last one ragged); ``block_rows = 0``
    means one block per slab.  A block's maximum, its descale and every
    code are decided on the float64 values.  Returns (codes uint8
    [Z, N, d], scales float32 [Z, nblocks]) with x_rot ~= decode(codes) * scale.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if x.ndim != 3:
        raise ValueError("x must be [Z, N, d]")
    Z, N, d = x.shape
    if signs is not None:
        x = rotate_fp64(x, signs)
    br = N if block_rows == 0 else int(block_rows)
    if br <= 0:
        raise ValueError("block_rows must be >= 0")
    nb = max(1, -(-N // br))
    scales = np.ones((Z, nb), dtype=np.float32)
    codes = np.zeros((Z, N, d), dtype=np.uint8)
    for b in range(nb):
        blk = x[:, b * br:(b + 1) * br, :]
        if blk.shape[1] == 0:
            continue
        amax = np.abs(blk).reshape(Z, -1).max(axis=1)
        s = block_scale(amax)
        scales[:, b] = s
        codes[:, b * br:(b + 1) * br, :] = e4m3_encode_f64(blk / s.astype(np.float64)[:, None, None])
    return codes, scales


def dequantize_blocks(codes, scales, block_rows: int) -> np.ndarray:
    """decode(codes) * scale per block, in float32 (exact: the scales are powers of two)."""
    codes = np.asarray(codes)
    Z, N, d = codes.shape
    br = N if block_rows == 0 else int(block_rows)
    s = np.repeat(np.asarray(scales, dtype=np.float32), br, axis=1)[:, :N]
    return e4m3_decode(codes) * s[:, :, None]


def quantized_attention(q, k, v, signs, *, causal: bool, p_scale: float, reverse: bool,
                        block_n: int = 128, rows=None, n_sink: int = 4):
    """The whole quantised path on float32 inputs q [B,H,N,d], k, v [B,Hkv,N,d].

    Steps (each as defined above): rotate Q, K, V by R when ``signs`` is
    given; cast Q and K with a scale per 128-row block and V with a scale per
    (batch, head); run the blockwise P-cast attention of the emulator on the
    dequantised values (exact: the scales are powers of two); rotate the
    output back by R^T (float64 definition) and round it to bfloat16
    (through float32).  Returns a dict with
    o (float32 values of the bfloat16 output, [B,H,R,d]), lse, the emulator
    result in the rotated frame and the codes and scales of Q, K and V.
    """
    from . import bf16_bits_to_float, bf16_round_bits, emulate

    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    v = np.asarray(v, dtype=np.float32)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    qc, qs = quantize_blocks(q.reshape(B * H, N, d), 128, signs)
    kc, ks = quantize_blocks(k.reshape(B * Hkv, N, d), 128, signs)
    vc, vs = quantize_blocks(v.reshape(B * Hkv, N, d), 0, signs)
    qd = dequantize_blocks(qc, qs, 128).reshape(B, H, N, d)
    kd = dequantize_blocks(kc, ks, 128).reshape(B, Hkv, N, d)
    vd = dequantize_blocks(vc, vs, 0).reshape(B, Hkv, N, d)
    res = emulate(qd, kd, vd, causal=causal, block_n=block_n, p_scale=p_scale, reverse=reverse,
                  n_sink=n_sink, rows=rows)
    o32 = res.o_f32 if signs is None else unrotate_fp64(res.o_f32, signs).astype(np.float32)
    o = bf16_bits_to_float(bf16_round_bits(o32))
    return {"o": o, "lse": res.lse, "rotated": res,
            "q": (qc.reshape(B, H, N, d), qs), "k": (kc.reshape(B, Hkv, N, d), ks),
            "v": (vc.reshape(B, Hkv, N, d), vs)}
