"""Comparison of E4M3 codes and descales computed through a float32 rotation
(the quantisation kernel) with the oracle's, which takes the rotation from its
float64 definition (oracle.quantize).

A float32 evaluation of y = x R, R = diag(signs) H_d / sqrt(d), by any radix-2
fast Walsh-Hadamard transform forms every output as a sum of the d signed
inputs over a binary tree of depth L = log2(d), one rounding per add, then one
multiply by float32(1/sqrt(d)) (itself within half an ulp of 1/sqrt(d)).  The
standard error analysis of such a sum gives, for output i,

    |y_f32_i - y_i| <= ((1 + u)^(L + 2) - 1) * sum_j |x_j| / sqrt(d),   u = 2^-24,

whatever the order of the stages.  The float64 reference carries its own
error, bounded the same way with u = 2^-53 and depth d (a plain matrix
product); both are added.  From that bound:

  * a block's maximum moves by at most the largest bound in the block, so its
    descale may be the neighbouring power of two only when the float64 maximum
    lies that close to a boundary 448 * 2^e;
  * rounding is monotone, so a code's value must lie between the E4M3
    roundings of the two ends of the interval of possible float32 values;
    where both ends round alike (the float64 value is not that close to a
    rounding boundary) the code is fixed.  Values, not bytes, are compared,
    so +0 and -0 are the same code here.

``compare_codes`` checks exactly that and returns how many elements were
ambiguous, so that a test can also require them to be rare.
"""
from __future__ import annotations

import numpy as np

import oracle
from oracle import quantize as Qz


def rotation_error_bound(x, rotate: bool) -> np.ndarray:
    """Per-element bound on |float32 rotation - exact rotation| for rows x [..., d] (float32 values).

    Without rotation the values are used as they are (bound 0)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    d = x.shape[-1]
    if not rotate:
        return np.zeros(x.shape)
    L = int(round(np.log2(d)))
    l1 = np.abs(x).sum(axis=-1, keepdims=True) / np.sqrt(d)
    g32 = (1.0 + 2.0 ** -24) ** (L + 2) - 1.0
    g64 = (1.0 + 2.0 ** -53) ** (d + 2) - 1.0
    return np.broadcast_to((g32 + g64) * l1, x.shape) * (1.0 + 1e-12)


def compare_codes(x, block_rows: int, signs, codes_got, scales_got):
    """Check codes/scales of x [Z, N, d] against the oracle with the allowance above.

    Returns (n_ambiguous_elements, n_ambiguous_blocks, n_code_mismatches,
    n_scale_mismatches): mismatches are disagreements outside the allowance
    (zero for a correct implementation)."""
    x = np.asarray(x, dtype=np.float32)
    Z, N, d = x.shape
    codes_got = np.asarray(codes_got, dtype=np.uint8)
    scales_got = np.asarray(scales_got, dtype=np.float32)
    y = x.astype(np.float64) if signs is None else Qz.rotate_fp64(x, signs)
    beta = rotation_error_bound(x, signs is not None)
    br = N if block_rows == 0 else int(block_rows)
    nb = max(1, -(-N // br))
    if scales_got.shape != (Z, nb) or codes_got.shape != (Z, N, d):
        raise ValueError("shape mismatch")
    amb_el = amb_blk = bad_codes = bad_scales = 0
    for b in range(nb):
        sl = slice(b * br, (b + 1) * br)
        yb, bb = y[:, sl], beta[:, sl]
        if yb.shape[1] == 0:
            continue
        amax = np.abs(yb).reshape(Z, -1).max(axis=1)
        bmax = bb.reshape(Z, -1).max(axis=1)
        s_lo = Qz.block_scale(np.maximum(amax - bmax, 0.0))
        s_hi = Qz.block_scale(amax + bmax)
        s_got = scales_got[:, b]
        ok_s = (s_got == s_lo) | (s_got == s_hi)
        bad_scales += int((~ok_s).sum())
        amb_blk += int((s_lo != s_hi).sum())
        s = s_got.astype(np.float64)[:, None, None]
        lo = oracle.e4m3_decode(oracle.e4m3_encode_f64((yb - bb) / s))
        hi = oracle.e4m3_decode(oracle.e4m3_encode_f64((yb + bb) / s))
        got = oracle.e4m3_decode(codes_got[:, sl])
        amb_el += int((lo != hi).sum())
        bad_codes += int(((got < lo) | (got > hi) | np.isnan(got)).sum())
    return amb_el, amb_blk, bad_codes, bad_scales
