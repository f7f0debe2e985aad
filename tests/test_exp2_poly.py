"""The polynomial exponential the kernels use for part of the exp2 work:
its constants in sm100_ptx.cuh are the float32 Remez fit that
gen_exp2_poly.py reproduces, and its relative error (a few 1e-6) stays far
below what an E4M3 cast (3 mantissa bits) or a float32 row sum would notice,
over the whole range of arguments the kernel passes."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "softmax_cast_precision_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def header_coefficients():
    text = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    body = text[text.index("exp2_poly2"):text.index("ex2_approx")]
    vals = [float.fromhex(h) for h in re.findall(r"(0x1\.[0-9a-f]+p[-+]\d+)f", body)]
    # Horner order in the source: highest degree first (each literal appears twice)
    uniq = []
    for v in vals:
        if not uniq or uniq[-1] != v:
            uniq.append(v)
    return np.array(uniq[::-1], dtype=np.float32)


def test_header_constants_are_the_fit():
    gen = _gen()
    c = gen.coefficients_f32()
    assert np.array_equal(header_coefficients(), c)


def test_polynomial_error_bound():
    gen = _gen()
    c = header_coefficients()
    assert gen.max_rel_error_f32(c) < 3e-6


def test_full_reduction_matches_exp2():
    # Emulate the kernel's reduction in float32: j = round(x), f = x - j,
    # 2^f by Horner, 2^j by exponent add; compare with exact 2^x.
    c = header_coefficients()
    # Arguments are x - m + log2(S): at most log2(S) <= 64.
    x = np.concatenate([np.linspace(-125, 64, 300001), -np.logspace(-8, 2, 20001),
                        np.logspace(-8, 1.8, 20001)]).astype(np.float32)
    xr = np.maximum(x, np.float32(-125.0))
    t = (xr + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (xr - j).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    q = np.full_like(f, c[-1])
    for ci in c[-2::-1]:
        q = (q * f + ci).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    y = bits.view(np.float32).astype(np.float64)
    ref = 2.0 ** x.astype(np.float64)
    assert np.max(np.abs(y / ref - 1.0)) < 3.2e-6
