"""The polynomial exponential the kernels use for part of the exp2 work:
its constants in sm100_ptx.cuh are the float32 Remez fit that
gen_exp2_poly.py reproduces, and its error stays at the level of the
hardware approximation (a few float32 ulp) over the whole reduced range."""
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
    # Horner order in the source: c5, c4, c3, c2, c1, c0 (each literal appears twice)
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
    assert gen.max_rel_error_f32(c) < 3e-7


def test_full_reduction_matches_exp2():
    # Emulate the kernel's reduction in float32: j = round(x), f = x - j,
    # 2^f by Horner, 2^j by exponent add; compare with exact 2^x.
    c = header_coefficients()
    x = np.concatenate([np.linspace(-125, 0, 200001), -np.logspace(-8, 2, 20001)]).astype(np.float32)
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
    assert np.max(np.abs(y / ref - 1.0)) < 4e-7
