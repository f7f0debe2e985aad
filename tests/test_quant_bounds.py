"""CPU check of the code comparison in quant_bounds (used by the GPU tests of
the quantisation kernel), in both directions:

  * a numpy model of a float32 fast-transform quantiser -- radix-2 stages in
    either order, one multiply by float32(1/sqrt(d)), float32 block maxima,
    the descale rule and round-to-nearest-even casts -- lies inside the
    allowance, with ambiguous elements present but rare;
  * its float32 transform lies inside the error bound the allowance uses;
  * planted mistakes (a swapped butterfly sign, a descale off by one power of
    two, a missing sign flip, a transposed index) fall far outside it.
"""
import numpy as np
import pytest

import oracle
from oracle import quantize as Qz
import synthetic
from quant_bounds import compare_codes, rotation_error_bound


def _fwht_f32(x, stage_order="up", swap_sign=False):
    y = np.array(x, dtype=np.float32, copy=True)
    d = y.shape[-1]
    lead = y.shape[:-1]
    hs = [1 << i for i in range(int(np.log2(d)))]
    if stage_order == "down":
        hs = hs[::-1]
    for h in hs:
        z = y.reshape(*lead, d // (2 * h), 2, h)
        a = z[..., 0, :].copy()
        b = z[..., 1, :].copy()
        z[..., 0, :] = (a - b) if swap_sign else (a + b)
        z[..., 1, :] = (a + b) if swap_sign else (a - b)
        y = z.reshape(*lead, d)
    return y


def _model(x, block_rows, signs, stage_order="up", mistake=None):
    """float32 quantiser model: returns (codes, scales)."""
    x = np.asarray(x, dtype=np.float32)
    Z, N, d = x.shape
    if signs is not None:
        sg = np.asarray(signs, dtype=np.float32)
        if mistake == "no_signs":
            sg = np.ones_like(sg)
        xin = x * sg
        if mistake == "transpose_index":
            xin = xin[..., ::-1]
        y = _fwht_f32(xin, stage_order, swap_sign=(mistake == "swap_sign")) * np.float32(1.0 / np.sqrt(d))
    else:
        y = x
    br = N if block_rows == 0 else block_rows
    nb = max(1, -(-N // br))
    scales = np.ones((Z, nb), dtype=np.float32)
    codes = np.zeros((Z, N, d), dtype=np.uint8)
    for b in range(nb):
        blk = y[:, b * br:(b + 1) * br]
        amax = np.abs(blk).reshape(Z, -1).max(axis=1)
        s = Qz.block_scale(amax.astype(np.float64))
        if mistake == "descale_off":
            s = s * np.float32(2.0)
        scales[:, b] = s
        codes[:, b * br:(b + 1) * br] = oracle.e4m3_encode(blk / s[:, None, None])
    return codes, scales


def _inputs(d, seed, Z=4, N=300):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((Z, N, d)) * np.exp(rng.uniform(-4, 4, (Z, 1, 1)))).astype(np.float32)
    x[:, :, 3] *= 30.0
    return x


@pytest.mark.parametrize("d", [64, 128])
def test_float32_transform_inside_bound(d):
    x = _inputs(d, 1)
    s = synthetic.hadamard_signs(d, 2)
    exact = Qz.rotate_fp64(x, s)
    bound = rotation_error_bound(x, True)
    for order in ("up", "down"):
        y32 = (_fwht_f32(x * s, order) * np.float32(1.0 / np.sqrt(d))).astype(np.float64)
        err = np.abs(y32 - exact)
        assert np.all(err <= bound)
        assert err.max() > 0.02 * bound.max()  # the bound is not vacuous
    bad = (_fwht_f32(x * s, "up", swap_sign=True) * np.float32(1.0 / np.sqrt(d))).astype(np.float64)
    assert np.abs(bad - exact).max() > 1e4 * bound.max()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block_rows", [128, 37, 0])
@pytest.mark.parametrize("order", ["up", "down"])
def test_float32_model_passes(d, block_rows, order):
    x = _inputs(d, 3 + block_rows)
    s = synthetic.hadamard_signs(d, 4)
    codes, scales = _model(x, block_rows, s, order)
    amb, amb_blk, bad_c, bad_s = compare_codes(x, block_rows, s, codes, scales)
    assert bad_c == 0 and bad_s == 0
    assert amb < 1e-3 * x.size  # ambiguity is rare
    # without rotation nothing is ambiguous: the codes are fixed
    codes0, scales0 = _model(x, block_rows, None)
    assert compare_codes(x, block_rows, None, codes0, scales0) == (0, 0, 0, 0)


def test_ambiguous_elements_occur_and_are_accepted():
    # enough elements that some float32 values land on the other side of a
    # rounding boundary than the float64 value; the allowance must cover them
    d = 128
    x = _inputs(d, 9, Z=8, N=1024)
    s = synthetic.hadamard_signs(d, 10)
    codes, scales = _model(x, 128, s)
    ref_codes, ref_scales = Qz.quantize_blocks(x, 128, s)
    differ = int((oracle.e4m3_decode(codes) != oracle.e4m3_decode(ref_codes)).sum())
    amb, _, bad_c, bad_s = compare_codes(x, 128, s, codes, scales)
    assert bad_c == 0 and bad_s == 0
    assert amb >= differ
    assert amb > 0


@pytest.mark.parametrize("mistake", ["swap_sign", "descale_off", "no_signs", "transpose_index"])
def test_planted_mistakes_fail(mistake):
    d = 128
    x = _inputs(d, 11)
    s = synthetic.hadamard_signs(d, 12)
    codes, scales = _model(x, 128, s, mistake=mistake)
    _, _, bad_c, bad_s = compare_codes(x, 128, s, codes, scales)
    assert bad_c > 0.1 * x.size or bad_s > 0
