"""Pins of the quantisation-step oracle (oracle.quantize) against facts fixed by
the mathematics, independent of its own formulas:

  * the Hadamard matrix against SciPy's, and H H^T = d I;
  * R orthogonal: rotate then unrotate is the identity; a one-hot vector
    becomes flat (every |component| = 1/sqrt(d)), and its codes follow in
    closed form: all of magnitude 448 at the right scale, with the signs of
    the signs vector times a row of H (a swapped index, sign or transpose
    changes them);
  * attention is invariant: rotating Q, K and V and rotating the output back
    gives the same output as unrotated attention;
  * the block scale: a power of two with amax/scale in (224, 448], exact at
    the boundaries amax = 448 * 2^e;
  * the cast: every dequantised value within half an E4M3 step of the input;
  * the page's claim, as a direction: with outlier channels, rotation before
    the cast lowers the output error ("Attenzione flash e domanda sulla
    lunghezza della sequenza", section "FA3: Meccanica della tramoggia",
    point 3).
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle import quantize as Qz
import synthetic


@pytest.mark.parametrize("d", [2, 8, 64, 128])
def test_hadamard_matrix(d):
    h = Qz.hadamard_fp64(d)
    assert np.array_equal(h, scipy.linalg.hadamard(d).astype(np.float64))
    assert np.array_equal(h @ h.T, d * np.eye(d))


@pytest.mark.parametrize("d", [64, 128])
def test_rotation_is_orthogonal(d):
    rng = np.random.default_rng(2)
    s = synthetic.hadamard_signs(d, 7)
    x = rng.standard_normal((20, d))
    y = Qz.rotate_fp64(x, s)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    assert np.allclose(Qz.unrotate_fp64(y, s), x, atol=1e-12)


def test_one_hot_becomes_flat():
    d = 128
    s = synthetic.hadamard_signs(d, 3)
    for i in (0, 5, 127):
        e = np.zeros(d, dtype=np.float32)
        e[i] = 1.0
        y = Qz.rotate_fp64(e, s)
        assert np.allclose(np.abs(y), 1.0 / np.sqrt(d), atol=1e-15)


@pytest.mark.parametrize("d", [64, 128])
def test_one_hot_codes_closed_form(d):
    # x = 256 sqrt(d) e_i (float32): the rotated row is 256 * signs[i] * H[i, :]
    # up to float32 rounding of sqrt(d), so the block scale is 1 and every code
    # is +-256 (0x78 / 0xF8) with the sign of signs[i] * H[i, j] (Sylvester:
    # H[i, j] = (-1)^popcount(i & j)).
    s = synthetic.hadamard_signs(d, 5)
    for i in (0, 1, d // 2 + 3, d - 1):
        x = np.zeros((1, 4, d), dtype=np.float32)
        x[0, 2, i] = np.float32(256.0 * np.sqrt(d))
        codes, scales = Qz.quantize_blocks(x, 0, s)
        assert scales[0, 0] == 1.0
        want = np.array([0x78 if s[i] * (-1) ** bin(i & j).count("1") > 0 else 0xF8 for j in range(d)],
                        dtype=np.uint8)
        assert np.array_equal(codes[0, 2], want)
        assert np.all(oracle.e4m3_decode(codes[0, [0, 1, 3]]) == 0.0)


def test_attention_is_rotation_invariant():
    rng = np.random.default_rng(4)
    B, H, Hkv, N, d = 1, 2, 1, 70, 64
    q = rng.standard_normal((B, H, N, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    s = synthetic.hadamard_signs(d, 9)
    o_ref, lse_ref = oracle.attention_fp64(q, k, v, causal=True)
    qr, kr, vr = (Qz.rotate_fp64(x, s).astype(np.float32) for x in (q, k, v))
    o_rot, lse_rot = oracle.attention_fp64(qr, kr, vr, causal=True)
    assert np.allclose(Qz.unrotate_fp64(o_rot, s), o_ref, atol=2e-6)
    assert np.allclose(lse_rot, lse_ref, atol=2e-6)


def test_block_scale_rule():
    for e in range(-20, 21):
        a = 448.0 * 2.0 ** e
        assert Qz.block_scale(a) == np.float32(2.0 ** e)
        assert Qz.block_scale(np.nextafter(a, np.inf)) == np.float32(2.0 ** (e + 1))
        assert Qz.block_scale(np.nextafter(a, 0)) == np.float32(2.0 ** e)
    assert Qz.block_scale(0.0) == 1.0
    # the floor: tiny blocks get 2^-126, and then amax / s < 224
    assert Qz.block_scale(448.0 * 2.0 ** -127) == np.float32(2.0 ** -126)
    assert Qz.block_scale(1e-40) == np.float32(2.0 ** -126)
    rng = np.random.default_rng(5)
    amax = np.exp(rng.uniform(-30, 30, 10000))
    s = Qz.block_scale(amax).astype(np.float64)
    assert np.all(np.log2(s) == np.round(np.log2(s)))
    r = amax / s
    assert np.all((r > 224.0) & (r <= 448.0))
    with pytest.raises(ValueError):
        Qz.block_scale(-1.0)


@pytest.mark.parametrize("block_rows", [128, 0])
def test_cast_within_half_step(block_rows):
    rng = np.random.default_rng(6)
    Z, N, d = 3, 300, 128
    x = (rng.standard_normal((Z, N, d)) * np.exp(rng.uniform(-5, 5, (Z, 1, 1)))).astype(np.float32)
    x[1, 128:256] = 0.0  # an all-zero block
    codes, scales = Qz.quantize_blocks(x, block_rows)
    nb = 3 if block_rows else 1
    assert scales.shape == (Z, nb)
    deq = Qz.dequantize_blocks(codes, scales, block_rows)
    br = block_rows or N
    for z in range(Z):
        for b in range(nb):
            blk = x[z, b * br:(b + 1) * br]
            s = float(scales[z, b])
            amax = float(np.abs(blk).max())
            if amax == 0.0:
                assert s == 1.0 and np.all(codes[z, b * br:(b + 1) * br] == 0)
                continue
            assert 224.0 < amax / s <= 448.0
            y = blk.astype(np.float64) / s
            err = np.abs(deq[z, b * br:(b + 1) * br].astype(np.float64) / s - y)
            # half an E4M3 step: 2^(floor(log2|y|) - 4) for normals, 2^-10 below 2^-6
            half = np.where(np.abs(y) >= 2.0 ** -6,
                            2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-300))) - 4), 2.0 ** -10)
            assert np.all(err <= half * (1 + 1e-12))
            # the largest value keeps its magnitude (no saturation, no collapse)
            assert np.abs(deq[z, b * br:(b + 1) * br]).max() >= amax * (1 - 2 ** -4)


def test_rotation_helps_with_outlier_channels():
    B, H, Hkv, N, d = 1, 2, 2, 512, 128
    q, k, v, _ = synthetic.make_wide_inputs(B, H, Hkv, N, d, 3.0, seed=11, outliers=4, outlier_gain=40.0)
    rows = np.arange(0, N, 8)
    o_ref, _ = oracle.attention_fp64(q, k, v, causal=True, rows=rows)
    s = synthetic.hadamard_signs(d, 12)
    plain = Qz.quantized_attention(q, k, v, None, causal=True, p_scale=256.0, reverse=True, rows=rows)
    rot = Qz.quantized_attention(q, k, v, s, causal=True, p_scale=256.0, reverse=True, rows=rows)
    e_plain = np.sqrt(np.mean((plain["o"] - o_ref) ** 2))
    e_rot = np.sqrt(np.mean((rot["o"] - o_ref) ** 2))
    assert e_rot < e_plain / 1.5, (e_plain, e_rot)


def test_quantized_path_without_rotation_is_plain_emulation_of_the_casts():
    # With unit-variance inputs the cast of a block is x -> s * E4M3(x / s); the
    # pipeline must equal the emulator run on exactly those values.
    B, H, Hkv, N, d = 1, 1, 1, 200, 64
    q, k, v, _ = synthetic.make_wide_inputs(B, H, Hkv, N, d, 5.0, seed=13)
    res = Qz.quantized_attention(q, k, v, None, causal=False, p_scale=256.0, reverse=False, block_n=64)
    qd = Qz.dequantize_blocks(res["q"][0].reshape(1, N, d), res["q"][1], 128).reshape(q.shape)
    kd = Qz.dequantize_blocks(res["k"][0].reshape(1, N, d), res["k"][1], 128).reshape(k.shape)
    vd = Qz.dequantize_blocks(res["v"][0].reshape(1, N, d), res["v"][1], 0).reshape(v.shape)
    direct = oracle.emulate(qd, kd, vd, causal=False, block_n=64, p_scale=256.0, reverse=False)
    assert np.array_equal(direct.o, res["o"])
    # and the dequantised values are the cast values themselves
    s_q = float(res["q"][1][0, 0])
    assert np.array_equal(qd[0, 0, :128] / s_q, oracle.e4m3_round(q[0, 0, :128] / s_q))
