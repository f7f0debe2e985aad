"""GPU parity of the quantisation path (fp8attn_quantize, fp8attn_fwd_scaled)
against the oracle (oracle.quantize), through the C ABI.

  * Codes and descales: without the rotation both sides cast the same
    float32 values, so they match bit for bit.  With it, the oracle rotates by
    the float64 definition and the kernel by a float32 fast transform; every
    descale and code must then equal the oracle's except where the float64
    value lies within the float32 transform's error bound of a rounding
    boundary, where the neighbour is allowed too (tests/quant_bounds.py; the
    number of such elements is reported and must be rare).
  * The scaled forward pass is compared like the plain one: per element
    max|O_gpu - O_oracle| <= 1e-2 * max|V|, lse within 1e-3.
  * Rotation with outlier channels lowers the error against exact attention
    ("Attenzione flash e domanda sulla lunghezza della sequenza", section
    "FA3: Meccanica della tramoggia", point 3), on the GPU as in the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import quantize as Qz
import synthetic
from quant_bounds import compare_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return fp8attn


def _dev(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).cuda()


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("block_rows", [128, 0, 37])
@pytest.mark.parametrize("rotate", [True, False])
def test_quantize_bit_exact(fp8, d, dtype, block_rows, rotate):
    rng = np.random.default_rng(d + block_rows)
    Z, N = 3, 300
    x = (rng.standard_normal((Z, N, d)) * np.exp(rng.uniform(-4, 4, (Z, 1, 1)))).astype(np.float32)
    x[:, :, 3] *= 30.0  # an outlier channel
    x[1, 128:256] = 0.0
    x = torch.from_numpy(x).to(dtype).float().numpy()  # the values the GPU sees
    signs = synthetic.hadamard_signs(d, 21) if rotate else None
    codes, scales = fp8.quantize(_dev(x, dtype), block_rows, signs)
    torch.cuda.synchronize()
    got, s_got = codes.cpu().numpy(), scales.cpu().numpy()
    if not rotate:
        c_ref, s_ref = Qz.quantize_blocks(x, block_rows, None)
        assert np.array_equal(s_got, s_ref)
        assert np.array_equal(got, c_ref), f"{(got != c_ref).sum()} codes differ"
    amb, amb_blk, bad_codes, bad_scales = compare_codes(x, block_rows, signs, got, s_got)
    assert bad_scales == 0, f"{bad_scales} descales outside the allowance"
    assert bad_codes == 0, f"{bad_codes} codes outside the allowance ({amb} ambiguous)"
    assert amb <= 1e-3 * x.size, f"{amb} ambiguous elements"


def test_quantize_empty_and_tiny(fp8):
    x = torch.zeros((2, 0, 128), dtype=torch.bfloat16, device="cuda")
    codes, scales = fp8.quantize(x, 0)
    assert codes.shape == (2, 0, 128) and torch.equal(scales.cpu(), torch.ones(2, 1))
    x = torch.full((1, 5, 128), 1e-38, dtype=torch.float32, device="cuda")
    codes, scales = fp8.quantize(x, 128)
    c_ref, s_ref = Qz.quantize_blocks(x.cpu().numpy(), 128)
    assert np.array_equal(scales.cpu().numpy(), s_ref) and np.array_equal(codes.cpu().numpy(), c_ref)


def _case(fp8, B, H, Hkv, N, causal, S, order, rotate, outliers=0, delta=7.0, seed=31, rows=None):
    d = 128
    q, k, v, _ = synthetic.make_wide_inputs(B, H, Hkv, N, d, delta, seed=seed, outliers=outliers, outlier_gain=20.0)
    signs = synthetic.hadamard_signs(d, seed + 1) if rotate else None
    o, lse = fp8.fwd_wide(_dev(q, torch.bfloat16), _dev(k, torch.bfloat16), _dev(v, torch.bfloat16), causal=causal,
                          p_scale=S, kv_order=order, signs=signs)
    fp8.check_error()
    ref = Qz.quantized_attention(q, k, v, signs, causal=causal, p_scale=S, reverse=(order == "reverse"), rows=rows)
    rr = np.arange(N) if rows is None else np.asarray(rows)
    o_g = o.float().cpu().numpy()[:, :, rr]
    lse_g = lse.cpu().numpy()[:, :, rr]
    vmax = float(np.abs(v).max())
    err = float(np.abs(o_g - ref["o"]).max())
    assert err <= 1e-2 * vmax, f"max|dO| {err} > {1e-2 * vmax}"
    assert float(np.abs(lse_g - ref["lse"]).max()) <= 1e-3
    return q, k, v, o_g, rr


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("causal,order", [(True, "reverse"), (True, "forward"), (False, "reverse")])
def test_scaled_forward_matches_oracle(fp8, rotate, causal, order):
    _case(fp8, 1, 4, 2, 300, causal, 256.0, order, rotate)


@pytest.mark.parametrize("S", [1.0, 448.0])
def test_scaled_forward_other_scales(fp8, S):
    _case(fp8, 2, 2, 1, 200, True, S, "reverse", True, delta=5.0)


def test_scaled_forward_larger_sampled(fp8):
    N = 4096
    rows = synthetic.sampled_rows(N, 128)
    _case(fp8, 1, 8, 8, N, True, 256.0, "reverse", True, rows=rows)


def test_rotation_lowers_error_on_gpu(fp8):
    N = 512
    rows = np.arange(0, N, 4)
    errs = {}
    for rotate in (False, True):
        q, k, v, o_g, rr = _case(fp8, 1, 2, 2, N, True, 256.0, "reverse", rotate, outliers=4, delta=3.0, seed=41,
                                 rows=rows)
        o64, _ = oracle.attention_fp64(q, k, v, causal=True, rows=rr)
        errs[rotate] = float(np.sqrt(np.mean((o_g - o64) ** 2)))
    assert errs[True] < errs[False] / 1.5, errs


def test_unit_scales_match_plain_forward(fp8):
    q, k, v, _ = synthetic.make_inputs(1, 2, 2, 384, 128, 7.0, seed=51)
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    o_plain, lse_plain = fp8.fwd(qd, kd, vd, causal=True, p_scale=256.0, kv_order="reverse")
    ones = lambda *s: torch.ones(s, dtype=torch.float32, device="cuda")  # noqa: E731
    o_s, lse_s = fp8.fwd_scaled(qd, kd, vd, ones(2, 3), ones(2, 3), ones(2), causal=True, p_scale=256.0,
                                kv_order="reverse")
    fp8.check_error()
    vmax = float(np.abs(oracle.e4m3_decode(v)).max())
    assert float((o_s.float() - o_plain.float()).abs().max()) <= 1e-2 * vmax
    assert float((lse_s - lse_plain).abs().max()) <= 1e-4
