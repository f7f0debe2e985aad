"""The allocation-free entry point fp8attn_fwd_noalloc against fp8attn_fwd.

Both are called through the C ABI on the same seeded inputs.  The
allocation-free call is made twice in a row on one stream, into outputs
filled with NaN first, so the second call must find its work-unit counter
zeroed again.  Tolerances are those of the GPU parity tests: per element
max|dO| <= 1e-2 * max|V|, lse within 1e-3.

This file is collected last on purpose: it must pass in a fresh process (the
first call on the device does the entry point's set-up) and after every other
test has used the library.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return fp8attn


def _inputs(B, H, Hkv, N, d, seed):
    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, d, delta=7.0, seed=seed)
    vmax = float(np.abs(oracle.e4m3_decode(v)).max())
    return [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (q, k, v)], vmax


@pytest.mark.parametrize("B,H,Hkv,N,d,causal,S,order", [
    (1, 4, 2, 1000, 128, True, 256.0, "reverse"),     # ragged tail, GQA
    (2, 2, 2, 700, 128, False, 1.0, "forward"),       # several batches, non-causal
    (1, 16, 4, 4096, 128, True, 256.0, "reverse"),    # 256 work units: more than one per SM
    (1, 3, 1, 333, 64, True, 448.0, "forward"),       # d = 64 (kernel without scratch)
])
def test_noalloc_matches_fwd_twice_in_a_row(fp8, B, H, Hkv, N, d, causal, S, order):
    (q, k, v), vmax = _inputs(B, H, Hkv, N, d, seed=1000 + N)
    o_ref, lse_ref = fp8.fwd(q, k, v, causal=causal, p_scale=S, kv_order=order)
    fp8.check_error()
    outs = []
    for _ in range(2):
        o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
        fp8.fwd_noalloc(q, k, v, o, lse, causal=causal, p_scale=S, kv_order=order)
        outs.append((o, lse))
    fp8.check_error()
    for o, lse in outs:
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        err = float((o.float() - o_ref.float()).abs().max())
        assert err <= 1e-2 * vmax, f"max|dO| {err} > {1e-2 * vmax}"
        assert float((lse - lse_ref).abs().max()) <= 1e-3


def test_noalloc_without_lse_and_on_a_side_stream(fp8):
    (q, k, v), vmax = _inputs(1, 2, 1, 513, 128, seed=7)
    o_ref, _ = fp8.fwd(q, k, v, causal=True, p_scale=256.0, kv_order="reverse", with_lse=False)
    side = torch.cuda.Stream()
    o = torch.full_like(o_ref, float("nan"))
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fp8.fwd_noalloc(q, k, v, o, None, causal=True, p_scale=256.0, kv_order="reverse", stream=side)
    fp8.check_error(stream=side)
    assert float((o.float() - o_ref.float()).abs().max()) <= 1e-2 * vmax


def test_noalloc_leaves_free_device_memory_unchanged(fp8):
    (q, k, v), _ = _inputs(1, 8, 8, 2048, 128, seed=11)
    o = torch.empty((1, 8, 2048, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 8, 2048), dtype=torch.float32, device="cuda")
    fp8.fwd_noalloc(q, k, v, o, lse, causal=True)  # set-up already done or done here
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        fp8.fwd_noalloc(q, k, v, o, lse, causal=True)
    torch.cuda.synchronize()
    fp8.check_error()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_rejects_bad_output_tensors(fp8):
    (q, k, v), _ = _inputs(1, 2, 2, 256, 128, seed=3)
    with pytest.raises(ValueError):
        fp8.fwd_noalloc(q, k, v, torch.empty((1, 2, 256, 128), dtype=torch.float32, device="cuda"), causal=True)
    with pytest.raises(ValueError):
        fp8.fwd_noalloc(q, k, v, torch.empty((1, 2, 256, 64), dtype=torch.bfloat16, device="cuda"), causal=True)
