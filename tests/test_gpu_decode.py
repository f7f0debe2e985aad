"""GPU parity of the split-KV decode pass (fp8attn_decode) against the oracle
(oracle.decode.split_decode), through the C ABI: per element max|O_gpu -
O_oracle| <= 1e-2 max|V|, lse within 1e-3; and agreement with the prefill
kernel's last query row when a single split covers every key (both then run
the same tiles in the same order)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import decode as Dc
import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return fp8attn


def _inputs(B, H, Hkv, N, seed, delta=7.0):
    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, 128, delta, seed=seed)
    return np.ascontiguousarray(q[:, :, -1]), k, v


@pytest.mark.parametrize("B,H,Hkv,N,split,S,order", [
    (2, 8, 2, 1000, 3, 256.0, "reverse"),
    (1, 4, 4, 300, 1, 1.0, "forward"),
    (1, 8, 1, 2048, 4, 448.0, "forward"),
    (3, 2, 2, 129, 100, 256.0, "reverse"),
    (2, 16, 8, 5000, 7, 256.0, "reverse"),
])
def test_decode_matches_oracle(fp8, B, H, Hkv, N, split, S, order):
    q, k, v = _inputs(B, H, Hkv, N, seed=N + split)
    o, lse = fp8.decode(*(torch.from_numpy(x).cuda() for x in (q, k, v)), p_scale=S, kv_order=order,
                        split_tiles=split)
    fp8.check_error()
    ref = Dc.split_decode(q, k, v, p_scale=S, reverse=(order == "reverse"), split_tiles=split)
    vmax = float(np.abs(oracle.e4m3_decode(v)).max())
    err = float(np.abs(o.float().cpu().numpy() - ref["o"]).max())
    assert err <= 1e-2 * vmax, err
    assert float(np.abs(lse.cpu().numpy() - ref["lse"]).max()) <= 1e-3


def test_single_split_equals_prefill_last_row(fp8):
    B, H, Hkv, N = 1, 4, 2, 640
    qf, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, 128, 7.0, seed=91)
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (qf, k, v))
    o_pre, lse_pre = fp8.fwd(qd, kd, vd, causal=True, p_scale=256.0, kv_order="reverse")
    o_dec, lse_dec = fp8.decode(qd[:, :, -1].contiguous(), kd, vd, p_scale=256.0, kv_order="reverse",
                                split_tiles=1000)
    fp8.check_error()
    vmax = float(np.abs(oracle.e4m3_decode(v)).max())
    assert float((o_dec.float() - o_pre[:, :, -1].float()).abs().max()) <= 1e-2 * vmax
    assert float((lse_dec - lse_pre[:, :, -1]).abs().max()) <= 1e-4


def test_decode_larger_sampled_heads(fp8):
    B, H, Hkv, N = 4, 32, 8, 16384
    q, k, v = _inputs(B, H, Hkv, N, seed=93)
    o, lse = fp8.decode(*(torch.from_numpy(x).cuda() for x in (q, k, v)), p_scale=256.0, kv_order="reverse",
                        split_tiles=16)
    fp8.check_error()
    # the oracle on two (batch, kv-head) groups
    for b, hk in ((0, 0), (3, 7)):
        hs = slice(hk * 4, hk * 4 + 4)
        ref = Dc.split_decode(q[b:b + 1, hs], k[b:b + 1, hk:hk + 1], v[b:b + 1, hk:hk + 1], p_scale=256.0,
                              reverse=True, split_tiles=16)
        vmax = float(np.abs(oracle.e4m3_decode(v[b, hk])).max())
        assert float(np.abs(o[b:b + 1, hs].float().cpu().numpy() - ref["o"]).max()) <= 1e-2 * vmax
        assert float(np.abs(lse[b:b + 1, hs].cpu().numpy() - ref["lse"]).max()) <= 1e-3
