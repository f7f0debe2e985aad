"""The streamed host-tensor forward pass (C entry fp8attn_fwd_host, binding fwd_host).

CPU: the entry point validates its arguments before touching the device.
GPU: its outputs equal those of ``fwd`` on the same inputs bit for bit, for
every piece count: each (batch, head) slab is computed by the same kernel,
whatever piece it belongs to and whenever its piece lands.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic


def _call_host(fp8, pieces=0, qh=16, kh=16, vh=16, oh=16, lh=16, qd=16, kd=16, vd=16, od=16, ld=16, B=1, H=4, Hkv=2,
               N=256, d=128):
    P = ctypes.c_void_p
    return fp8.lib().fp8attn_fwd_host(P(qh), P(kh), P(vh), P(oh), P(lh), P(qd), P(kd), P(vd), P(od), P(ld), B, H, Hkv,
                                      N, d, 1, ctypes.c_float(256.0), 1, pieces, P(0))


@pytest.mark.parametrize("kw,expected", [
    (dict(pieces=-1), 1), (dict(pieces=33), 1), (dict(qh=0), 1), (dict(kh=0), 1), (dict(vh=0), 1), (dict(oh=0), 1),
    (dict(od=0), 1), (dict(od=8), 1), (dict(qd=0), 1), (dict(ld=0), 1), (dict(lh=0), 1), (dict(ld=18), 1),
    (dict(d=96), 2), (dict(H=3), 1), (dict(N=0), 0), (dict(N=0, qh=0, qd=0, kd=0, vd=0), 0),
])
def test_fwd_host_validation(kw, expected):
    from softmax_cast_precision_b200 import fp8attn

    assert _call_host(fp8attn, **kw) == expected


def test_fwd_host_binding_rejects_device_tensors_and_bad_outputs():
    from softmax_cast_precision_b200 import fp8attn

    q = torch.zeros((1, 2, 8, 128), dtype=torch.uint8)
    with pytest.raises(ValueError):
        fp8attn.fwd_host(q, q, q, causal=True, out=torch.zeros((1, 2, 8, 128), dtype=torch.float32))
    with pytest.raises(ValueError):
        fp8attn.fwd_host(q, q, q, causal=True, out=torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16),
                         lse_out=torch.zeros((1, 2, 9), dtype=torch.float32))


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,Hkv,N,d,pieces,with_lse", [
    (1, 8, 8, 1000, 128, 3, True),     # ragged N, three pieces
    (2, 4, 2, 300, 128, 0, True),      # two batch entries, grouped heads, the default piece count
    (1, 4, 4, 64, 128, 1, True),       # one piece: the in-order path
    (1, 16, 4, 2048, 128, 16, True),   # more pieces asked than kv heads: one kv head per piece
    (4, 8, 2, 1536, 128, 5, False),    # pieces across batch entries, no lse
    (1, 32, 32, 4096, 128, 12, True),  # the bench's piece count on a mid-size problem
    (1, 2, 2, 300, 64, 4, True),       # d = 64: the in-order path
])
def test_fwd_host_equals_fwd(B, H, Hkv, N, d, pieces, with_lse):
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, d, 7.0, seed=81 + pieces)
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    o_ref, l_ref = fp8attn.fwd(qh.cuda(), kh.cuda(), vh.cuda(), causal=True, p_scale=256.0, kv_order="reverse")
    for _ in range(2):  # the second call reuses the library's copy streams
        o_h, l_h = fp8attn.fwd_host(qh, kh, vh, causal=True, p_scale=256.0, kv_order="reverse", pieces=pieces,
                                    with_lse=with_lse)
        fp8attn.check_error()
        assert torch.equal(o_h, o_ref.cpu())
        if with_lse:
            assert torch.equal(l_h, l_ref.cpu())
            assert np.isfinite(l_h.numpy()).all()
        else:
            assert l_h is None


@pytest.mark.gpu
def test_fwd_host_pageable_buffers():
    """Pageable host memory: the copies no longer overlap, but the result is the same."""
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    q, k, v, _ = synthetic.make_inputs(1, 8, 4, 700, 128, 7.0, seed=90)
    qh, kh, vh = (torch.from_numpy(x) for x in (q, k, v))
    o_ref, l_ref = fp8attn.fwd(qh.cuda(), kh.cuda(), vh.cuda(), causal=True)
    oh = torch.empty((1, 8, 700, 128), dtype=torch.bfloat16)
    lh = torch.empty((1, 8, 700), dtype=torch.float32)
    o_h, l_h = fp8attn.fwd_host(qh, kh, vh, causal=True, pieces=4, out=oh, lse_out=lh)
    fp8attn.check_error()
    assert torch.equal(o_h, o_ref.cpu()) and torch.equal(l_h, l_ref.cpu())
