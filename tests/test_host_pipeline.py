"""The pipelined host-tensor forward pass (fp8attn.fwd_host).

CPU: the piece planner covers every (batch, kv head) exactly once, in order,
in near-equal contiguous ranges that never cross a batch entry.
GPU: its outputs equal those of
``fwd`` on the same inputs bit for bit, since every (batch, head) slab is
computed by the same kernel whatever the piece it belongs to.
"""
import numpy as np
import pytest
import torch

import synthetic


@pytest.mark.parametrize("B,H,Hkv,N,chunks", [(1, 32, 32, 32768, None), (4, 32, 8, 8192, None),
                                              (1, 32, 8, 131072, None), (2, 4, 2, 100, None), (1, 8, 8, 256, None),
                                              (3, 6, 3, 1000, 2), (1, 5, 5, 4096, 3), (2, 8, 8, 64, 100)])
def test_host_chunks_partition(B, H, Hkv, N, chunks):
    from softmax_cast_precision_b200.fp8attn import host_chunks

    pieces = host_chunks(B, H, Hkv, N, chunks)
    covered = [(b, g) for b, g0, g1 in pieces for g in range(g0, g1)]
    assert covered == [(b, g) for b in range(B) for g in range(Hkv)]
    sizes = [g1 - g0 for _, g0, g1 in pieces]
    assert min(sizes) >= 1
    for b in range(B):
        sz = [g1 - g0 for bb, g0, g1 in pieces if bb == b]
        assert max(sz) - min(sz) <= 1
    if chunks is None and B * H * N >= 8 * 2 * 148 * 256:
        assert len(pieces) >= 8  # large problems are cut into at least eight pieces


def test_host_chunks_rejects_bad_shapes():
    from softmax_cast_precision_b200.fp8attn import host_chunks

    for args in [(0, 4, 2, 10), (1, 4, 3, 10), (1, 4, 0, 10)]:
        with pytest.raises(ValueError):
            host_chunks(*args)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,Hkv,N,chunks", [(1, 8, 8, 1000, 3), (2, 4, 2, 300, None), (1, 4, 4, 64, 1)])
def test_fwd_host_equals_fwd(B, H, Hkv, N, chunks):
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, 128, 7.0, seed=81)
    qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    o_ref, l_ref = fp8attn.fwd(qh.cuda(), kh.cuda(), vh.cuda(), causal=True, p_scale=256.0, kv_order="reverse")
    o_h, l_h = fp8attn.fwd_host(qh, kh, vh, causal=True, p_scale=256.0, kv_order="reverse", chunks=chunks)
    fp8attn.check_error()
    assert torch.equal(o_h, o_ref.cpu()) and torch.equal(l_h, l_ref.cpu())
    assert np.isfinite(l_h.numpy()).all()
