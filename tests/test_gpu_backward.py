"""GPU parity of the backward pass (fp8attn_bwd) against the oracle's
backward (oracle.backward), through the C ABI.

Inputs: E4M3 q, k, v from the sink-structured generator, the forward outputs
o (bfloat16) and lse from the CPU emulator (never from the GPU), and a seeded
bfloat16 output gradient.  Both sides then compute the gradients of the same
function; the oracle in float64.

Tolerances: the per-element bounds of tests/backward_bounds.py, derived from
the kernels' arithmetic (float32 logits and exponentials, bfloat16 dS,
float32 accumulation, E4M3 rounding-boundary ambiguity of P S) and shown on
the CPU (tests/test_backward_bounds.py) to hold for a model of that
arithmetic and to fail for planted mistakes.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as Bw
import synthetic
from backward_bounds import error_bounds, violations

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return fp8attn


def _case(fp8, B, H, Hkv, N, causal, S, delta=5.0, seed=61):
    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, 128, delta, seed=seed)
    fwd = oracle.emulate(q, k, v, causal=causal, block_n=128, p_scale=S, reverse=True)
    o = oracle.bf16_bits_to_float(fwd.o_bf16)
    lse = fwd.lse
    do = synthetic.make_output_grad((B, H, N, 128), seed + 1)
    ref = Bw.backward(q, k, v, o, lse, do, causal=causal, p_scale=S)
    dev = lambda x, t: torch.from_numpy(np.ascontiguousarray(x)).to(t).cuda()  # noqa: E731
    dq, dk, dv, delta_g = fp8.bwd(dev(q, torch.uint8), dev(k, torch.uint8), dev(v, torch.uint8),
                                  dev(o, torch.bfloat16), dev(lse, torch.float32), dev(do, torch.bfloat16),
                                  causal=causal, p_scale=S)
    fp8.check_error()
    got = [t.cpu().numpy() for t in (dq, dk, dv, delta_g)]
    d_ref = np.sum(do.astype(np.float64) * o.astype(np.float64), axis=-1)
    bounds = error_bounds(q, k, v, o, lse, do, causal=causal, p_scale=S)
    for name, g, r, bd in zip(("dq", "dk", "dv", "delta"), got, ref + (d_ref,), bounds):
        n, worst = violations(g, r, bd)
        assert n == 0, f"{name}: {n} elements outside the bound (worst ratio {worst:.3g})"


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 2)])
def test_backward_matches_oracle(fp8, causal, H, Hkv):
    _case(fp8, 1, H, Hkv, 300, causal, 256.0)  # three tiles, the last one ragged


@pytest.mark.parametrize("S", [1.0, 448.0])
def test_backward_other_scales(fp8, S):
    _case(fp8, 2, 2, 1, 256, True, S, delta=7.0)


def test_backward_single_partial_tile(fp8):
    _case(fp8, 1, 1, 1, 5, True, 256.0)


def test_backward_several_tiles_gqa(fp8):
    _case(fp8, 1, 8, 2, 1024, True, 256.0, delta=7.0)
