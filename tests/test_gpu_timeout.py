"""The bounded waits of the persistent forward kernel, made to run out on
purpose (no fault, no trap, no hang).

fp8attn_test_withhold_load arms the next launch so that its producer skips the
first K tile: the waits for that tile give up after a short limit, the kernel
stops every role, lets its in-flight copies and products land, frees its
tensor memory and returns.  The host then reads FP8ATTN_ERR_TIMEOUT from
fp8attn_check_error, and the next normal call on the same stream is correct
(compared with the oracle like the other parity tests).
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


@pytest.mark.parametrize("counting", [False, True])
def test_wait_runs_out_and_the_next_call_is_correct(fp8, counting):
    q, k, v, _ = synthetic.make_inputs(1, 4, 2, 640, 128, 7.0, seed=91)
    qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
    stream = torch.cuda.current_stream()
    fp8.check_error()  # nothing pending from earlier tests
    fp8.test_withhold_load(20_000_000)  # 20 ms
    if counting:
        fp8.pzero_count(qd, kd, vd, causal=True, p_scale=256.0, kv_order="reverse", n_sink=4)
    else:
        fp8.fwd(qd, kd, vd, causal=True, p_scale=256.0, kv_order="reverse")
    with pytest.raises(fp8.Fp8AttnError) as exc:
        fp8.check_error()
    assert exc.value.status == fp8.ERR_TIMEOUT
    # the switch was consumed and the context is usable: a normal call on the same stream
    o, lse = fp8.fwd(qd, kd, vd, causal=True, p_scale=256.0, kv_order="reverse", stream=stream)
    fp8.check_error()
    ref = oracle.emulate(q, k, v, causal=True, block_n=128, p_scale=256.0, reverse=True)
    vmax = float(np.abs(oracle.e4m3_decode(v)).max())
    assert float(np.abs(o.float().cpu().numpy() - ref.o).max()) <= 1e-2 * vmax
    assert float(np.abs(lse.cpu().numpy() - ref.lse).max()) <= 1e-3
