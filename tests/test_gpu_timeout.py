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


_STREAMED_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import torch
import synthetic
from softmax_cast_precision_b200 import fp8attn as fp8
q, k, v, _ = synthetic.make_inputs(1, 8, 4, 1000, 128, 7.0, seed=93)
qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
fp8.check_error()
fp8.test_withhold_load(20_000_000)  # 20 ms
fp8.fwd_host(qh, kh, vh, causal=True, pieces=4)  # returns: every piece flag is raised by the CTAs that gave up
try:
    fp8.check_error()
    sys.exit("no timeout reported")
except fp8.Fp8AttnError as e:
    assert e.status == fp8.ERR_TIMEOUT, e.status
o_h, l_h = fp8.fwd_host(qh, kh, vh, causal=True, pieces=4)
fp8.check_error()
o_ref, l_ref = fp8.fwd(qh.cuda(), kh.cuda(), vh.cuda(), causal=True)
assert torch.equal(o_h, o_ref.cpu()) and torch.equal(l_h, l_ref.cpu())
print("ok")
"""


def test_streamed_call_returns_after_a_wait_runs_out(fp8):
    """fp8attn_fwd_host with a wait made to run out: the kernel raises every piece flag as it gives up, so the
    copy-out stream's waits end and the call returns; the next call matches fwd bit for bit.  Run in a child
    process with a time limit, so that a regression shows as a failure rather than a stuck test run."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _STREAMED_CHILD.format(root=root)], cwd=root, timeout=180,
                         capture_output=True, text=True)
    assert res.returncode == 0 and res.stdout.strip().endswith("ok"), res.stdout + res.stderr
