"""Pins of the split-KV decode oracle (oracle.decode) against facts fixed by the
mathematics:

  * without the cast, any split of the keys merges to exact attention (the
    online-softmax merge of "Attenzione flash e domanda sulla lunghezza della
    sequenza", section "La ricorrenza softmax online", is exact), output and
    log-sum-exp;
  * with the cast and one split covering every key, the result is the
    blockwise emulator's on the full key range;
  * with single-tile splits the KV order cannot matter: forward == reverse.
"""
import numpy as np
import pytest

import oracle
from oracle import decode as Dc
import synthetic


def _decode_inputs(B, H, Hkv, N, seed, delta=7.0):
    q, k, v, _ = synthetic.make_inputs(B, H, Hkv, N, 128, delta, seed=seed)
    return q[:, :, -1], k, v  # the last position's query attends to every key


@pytest.mark.parametrize("split_tiles", [1, 2, 5])
def test_merge_without_cast_is_exact(split_tiles):
    q, k, v = _decode_inputs(1, 4, 2, 700, seed=3)
    res = Dc.split_decode(q, k, v, p_scale=256.0, reverse=True, split_tiles=split_tiles, cast=False)
    # exact attention of the query row against all keys
    qfull = np.zeros((1, 4, 700, 128), dtype=np.float32)
    qfull[:, :, 0] = oracle.e4m3_decode(q)
    o64, lse64 = oracle.attention_fp64(qfull, k, v, causal=False, rows=[0])
    assert np.allclose(res["o_f64"], o64[:, :, 0], atol=2e-6)
    assert np.allclose(res["lse"], lse64[:, :, 0], atol=2e-6)


def test_one_split_is_the_full_emulation():
    q, k, v = _decode_inputs(2, 2, 1, 500, seed=4)
    res = Dc.split_decode(q, k, v, p_scale=256.0, reverse=True, split_tiles=100)
    qfull = np.zeros((2, 2, 500, 128), dtype=np.float32)
    qfull[:, :, 0] = oracle.e4m3_decode(q)
    ref = oracle.emulate(qfull, k, v, causal=False, block_n=128, p_scale=256.0, reverse=True, rows=[0])
    assert np.array_equal(res["o"], ref.o[:, :, 0])
    assert np.allclose(res["lse"], ref.lse[:, :, 0], atol=1e-6)


def test_single_tile_splits_ignore_order():
    q, k, v = _decode_inputs(1, 2, 2, 384, seed=5)
    f = Dc.split_decode(q, k, v, p_scale=1.0, reverse=False, split_tiles=1)
    r = Dc.split_decode(q, k, v, p_scale=1.0, reverse=True, split_tiles=1)
    assert np.array_equal(f["o"], r["o"]) and np.array_equal(f["lse"], r["lse"])


def test_order_matters_inside_a_split_when_casting():
    # S = 1, forward: the sink tile first collapses the later tiles; reverse
    # inside a multi-tile split does not (the P-cast summary's section 2).
    q, k, v = _decode_inputs(1, 4, 4, 1024, seed=6, delta=8.0)
    f = Dc.split_decode(q, k, v, p_scale=1.0, reverse=False, split_tiles=8)
    r = Dc.split_decode(q, k, v, p_scale=1.0, reverse=True, split_tiles=8)
    qfull = np.zeros((1, 4, 1024, 128), dtype=np.float32)
    qfull[:, :, 0] = oracle.e4m3_decode(q)
    o64, _ = oracle.attention_fp64(qfull, k, v, causal=False, rows=[0])
    ef = np.mean((f["o_f64"] - o64[:, :, 0]) ** 2)
    er = np.mean((r["o_f64"] - o64[:, :, 0]) ** 2)
    assert ef > er
