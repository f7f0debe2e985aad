"""CPU oracle for FP8 (E4M3) attention with a static P-cast scale.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the CPU-baseline
leg of the benchmark may import this package; the product path (the CUDA
library and its binding) never does, and the two share no code.

Contents
  * ``oracle.c`` (built here into ``liboracle.so``): the E4M3 codec, bfloat16
    rounding, exact FP64 attention and the blockwise E4M3 emulator.
  * ``closed_forms``: the analytic quantities of the P-cast paper -- the
    underflow fraction F(Delta, S), the collapse threshold Delta_c, the
    expected sink maximum delta_k and the normalised quantisation step d_p(S).

Every function cites the passage it follows; see ``oracle.c`` for the C side.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .closed_forms import (  # noqa: F401  (re-exported)
    LN2_TEN,
    delta_c,
    delta_k,
    dp_closed_form,
    dp_from_grid,
    f_forward,
    f_row,
)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O3", "-mavx2", "-mfma", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode_array.argtypes = [P, P, i64]
        lib.oracle_e4m3_encode_array_f64.argtypes = [P, P, i64]
        lib.oracle_e4m3_decode_array.argtypes = [P, P, i64]
        lib.oracle_bf16_round_array.argtypes = [P, P, i64]
        lib.oracle_attention_fp64.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, P, i32, P, P]
        lib.oracle_emulate.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32,
                                       i32, f32, i32, i32, i32, P, i32, P, P, P, P, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    """OpenMP threads the oracle's loops use."""
    return int(_load().oracle_num_threads())


# --------------------------------------------------------------------------
# E4M3 and bfloat16
# --------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Decode E4M3 bytes to float32 (exact; NaN for the NaN codes)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float32)
    _load().oracle_e4m3_decode_array(_ptr(c), _ptr(out), c.size)
    return out


def e4m3_encode(x) -> np.ndarray:
    """Round float32 values to E4M3 bytes (nearest-even, subnormals, satfinite)."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(a), _ptr(out), a.size)
    return out


def e4m3_encode_f64(x) -> np.ndarray:
    """Round float64 values to E4M3 bytes directly (same rule as ``e4m3_encode``)."""
    a = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array_f64(_ptr(a), _ptr(out), a.size)
    return out


def e4m3_round(x) -> np.ndarray:
    """The E4M3 value nearest to each float32 (the cast as a float32)."""
    return e4m3_decode(e4m3_encode(x))


def e4m3_decode_scalar(code: int) -> float:
    return float(_load().oracle_e4m3_decode(int(code)))


def e4m3_encode_scalar(x: float) -> int:
    return int(_load().oracle_e4m3_encode(float(x)))


def bf16_round_bits(x) -> np.ndarray:
    """bfloat16 bit patterns of float32 values, nearest-even."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_bf16_round_array(_ptr(a), _ptr(out), a.size)
    return out


def bf16_bits_to_float(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _rows_array(N: int, rows) -> np.ndarray:
    if rows is None:
        return np.arange(N, dtype=np.int32)
    r = np.ascontiguousarray(rows, dtype=np.int32)
    if r.ndim != 1 or r.size == 0 or r.min() < 0 or r.max() >= N:
        raise ValueError("rows must be a non-empty 1-D list of query positions in [0, N)")
    return r


def _values(x) -> np.ndarray:
    """Inputs as float32 values: E4M3 bytes are decoded, floats are taken as is."""
    a = np.asarray(x)
    if a.dtype == np.uint8:
        return e4m3_decode(a)
    return np.ascontiguousarray(a, dtype=np.float32)


def _shape(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.shape != k.shape:
        raise ValueError("q must be [B,H,N,d] and k, v [B,Hkv,N,d]")
    B, H, N, d = q.shape
    if k.shape[0] != B or k.shape[2] != N or k.shape[3] != d or H % k.shape[1]:
        raise ValueError("inconsistent q/k/v shapes")
    return B, H, k.shape[1], N, d


def attention_fp64(q, k, v, causal: bool, rows=None):
    """Exact attention in FP64 on the decoded inputs.

    Returns (o [B,H,nrows,d] float64, lse [B,H,nrows] float64) for the query
    positions ``rows`` (all positions if None).
    """
    qf, kf, vf = _values(q), _values(k), _values(v)
    B, H, Hkv, N, d = _shape(qf, kf, vf)
    r = _rows_array(N, rows)
    o = np.empty((B, H, r.size, d), dtype=np.float64)
    lse = np.empty((B, H, r.size), dtype=np.float64)
    _load().oracle_attention_fp64(_ptr(qf), _ptr(kf), _ptr(vf), B, H, Hkv, N, d, int(bool(causal)),
                                  _ptr(r), r.size, _ptr(o), _ptr(lse))
    return o, lse


class EmulatorResult:
    """Outputs of :func:`emulate` for the evaluated rows.

    o_f32     [B,H,R,d] float32  output before the bfloat16 rounding
    o_bf16    [B,H,R,d] uint16   bfloat16 bits of the output
    o         [B,H,R,d] float32  the bfloat16 output as float32
    lse       [B,H,R]   float32  natural-log softmax denominator
    zeros     [B,H,R,2] int64    visible non-sink keys whose P^ is 0 (sink block, other blocks)
    eligible  [B,H,R,2] int64    visible non-sink keys (sink block, other blocks)
    """

    def __init__(self, o_f32, o_bf16, lse, zeros, eligible, rows):
        self.o_f32, self.o_bf16, self.lse = o_f32, o_bf16, lse
        self.zeros, self.eligible, self.rows = zeros, eligible, rows
        self.o = bf16_bits_to_float(o_bf16)

    def zero_count(self, outside_sink_block_only: bool = False) -> np.ndarray:
        """Underflow count per (b, h), summed over the evaluated rows."""
        z = self.zeros[..., 1] if outside_sink_block_only else self.zeros.sum(-1)
        return z.sum(-1)


def emulate(q, k, v, *, causal: bool, block_n: int, p_scale: float, reverse: bool,
            cast: bool = True, n_sink: int = 4, rows=None) -> EmulatorResult:
    """Blockwise online-softmax attention with the E4M3 P-cast (see oracle.c)."""
    qf, kf, vf = _values(q), _values(k), _values(v)
    B, H, Hkv, N, d = _shape(qf, kf, vf)
    if block_n <= 0:
        raise ValueError("block_n must be positive")
    r = _rows_array(N, rows)
    R = r.size
    o_f32 = np.empty((B, H, R, d), dtype=np.float32)
    o_bf16 = np.empty((B, H, R, d), dtype=np.uint16)
    lse = np.empty((B, H, R), dtype=np.float32)
    zeros = np.empty((B, H, R, 2), dtype=np.int64)
    elig = np.empty((B, H, R, 2), dtype=np.int64)
    _load().oracle_emulate(_ptr(qf), _ptr(kf), _ptr(vf), B, H, Hkv, N, d, int(bool(causal)),
                           int(block_n), ctypes.c_float(p_scale), int(bool(reverse)), int(bool(cast)),
                           int(n_sink), _ptr(r), R, _ptr(o_f32), _ptr(o_bf16), _ptr(lse),
                           _ptr(zeros), _ptr(elig))
    return EmulatorResult(o_f32, o_bf16, lse, zeros, elig, r)
