"""Python binding of libfp8attn (argument marshalling only).

Every step of the attention passes runs in the CUDA library; this module
turns torch tensors into pointers, sizes and a stream, calls the C ABI, and
turns status codes into exceptions.  PyTorch supplies device memory, streams
and (for host inputs) the host<->device copies.

Layouts (see include/fp8attn.h): q [B,H,N,d], k and v [B,Hkv,N,d] as E4M3
(torch.float8_e4m3fn or uint8 bytes), o [B,H,N,d] bfloat16, lse [B,H,N]
float32.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8attn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_SCRATCH_LIMIT = range(6)
FORWARD, REVERSE = 0, 1

_lock = threading.Lock()
_lib = None


class Fp8AttnError(RuntimeError):
    """A libfp8attn call returned a non-OK status."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m softmax_cast_precision_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.fp8attn_fwd.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, P]
        L.fp8attn_fwd.restype = i32
        L.fp8attn_fwd_noalloc.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, P]
        L.fp8attn_fwd_noalloc.restype = i32
        L.fp8attn_fwd_host.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32, P]
        L.fp8attn_fwd_host.restype = i32
        L.fp8attn_quantize.argtypes = [P, i32, P, P, i32, i32, i32, i32, P, P]
        L.fp8attn_quantize.restype = i32
        L.fp8attn_fwd_scaled.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, P]
        L.fp8attn_fwd_scaled.restype = i32
        L.fp8attn_fwd_bf16qk.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, P]
        L.fp8attn_fwd_bf16qk.restype = i32
        u64 = ctypes.c_ulonglong
        L.fp8attn_decode.argtypes = [P, P, P, P, P, P, u64, i32, i32, i32, i32, i32, f32, i32, i32, P]
        L.fp8attn_decode.restype = i32
        L.fp8attn_decode_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.fp8attn_decode_workspace_bytes.restype = u64
        L.fp8attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, P]
        L.fp8attn_bwd.restype = i32
        L.fp8attn_pzero_count.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32, P]
        L.fp8attn_pzero_count.restype = i32
        L.fp8attn_kv_tile.argtypes = [i32]
        L.fp8attn_kv_tile.restype = i32
        L.fp8attn_status_str.argtypes = [i32]
        L.fp8attn_status_str.restype = ctypes.c_char_p
        L.fp8attn_check_error.argtypes = [P]
        L.fp8attn_check_error.restype = i32
        L.fp8attn_version.restype = i32
        L.fp8attn_test_withhold_load.argtypes = [u64]
        L.fp8attn_test_withhold_load.restype = i32
        _lib = L
        return L


def status_str(status: int) -> str:
    return lib().fp8attn_status_str(int(status)).decode()


def kv_tile(d: int) -> int:
    """Keys per KV block for head dimension d (0 if unsupported)."""
    return int(lib().fp8attn_kv_tile(int(d)))


def _order(kv_order) -> int:
    if kv_order in (0, "forward", "fwd"):
        return FORWARD
    if kv_order in (1, "reverse", "rev"):
        return REVERSE
    raise ValueError(f"kv_order must be 'forward'/0 or 'reverse'/1, got {kv_order!r}")


def _bytes(t: torch.Tensor) -> torch.Tensor:
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError("q, k, v must be torch.float8_e4m3fn or uint8 (E4M3 bytes)")
    return t.contiguous()


def _shapes(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q must be [B,H,N,d]; k and v [B,Hkv,N,d]")
    B, H, N, d = q.shape
    if k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError("q, k, v disagree on B, N or d")
    return int(B), int(H), int(k.shape[1]), int(N), int(d)


def _stream_ptr(device: torch.device, stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _on_device(device: torch.device):
    """Make ``device`` current for a library call: the library takes its per-device state (SM count, pools,
    scratch, error word) from the current device."""
    return torch.cuda.device(device)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr() if t is not None and t.numel() else 0)


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, p_scale: float = 256.0,
        kv_order="reverse", with_lse: bool = True, out: torch.Tensor | None = None,
        lse_out: torch.Tensor | None = None, stream=None, device=None):
    """Attention forward pass with the static P-cast scale ``p_scale``.

    Device inputs run in place on their device; host inputs are copied to
    ``device`` (default cuda:0), computed there, and the results copied back
    to the host.  Returns (o, lse) (lse is None when ``with_lse`` is False).
    """
    q, k, v = _bytes(q), _bytes(k), _bytes(v)
    B, H, Hkv, N, d = _shapes(q, k, v)
    if not q.is_cuda:
        # Host inputs: the copies in, the pass and the copies out all go on one stream (the given one, else
        # the device's current stream), which the call waits for before returning.
        dev = torch.device(device if device is not None else "cuda:0")
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        with torch.cuda.stream(s):
            qd, kd, vd = (x.to(dev, non_blocking=True) for x in (q, k, v))
            o_d, lse_d = fwd(qd, kd, vd, causal=causal, p_scale=p_scale, kv_order=kv_order, with_lse=with_lse,
                             stream=s)
            o_h = out if out is not None else torch.empty(o_d.shape, dtype=o_d.dtype, pin_memory=True)
            o_h.copy_(o_d, non_blocking=True)
            lse_h = None
            if lse_d is not None:
                lse_h = lse_out if lse_out is not None else torch.empty(lse_d.shape, dtype=lse_d.dtype,
                                                                        pin_memory=True)
                lse_h.copy_(lse_d, non_blocking=True)
        s.synchronize()
        return o_h, lse_h
    dev = q.device
    if k.device != dev or v.device != dev:
        raise ValueError("q, k, v must be on the same device")
    o = out if out is not None else torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = None
    if with_lse:
        lse = lse_out if lse_out is not None else torch.empty((B, H, N), dtype=torch.float32, device=dev)
    with _on_device(q.device):
        st = lib().fp8attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, N, d, int(bool(causal)),
                               ctypes.c_float(p_scale), _order(kv_order), _stream_ptr(dev, stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_fwd")
    return o, lse


def fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, p_scale: float = 256.0,
             kv_order="reverse", pieces: int = 0, with_lse: bool = True, device=None, out: torch.Tensor | None = None,
             lse_out: torch.Tensor | None = None, stream=None):
    """Forward pass of host tensors, the copies overlapped with the computation (C entry ``fp8attn_fwd_host``).

    q [B,H,N,d], k, v [B,Hkv,N,d] are E4M3 host tensors (pinned, for the copies to overlap).  The library cuts
    the problem into ``pieces`` pieces of whole kv heads (0: its default), copies each in on a copy stream of its
    own, runs one persistent pass on ``stream`` (default: the device's current stream) that takes the pieces in
    order as they land, and copies each piece's outputs back as soon as they are stored.  Device staging buffers
    are allocated here.  Returns host (o, lse): ``out`` (bfloat16 [B,H,N,d]) and ``lse_out`` (float32 [B,H,N])
    when given (pinned, for the copies to overlap), else new pinned tensors; lse is None when ``with_lse`` is
    False.  The call returns once both are complete.
    """
    q, k, v = _bytes(q), _bytes(k), _bytes(v)
    B, H, Hkv, N, d = _shapes(q, k, v)
    if q.is_cuda or k.is_cuda or v.is_cuda:
        raise ValueError("fwd_host takes host tensors")
    if not all(t.is_contiguous() for t in (q, k, v)):
        raise ValueError("fwd_host takes contiguous q, k, v")
    dev = torch.device(device if device is not None else "cuda:0")
    if ((out is not None and (out.is_cuda or out.dtype != torch.bfloat16 or tuple(out.shape) != (B, H, N, d)
                              or not out.is_contiguous()))
            or (with_lse and lse_out is not None and (lse_out.is_cuda or lse_out.dtype != torch.float32
                                                      or tuple(lse_out.shape) != (B, H, N)
                                                      or not lse_out.is_contiguous()))):
        raise ValueError("out / lse_out must be contiguous host tensors: bfloat16 [B,H,N,d] and float32 [B,H,N]")
    o_h = out if out is not None else torch.empty((B, H, N, d), dtype=torch.bfloat16, pin_memory=True)
    lse_h = None
    if with_lse:
        lse_h = lse_out if lse_out is not None else torch.empty((B, H, N), dtype=torch.float32, pin_memory=True)
    if B * H * N == 0:
        return o_h, lse_h
    qd, kd, vd = (torch.empty(t.shape, dtype=torch.uint8, device=dev) for t in (q, k, v))
    od = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lsed = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse_h is not None else None
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    with _on_device(dev):
        st = lib().fp8attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o_h), _ptr(lse_h), _ptr(qd), _ptr(kd), _ptr(vd),
                                    _ptr(od), _ptr(lsed), B, H, Hkv, N, d, int(bool(causal)), ctypes.c_float(p_scale),
                                    _order(kv_order), int(pieces), ctypes.c_void_p(s.cuda_stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_fwd_host")
    s.synchronize()
    return o_h, lse_h


def fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                lse_out: torch.Tensor | None = None, *, causal: bool, p_scale: float = 256.0,
                kv_order="reverse", stream=None) -> None:
    """The allocation-free forward pass (C entry point ``fp8attn_fwd_noalloc``).

    For callers that cannot let the library allocate device memory.  All
    tensors are the caller's, on one device: ``out`` bf16 [B,H,N,d] and the
    optional ``lse_out`` float32 [B,H,N], both contiguous, are written in
    place.  Every call on a device shares one fixed scratch array, so calls
    must not overlap (keep them on one stream); the first call on a device
    does a one-time set-up and should come before any stream capture.
    q, k and v must be contiguous: this wrapper makes no copies.
    """
    if not all(t.is_contiguous() for t in (q, k, v)):
        raise ValueError("fwd_noalloc takes contiguous q, k, v")
    q, k, v = _bytes(q), _bytes(k), _bytes(v)
    B, H, Hkv, N, d = _shapes(q, k, v)
    if not q.is_cuda or k.device != q.device or v.device != q.device:
        raise ValueError("fwd_noalloc takes device tensors on one device")
    if (out.device != q.device or out.dtype != torch.bfloat16 or tuple(out.shape) != (B, H, N, d)
            or not out.is_contiguous()):
        raise ValueError("out must be a contiguous bfloat16 [B,H,N,d] tensor on the inputs' device")
    if lse_out is not None and (lse_out.device != q.device or lse_out.dtype != torch.float32
                                or tuple(lse_out.shape) != (B, H, N) or not lse_out.is_contiguous()):
        raise ValueError("lse_out must be a contiguous float32 [B,H,N] tensor on the inputs' device")
    with _on_device(q.device):
        st = lib().fp8attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse_out), B, H, Hkv, N, d,
                                       int(bool(causal)), ctypes.c_float(p_scale), _order(kv_order),
                                       _stream_ptr(q.device, stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_fwd_noalloc")


def fwd_bf16qk(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, p_scale: float = 256.0,
               kv_order="reverse", with_lse: bool = True, stream=None):
    """Forward pass with bfloat16 q [B,H,N,128], k [B,Hkv,N,128] and E4M3 v [B,Hkv,N,128] (device
    tensors): S = Q K^T on the 16-bit tensor-core path, then the same P-cast and P V as ``fwd``."""
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16:
        raise TypeError("q and k must be bfloat16")
    v = _bytes(v)
    q, k = q.contiguous(), k.contiguous()
    B, H, Hkv, N, d = _shapes(q, k, v)
    if not q.is_cuda:
        raise ValueError("fwd_bf16qk takes device tensors")
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if with_lse else None
    with _on_device(q.device):
        st = lib().fp8attn_fwd_bf16qk(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, N, d, int(bool(causal)),
                                      ctypes.c_float(p_scale), _order(kv_order), _stream_ptr(q.device, stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_fwd_bf16qk")
    return o, lse


def decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, p_scale: float = 256.0, kv_order="reverse",
           split_tiles: int = 16, with_lse: bool = True, workspace: torch.Tensor | None = None, stream=None):
    """Decode step: q [B,H,d] (one query row per head) against k, v [B,Hkv,N,d], all E4M3 on the GPU.

    The keys are processed in splits of ``split_tiles`` 128-key tiles that are
    merged exactly; returns (o [B,H,d] bfloat16, lse [B,H] or None).
    """
    q, k, v = _bytes(q), _bytes(k), _bytes(v)
    if q.dim() != 3 or k.dim() != 4 or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q must be [B,H,d]; k and v [B,Hkv,N,d]")
    B, H, d = (int(x) for x in q.shape)
    Hkv, N = int(k.shape[1]), int(k.shape[2])
    if not q.is_cuda:
        raise ValueError("decode takes device tensors")
    need = int(lib().fp8attn_decode_workspace_bytes(B, H, N, int(split_tiles)))
    with torch.cuda.stream(stream):  # a workspace made here is allocated on the stream that uses it
        ws = workspace if workspace is not None else torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        o = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device)
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if with_lse else None
        st = lib().fp8attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(ws),
                                  ws.numel() * ws.element_size(), B, H, Hkv, N, d, ctypes.c_float(p_scale),
                                  _order(kv_order), int(split_tiles), _stream_ptr(q.device, stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_decode")
    return o, lse


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
        dout: torch.Tensor, *, causal: bool, p_scale: float = 256.0, stream=None):
    """Backward pass of ``fwd`` (see fp8attn_bwd): gradients of the P-cast attention.

    q, k, v are the forward's E4M3 inputs, o (bfloat16 [B,H,N,d]) and lse
    (float32 [B,H,N]) its outputs, dout the bfloat16 output gradient; all on
    one GPU.  Returns (dq [B,H,N,d], dk [B,Hkv,N,d], dv [B,Hkv,N,d], delta
    [B,H,N]), all float32, delta_i = dout_i . o_i.
    """
    q, k, v = _bytes(q), _bytes(k), _bytes(v)
    B, H, Hkv, N, d = _shapes(q, k, v)
    if not q.is_cuda or any(t.device != q.device for t in (k, v, o, lse, dout)):
        raise ValueError("bwd takes device tensors on one device")
    if o.dtype != torch.bfloat16 or dout.dtype != torch.bfloat16 or lse.dtype != torch.float32:
        raise TypeError("o and dout must be bfloat16, lse float32")
    if tuple(o.shape) != (B, H, N, d) or tuple(dout.shape) != (B, H, N, d) or tuple(lse.shape) != (B, H, N):
        raise ValueError("o and dout must be [B,H,N,d] and lse [B,H,N]")
    o, lse, dout = o.contiguous(), lse.contiguous(), dout.contiguous()
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty((B, H, N, d), **f32)
    dk = torch.empty((B, Hkv, N, d), **f32)
    dv = torch.empty((B, Hkv, N, d), **f32)
    delta = torch.empty((B, H, N), **f32)
    with _on_device(q.device):
        st = lib().fp8attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(delta), B, H, Hkv, N, d, int(bool(causal)), ctypes.c_float(p_scale),
                               _stream_ptr(q.device, stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_bwd")
    return dq, dk, dv, delta


def _host_signs(signs, d: int):
    """Signs as a host float32 array kept alive for the call (None -> NULL)."""
    if signs is None:
        return None, ctypes.c_void_p(0)
    a = torch.as_tensor(signs, dtype=torch.float32).detach().cpu().contiguous().reshape(-1)
    if a.numel() != d:
        raise ValueError(f"signs must have {d} entries")
    return a, ctypes.c_void_p(a.data_ptr())


def quantize(x: torch.Tensor, block_rows: int, signs=None, *, out: torch.Tensor | None = None,
             scales: torch.Tensor | None = None, stream=None):
    """E4M3 codes and per-block descales of x [..., N, d] (bfloat16 or float32, on the GPU).

    Rows are rotated by R = diag(signs) H_d / sqrt(d) first when ``signs``
    (d values of +-1) is given.  ``block_rows`` rows of one slab share a
    descale (0: one per slab).  Returns (codes uint8 of x's shape, scales
    float32 [Z, nblocks]) with Z the product of the leading dimensions.
    """
    if not x.is_cuda:
        raise ValueError("quantize takes a device tensor")
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("x must be bfloat16 or float32")
    x = x.contiguous()
    N, d = int(x.shape[-2]), int(x.shape[-1])
    Z = math.prod(int(n) for n in x.shape[:-2])
    nb = 1 if block_rows == 0 else -(-N // block_rows)
    codes = out if out is not None else torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    sc = scales if scales is not None else torch.empty((Z, nb), dtype=torch.float32, device=x.device)
    keep, sp = _host_signs(signs, d)
    with _on_device(x.device):
        st = lib().fp8attn_quantize(_ptr(x), 0 if x.dtype == torch.bfloat16 else 1, _ptr(codes), _ptr(sc), Z, N, d,
                                    int(block_rows), sp, _stream_ptr(x.device, stream))
    del keep
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_quantize")
    return codes, sc


def fwd_scaled(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_scales: torch.Tensor, k_scales: torch.Tensor,
               v_scales: torch.Tensor, *, causal: bool, p_scale: float = 256.0, kv_order="reverse", signs=None,
               with_lse: bool = True, stream=None):
    """Forward pass on quantised q, k, v (E4M3 codes) with their descales; see fp8attn_fwd_scaled."""
    q, k, v = _bytes(q), _bytes(k), _bytes(v)
    B, H, Hkv, N, d = _shapes(q, k, v)
    if not q.is_cuda:
        raise ValueError("fwd_scaled takes device tensors")
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if with_lse else None
    qs, ks, vs = (t.contiguous().float() for t in (q_scales, k_scales, v_scales))
    keep, sp = _host_signs(signs, d)
    with _on_device(q.device):
        st = lib().fp8attn_fwd_scaled(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(qs), _ptr(ks), _ptr(vs), sp,
                                      B, H, Hkv, N, d, int(bool(causal)), ctypes.c_float(p_scale), _order(kv_order),
                                      _stream_ptr(q.device, stream))
    del keep
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_fwd_scaled")
    return o, lse


def fwd_wide(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, p_scale: float = 256.0,
             kv_order="reverse", signs=None, with_lse: bool = True, stream=None):
    """Attention on bfloat16/float32 q [B,H,N,d], k, v [B,Hkv,N,d]: quantise (Q, K per 128-row
    block, V per head, rotated by ``signs`` when given), then the scaled forward pass.

    The intermediate codes and scales are allocated on ``stream`` (when given), the stream that
    reads them, so the caching allocator cannot hand their memory out while the pass still runs."""
    with torch.cuda.stream(stream):
        qc, qs = quantize(q, 128, signs, stream=stream)
        kc, ks = quantize(k, 128, signs, stream=stream)
        vc, vs = quantize(v, 0, signs, stream=stream)
        return fwd_scaled(qc, kc, vc, qs, ks, vs, causal=causal, p_scale=p_scale, kv_order=kv_order,
                          signs=signs, with_lse=with_lse, stream=stream)


def pzero_count(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, p_scale: float = 256.0,
                kv_order="reverse", n_sink: int = 4, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Per-(b, h) count of visible keys j >= n_sink whose E4M3(P * S) is zero.

    Returns an int64 tensor [B, H] on the inputs' device.
    """
    q, k, v = _bytes(q), _bytes(k), _bytes(v)
    B, H, Hkv, N, d = _shapes(q, k, v)
    if not q.is_cuda:
        raise ValueError("pzero_count takes device tensors")
    counts = out if out is not None else torch.empty((B, H), dtype=torch.int64, device=q.device)
    with _on_device(q.device):
        st = lib().fp8attn_pzero_count(_ptr(q), _ptr(k), _ptr(v), _ptr(counts), B, H, Hkv, N, d, int(bool(causal)),
                                       ctypes.c_float(p_scale), _order(kv_order), int(n_sink),
                                       _stream_ptr(q.device, stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_pzero_count")
    return counts


def check_error(stream=None, device=None) -> None:
    """Synchronise and raise if a device-side bounded wait ran out."""
    dev = torch.device(device if device is not None else "cuda:0")
    st = lib().fp8attn_check_error(_stream_ptr(dev, stream))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_check_error")


def test_withhold_load(wait_limit_ns: int) -> None:
    """Test switch: the next d = 128 forward launch skips its first K tile load and its waits give up after
    ``wait_limit_ns`` (see fp8attn_test_withhold_load); check_error() then raises with ERR_TIMEOUT."""
    st = lib().fp8attn_test_withhold_load(int(wait_limit_ns))
    if st != OK:
        raise Fp8AttnError(st, "fp8attn_test_withhold_load")


def raw_call(name: str, *args) -> int:
    """Call a C-ABI entry point with raw arguments (pointers as ints); returns the status."""
    return int(getattr(lib(), name)(*args))
