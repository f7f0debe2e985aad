"""CPU checks of the C-ABI library: it loads without a GPU, exports every
entry point include/fp8attn.h declares, and rejects invalid arguments before
touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8attn.h")


@pytest.fixture(scope="module")
def fp8():
    from softmax_cast_precision_b200 import build

    build.build()
    from softmax_cast_precision_b200 import fp8attn

    return fp8attn


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8attn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["fp8attn_fwd", "fp8attn_fwd_noalloc", "fp8attn_fwd_scaled", "fp8attn_quantize",
                     "fp8attn_fwd_bf16qk", "fp8attn_decode", "fp8attn_decode_workspace_bytes",
                     "fp8attn_bwd", "fp8attn_pzero_count", "fp8attn_kv_tile", "fp8attn_status_str",
                     "fp8attn_check_error"]:
        assert required in names


def test_library_exports_every_declared_symbol(fp8):
    lib = fp8.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", fp8.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (fp8attn_\w+)", out))
    assert set(declared_functions()) <= exported


def test_library_has_no_oracle_or_torch_dependency(fp8):
    out = subprocess.run(["ldd", fp8.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in out and "torch" not in out and "libcuda.so" not in out


def test_host_only_queries(fp8):
    assert fp8.kv_tile(128) == 128
    assert fp8.kv_tile(64) == 64
    assert fp8.kv_tile(96) == 0
    assert fp8.status_str(0) == "ok"
    assert fp8.status_str(4) == "device wait timed out"
    assert fp8.status_str(99) == "unknown status"
    assert fp8.lib().fp8attn_version() >= 100


def _call_fwd(fp8, q=16, k=16, v=16, o=16, B=1, H=2, Hkv=1, N=128, d=128, causal=0, S=256.0, order=1,
              entry="fp8attn_fwd"):
    P = ctypes.c_void_p
    return getattr(fp8.lib(), entry)(P(q), P(k), P(v), P(o), P(0), B, H, Hkv, N, d, causal, ctypes.c_float(S),
                                     order, P(0))


@pytest.mark.parametrize("kw,expected", [
    (dict(d=96), 2), (dict(d=0), 2), (dict(H=3, Hkv=2), 1), (dict(Hkv=0), 1), (dict(H=0), 1),
    (dict(B=-1), 1), (dict(N=-5), 1), (dict(S=0.0), 1), (dict(S=-1.0), 1), (dict(S=float("inf")), 1),
    (dict(S=float("nan")), 1), (dict(S=2.0**65), 1), (dict(S=2.0**-65), 1), (dict(order=2), 1), (dict(q=0), 1), (dict(k=8), 1), (dict(v=4), 1),
    (dict(o=0), 1), (dict(o=24), 1), (dict(B=70000), 2),
])
@pytest.mark.parametrize("entry", ["fp8attn_fwd", "fp8attn_fwd_noalloc", "fp8attn_fwd_bf16qk"])
def test_invalid_arguments_rejected_without_launch(fp8, kw, expected, entry):
    assert _call_fwd(fp8, entry=entry, **kw) == expected


def _header_define(name):
    m = re.search(rf"#define {name} (\d+)", open(HEADER).read())
    return int(m.group(1))


def test_noalloc_limits_and_rejection(fp8):
    assert _header_define("FP8ATTN_NOALLOC_SCRATCH_BYTES") == 256
    max_units = _header_define("FP8ATTN_NOALLOC_MAX_UNITS")
    assert max_units == 2**31 - 2**16  # the 32-bit counter ends at units + grid (< 2^16 CTAs)
    assert fp8.status_str(fp8.ERR_SCRATCH_LIMIT).startswith("problem too large")
    # 65535 x 65535 heads of one row: 4.29e9 work units, rejected before any device work.
    assert _call_fwd(fp8, B=65535, H=65535, Hkv=65535, N=1, entry="fp8attn_fwd_noalloc") == fp8.ERR_SCRATCH_LIMIT
    # d = 64 runs a kernel without scratch and does not hit this limit (only the size checks
    # shared with fp8attn_fwd, which reject this shape as unsupported).
    assert _call_fwd(fp8, B=65535, H=65535, Hkv=65535, N=300, d=64,
                     entry="fp8attn_fwd_noalloc") == fp8.ERR_UNSUPPORTED
    assert _call_fwd(fp8, N=0, q=0, k=0, v=0, o=0, entry="fp8attn_fwd_noalloc") == 0


def test_empty_problems_are_noops(fp8):
    # nothing to compute: valid, nothing launched, no device needed
    assert _call_fwd(fp8, N=0) == 0
    assert _call_fwd(fp8, B=0) == 0
    assert _call_fwd(fp8, N=0, q=0, k=0, v=0, o=0) == 0
    P = ctypes.c_void_p
    assert fp8.lib().fp8attn_pzero_count(P(16), P(16), P(16), P(0), 0, 2, 1, 128, 128, 0, ctypes.c_float(256.0), 1,
                                         4, P(0)) == 0
    assert fp8.lib().fp8attn_pzero_count(P(16), P(16), P(16), P(16), 1, 2, 1, 128, 128, 0, ctypes.c_float(256.0), 1,
                                         -1, P(0)) == 1


def test_binding_raises_without_fallback(fp8, monkeypatch):
    import softmax_cast_precision_b200.fp8attn as mod

    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "LIB_PATH", "/nonexistent/libfp8attn.so")
    with pytest.raises(RuntimeError, match="no fallback"):
        mod.lib()


def _call_quantize(fp8, x=16, dtype=0, xq=16, scales=16, Z=2, N=300, d=128, block_rows=128, signs=None):
    P = ctypes.c_void_p
    sp = P(0)
    keep = None
    if signs is not None:
        keep = (ctypes.c_float * len(signs))(*signs)
        sp = ctypes.cast(keep, P)
    return fp8.lib().fp8attn_quantize(P(x), dtype, P(xq), P(scales), Z, N, d, block_rows, sp, P(0))


@pytest.mark.parametrize("kw,expected", [
    (dict(d=96), 2), (dict(d=256), 2), (dict(dtype=2), 1), (dict(block_rows=-1), 1), (dict(block_rows=129), 1),
    (dict(Z=-1), 1), (dict(N=-1), 1), (dict(x=0), 1), (dict(x=8), 1), (dict(xq=8), 1), (dict(scales=0), 1),
    (dict(scales=2), 1), (dict(Z=70000), 2), (dict(signs=[1.0] * 127 + [0.5]), 1),
    (dict(Z=65535, N=20000, d=64, block_rows=1), 2),  # more than 2^30 blocks
    (dict(Z=0), 0), (dict(N=0), 0), (dict(N=0, x=0, xq=0), 0),
])
def test_quantize_validation(fp8, kw, expected):
    assert _call_quantize(fp8, **kw) == expected


def _call_fwd_scaled(fp8, qs=16, ks=16, vs=16, d=128, signs=None, N=128, S=256.0):
    P = ctypes.c_void_p
    sp = P(0)
    keep = None
    if signs is not None:
        keep = (ctypes.c_float * len(signs))(*signs)
        sp = ctypes.cast(keep, P)
    return fp8.lib().fp8attn_fwd_scaled(P(16), P(16), P(16), P(16), P(0), P(qs), P(ks), P(vs), sp, 1, 2, 1, N, d, 1,
                                        ctypes.c_float(S), 1, P(0))


@pytest.mark.parametrize("kw,expected", [
    (dict(d=64), 2), (dict(d=96), 2), (dict(qs=0), 1), (dict(ks=2), 1), (dict(vs=0), 1), (dict(S=0.0), 1),
    (dict(signs=[1.0, -1.0] * 63 + [2.0, 1.0]), 1), (dict(N=0, qs=0, ks=0, vs=0), 0),
])
def test_fwd_scaled_validation(fp8, kw, expected):
    assert _call_fwd_scaled(fp8, **kw) == expected


def test_bf16qk_is_d128_only(fp8):
    assert _call_fwd(fp8, d=64, entry="fp8attn_fwd_bf16qk") == fp8.ERR_UNSUPPORTED


def test_decode_workspace_and_validation(fp8):
    L = fp8.lib()
    assert L.fp8attn_decode_workspace_bytes(2, 8, 1000, 3) == 2 * 8 * 3 * 130 * 4  # 8 tiles -> 3 splits
    assert L.fp8attn_decode_workspace_bytes(0, 8, 1000, 3) == 0
    assert L.fp8attn_decode_workspace_bytes(1, 8, 1000, 0) == 0
    P = ctypes.c_void_p

    def call(d=128, H=8, Hkv=2, N=1000, split=3, ws=16, wsb=10 ** 6, S=256.0, order=1, B=1):
        return L.fp8attn_decode(P(16), P(16), P(16), P(16), P(0), P(ws), wsb, B, H, Hkv, N, d, ctypes.c_float(S),
                                order, split, P(0))
    assert call(d=64) == fp8.ERR_UNSUPPORTED
    assert call(H=32, Hkv=2) == fp8.ERR_UNSUPPORTED  # 16 query heads per kv head
    assert call(H=6, Hkv=4) == fp8.ERR_INVALID_ARG
    assert call(split=0) == fp8.ERR_INVALID_ARG
    assert call(wsb=100) == fp8.ERR_INVALID_ARG
    assert call(ws=0) == fp8.ERR_INVALID_ARG
    assert call(ws=8) == fp8.ERR_INVALID_ARG
    assert call(N=0) == fp8.ERR_INVALID_ARG
    assert call(S=0.0) == fp8.ERR_INVALID_ARG
    assert call(order=3) == fp8.ERR_INVALID_ARG
    assert call(B=0) == fp8.OK


def test_binding_rejects_bad_arguments_before_calling_the_library(fp8):
    import torch

    b16 = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16)
    u8 = torch.zeros((1, 2, 8, 128), dtype=torch.uint8)
    with pytest.raises(TypeError):
        fp8.fwd_bf16qk(u8, u8, u8, causal=True)  # q, k must be bfloat16
    with pytest.raises(ValueError):
        fp8.fwd_bf16qk(b16, b16, u8, causal=True)  # host tensors
    with pytest.raises(ValueError):
        fp8.quantize(b16, 128)  # host tensor
    with pytest.raises(ValueError):
        fp8.quantize(torch.zeros((2, 8, 128), dtype=torch.float16), 128)  # host tensor (checked first)
    with pytest.raises(ValueError):
        fp8.decode(u8, u8, u8)  # q must be [B, H, d]
    with pytest.raises(ValueError):
        fp8.decode(torch.zeros((1, 2, 128), dtype=torch.uint8), u8, u8)  # host tensors
    with pytest.raises(ValueError):
        fp8.fwd(u8, u8[:, :1], u8, causal=True, kv_order="sideways")
    with pytest.raises(ValueError):
        fp8.fwd_noalloc(u8.cuda() if torch.cuda.is_available() else u8, u8, u8, torch.empty(0), causal=True)


def test_bwd_validation(fp8):
    """fp8attn_bwd rejects bad sizes, scales, pointers and alignments before any CUDA call."""
    L = fp8.lib()
    P = ctypes.c_void_p

    def call(d=128, B=1, H=8, Hkv=2, N=300, S=256.0, q=16, o=16, lse=16, dq=16, delta=16):
        return L.fp8attn_bwd(P(q), P(16), P(16), P(o), P(lse), P(16), P(dq), P(16), P(16), P(delta), B, H, Hkv, N,
                             d, 1, ctypes.c_float(S), P(0))
    assert call(d=64) == fp8.ERR_UNSUPPORTED
    assert call(H=6, Hkv=4) == fp8.ERR_INVALID_ARG
    assert call(Hkv=0) == fp8.ERR_INVALID_ARG
    assert call(N=-1) == fp8.ERR_INVALID_ARG
    assert call(S=0.0) == fp8.ERR_INVALID_ARG
    assert call(S=float("nan")) == fp8.ERR_INVALID_ARG
    assert call(S=2.0 ** 65) == fp8.ERR_INVALID_ARG
    assert call(B=70000) == fp8.ERR_UNSUPPORTED
    assert call(B=65535, H=65535, Hkv=65535, N=8) == fp8.ERR_UNSUPPORTED  # more than 2^34 rows
    assert call(q=0) == fp8.ERR_INVALID_ARG
    assert call(q=8) == fp8.ERR_INVALID_ARG  # not 16-byte aligned
    assert call(o=24) == fp8.ERR_INVALID_ARG
    assert call(dq=0) == fp8.ERR_INVALID_ARG
    assert call(lse=2) == fp8.ERR_INVALID_ARG
    assert call(delta=0) == fp8.ERR_INVALID_ARG
    assert call(B=0) == fp8.OK and call(N=0) == fp8.OK  # empty problems launch nothing


def test_bwd_binding_checks(fp8):
    import torch

    u8 = torch.zeros((1, 2, 8, 128), dtype=torch.uint8)
    b16 = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16)
    lse = torch.zeros((1, 2, 8), dtype=torch.float32)
    with pytest.raises(ValueError):
        fp8.bwd(u8, u8, u8, b16, lse, b16, causal=True)  # host tensors
    with pytest.raises(ValueError):
        fp8.bwd(u8, u8[:, :, :4], u8, b16, lse, b16, causal=True)  # k disagrees on N


def test_withhold_switch_validation(fp8):
    L = fp8.lib()
    assert L.fp8attn_test_withhold_load(0) == fp8.ERR_INVALID_ARG
    assert L.fp8attn_test_withhold_load(2_000_000_001) == fp8.ERR_INVALID_ARG
