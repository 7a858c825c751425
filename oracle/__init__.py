"""Plain CPU oracle for MX block-32 quantization (test infrastructure only).

This package wraps ``libmx_oracle.so``, the scalar C++ restatement in
``mx_oracle.cpp``. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it; the product library never imports, links
or calls it, and it imports nothing from the product package.

Arrays are numpy: bf16 tensors travel as ``uint16`` bit patterns, codes and
scale bytes as ``uint8``. Every function mirrors one exported C function of the
oracle; see the comments there for the definition each one follows.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, oracle_library_path

E2M1, E4M3, E5M2, E3M2, E2M3, INT8 = 0, 1, 2, 3, 4, 5
E2M1_B16, NVFP4 = 6, 7   # block-16 comparison formats (E8M0 / E4M3 scales)


def block_size(fmt: int) -> int:
    return 16 if fmt in (E2M1_B16, NVFP4) else 32


def packed_fp4(fmt: int) -> bool:
    return fmt in (E2M1, E2M1_B16, NVFP4)
FLOOR, CEIL, OAS_RULE, OAS = 0, 1, 2, 3
MBS_STATIC, MBS_DYNAMIC = 1 << 4, 2 << 4

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = oracle_library_path()
    if not os.path.exists(path):
        build_oracle()
    lib = ctypes.CDLL(path)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    dp = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    c_int = ctypes.c_int
    lib.oracle_set_threads.argtypes = [c_int]
    lib.oracle_get_threads.restype = c_int
    lib.oracle_decode_bf16.argtypes = [ctypes.c_uint16]
    lib.oracle_decode_bf16.restype = ctypes.c_double
    lib.oracle_encode_bf16_rne.argtypes = [ctypes.c_double]
    lib.oracle_encode_bf16_rne.restype = ctypes.c_uint16
    for name in ("oracle_decode_e2m1", "oracle_decode_e4m3", "oracle_decode_e8m0"):
        getattr(lib, name).argtypes = [c_int]
        getattr(lib, name).restype = ctypes.c_double
    lib.oracle_decode_element.argtypes = [c_int, c_int]
    lib.oracle_decode_element.restype = ctypes.c_double
    lib.oracle_round_element.argtypes = [ctypes.c_double, ctypes.c_double, c_int]
    lib.oracle_round_element.restype = c_int
    lib.oracle_round_array.argtypes = [dp, i64, ctypes.c_double, c_int,
                                       ctypes.POINTER(ctypes.c_int32)]
    lib.oracle_block_scale.argtypes = [u16p, c_int, c_int, c_int]
    lib.oracle_block_scale.restype = c_int
    lib.oracle_macro_k.argtypes = [u16p, c_int, c_int]
    lib.oracle_macro_k.restype = c_int
    lib.oracle_quantize.argtypes = [u16p, i64, i64, c_int, c_int, u8p, u8p, u8p]
    lib.oracle_dequantize.argtypes = [u8p, u8p, u8p, i64, i64, c_int, c_int, ctypes.c_void_p]
    lib.oracle_fake_quant_fwd.argtypes = [u16p, i64, i64, c_int, c_int, u16p, u8p]
    lib.oracle_fake_quant_bwd.argtypes = [u16p, u16p, i64, i64, c_int, c_int, u16p]
    lib.oracle_block_error.argtypes = [u16p, i64, i64, c_int, c_int, dp, dp]
    fp = ctypes.POINTER(ctypes.c_float)
    lib.oracle_bat_apply.argtypes = [u16p, i64, i64, c_int, fp, fp, fp, fp, u16p, fp]
    _lib = lib
    return lib


def _ptr(a, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _bf16(x):
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 inputs travel as uint16 bit patterns"
    return x


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return _load().oracle_get_threads()


def decode_bf16(b: int) -> float:
    return _load().oracle_decode_bf16(int(b))


def encode_bf16_rne(v: float) -> int:
    return _load().oracle_encode_bf16_rne(float(v))


def decode_e2m1(code: int) -> float:
    return _load().oracle_decode_e2m1(int(code))


def decode_e4m3(code: int) -> float:
    return _load().oracle_decode_e4m3(int(code))


def decode_element(code: int, fmt: int) -> float:
    return _load().oracle_decode_element(int(code), int(fmt))


def decode_e8m0(b: int) -> float:
    return _load().oracle_decode_e8m0(int(b))


def round_element(v: float, X: float, fmt: int) -> int:
    return _load().oracle_round_element(float(v), float(X), int(fmt))


def round_array(v, X: float, fmt: int):
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.zeros(v.size, np.int32)
    _load().oracle_round_array(_ptr(v, ctypes.c_double), v.size, float(X), int(fmt),
                               _ptr(out, ctypes.c_int32))
    return out.reshape(v.shape)


def block_scale(x32, fmt: int, rule: int, k: int = 0) -> int:
    x32 = _bf16(x32)
    assert x32.size == 32
    return _load().oracle_block_scale(_ptr(x32, ctypes.c_uint16), fmt, rule, k)


def macro_k(x128, fmt: int, scaling: int) -> int:
    x128 = _bf16(x128)
    assert x128.size == 128
    return _load().oracle_macro_k(_ptr(x128, ctypes.c_uint16), fmt, scaling)


def _shape(x, scaling=0, fmt=E2M1):
    rows, cols = (1, x.shape[0]) if x.ndim == 1 else (int(np.prod(x.shape[:-1])), x.shape[-1])
    assert cols % block_size(fmt) == 0, "rows must hold whole blocks"
    assert not (scaling >> 4) or cols % 128 == 0, "MBS needs whole 128-element macro blocks"
    return rows, cols


def quantize(x, fmt: int = E2M1, scaling: int = FLOOR):
    """Returns (codes, scales, macro); macro is None without MBS."""
    x = _bf16(x)
    rows, cols = _shape(x, scaling, fmt)
    bs = block_size(fmt)
    ncode = rows * cols // 2 if packed_fp4(fmt) else rows * cols
    codes = np.zeros(ncode, np.uint8)
    scales = np.zeros(rows * cols // bs, np.uint8)
    macro = np.zeros(rows * cols // 128, np.uint8) if scaling >> 4 else None
    _load().oracle_quantize(_ptr(x, ctypes.c_uint16), rows, cols, fmt, scaling,
                            _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint8),
                            _ptr(macro, ctypes.c_uint8))
    ccols = cols // 2 if packed_fp4(fmt) else cols
    codes = codes.reshape(*x.shape[:-1], ccols)
    scales = scales.reshape(*x.shape[:-1], cols // bs)
    if macro is not None:
        macro = macro.reshape(*x.shape[:-1], cols // 128)
    return codes, scales, macro


def dequantize(codes, scales, macro, rows: int, cols: int, fmt: int = E2M1, out_fp32: bool = False):
    """Returns uint16 (bf16 bits) or uint32 (float bits) of shape [rows, cols]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    if macro is not None:
        macro = np.ascontiguousarray(macro, dtype=np.uint8)
    out = np.zeros(rows * cols, np.uint32 if out_fp32 else np.uint16)
    _load().oracle_dequantize(_ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint8),
                              _ptr(macro, ctypes.c_uint8), rows, cols, fmt, int(out_fp32),
                              out.ctypes.data_as(ctypes.c_void_p))
    return out.reshape(rows, cols)


def fake_quant_fwd(x, fmt: int = E2M1, scaling: int = FLOOR, want_scales: bool = False):
    x = _bf16(x)
    rows, cols = _shape(x, scaling, fmt)
    y = np.zeros(rows * cols, np.uint16)
    scales = np.zeros(rows * cols // block_size(fmt), np.uint8) if want_scales else None
    _load().oracle_fake_quant_fwd(_ptr(x, ctypes.c_uint16), rows, cols, fmt, scaling,
                                  _ptr(y, ctypes.c_uint16), _ptr(scales, ctypes.c_uint8))
    y = y.reshape(x.shape)
    if want_scales:
        return y, scales.reshape(*x.shape[:-1], cols // block_size(fmt))
    return y


def fake_quant_bwd(x, gy, fmt: int = E2M1, scaling: int = FLOOR):
    x = _bf16(x)
    gy = _bf16(gy)
    assert gy.shape == x.shape
    rows, cols = _shape(x, scaling, fmt)
    gx = np.zeros(rows * cols, np.uint16)
    _load().oracle_fake_quant_bwd(_ptr(x, ctypes.c_uint16), _ptr(gy, ctypes.c_uint16), rows, cols,
                                  fmt, scaling, _ptr(gx, ctypes.c_uint16))
    return gx.reshape(x.shape)


def block_error(x, fmt: int = E2M1, scaling: int = FLOOR, want_blocks: bool = True):
    """Returns (block_sse [rows, cols/32] float64 or None, sum_d2, sum_x2)."""
    x = _bf16(x)
    rows, cols = _shape(x, scaling, fmt)
    bs = np.zeros(rows * cols // block_size(fmt), np.float64) if want_blocks else None
    totals = np.zeros(2, np.float64)
    _load().oracle_block_error(_ptr(x, ctypes.c_uint16), rows, cols, fmt, scaling,
                               _ptr(bs, ctypes.c_double), _ptr(totals, ctypes.c_double))
    if bs is not None:
        bs = bs.reshape(*x.shape[:-1], cols // block_size(fmt))
    return bs, float(totals[0]), float(totals[1])


def bat_apply(x, a: int, A, B, beta_min=None, beta_max=None, want_f32: bool = False):
    """BATQuant apply step: y = x diag(B_j (x) A) per 32-element block, clipped
    to [beta_min_j min y, beta_max_j max y], rounded to bf16. A: [a, a]
    float32; B: [cols/32, b, b] float32 (b = 32 / a); beta_*: [cols/32] float32
    or both None. Returns the bf16 bits (and the fp32 values if asked)."""
    x = _bf16(x)
    rows, cols = _shape(x)
    assert a in (1, 2, 4, 8, 16, 32)
    b = 32 // a
    A = np.ascontiguousarray(A, dtype=np.float32)
    B = np.ascontiguousarray(B, dtype=np.float32)
    assert A.shape == (a, a) and B.shape == (cols // 32, b, b)
    assert (beta_min is None) == (beta_max is None), "both clip thresholds or neither"
    if beta_min is not None:
        beta_min = np.ascontiguousarray(beta_min, dtype=np.float32)
        beta_max = np.ascontiguousarray(beta_max, dtype=np.float32)
        assert beta_min.shape == beta_max.shape == (cols // 32,)
    y = np.zeros(rows * cols, np.uint16)
    yf = np.zeros(rows * cols, np.float32) if want_f32 else None
    fp = ctypes.c_float
    _load().oracle_bat_apply(_ptr(x, ctypes.c_uint16), rows, cols, int(a), _ptr(A, fp), _ptr(B, fp),
                             _ptr(beta_min, fp), _ptr(beta_max, fp), _ptr(y, ctypes.c_uint16),
                             _ptr(yf, fp))
    y = y.reshape(x.shape)
    if want_f32:
        return y, yf.reshape(x.shape)
    return y


def bat_quantize(x, a: int, A, B, beta_min=None, beta_max=None, fmt: int = E2M1,
                 scaling: int = FLOOR):
    """BATQuant: the apply step, then MX quantization of its bf16 result."""
    return quantize(bat_apply(x, a, A, B, beta_min, beta_max), fmt, scaling)
