"""B200-native OCP Microscaling (MX) block-32 quantization.

A thin Python binding over ``libmx.so`` (C ABI in ``include/mx.h``): argument
marshalling only. Every step of quantize / dequantize / fake-quant / error runs
in the library's sm_100a kernels; PyTorch provides device memory and streams.
There is no CPU fallback: without the built library, or on a machine whose
tensors are not on a CUDA device, the calls raise.

Two layers, both exported here:

* ``mx_quantize``, ``mx_dequantize``, ``mx_fake_quant_fwd``,
  ``mx_fake_quant_bwd``, ``mx_block_error``, ``mx_bat_apply``,
  ``mx_bat_quantize``, ``mx_scale_bytes``, ``mx_status_string``: the C
  functions with their C names and arguments (raw pointers as ints, stream as
  an int handle), returning the status code.
* ``quantize``, ``dequantize``, ``fake_quant``, ``fake_quant_bwd``,
  ``block_error``, ``bat_apply``, ``bat_quantize`` (BATQuant's block
  transform and clip, alone or fused with quantize):
  tensor-level calls that check tensors, allocate outputs
  with torch on the input's device, launch on the current CUDA stream and
  raise ``MXError`` on a nonzero status. ``quantize`` and ``dequantize`` also
  take CPU tensors: the binding then copies the input to the GPU, launches,
  and copies the outputs back (pinned host memory makes those copies async).
* ``MXFakeQuantize``: an autograd function (forward fake-quant, straight-
  through backward) for quantization-aware training of activations and
  weights alike.
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "E2M1", "E4M3", "E5M2", "E3M2", "E2M3", "INT8", "FLOOR", "CEIL", "OAS_RULE", "OAS", "MBS_STATIC", "MBS_DYNAMIC",
    "MXError", "library_path", "load_library",
    "mx_quantize", "mx_dequantize", "mx_fake_quant_fwd", "mx_fake_quant_bwd",
    "mx_block_error", "mx_status_string", "mx_version", "mx_scale_bytes", "MMA_SCALES",
    "E2M1_B16", "NVFP4", "block_size",
    "quantize", "dequantize", "fake_quant", "fake_quant_bwd", "block_error", "MXFakeQuantize",
    "mx_bat_apply", "mx_bat_quantize", "bat_apply", "bat_quantize",
    "mx_gemm", "mx_quant_gemm", "gemm", "quant_gemm", "GEMM_A_ON_CHIP", "mx_quant_gemm_noalloc",
    "MXFP4_FORMAT", "MXFP8_FORMAT",
]

# formats (mx_format_t)
E2M1 = 0   # MXFP4
E4M3 = 1   # MXFP8
E5M2 = 2   # MXFP8
E3M2 = 3   # MXFP6 (one code per byte, low 6 bits)
E2M3 = 4   # MXFP6
INT8 = 5   # MXINT8 (i * 2^-6)
# OR into `scaling`: scale bytes in the tiled layout of block-scaled tensor-core
# GEMMs (a flat uint8 buffer of mx_scale_bytes(rows, cols, format, scaling) bytes)
MMA_SCALES = 1 << 8
# OR into mx_quant_gemm's out_fp32: A quantized in the GEMM's prologue, on chip
GEMM_A_ON_CHIP = 1 << 9
E2M1_B16 = 6  # MXFP4 at block 16 (E8M0 scales [..., cols/16])
NVFP4 = 7     # E2M1 at block 16 with E4M3 scales amax/6 (FLOOR only)
_PACKED = (E2M1, E2M1_B16, NVFP4)


def block_size(format: int) -> int:
    """Elements per scale byte: 16 for the block-16 formats, else 32."""
    return 16 if format in (E2M1_B16, NVFP4) else 32
MXFP4_FORMAT = E2M1
MXFP8_FORMAT = E4M3
# scaling (mx_scaling_t)
FLOOR, CEIL, OAS_RULE, OAS = 0, 1, 2, 3
MBS_STATIC, MBS_DYNAMIC = 1 << 4, 2 << 4

_STATUS = {0: "MX_OK", 1: "MX_ERR_INVALID_ARG", 2: "MX_ERR_SHAPE", 3: "MX_ERR_ALIGN",
           4: "MX_ERR_UNSUPPORTED", 5: "MX_ERR_CUDA", 6: "MX_ERR_TOO_LARGE"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


class MXError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)} ({mx_status_string(status)})")


def library_path() -> str:
    return os.path.join(_HERE, "libmx.so")


def load_library():
    """Loads libmx.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m fp8_quantization_mx_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.mx_quantize.argtypes = [vp, i64, i64, c_int, c_int, vp, vp, vp, vp]
    lib.mx_dequantize.argtypes = [vp, vp, vp, i64, i64, c_int, c_int, vp, vp]
    lib.mx_fake_quant_fwd.argtypes = [vp, i64, i64, c_int, c_int, vp, vp, vp]
    lib.mx_fake_quant_bwd.argtypes = [vp, vp, i64, i64, c_int, c_int, vp, vp]
    lib.mx_block_error.argtypes = [vp, i64, i64, c_int, c_int, vp, vp, vp]
    for f in ("mx_quantize", "mx_dequantize", "mx_fake_quant_fwd", "mx_fake_quant_bwd",
              "mx_block_error"):
        getattr(lib, f).restype = c_int
    lib.mx_status_string.argtypes = [c_int]
    lib.mx_status_string.restype = ctypes.c_char_p
    lib.mx_version.restype = c_int
    lib.mx_scale_bytes.argtypes = [i64, i64, c_int, c_int]
    lib.mx_scale_bytes.restype = i64
    lib.mx_bat_apply.argtypes = [vp, i64, i64, c_int, vp, vp, vp, vp, vp, vp]
    lib.mx_bat_quantize.argtypes = [vp, i64, i64, c_int, vp, vp, vp, vp, c_int, c_int, vp, vp, vp, vp]
    lib.mx_bat_apply.restype = c_int
    lib.mx_bat_quantize.restype = c_int
    lib.mx_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, c_int, vp, vp, vp]
    lib.mx_quant_gemm.argtypes = [vp, c_int, vp, vp, i64, i64, i64, c_int, vp, vp, vp, vp, vp]
    lib.mx_gemm.restype = c_int
    lib.mx_quant_gemm.restype = c_int
    lib.mx_quant_gemm_noalloc.argtypes = [vp, c_int, vp, vp, i64, i64, i64, c_int, vp, vp, vp]
    lib.mx_quant_gemm_noalloc.restype = c_int
    _lib = lib
    return lib


# ---------------------------------------------------------------- C layer --

def mx_quantize(x, rows, cols, format, scaling, codes, scales, macro, stream=0) -> int:
    return load_library().mx_quantize(x, rows, cols, format, scaling, codes, scales, macro, stream)


def mx_dequantize(codes, scales, macro, rows, cols, format, out_fp32, out, stream=0) -> int:
    return load_library().mx_dequantize(codes, scales, macro, rows, cols, format, out_fp32, out,
                                        stream)


def mx_fake_quant_fwd(x, rows, cols, format, scaling, y, scales_out, stream=0) -> int:
    return load_library().mx_fake_quant_fwd(x, rows, cols, format, scaling, y, scales_out, stream)


def mx_fake_quant_bwd(x, grad_y, rows, cols, format, scaling, grad_x, stream=0) -> int:
    return load_library().mx_fake_quant_bwd(x, grad_y, rows, cols, format, scaling, grad_x, stream)


def mx_block_error(x, rows, cols, format, scaling, block_sse, totals, stream=0) -> int:
    return load_library().mx_block_error(x, rows, cols, format, scaling, block_sse, totals, stream)


def mx_bat_apply(x, rows, cols, a_dim, A, B, beta_min, beta_max, y, stream=0) -> int:
    return load_library().mx_bat_apply(x, rows, cols, a_dim, A, B, beta_min, beta_max, y, stream)


def mx_bat_quantize(x, rows, cols, a_dim, A, B, beta_min, beta_max, format, scaling, codes, scales,
                    macro, stream=0) -> int:
    return load_library().mx_bat_quantize(x, rows, cols, a_dim, A, B, beta_min, beta_max, format,
                                          scaling, codes, scales, macro, stream)


def mx_gemm(a_codes, a_scales, b_codes, b_scales, M, N, K, out_fp32, d, status, stream=0) -> int:
    return load_library().mx_gemm(a_codes, a_scales, b_codes, b_scales, M, N, K, out_fp32, d, status,
                                  stream)


def mx_quant_gemm(a, scaling, b_codes, b_scales, M, N, K, out_fp32, d, a_codes_out, a_scales_out,
                  status, stream=0) -> int:
    return load_library().mx_quant_gemm(a, scaling, b_codes, b_scales, M, N, K, out_fp32, d,
                                        a_codes_out, a_scales_out, status, stream)


def mx_quant_gemm_noalloc(a, scaling, b_codes, b_scales, M, N, K, out_fp32, d, status,
                          stream=0) -> int:
    """mx_quant_gemm (staged, no A buffers) with its scratch in the library's
    fixed device array: for callers that may not allocate device memory
    while they run. Calls that overlap on the GPU race on that array."""
    return load_library().mx_quant_gemm_noalloc(a, scaling, b_codes, b_scales, M, N, K, out_fp32,
                                                d, status, stream)


def mx_status_string(status: int) -> str:
    return load_library().mx_status_string(int(status)).decode()


def mx_version() -> int:
    return load_library().mx_version()


def mx_scale_bytes(rows, cols, format, scaling) -> int:
    return load_library().mx_scale_bytes(rows, cols, format, scaling)


# ----------------------------------------------------------- tensor layer --

def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise MXError(status, where)


def _rows_cols(x: torch.Tensor):
    if x.dim() == 0:
        raise ValueError("expected at least a 1-D tensor")
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    return rows, cols


def _cuda_bf16(x: torch.Tensor, name: str):
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if x.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {x.dtype}")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")


def _check_buf(t, name: str, device, dtype, need: int):
    """A caller-supplied buffer must be a contiguous ``dtype`` tensor on
    ``device`` holding at least ``need`` elements: the kernels write through
    its raw pointer, so a host tensor, a short buffer or a narrower dtype
    would be written out of bounds."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if t.device != torch.device(device):
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < need:
        raise ValueError(f"{name} holds {t.numel()} elements, needs at least {need}")


def _scale_count(rows, cols, format, scaling) -> int:
    if scaling & MMA_SCALES:
        return mx_scale_bytes(rows, cols, format, scaling)
    return rows * (cols // block_size(format))


def _quantize_buffers(device, lead, rows, cols, format, scaling, out):
    """The (codes, scales, macro) a quantize call writes: new tensors on
    ``device`` when ``out`` is None, else ``out`` after checking each buffer
    against what the kernels write (device, uint8, contiguous, size)."""
    mbs = ((scaling >> 4) & 3) != 0
    ccols = cols // 2 if format in _PACKED else cols
    if out is None:
        codes = torch.empty(*lead, ccols, dtype=torch.uint8, device=device)
        scales = _scales_buffer(lead, rows, cols, format, scaling, device)
        macro = torch.empty(*lead, cols // 128, dtype=torch.uint8, device=device) if mbs else None
        return codes, scales, macro
    if len(out) != 3:
        raise ValueError("out must be (codes, scales, macro)")
    codes, scales, macro = out
    _check_buf(codes, "codes", device, torch.uint8, rows * ccols)
    _check_buf(scales, "scales", device, torch.uint8, _scale_count(rows, cols, format, scaling))
    if mbs:
        _check_buf(macro, "macro", device, torch.uint8, rows * (cols // 128))
    return codes, scales, macro


def quantize(x: torch.Tensor, format: int = E2M1, scaling: int = FLOOR, out=None):
    """MX-quantizes bf16 ``x`` [..., cols] along its last dimension.

    Returns ``(codes, scales, macro)``: codes uint8 [..., cols/2] (MXFP4, two
    codes per byte, even element in the low nibble) or [..., cols] (every other
    format, one code per byte); scales uint8 [..., cols/32] (E8M0); macro uint8 [..., cols/128]
    with Macro Block Scaling, else None. ``out`` may supply the three buffers.
    A CPU ``x`` is copied to the current GPU and the outputs come back to the
    CPU: into ``out`` (host tensors) when given, else into new tensors (pinned
    when ``x`` is pinned). A pinned ``x`` is moved in row chunks so that its
    upload, the kernels and the download of earlier chunks overlap (PCIe is
    full duplex); the current stream waits for all of it, so the call orders
    like a single kernel on the current stream.
    """
    if not x.is_cuda:
        if out is not None:
            rows, cols = _rows_cols(x)
            _quantize_buffers(torch.device("cpu"), x.shape[:-1], rows, cols, format, scaling, out)
        dev = torch.device("cuda", torch.cuda.current_device())
        if x.is_pinned() and x.numel() * 2 >= 2 * _CHUNK_BYTES:
            return _quantize_host_pipelined(x, format, scaling, out, dev)
        xd = x.to(dev, non_blocking=x.is_pinned())
        res = quantize(xd, format, scaling)
        if out is None:
            return tuple(None if t is None else _to_host(t, x.is_pinned()) for t in res)
        for h, d in zip(out, res):
            if h is not None and d is not None:
                h.copy_(d, non_blocking=h.is_pinned())
        return out
    _cuda_bf16(x, "x")
    rows, cols = _rows_cols(x)
    codes, scales, macro = _quantize_buffers(x.device, x.shape[:-1], rows, cols, format, scaling,
                                             out)
    with torch.cuda.device(x.device):
        _check(mx_quantize(_ptr(x), rows, cols, format, scaling, _ptr(codes), _ptr(scales),
                           _ptr(macro), _stream(x.device)), "mx_quantize")
    return codes, scales, macro


# host <-> device pipelining of quantize on pinned host tensors
_CHUNK_BYTES = 64 << 20
_SIDE_STREAMS = {}


def _side_streams(dev):
    if dev.index not in _SIDE_STREAMS:
        with torch.cuda.device(dev):
            _SIDE_STREAMS[dev.index] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    return _SIDE_STREAMS[dev.index]


def _quantize_host_pipelined(x, format, scaling, out, dev):
    rows, cols = _rows_cols(x)
    lead = x.shape[:-1]
    mbs = ((scaling >> 4) & 3) != 0
    mma = (scaling & MMA_SCALES) != 0
    ccols = cols // 2 if format in _PACKED else cols
    bs = block_size(format)
    if out is not None:
        _quantize_buffers(torch.device("cpu"), lead, rows, cols, format, scaling, out)
    if out is None:
        hc = torch.empty(*lead, ccols, dtype=torch.uint8, pin_memory=True)
        hs = (torch.empty(mx_scale_bytes(rows, cols, format, scaling), dtype=torch.uint8,
                          pin_memory=True) if mma else
              torch.empty(*lead, cols // bs, dtype=torch.uint8, pin_memory=True))
        hm = torch.empty(*lead, cols // 128, dtype=torch.uint8, pin_memory=True) if mbs else None
    else:
        hc, hs, hm = out
    # chunks of whole 128-row bands (tiled scales then stay contiguous per chunk)
    chunk = max(128, (_CHUNK_BYTES // max(1, cols * 2)) // 128 * 128)
    with torch.cuda.device(dev):
        cur = torch.cuda.current_stream(dev)
        s_in, s_out = _side_streams(dev)
        xd = torch.empty(rows, cols, dtype=torch.bfloat16, device=dev)
        cd = torch.empty(rows, ccols, dtype=torch.uint8, device=dev)
        sd = torch.empty(hs.numel(), dtype=torch.uint8, device=dev)
        md = torch.empty(rows, cols // 128, dtype=torch.uint8, device=dev) if mbs else None
        x2, hc2, hs1 = x.reshape(rows, cols), hc.reshape(rows, ccols), hs.reshape(-1)
        hm2 = hm.reshape(rows, cols // 128) if mbs else None
        nct = (cols // bs + 3) // 4
        s_in.wait_stream(cur)
        s_out.wait_stream(cur)
        for r0 in range(0, rows, chunk):
            r1 = min(rows, r0 + chunk)
            with torch.cuda.stream(s_in):
                xd[r0:r1].copy_(x2[r0:r1], non_blocking=True)
            cur.wait_stream(s_in)
            # scale bytes of rows [r0, r1): a contiguous range in either layout
            s0 = (r0 // 128) * nct * 512 if mma else r0 * (cols // bs)
            s1 = s0 + mx_scale_bytes(r1 - r0, cols, format, scaling)
            _check(mx_quantize(_ptr(xd[r0:r1]), r1 - r0, cols, format, scaling, _ptr(cd[r0:r1]),
                               _ptr(sd[s0:s1]), _ptr(md[r0:r1]) if mbs else None, cur.cuda_stream),
                   "mx_quantize")
            s_out.wait_stream(cur)
            with torch.cuda.stream(s_out):
                hc2[r0:r1].copy_(cd[r0:r1], non_blocking=True)
                hs1[s0:s1].copy_(sd[s0:s1], non_blocking=True)
                if mbs:
                    hm2[r0:r1].copy_(md[r0:r1], non_blocking=True)
        # The device buffers were allocated on the current stream, which now
        # waits for everything the side streams did with them (and waited for
        # every upload before the kernels): any later reuse of their memory on
        # the current stream is ordered after that work, so they need no
        # record_stream (which would keep the allocator from reusing them).
        cur.wait_stream(s_out)
    return hc, hs, hm


def _to_host(t: torch.Tensor, pinned: bool) -> torch.Tensor:
    if pinned:
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t, non_blocking=True)
        return h
    return t.cpu()


def _scales_buffer(lead, rows, cols, format, scaling, device):
    if scaling & MMA_SCALES:
        return torch.empty(mx_scale_bytes(rows, cols, format, scaling), dtype=torch.uint8,
                           device=device)
    return torch.empty(*lead, cols // block_size(format), dtype=torch.uint8, device=device)


def dequantize(codes: torch.Tensor, scales: torch.Tensor, macro=None, format: int = E2M1,
               out_dtype=torch.bfloat16, out=None, mma_scales: bool = False):
    """Inverse of ``quantize``: value(code) * f * 2^(scale - 127) as bf16 or fp32.
    ``mma_scales``: ``scales`` is in the MMA_SCALES layout."""
    if not codes.is_cuda:
        dev = torch.device("cuda", torch.cuda.current_device())
        pinned = codes.is_pinned()
        args = [None if t is None else t.to(dev, non_blocking=pinned) for t in (codes, scales, macro)]
        res = dequantize(*args, format=format, out_dtype=out_dtype, mma_scales=mma_scales)
        if out is None:
            return _to_host(res, pinned)
        out.copy_(res, non_blocking=out.is_pinned())
        return out
    if codes.dim() == 0:
        raise ValueError("codes must be at least 1-D")
    cols = codes.shape[-1] * 2 if format in _PACKED else codes.shape[-1]
    rows = codes.numel() * (2 if format in _PACKED else 1) // cols if cols else 0
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    dev = codes.device
    _check_buf(codes, "codes", dev, torch.uint8, codes.numel())
    if cols % block_size(format) == 0:
        flags = MMA_SCALES if mma_scales else 0
        _check_buf(scales, "scales", dev, torch.uint8, _scale_count(rows, cols, format, flags))
    else:
        _check_buf(scales, "scales", dev, torch.uint8, 0)   # the library rejects the shape
    if macro is not None:
        _check_buf(macro, "macro", dev, torch.uint8, rows * (cols // 128))
    if out is None:
        out = torch.empty(*codes.shape[:-1], cols, dtype=out_dtype, device=dev)
    else:
        _check_buf(out, "out", dev, out_dtype, rows * cols)
    with torch.cuda.device(codes.device):
        flags = int(out_dtype == torch.float32) | (MMA_SCALES if mma_scales else 0)
        _check(mx_dequantize(_ptr(codes), _ptr(scales), _ptr(macro), rows, cols, format,
                             flags, _ptr(out), _stream(codes.device)),
               "mx_dequantize")
    return out


def fake_quant(x: torch.Tensor, format: int = E2M1, scaling: int = FLOOR, out=None,
               return_scales: bool = False):
    """QAT forward: dequantize(quantize(x)) in one kernel, bf16 out."""
    _cuda_bf16(x, "x")
    rows, cols = _rows_cols(x)
    if out is not None:
        _check_buf(out, "out", x.device, torch.bfloat16, x.numel())
    y = torch.empty_like(x) if out is None else out
    scales = _scales_buffer(x.shape[:-1], rows, cols, format, scaling, x.device) if return_scales else None
    with torch.cuda.device(x.device):
        _check(mx_fake_quant_fwd(_ptr(x), rows, cols, format, scaling, _ptr(y), _ptr(scales),
                                 _stream(x.device)), "mx_fake_quant_fwd")
    return (y, scales) if return_scales else y


def fake_quant_bwd(x: torch.Tensor, grad_y: torch.Tensor, format: int = E2M1,
                   scaling: int = FLOOR, out=None):
    """Straight-through backward: grad_y where |x| <= maxv * X, else 0."""
    _cuda_bf16(x, "x")
    _cuda_bf16(grad_y, "grad_y")
    if grad_y.shape != x.shape:
        raise ValueError("grad_y must have the shape of x")
    if grad_y.device != x.device:
        raise ValueError(f"grad_y must be on {x.device}, got {grad_y.device}")
    rows, cols = _rows_cols(x)
    if out is not None:
        _check_buf(out, "out", x.device, torch.bfloat16, x.numel())
    gx = torch.empty_like(x) if out is None else out
    with torch.cuda.device(x.device):
        _check(mx_fake_quant_bwd(_ptr(x), _ptr(grad_y), rows, cols, format, scaling, _ptr(gx),
                                 _stream(x.device)), "mx_fake_quant_bwd")
    return gx


def block_error(x: torch.Tensor, format: int = E2M1, scaling: int = FLOOR,
                per_block: bool = True):
    """Returns (block_sse float32 [..., cols/32] or None, totals float64 [2]).

    totals = {sum (x - y)^2, sum x^2} with y the exact dequantized value;
    MSE = totals[0] / numel, SQNR = 10 log10(totals[1] / totals[0]).
    """
    _cuda_bf16(x, "x")
    rows, cols = _rows_cols(x)
    bs = (torch.empty(*x.shape[:-1], cols // block_size(format), dtype=torch.float32, device=x.device)
          if per_block else None)
    totals = torch.empty(2, dtype=torch.float64, device=x.device)
    with torch.cuda.device(x.device):
        _check(mx_block_error(_ptr(x), rows, cols, format, scaling, _ptr(bs), _ptr(totals),
                              _stream(x.device)), "mx_block_error")
    return bs, totals


def _bat_params(x, A, B, beta_min, beta_max):
    """Checks the BATQuant parameters against x; returns (a, cols)."""
    rows, cols = _rows_cols(x)
    for name, t in (("A", A), ("B", B), ("beta_min", beta_min), ("beta_max", beta_max)):
        if t is None:
            continue
        if t.dtype != torch.float32 or not t.is_contiguous() or t.device != x.device:
            raise ValueError(f"{name} must be a contiguous float32 tensor on {x.device}")
    a = A.shape[0] if A.dim() == 2 else -1
    if A.dim() != 2 or A.shape[1] != a or a not in (1, 2, 4, 8, 16, 32):
        raise ValueError("A must be [a, a] with a in 1, 2, 4, 8, 16, 32")
    b = 32 // a
    if tuple(B.shape) != (cols // 32, b, b):
        raise ValueError(f"B must be [cols/32, {b}, {b}], got {tuple(B.shape)}")
    if (beta_min is None) != (beta_max is None):
        raise ValueError("give both clip thresholds or neither")
    if beta_min is not None and (beta_min.numel() != cols // 32 or beta_max.numel() != cols // 32):
        raise ValueError("beta_min / beta_max must hold cols/32 values")
    return a


def bat_apply(x: torch.Tensor, A: torch.Tensor, B: torch.Tensor, beta_min=None, beta_max=None,
              out=None):
    """BATQuant apply step: each 32-element block j of every row times
    B[j] (x) A, clipped to [beta_min[j] min, beta_max[j] max] of the block,
    as bf16 (see mx_bat_apply in include/mx.h for the exact arithmetic)."""
    _cuda_bf16(x, "x")
    rows, cols = _rows_cols(x)
    a = _bat_params(x, A, B, beta_min, beta_max)
    if out is not None:
        _check_buf(out, "out", x.device, torch.bfloat16, x.numel())
    y = torch.empty_like(x) if out is None else out
    with torch.cuda.device(x.device):
        _check(mx_bat_apply(_ptr(x), rows, cols, a, _ptr(A), _ptr(B), _ptr(beta_min), _ptr(beta_max),
                            _ptr(y), _stream(x.device)), "mx_bat_apply")
    return y


def bat_quantize(x: torch.Tensor, A: torch.Tensor, B: torch.Tensor, beta_min=None, beta_max=None,
                 format: int = E2M1, scaling: int = FLOOR, out=None):
    """BATQuant: bat_apply fused with quantize in one kernel; returns what
    quantize returns for the transformed rows."""
    _cuda_bf16(x, "x")
    rows, cols = _rows_cols(x)
    a = _bat_params(x, A, B, beta_min, beta_max)
    codes, scales, macro = _quantize_buffers(x.device, x.shape[:-1], rows, cols, format, scaling,
                                             out)
    with torch.cuda.device(x.device):
        _check(mx_bat_quantize(_ptr(x), rows, cols, a, _ptr(A), _ptr(B), _ptr(beta_min),
                               _ptr(beta_max), format, scaling, _ptr(codes), _ptr(scales),
                               _ptr(macro), _stream(x.device)), "mx_bat_quantize")
    return codes, scales, macro


class MXFakeQuantize(torch.autograd.Function):
    """y = fake_quant(x) with the straight-through gradient of the forward's mask."""

    @staticmethod
    def forward(ctx, x, format=E2M1, scaling=FLOOR):
        ctx.save_for_backward(x)
        ctx.format = format
        ctx.scaling = scaling
        return fake_quant(x.contiguous(), format, scaling)

    @staticmethod
    def backward(ctx, grad_y):
        (x,) = ctx.saved_tensors
        gx = fake_quant_bwd(x.contiguous(), grad_y.contiguous(), ctx.format, ctx.scaling)
        return gx, None, None


# ---------------------------------------------------- block-scaled GEMM --

def _gemm_operand_b(b_codes, b_scales, K, device):
    """B: MXFP4 codes [N, K/2] and its scales in the MMA_SCALES layout."""
    if b_codes.dim() != 2 or b_codes.shape[1] * 2 != K:
        raise ValueError(f"b_codes must be [N, K/2] = [N, {K // 2}]")
    N = b_codes.shape[0]
    _check_buf(b_codes, "b_codes", device, torch.uint8, N * (K // 2))
    _check_buf(b_scales, "b_scales", device, torch.uint8,
               max(0, mx_scale_bytes(N, K, E2M1, MMA_SCALES)))
    return N


def _gemm_out(M, N, out_dtype, out, device):
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    if out is None:
        return torch.empty(M, N, dtype=out_dtype, device=device)
    _check_buf(out, "out", device, out_dtype, M * N)
    return out


def _gemm_status(status, device):
    if status is None:
        return None
    _check_buf(status, "status", device, torch.int32, 1)
    return status


def gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor,
         b_scales: torch.Tensor, out_dtype=torch.bfloat16, out=None, status=None):
    """D = A B^T on the tensor cores, A [M, K] and B [N, K] both MXFP4: codes
    (as ``quantize`` writes them) and scales in the MMA_SCALES layout.
    ``status``: an optional int32 device tensor the kernel sets nonzero if one
    of its waits timed out. Returns D [M, N] (bf16 or float32)."""
    if not a_codes.is_cuda:
        raise ValueError("a_codes must be a CUDA tensor")
    dev = a_codes.device
    if a_codes.dim() != 2:
        raise ValueError("a_codes must be [M, K/2]")
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    _check_buf(a_codes, "a_codes", dev, torch.uint8, M * (K // 2))
    _check_buf(a_scales, "a_scales", dev, torch.uint8, max(0, mx_scale_bytes(M, K, E2M1, MMA_SCALES)))
    N = _gemm_operand_b(b_codes, b_scales, K, dev)
    d = _gemm_out(M, N, out_dtype, out, dev)
    st = _gemm_status(status, dev)
    with torch.cuda.device(dev):
        _check(mx_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K,
                       int(out_dtype == torch.float32), _ptr(d), _ptr(st), _stream(dev)), "mx_gemm")
    return d


def quant_gemm(a: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor,
               scaling: int = FLOOR, out_dtype=torch.bfloat16, out=None, a_out=None, status=None,
               on_chip: bool = False):
    """D = MXFP4(a) B^T with bf16 ``a`` [M, K] quantized within the same
    launch (``scaling``: FLOOR, CEIL, OAS_RULE or OAS). ``a_out`` = (codes
    [M, K/2], tiled scales) also receives A's quantized form when given.
    ``on_chip``: quantize inside the GEMM's prologue (thread-block clusters)
    instead of staging A through L2. Returns D."""
    _cuda_bf16(a, "a")
    if a.dim() != 2:
        raise ValueError("a must be [M, K]")
    M, K = a.shape
    dev = a.device
    N = _gemm_operand_b(b_codes, b_scales, K, dev)
    d = _gemm_out(M, N, out_dtype, out, dev)
    ac = asc = None
    if a_out is not None:
        ac, asc = a_out
        _check_buf(ac, "a_out codes", dev, torch.uint8, M * (K // 2))
        _check_buf(asc, "a_out scales", dev, torch.uint8, max(0, mx_scale_bytes(M, K, E2M1, MMA_SCALES)))
    st = _gemm_status(status, dev)
    with torch.cuda.device(dev):
        flags = int(out_dtype == torch.float32) | (GEMM_A_ON_CHIP if on_chip else 0)
        _check(mx_quant_gemm(_ptr(a), scaling, _ptr(b_codes), _ptr(b_scales), M, N, K, flags,
                             _ptr(d), _ptr(ac), _ptr(asc), _ptr(st), _stream(dev)),
               "mx_quant_gemm")
    return d
