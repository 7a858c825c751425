"""The C ABI on a host without a GPU: the library loads, exports every symbol
include/mx.h declares, and rejects bad arguments before touching CUDA.

Every call here fails validation (or is empty) and returns before any CUDA
call, so no kernel is launched; the fake device addresses are never
dereferenced.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mx.h")

OK, INVALID, SHAPE, ALIGN, UNSUPPORTED, CUDA_ERR = 0, 1, 2, 3, 4, 5
A = 0x10000          # a 256-byte aligned fake device address (never dereferenced)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mx_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("mx_quantize", "mx_dequantize", "mx_fake_quant_fwd", "mx_fake_quant_bwd",
              "mx_block_error", "mx_status_string", "mx_version"):
        assert n in names


def test_library_exports_every_declared_symbol(mx):
    lib = ctypes.CDLL(mx.library_path())
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(mx):
    for s in range(7):
        assert mx.mx_status_string(s)
    assert mx.mx_status_string(99) == "unknown status"
    assert mx.mx_version() >> 16 == 1


def test_product_does_not_use_the_oracle():
    """The package neither imports the oracle nor includes or loads its code."""
    pkg = os.path.join(ROOT, "fp8_quantization_mx_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith(".py"):
                text = open(path).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "libmx_oracle" not in text and "mx_oracle" not in text, f
            if f.endswith((".cu", ".cuh", ".h", ".cpp")):
                text = open(path).read()
                assert "oracle" not in text, f


@pytest.mark.parametrize("fmt,scaling,status", [
    (8, 0, UNSUPPORTED), (0, 4, UNSUPPORTED), (0, 0x30, UNSUPPORTED), (0, 0x40, UNSUPPORTED),
    # block-16 formats: MXFP4-B16 has no MBS, NVFP4 has its one rule
    (6, 0x11, UNSUPPORTED), (6, 0x12, UNSUPPORTED), (7, 1, UNSUPPORTED), (7, 3, UNSUPPORTED),
    (7, 0x10, UNSUPPORTED),
    (1, 2, UNSUPPORTED), (1, 0x10, UNSUPPORTED), (0, 0x11, UNSUPPORTED),
    (0, 0x12, UNSUPPORTED), (-1, 0, UNSUPPORTED), (0, -1, UNSUPPORTED),
    # one-byte formats: no OAS_RULE, no macro blocks; INT8 has no OAS
    (2, 2, UNSUPPORTED), (3, 0x20, UNSUPPORTED), (4, 0x13, UNSUPPORTED), (5, 3, UNSUPPORTED),
    (5, 2, UNSUPPORTED), (2, 0x10, UNSUPPORTED),
])
def test_quantize_rejects_modes(mx, fmt, scaling, status):
    assert mx.mx_quantize(A, 4, 128, fmt, scaling, A, A, A, 0) == status


def test_quantize_rejects_shapes_and_pointers(mx):
    q = mx.mx_quantize
    assert q(A, 4, 33, 0, 0, A, A, None, 0) == SHAPE
    assert q(A, 4, 96, 0, 0x10, A, A, A, 0) == SHAPE        # MBS needs cols % 128
    assert q(A, -1, 32, 0, 0, A, A, None, 0) == INVALID
    assert q(A, 4, -32, 0, 0, A, A, None, 0) == INVALID
    assert q(A, 1 << 40, 1 << 10, 0, 0, A, A, None, 0) == INVALID   # too many elements
    assert q(None, 4, 32, 0, 0, A, A, None, 0) == INVALID
    assert q(A, 4, 32, 0, 0, None, A, None, 0) == INVALID
    assert q(A, 4, 32, 0, 0, A, None, None, 0) == INVALID
    assert q(A, 4, 128, 0, 0x10, A, A, None, 0) == INVALID   # MBS needs macro
    assert q(A + 8, 4, 32, 0, 0, A, A, None, 0) == ALIGN
    assert q(A + 16, 4, 32, 0, 0, A, A, None, 0) == ALIGN     # x needs 32 bytes
    assert q(A, 4, 32, 0, 0, A + 4, A, None, 0) == ALIGN
    assert q(A, 4, 32, 0, 0, A + 8, A, None, 0) == ALIGN      # codes need 16
    # scales and macro may sit at any byte address: this one only fails on x
    assert q(A + 2, 4, 128, 0, 0x10, A, A + 1, A + 3, 0) == ALIGN
    # empty inputs are valid and launch nothing (pointers are not needed)
    assert q(None, 0, 32, 0, 0, None, None, None, 0) == OK
    assert q(None, 5, 0, 0, 0, None, None, None, 0) == OK


def test_other_entry_points_validate(mx):
    assert mx.mx_dequantize(A, A, None, 4, 33, 0, 0, A, 0) == SHAPE
    assert mx.mx_dequantize(A, A, A, 4, 96, 0, 0, A, 0) == SHAPE
    assert mx.mx_dequantize(A, A, A, 4, 128, 1, 0, A, 0) == UNSUPPORTED   # FP8 has no MBS
    assert mx.mx_dequantize(A, A, None, 4, 32, 0, 2, A, 0) == INVALID
    assert mx.mx_dequantize(A, A, None, 4, 32, 8, 0, A, 0) == UNSUPPORTED
    assert mx.mx_dequantize(A, A, None, 4, 24, 7, 0, A, 0) == SHAPE       # NVFP4: cols % 16
    assert mx.mx_quantize(A, 4, 24, 6, 0, A, A, None, 0) == SHAPE
    assert mx.mx_dequantize(A, A, A, 4, 128, 5, 0, A, 0) == UNSUPPORTED   # only FP4 has MBS
    assert mx.mx_dequantize(A + 8, A, None, 4, 32, 0, 0, A, 0) == ALIGN
    assert mx.mx_dequantize(A, None, None, 4, 32, 0, 0, A, 0) == INVALID
    assert mx.mx_dequantize(None, None, None, 0, 32, 0, 0, None, 0) == OK
    assert mx.mx_fake_quant_fwd(A, 4, 32, 5, 3, A, None, 0) == UNSUPPORTED
    assert mx.mx_fake_quant_fwd(A, 4, 48, 0, 0, A, None, 0) == SHAPE
    assert mx.mx_fake_quant_fwd(A, 4, 32, 0, 0, None, None, 0) == INVALID
    assert mx.mx_fake_quant_fwd(A, 4, 32, 0, 0, A + 8, None, 0) == ALIGN
    assert mx.mx_fake_quant_fwd(A, 4, 32, 0, 0, A + 16, None, 0) == ALIGN
    assert mx.mx_dequantize(A, A, None, 4, 32, 0, 0, A + 16, 0) == ALIGN
    assert mx.mx_fake_quant_bwd(A, A, 4, 32, 0, 0, A + 8, 0) == ALIGN
    assert mx.mx_fake_quant_bwd(A, None, 4, 32, 0, 0, A, 0) == INVALID
    assert mx.mx_fake_quant_bwd(A, A, 4, 64, 0, 0x20, A, 0) == SHAPE
    assert mx.mx_block_error(A, 4, 32, 0, 0, None, None, 0) == INVALID
    assert mx.mx_block_error(A, 4, 32, 0, 0, None, A + 4, 0) == ALIGN
    assert mx.mx_block_error(A, 4, 32, 0, 0, A + 2, A, 0) == ALIGN
    assert mx.mx_block_error(A, 4, 32, 1, 0x20, None, A, 0) == UNSUPPORTED


def test_gemm_entry_points_validate(mx):
    """Both GEMM entry points check shapes, flags and alignment before any
    CUDA call; the on-chip flag is taken off out_fp32 before the check."""
    on_chip = mx.GEMM_A_ON_CHIP
    g, q = mx.mx_gemm, mx.mx_quant_gemm
    assert g(A, A, A, A, 128, 64, 384, 0, A, None, 0) == SHAPE                  # K % 256
    assert g(A, A, A, A, 128, 60, 256, 0, A, None, 0) == SHAPE                  # N % 8
    assert g(A, A, A, A, 128, 64, 256, 2, A, None, 0) == INVALID                # out_fp32
    assert g(A, A, A, A, 128, 64, 256, on_chip, A, None, 0) == INVALID          # no flag here
    assert g(A + 8, A, A, A, 128, 64, 256, 0, A, None, 0) == ALIGN              # codes: 16 B
    assert g(A, None, A, A, 128, 64, 256, 0, A, None, 0) == INVALID
    assert g(A, A, A, A, -1, 64, 256, 0, A, None, 0) == INVALID
    assert g(None, None, None, None, 0, 64, 256, 0, None, None, 0) == OK         # M == 0
    assert q(A, 0x10, A, A, 128, 64, 256, 0, A, None, None, None, 0) == UNSUPPORTED   # MBS
    assert q(A, 0, A, A, 128, 64, 384, on_chip, A, None, None, None, 0) == SHAPE
    assert q(A, 0, A, A, 128, 64, 256, 2 | on_chip, A, None, None, None, 0) == INVALID
    assert q(A + 16, 0, A, A, 128, 64, 256, on_chip | 1, A, None, None, None, 0) == ALIGN
    assert q(A, 0, A, A, 128, 64, 256, 0, A, A + 8, None, None, 0) == ALIGN     # codes out
    assert q(A, 0, A, A, 128, 64, 256, 0, A, None, A + 8, None, 0) == ALIGN     # scales out
    assert q(A, 0, A, A, 128, 64, 256, 0, A, None, None, A + 2, 0) == ALIGN     # status


def test_noalloc_quant_gemm_validates_and_refuses_what_its_scratch_cannot_hold(mx):
    """The no-allocation quantize + GEMM checks its arguments like mx_quant_gemm
    and refuses problems whose scratch exceeds its fixed array, before any
    CUDA call."""
    TOO_LARGE = 6
    f = mx.mx_quant_gemm_noalloc
    assert f(A, 0, A, A, 8192, 64, 8192, 0, A, None, 0) == TOO_LARGE      # 32 MiB of codes
    assert f(A, 0, A, A, 1, 64, 2 ** 22, 0, A, None, 0) == TOO_LARGE      # one padded band of scales
    assert f(A, 0x10, A, A, 128, 64, 256, 0, A, None, 0) == UNSUPPORTED   # MBS: no
    assert f(A, 0, A, A, 128, 60, 256, 0, A, None, 0) == SHAPE            # N % 8
    assert f(A, 0, A, A, 128, 64, 384, 0, A, None, 0) == SHAPE            # K % 256
    assert f(A, 0, A, A, 128, 64, 256, 1 << 9, A, None, 0) == INVALID     # no on-chip flag
    assert f(A + 16, 0, A, A, 128, 64, 256, 0, A, None, 0) == ALIGN       # bf16 A: 32 bytes
    assert f(None, 0, A, A, 128, 64, 256, 0, A, None, 0) == INVALID
    assert f(A, 0, A, A, 0, 64, 256, 0, None, None, 0) == OK              # M == 0: nothing


def test_binding_refuses_cpu_tensors_for_device_only_calls(mx):
    import torch
    x = torch.zeros(2, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mx.fake_quant(x)
    with pytest.raises(ValueError):
        mx.block_error(x)


def test_scale_bytes_and_mma_layout_flag(mx):
    MMA = 1 << 8
    sb = lambda r, c, s, f=0: mx.mx_scale_bytes(r, c, f, s)
    assert sb(4, 128, 0) == 16
    assert sb(4, 128, MMA) == 128 * 4                  # one 128 x 4 tile
    assert sb(300, 224, MMA) == 384 * 8                # rows -> 384, 7 block columns -> 8
    assert sb(256, 512, MMA | 3) == 256 * 16
    assert sb(0, 64, MMA) == 0
    assert sb(4, 33, MMA) == -1 and sb(-1, 32, 0) == -1
    assert sb(4, 48, 0, 7) == 12 and sb(4, 48, 0, 1) == -1   # block 16 (NVFP4) vs 32
    assert sb(4, 48, MMA, 6) == 128 * 4 and sb(4, 32, 0, 8) == -1
    # the flag is accepted by quantize / fake-quant (checked before any launch) ...
    assert mx.mx_quantize(A, 4, 33, 0, MMA, A, A, None, 0) == SHAPE
    assert mx.mx_quantize(None, 0, 32, 1, MMA | 1, None, None, None, 0) == OK
    assert mx.mx_quantize(A, 4, 128, 0, MMA | 0x200, A, A, A, 0) == UNSUPPORTED
    # ... and by dequantize as a flags bit; block error has no scale output
    assert mx.mx_dequantize(A, A, None, 4, 33, 0, MMA | 1, A, 0) == SHAPE
    assert mx.mx_dequantize(A, A, None, 4, 32, 0, MMA | 2, A, 0) == INVALID
    assert mx.mx_block_error(A, 4, 32, 0, MMA, None, A, 0) == UNSUPPORTED


def test_bat_entry_points_validate(mx):
    ap, qz = mx.mx_bat_apply, mx.mx_bat_quantize
    # a must divide 32 as a power of two
    for bad in (0, 3, 64, -1):
        assert ap(A, 4, 32, bad, A, A, None, None, A, 0) == INVALID
        assert qz(A, 4, 32, bad, A, A, None, None, 0, 0, A, A, None, 0) == INVALID
    assert ap(A, 4, 48, 8, A, A, None, None, A, 0) == SHAPE
    assert ap(A, 4, 32, 8, None, A, None, None, A, 0) == INVALID
    assert ap(A, 4, 32, 8, A, None, None, None, A, 0) == INVALID
    assert ap(A, 4, 32, 8, A, A, A, None, A, 0) == INVALID        # one threshold array alone
    assert ap(A, 4, 32, 8, A, A, None, A, A, 0) == INVALID
    assert ap(A, 4, 32, 8, A + 4, A, None, None, A, 0) == ALIGN   # A, B: 16 bytes
    assert ap(A, 4, 32, 8, A, A + 8, None, None, A, 0) == ALIGN
    assert ap(A, 4, 32, 8, A, A, A + 2, A, A, 0) == ALIGN        # thresholds: 4 bytes
    assert ap(A + 16, 4, 32, 8, A, A, None, None, A, 0) == ALIGN
    assert ap(A, 4, 32, 8, A, A, None, None, A + 16, 0) == ALIGN
    assert ap(A, 4, 32, 8, A, A, None, None, None, 0) == INVALID
    assert ap(None, 0, 32, 8, None, None, None, None, None, 0) == OK
    # quantize: 32-element formats, no MBS-Dynamic; the mx_quantize mode rules
    assert qz(A, 4, 128, 8, A, A, None, None, 6, 0, A, A, None, 0) == UNSUPPORTED
    assert qz(A, 4, 128, 8, A, A, None, None, 7, 0, A, A, None, 0) == UNSUPPORTED
    assert qz(A, 4, 128, 8, A, A, None, None, 0, 0x20, A, A, A, 0) == UNSUPPORTED
    assert qz(A, 4, 128, 8, A, A, None, None, 0, 0x23, A, A, A, 0) == UNSUPPORTED
    assert qz(A, 4, 128, 8, A, A, None, None, 5, 3, A, A, None, 0) == UNSUPPORTED
    assert qz(A, 4, 96, 8, A, A, None, None, 0, 0x10, A, A, A, 0) == SHAPE
    assert qz(A, 4, 128, 8, A, A, None, None, 0, 0x10, A, A, None, 0) == INVALID
    assert qz(A, 4, 128, 8, A, A, None, None, 0, 0, A + 8, A, None, 0) == ALIGN
    assert qz(A, 4, 128, 8, None, A, None, None, 0, 0, A, A, None, 0) == INVALID
    assert qz(None, 0, 128, 8, None, None, None, None, 0, 0, None, None, None, 0) == OK


# -------------------------------------------- caller-supplied buffers ----

def test_binding_checks_every_output_buffer(mx):
    """Buffers passed as ``out`` are checked (device, dtype, contiguity,
    size) before the C call: the kernels write through their raw pointers.
    The checks run here against CPU tensors, with ``meta`` tensors standing
    in for a buffer on the wrong device; nothing is launched."""
    import torch
    cpu = torch.device("cpu")
    u8 = lambda *s: torch.zeros(*s, dtype=torch.uint8)
    lead, rows, cols = (4,), 4, 256
    chk = lambda out, fmt=0, sc=0: mx._quantize_buffers(cpu, lead, rows, cols, fmt, sc, out)
    chk((u8(4, 128), u8(4, 8), None))                              # exact sizes pass
    chk((u8(4, 128), u8(4, 8), u8(4, 2)), 0, mx.MBS_STATIC)
    chk((u8(4, 256), u8(4, 8), None), mx.E4M3)
    chk((u8(512), u8(1024), None), 0, mx.MMA_SCALES)               # two padded 128 x 4 tiles
    bad = [
        ((u8(4, 127), u8(4, 8), None), 0, 0),                      # codes one byte short
        ((u8(4, 128), u8(4, 7), None), 0, 0),                      # scales short
        ((u8(4, 128), u8(1023), None), 0, mx.MMA_SCALES),          # tiled scales need 1024
        ((u8(4, 128), u8(4, 8), None), 0, mx.MBS_STATIC),          # macro missing
        ((u8(4, 128), u8(4, 8), u8(4, 1)), 0, mx.MBS_DYNAMIC),     # macro short
        ((u8(4, 128), u8(4, 8), None), mx.E4M3, 0),                # FP8 codes are 1 B/elem
        ((torch.zeros(4, 128, dtype=torch.int16), u8(4, 8), None), 0, 0),
        ((u8(4, 256)[:, ::2], u8(4, 8), None), 0, 0),              # not contiguous
        ((torch.empty(4, 128, dtype=torch.uint8, device="meta"), u8(4, 8), None), 0, 0),
        ((u8(4, 128), u8(4, 8)), 0, 0),                            # not a triple
    ]
    for out, fmt, sc in bad:
        with pytest.raises(ValueError):
            chk(out, fmt, sc)
    with pytest.raises(ValueError):
        mx._check_buf(torch.zeros(8, dtype=torch.bfloat16), "out", cpu, torch.float32, 8)
    with pytest.raises(ValueError):
        mx._check_buf(torch.zeros(7, dtype=torch.float32), "out", cpu, torch.float32, 8)
    mx._check_buf(torch.zeros(8, dtype=torch.float32), "out", cpu, torch.float32, 8)


def test_binding_checks_host_path_buffers(mx):
    """A CPU input with CPU ``out`` buffers: the same checks, before any copy."""
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    short = (torch.zeros(4, 31, dtype=torch.uint8), torch.zeros(4, 2, dtype=torch.uint8), None)
    with pytest.raises(ValueError):
        mx.quantize(x, out=short)


def test_launch_failure_returns_mx_err_cuda(mx):
    """With no CUDA device visible, a call that passes validation fails at its
    first CUDA runtime call and returns MX_ERR_CUDA (nothing is written; the
    fake addresses are never dereferenced because no kernel can start). Runs
    in a child process that sees no device, on a host with or without GPUs."""
    import subprocess
    import sys
    code = (
        "import ctypes, sys\n"
        f"lib = ctypes.CDLL({mx.library_path()!r})\n"
        "vp, i64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int\n"
        "lib.mx_quantize.argtypes = [vp, i64, i64, ci, ci, vp, vp, vp, vp]\n"
        "lib.mx_block_error.argtypes = [vp, i64, i64, ci, ci, vp, vp, vp]\n"
        "lib.mx_dequantize.argtypes = [vp, vp, vp, i64, i64, ci, ci, vp, vp]\n"
        f"A = {A}\n"
        "print(lib.mx_quantize(A, 4, 128, 0, 0, A, A, None, None),\n"
        "      lib.mx_quantize(A, 4, 128, 0, 3 | 256, A, A, None, None),\n"
        "      lib.mx_block_error(A, 4, 128, 0, 0, None, A, None),\n"
        "      lib.mx_dequantize(A, A, None, 4, 128, 1, 0, A, None))\n")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split() == [str(CUDA_ERR)] * 4
