"""The MMA_SCALES layout: E8M0 bytes in the tiled order block-scaled tensor-core
GEMMs consume on sm_100.

* The layout is restated here from its definition, independently of the
  kernels: 128-row x 4-block-column tiles of 512 bytes, row-major over the
  tiles, and inside a tile the byte (r % 32) * 16 + (r / 32 % 4) * 4 + j % 4,
  zero padding. The kernels' bytes must be the oracle's plain scales moved
  there, with the padding cleared.
* A library block-scaled GEMM (torch's scaled_mm with 1x32 E8M0 block scaling,
  which runs cuBLASLt's MX kernels on sm_100) fed with our codes and scales
  must reproduce dequantize(A) @ dequantize(B)^T. That pins the layout to what
  the hardware reads, not just to our reading of it.
"""

import numpy as np
import pytest
import torch

from fp8_quantization_mx_b200 import inputs

pytestmark = pytest.mark.gpu

E2M1, E4M3, E5M2, E2M3, INT8 = 0, 1, 2, 4, 5
FLOOR, CEIL, OAS = 0, 1, 3
MMA = 1 << 8


def tiled(plain, rows, cols):
    """Plain [rows, cols/32] scale bytes -> the tiled layout (numpy restatement)."""
    bpr = cols // 32
    rt, ct = -(-rows // 128), -(-bpr // 4)
    out = np.zeros(rt * ct * 512, np.uint8)
    r = np.arange(rows)[:, None]
    j = np.arange(bpr)[None, :]
    off = ((r // 128) * ct + j // 4) * 512 + (r % 32) * 16 + (r // 32 % 4) * 4 + j % 4
    out[off.ravel()] = plain.reshape(rows, bpr).ravel()
    return out


@pytest.mark.parametrize("shape", [(300, 224), (128, 128), (256, 2048), (5, 96)])
@pytest.mark.parametrize("fm", [(E2M1, FLOOR), (E2M1, OAS | 16), (E4M3, OAS), (E2M3, CEIL),
                                (INT8, FLOOR)])
def test_tiled_scales_are_the_plain_ones_moved(mx, oracle_mod, cuda, shape, fm):
    rows, cols = shape
    fmt, m = fm
    if (m >> 4) and cols % 128:
        pytest.skip("MBS needs cols % 128 == 0")
    x = inputs.random_bf16_bits((rows, cols), seed=rows + cols).to(cuda)
    n = mx.mx_scale_bytes(rows, cols, fmt, MMA)
    # canary-filled buffer: the padding must come back as zeros
    sbuf = torch.full((n,), 0xA5, dtype=torch.uint8, device=cuda)
    codes = torch.empty(rows, cols // 2 if fmt == E2M1 else cols, dtype=torch.uint8, device=cuda)
    mac = torch.empty(rows, cols // 128, dtype=torch.uint8, device=cuda) if m >> 4 else None
    mx.quantize(x, fmt, m | MMA, out=(codes, sbuf, mac))
    y_t = mx.dequantize(codes, sbuf, mac, fmt, mma_scales=True)
    c_p, s_p, _ = mx.quantize(x, fmt, m)
    y_p = mx.dequantize(c_p, s_p, mac, fmt)
    yf, sf = mx.fake_quant(x, fmt, m | MMA, return_scales=True)
    torch.cuda.synchronize()
    oc, os_, _ = oracle_mod.quantize(inputs.bf16_bits_numpy(x.cpu()), fmt, m)
    want = tiled(os_, rows, cols)
    assert np.array_equal(sbuf.cpu().numpy(), want)
    assert np.array_equal(sf.cpu().numpy(), want)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert torch.equal(y_t, y_p)


def _scaled_mm_or_skip(a, b, sa, sb):
    F = torch.nn.functional
    try:
        return F.scaled_mm(a, b, sa, F.ScalingType.BlockWise1x32, sb, F.ScalingType.BlockWise1x32,
                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                           swizzle_b=F.SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.bfloat16)
    except (RuntimeError, NotImplementedError, TypeError) as e:
        pytest.skip(f"block-scaled scaled_mm unavailable here: {str(e).splitlines()[0][:160]}")


@pytest.mark.parametrize("M,N,K", [(256, 384, 512), (200, 128, 1024)])
def test_mxfp8_tiled_scales_drive_a_block_scaled_gemm(mx, cuda, M, N, K):
    a = (inputs.normal_weight(M, K, seed=7, device=cuda, std=1.0))
    b = (inputs.normal_weight(N, K, seed=8, device=cuda, std=0.05))
    ca, sa, _ = mx.quantize(a, E4M3, FLOOR | MMA)
    cb, sb, _ = mx.quantize(b, E4M3, FLOOR | MMA)
    out = _scaled_mm_or_skip(ca.view(torch.float8_e4m3fn), cb.view(torch.float8_e4m3fn).t(),
                             sa.view(torch.float8_e8m0fnu), sb.view(torch.float8_e8m0fnu))
    ya = mx.dequantize(ca, sa, None, E4M3, torch.float32, mma_scales=True)
    yb = mx.dequantize(cb, sb, None, E4M3, torch.float32, mma_scales=True)
    torch.cuda.synchronize()
    ref = ya.double().cpu() @ yb.double().cpu().t()
    got = out.double().cpu()
    tol = 1e-2 * ref.abs().max().item()
    assert (got - ref).abs().max().item() <= tol
    # bf16 output rounding gives ~0.1-0.2% on average; a wrong layout, which
    # pairs most blocks with another block's scale, gives errors of order 100%
    assert (got - ref).abs().mean().item() <= 1e-2 * ref.abs().mean().item()


def test_mxfp4_tiled_scales_drive_a_block_scaled_gemm(mx, cuda):
    M, N, K = 256, 256, 512
    a = inputs.normal_weight(M, K, seed=9, device=cuda, std=1.0)
    b = inputs.normal_weight(N, K, seed=10, device=cuda, std=1.0)
    ca, sa, _ = mx.quantize(a, E2M1, FLOOR | MMA)
    cb, sb, _ = mx.quantize(b, E2M1, FLOOR | MMA)
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("no packed FP4 dtype in this torch")
    out = _scaled_mm_or_skip(ca.view(torch.float4_e2m1fn_x2), cb.view(torch.float4_e2m1fn_x2).t(),
                             sa.view(torch.float8_e8m0fnu), sb.view(torch.float8_e8m0fnu))
    ya = mx.dequantize(ca, sa, None, E2M1, torch.float32, mma_scales=True)
    yb = mx.dequantize(cb, sb, None, E2M1, torch.float32, mma_scales=True)
    torch.cuda.synchronize()
    ref = ya.double().cpu() @ yb.double().cpu().t()
    got = out.double().cpu()
    assert (got - ref).abs().max().item() <= 1e-2 * ref.abs().max().item()
    assert (got - ref).abs().mean().item() <= 1e-2 * ref.abs().mean().item()


def test_nvfp4_tiled_scales_drive_a_block_scaled_gemm(mx, cuda):
    """NVFP4 (E2M1, block 16, E4M3 scales) through the library's single-level
    1x16 block-scaled GEMM: checks the encoding and the layout at block 16."""
    NVFP4 = 7
    M, N, K = 256, 128, 512
    a = inputs.normal_weight(M, K, seed=11, device=cuda, std=1.0)
    b = inputs.normal_weight(N, K, seed=12, device=cuda, std=1.0)
    ca, sa, _ = mx.quantize(a, NVFP4, FLOOR | MMA)
    cb, sb, _ = mx.quantize(b, NVFP4, FLOOR | MMA)
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("no packed FP4 dtype in this torch")
    F = torch.nn.functional
    try:
        out = F.scaled_mm(ca.view(torch.float4_e2m1fn_x2), cb.view(torch.float4_e2m1fn_x2).t(),
                          sa.view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                          sb.view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                          swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                          swizzle_b=F.SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.bfloat16)
    except (RuntimeError, NotImplementedError, TypeError) as e:
        pytest.skip(f"NVFP4 scaled_mm unavailable here: {str(e).splitlines()[0][:160]}")
    ya = mx.dequantize(ca, sa, None, NVFP4, torch.float32, mma_scales=True)
    yb = mx.dequantize(cb, sb, None, NVFP4, torch.float32, mma_scales=True)
    torch.cuda.synchronize()
    ref = ya.double().cpu() @ yb.double().cpu().t()
    got = out.double().cpu()
    assert (got - ref).abs().max().item() <= 1e-2 * ref.abs().max().item()
    assert (got - ref).abs().mean().item() <= 1e-2 * ref.abs().mean().item()
