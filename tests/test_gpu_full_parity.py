"""Whole-tensor parity at the workload sizes: every output of the CUDA path
(through the C ABI) against the CPU oracle on the same seeded tensors.

Codes, scale bytes, macro factors, dequantized values, fake-quant outputs and
straight-through gradients are compared bit for bit over the whole tensor;
per-block squared errors and the totals {sum d^2, sum x^2} (hence MSE and
SQNR) within a relative 1e-6. The one exception is MBS-Dynamic, whose oracle
evaluates all 256 factors element by element (about 3 CPU-minutes for the
8192 x 4096 tensor): the GPU still runs the whole tensor, and 256 rows spread
over it are compared.

Workloads (fp8_quantization_mx_b200.inputs):
  mlp_weight   bf16 [8192, 3072], N(0, 0.02^2): MXFP8 and the other one-byte
               formats, quantize and dequantize
  qat_act      bf16 [16384, 3072], Student-t(3) * 0.5, and qat_weight bf16
               [8192, 3072], N(0, 0.02^2): MXFP4 fake-quant forward and
               straight-through backward (and the block-16 formats on qat_act)
  heavy_tail   bf16 [8192, 4096], N(0, 1) with 16 outlier channels x100 and
               0.05% spikes x20: MXFP4 under every scaling mode, quantize,
               dequantize and block error
  moe_w13      bf16 [128, 1536, 2048] (403M elements), N(0, 0.02^2) with
               per-expert U(0.5, 2) scales: MXFP4 quantize and dequantize
"""

import os

import numpy as np
import pytest
import torch

from fp8_quantization_mx_b200 import inputs

pytestmark = pytest.mark.gpu

E2M1, E4M3, E5M2, E3M2, E2M3, INT8, E2M1_B16, NVFP4 = 0, 1, 2, 3, 4, 5, 6, 7
FLOOR, CEIL, OAS_RULE, OAS = 0, 1, 2, 3
MBS_STATIC, MBS_DYNAMIC = 16, 32
BYTE_FMTS = [E4M3, E5M2, E3M2, E2M3, INT8]
FMT_NAMES = {E2M1: "fp4", E4M3: "e4m3", E5M2: "e5m2", E3M2: "e3m2", E2M3: "e2m3", INT8: "int8",
             E2M1_B16: "fp4b16", NVFP4: "nvfp4"}
MODE_NAMES = {FLOOR: "FLOOR", CEIL: "CEIL", OAS_RULE: "OAS_RULE", OAS: "OAS",
              MBS_STATIC: "MBS_STATIC", OAS | MBS_STATIC: "OAS+MBS_STATIC",
              MBS_DYNAMIC: "MBS_DYNAMIC", OAS | MBS_DYNAMIC: "OAS+MBS_DYNAMIC"}
REL = 1e-6


def bits(t):
    return inputs.bf16_bits_numpy(t)


def host(t):
    return t.detach().cpu().numpy()


@pytest.fixture(scope="module")
def oracle_all(oracle_mod):
    """The oracle on every host core for the duration of this module."""
    before = oracle_mod.get_threads()
    oracle_mod.set_threads(len(os.sched_getaffinity(0)))
    yield oracle_mod
    oracle_mod.set_threads(before)


def assert_block_sse(gpu_bs, oracle_bs):
    """Per-block SSE: the kernel writes float, the oracle sums in double; both
    overflow a float for the same huge blocks."""
    want = np.asarray(oracle_bs, np.float64).astype(np.float32).astype(np.float64)
    got = host(gpu_bs).astype(np.float64).reshape(want.shape)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(np.isinf(got), np.isinf(want))
    fin = np.isfinite(want)
    # a relative bound on every block (zero blocks must be exactly zero)
    assert np.allclose(got[fin], np.asarray(oracle_bs, np.float64)[fin], rtol=REL, atol=0)


def assert_totals(tot, osd, osx, n):
    t = host(tot)
    assert np.isclose(t[0], osd, rtol=REL, atol=0), (t[0], osd)
    assert np.isclose(t[1], osx, rtol=REL, atol=0), (t[1], osx)
    # the published statistics follow: MSE = sum d^2 / N, SQNR = 10 log10(sum x^2 / sum d^2)
    assert np.isclose(t[0] / n, osd / n, rtol=REL, atol=0)
    if osd > 0:
        sq_gpu, sq_ora = 10 * np.log10(t[1] / t[0]), 10 * np.log10(osx / osd)
        assert abs(sq_gpu - sq_ora) <= REL * abs(sq_ora) + 1e-9


# ----------------------------------------------- MXFP8 / one-byte formats --

@pytest.fixture(scope="module")
def mlp_weight(cuda):
    x = inputs.mlp_weight(device=cuda)
    return x, bits(x)


@pytest.mark.parametrize("fmt", BYTE_FMTS, ids=lambda f: FMT_NAMES[f])
def test_mlp_weight_whole_tensor(mx, oracle_all, mlp_weight, fmt):
    x, xb = mlp_weight
    rows, cols = x.shape
    c, s, _ = mx.quantize(x, fmt, FLOOR)
    y = mx.dequantize(c, s, None, fmt)
    torch.cuda.synchronize()
    oc, os_, _ = oracle_all.quantize(xb, fmt, FLOOR)
    assert np.array_equal(host(s), os_), "scale bytes"
    assert np.array_equal(host(c), oc), "codes"
    assert np.array_equal(bits(y), oracle_all.dequantize(oc, os_, None, rows, cols, fmt)), \
        "dequantized bf16"


# ------------------------------------------------------------ QAT tensors --

@pytest.mark.parametrize("which", ["qat_act", "qat_weight"])
def test_qat_whole_tensor(mx, oracle_all, cuda, which):
    x = getattr(inputs, which)(device=cuda)
    g = inputs.qat_grad(*x.shape, device=cuda)
    y, s = mx.fake_quant(x, E2M1, FLOOR, return_scales=True)
    gx = mx.fake_quant_bwd(x, g, E2M1, FLOOR)
    torch.cuda.synchronize()
    xb = bits(x)
    oy, os_ = oracle_all.fake_quant_fwd(xb, E2M1, FLOOR, want_scales=True)
    assert np.array_equal(bits(y), oy), "fake-quant forward"
    assert np.array_equal(host(s), os_), "scales_out"
    del oy
    assert np.array_equal(bits(gx), oracle_all.fake_quant_bwd(xb, bits(g), E2M1, FLOOR)), \
        "straight-through backward"


@pytest.mark.parametrize("fm", [(E2M1_B16, OAS), (E2M1_B16, FLOOR), (NVFP4, FLOOR)],
                         ids=["fp4b16-OAS", "fp4b16-FLOOR", "nvfp4-FLOOR"])
def test_qat_act_block16_whole_tensor(mx, oracle_all, cuda, fm):
    fmt, m = fm
    x = inputs.qat_act(device=cuda)
    c, s, _ = mx.quantize(x, fmt, m)
    bs, tot = mx.block_error(x, fmt, m)
    torch.cuda.synchronize()
    xb = bits(x)
    oc, os_, _ = oracle_all.quantize(xb, fmt, m)
    assert np.array_equal(host(s), os_), "scale bytes"
    assert np.array_equal(host(c), oc), "codes"
    obs, osd, osx = oracle_all.block_error(xb, fmt, m)
    assert_block_sse(bs, obs)
    assert_totals(tot, osd, osx, x.numel())


# ----------------------------------------------- heavy-tail, every mode --

@pytest.fixture(scope="module")
def heavy_tail(cuda):
    x = inputs.heavy_tail(device=cuda)
    return x, bits(x)


@pytest.mark.parametrize("m", [FLOOR, CEIL, OAS_RULE, OAS, MBS_STATIC, OAS | MBS_STATIC],
                         ids=lambda m: MODE_NAMES[m])
def test_heavy_tail_whole_tensor(mx, oracle_all, heavy_tail, m):
    x, xb = heavy_tail
    rows, cols = x.shape
    c, s, mac = mx.quantize(x, E2M1, m)
    yf = mx.dequantize(c, s, mac, E2M1, torch.float32)
    bs, tot = mx.block_error(x, E2M1, m)
    torch.cuda.synchronize()
    oc, os_, omac = oracle_all.quantize(xb, E2M1, m)
    assert np.array_equal(host(s), os_), "scale bytes"
    assert np.array_equal(host(c), oc), "codes"
    if m >> 4:
        assert np.array_equal(host(mac), omac), "macro factors"
    want = oracle_all.dequantize(oc, os_, omac, rows, cols, E2M1, out_fp32=True)
    assert np.array_equal(host(yf.view(torch.int32)).view(np.uint32), want), "dequantized float"
    obs, osd, osx = oracle_all.block_error(xb, E2M1, m)
    assert_block_sse(bs, obs)
    assert_totals(tot, osd, osx, x.numel())


@pytest.mark.parametrize("m", [MBS_DYNAMIC, OAS | MBS_DYNAMIC], ids=lambda m: MODE_NAMES[m])
def test_heavy_tail_mbs_dynamic(mx, oracle_all, heavy_tail, m):
    """The whole tensor on the GPU; 256 rows (one in every 32, at a varying
    offset) against the oracle. The sum of x^2 is mode-independent and is
    compared over the whole tensor; the sum of d^2 over the sampled rows."""
    x, xb = heavy_tail
    rows, cols = x.shape
    c, s, mac = mx.quantize(x, E2M1, m)
    bs, tot = mx.block_error(x, E2M1, m)
    _, tot_static = mx.block_error(x, E2M1, (m & 15) | MBS_STATIC)
    torch.cuda.synchronize()
    r = np.arange(0, rows, 32) + (np.arange(rows // 32) * 7) % 32
    r[-1] = rows - 1
    xs = np.ascontiguousarray(xb[r])
    oc, os_, omac = oracle_all.quantize(xs, E2M1, m)
    assert np.array_equal(host(s[r]), os_), "scale bytes"
    assert np.array_equal(host(c[r]), oc), "codes"
    assert np.array_equal(host(mac[r]), omac), "macro factors"
    obs, osd_rows, _ = oracle_all.block_error(xs, E2M1, m)
    assert_block_sse(bs[r], obs)
    assert np.isclose(host(bs[r]).astype(np.float64).sum(), osd_rows, rtol=REL)
    _, _, osx = oracle_all.block_error(xb, E2M1, FLOOR, want_blocks=False)
    assert np.isclose(host(tot)[1], osx, rtol=REL, atol=0)
    # the dynamic factor is the argmin over a set holding the static one
    assert host(tot)[0] <= host(tot_static)[0] * (1 + REL)


# ---------------------------------------------------- MoE w13 stack (C5) --

def test_moe_w13_whole_stack(mx, oracle_all, cuda):
    x = inputs.moe_w13(device=cuda).view(-1, 2048)
    rows, cols = x.shape
    c, s, _ = mx.quantize(x, E2M1, FLOOR)
    y = mx.dequantize(c, s, None, E2M1)
    torch.cuda.synchronize()
    xb = bits(x)
    del x
    oc, os_, _ = oracle_all.quantize(xb, E2M1, FLOOR)
    del xb
    assert np.array_equal(host(s), os_), "scale bytes"
    assert np.array_equal(host(c), oc), "codes"
    del c, s
    yb = bits(y)
    del y
    assert np.array_equal(yb, oracle_all.dequantize(oc, os_, None, rows, cols, E2M1)), \
        "dequantized bf16"
