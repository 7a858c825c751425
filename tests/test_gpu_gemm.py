"""The block-scaled MXFP4 GEMM (D = A B^T on the tensor cores) and its fused
activation quantizer, through the C ABI, against the oracle.

"Unveiling the Potential of Quantization with MXFP4", sections 2.B and 4: the
MX scale work next to the tensor-core GEMM; "[vLLM] MXFP8/MXFP4", MXFP4 MoE
section: SM100 kernels consume MXFP4 operands and E8M0 scales.

* The quantizer inside the GEMM: A's codes and (tiled) scales, written out by
  the kernel, equal the oracle's quantization of A bit for bit, under every
  rule the GEMM takes.
* Integer cases: operands on the E2M1 grid with scale 2^0, so every product
  is a multiple of 1/4 and every partial sum stays below 2^22: the product is
  exact in fp32 whatever order the tensor cores sum in, and D must equal it
  (one rounding to bf16).
* Random cases: D against the fp64 product of the oracle's dequantized
  operands, within a bound proportional to the sum of |a_k b_k| (the tensor
  cores' accumulation order and internal precision are not specified).
* The fused GEMM, in both forms (A quantized on chip and shared across a
  cluster; A quantized into the caller's buffers and the GEMM run on them in
  the same cooperative launch), equals the unfused one (quantize, then the
  GEMM on the quantized operands) bit for bit: both feed the same operands to
  the same MMA sequence.
"""

import numpy as np
import pytest
import torch

from fp8_quantization_mx_b200 import inputs

pytestmark = pytest.mark.gpu

E2M1 = 0
FLOOR, CEIL, OAS_RULE, OAS = 0, 1, 2, 3
MMA = 1 << 8
RULES = [FLOOR, CEIL, OAS_RULE, OAS]
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
# (M, N, K): one tile; ragged M and N; a single row; several K-blocks and
# 128-wide N tiles; the MoE w13 expert shape (N = 2I = 1536, K = H = 2048);
# more tiles than SMs, so that persistent CTAs take several tiles (256-wide,
# one with a last N tile 8 columns wide)
SHAPES = [(128, 128, 256), (200, 264, 512), (1, 8, 256), (300, 520, 1024), (16, 1536, 2048),
          (260, 400, 768), (1536, 4096, 512), (2200, 2056, 256)]


def bits(t):
    return inputs.bf16_bits_numpy(t)


def host(t):
    return t.detach().cpu().numpy()


def untile(tiled, rows, K):
    """Plain [rows, K/32] scale bytes from the MMA tiled layout."""
    tiled = np.asarray(tiled).reshape(-1)
    nb = K // 32
    T = (nb + 3) // 4
    r = np.arange(rows)[:, None]
    j = np.arange(nb)[None, :]
    off = ((r // 128) * T + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
    return tiled[off]


def grid_matrix(rows, cols, seed):
    """Values on the E2M1 grid, every 32-block holding a +-6: FLOOR scale 2^0
    and an exact quantization."""
    rng = np.random.default_rng(seed)
    v = GRID[rng.integers(0, 8, (rows, cols))] * rng.choice([-1.0, 1.0], (rows, cols))
    v[:, ::32] = 6.0 * rng.choice([-1.0, 1.0], (rows, cols // 32))
    return v, torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)


def weights(mx, w, cuda):
    """B operand: MXFP4 codes and tiled scales of a bf16 weight [N, K]."""
    c, s, _ = mx.quantize(w.to(cuda), E2M1, FLOOR | MMA)
    return c, s


def dequant64(oracle_mod, codes, plain_scales, rows, K):
    y = oracle_mod.dequantize(host(codes) if torch.is_tensor(codes) else codes, plain_scales, None,
                              rows, K, E2M1, out_fp32=True)
    return y.view(np.float32).astype(np.float64)


def a_buffers(mx, cuda, M, K):
    """Caller buffers for A's quantized form (codes, tiled scales)."""
    return (torch.empty(M, K // 2, dtype=torch.uint8, device=cuda),
            torch.empty(mx.mx_scale_bytes(M, K, E2M1, MMA), dtype=torch.uint8, device=cuda))


# The forms of mx_quant_gemm: quantized in the GEMM's prologue on chip; staged
# through scratch the library allocates; staged through the caller's buffers.
FORMS = ["on-chip", "scratch", "staged"]


def quant_gemm_form(mx, cuda, form, a, bc, bs, rule, **kw):
    """mx_quant_gemm in one of FORMS; returns (D, the caller's A buffers or None)."""
    M, K = a.shape
    buf = a_buffers(mx, cuda, M, K) if form == "staged" else None
    d = mx.quant_gemm(a, bc, bs, rule, a_out=buf, on_chip=form == "on-chip", **kw)
    return d, buf


@pytest.mark.parametrize("fused", FORMS + ["prequantized"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_integer_cases_are_exact(mx, cuda, shape, fused):
    M, N, K = shape
    av, a = grid_matrix(M, K, seed=M + K)
    bv, b = grid_matrix(N, K, seed=N + 7 * K)
    exact = av @ bv.T                       # every partial sum exact in fp32
    assert np.abs(exact).max() < 2 ** 22
    bc, bs = weights(mx, b, cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    outs = {}
    for dt in (torch.float32, torch.bfloat16):
        if fused in FORMS:
            outs[dt], _ = quant_gemm_form(mx, cuda, fused, a.to(cuda), bc, bs, FLOOR, out_dtype=dt,
                                          status=status)
        else:
            ac, as_, _ = mx.quantize(a.to(cuda), E2M1, FLOOR | MMA)
            outs[dt] = mx.gemm(ac, as_, bc, bs, out_dtype=dt, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert np.array_equal(host(outs[torch.float32]).astype(np.float64), exact)
    want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(bits(outs[torch.bfloat16]), bits(want))


# Long persistent runs: ~256 units over the clusters, each unit 12 K-blocks,
# so every stage of the ring is refilled by changing owners many times over;
# staged, 32 bands of A counted ready while seven waves of tiles run.
BIG = [(4096, 8192, 3072)]


@pytest.mark.parametrize("form", ["on-chip", "scratch"])
@pytest.mark.parametrize("shape", BIG, ids=lambda s: "x".join(map(str, s)))
def test_integer_cases_are_exact_many_units(mx, cuda, shape, form):
    M, N, K = shape
    av, a = grid_matrix(M, K, seed=5)
    bv, b = grid_matrix(N, K, seed=6)
    exact = av @ bv.T
    bc, bs = weights(mx, b, cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    d, _ = quant_gemm_form(mx, cuda, form, a.to(cuda), bc, bs, FLOOR, out_dtype=torch.float32,
                           status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert np.array_equal(host(d).astype(np.float64), exact)


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("rule", [FLOOR, OAS], ids=["FLOOR", "OAS"])
@pytest.mark.parametrize("shape", BIG, ids=lambda s: "x".join(map(str, s)))
def test_fused_equals_quantize_then_gemm_many_units(mx, cuda, shape, rule, form):
    M, N, K = shape
    a = inputs.heavy_tail(M, K, seed=rule + 9).to(cuda)
    bc, bs = weights(mx, inputs.normal_weight(N, K, seed=11), cuda)
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    d_fused, buf = quant_gemm_form(mx, cuda, form, a, bc, bs, rule, out_dtype=torch.float32,
                                   status=status)
    ac, as_, _ = mx.quantize(a, E2M1, rule | MMA)
    d_two = mx.gemm(ac, as_, bc, bs, out_dtype=torch.float32, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(d_fused.view(torch.int32), d_two.view(torch.int32))
    if buf is not None:
        assert torch.equal(buf[0], ac) and torch.equal(buf[1], as_)


@pytest.mark.parametrize("rule", RULES, ids=["FLOOR", "CEIL", "OAS_RULE", "OAS"])
def test_fused_quantizer_writes_the_oracle_quantization(mx, oracle_mod, cuda, rule):
    M, N, K = 300, 136, 1024
    a = inputs.heavy_tail(M, K, seed=rule + 40)
    bc, bs = weights(mx, inputs.normal_weight(N, K, seed=3), cuda)
    ac = torch.full((M, K // 2), 0xA5, dtype=torch.uint8, device=cuda)
    asc = torch.full((mx.mx_scale_bytes(M, K, E2M1, MMA),), 0x5A, dtype=torch.uint8, device=cuda)
    mx.quant_gemm(a.to(cuda), bc, bs, rule, a_out=(ac, asc))
    torch.cuda.synchronize()
    oc, os_, _ = oracle_mod.quantize(bits(a), E2M1, rule)
    assert np.array_equal(host(ac), oc), "codes"
    tiled = host(asc)
    assert np.array_equal(untile(tiled, M, K), os_), "scale bytes"
    # the padding rows of the last 128-row band hold zero bytes
    pad = np.ones(tiled.size, bool)
    nb = K // 32
    T = nb // 4
    r = np.arange(M)[:, None]
    j = np.arange(nb)[None, :]
    pad[(((r // 128) * T + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4).ravel()] = False
    assert np.all(tiled[pad] == 0)


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("rule", RULES, ids=["FLOOR", "CEIL", "OAS_RULE", "OAS"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fused_equals_quantize_then_gemm(mx, cuda, shape, rule, form):
    M, N, K = shape
    a = inputs.heavy_tail(M, K, seed=M * 3 + rule).to(cuda)
    bc, bs = weights(mx, inputs.normal_weight(N, K, seed=N), cuda)
    d_fused, buf = quant_gemm_form(mx, cuda, form, a, bc, bs, rule, out_dtype=torch.float32)
    ac, as_, _ = mx.quantize(a, E2M1, rule | MMA)
    d_two = mx.gemm(ac, as_, bc, bs, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(d_fused.view(torch.int32), d_two.view(torch.int32))
    if buf is not None:   # A's quantized form, padding included, is mx_quantize's
        assert torch.equal(buf[0], ac) and torch.equal(buf[1], as_)


@pytest.mark.parametrize("on_chip", [False, True], ids=["staged", "on-chip"])
@pytest.mark.parametrize("part", ["codes", "scales"])
@pytest.mark.parametrize("shape", [(300, 520, 1024), (1536, 4096, 512)],
                         ids=lambda s: "x".join(map(str, s)))
def test_one_buffer_receives_its_part(mx, cuda, shape, part, on_chip):
    """Only one of A's buffers given: it receives mx_quantize's bytes (the
    other part goes to scratch, staged, or stays on chip) and D is unchanged."""
    M, N, K = shape
    a = inputs.heavy_tail(M, K, seed=M + 5).to(cuda)
    bc, bs = weights(mx, inputs.normal_weight(N, K, seed=N + 1), cuda)
    ac, as_, _ = mx.quantize(a, E2M1, OAS | MMA)
    codes, scales = a_buffers(mx, cuda, M, K)
    buf = codes if part == "codes" else scales
    buf.fill_(0xA5)
    d = torch.empty(M, N, dtype=torch.float32, device=cuda)
    flags = 1 | (mx.GEMM_A_ON_CHIP if on_chip else 0)
    st = mx.mx_quant_gemm(a.data_ptr(), OAS, bc.data_ptr(), bs.data_ptr(), M, N, K, flags,
                          d.data_ptr(), codes.data_ptr() if part == "codes" else None,
                          scales.data_ptr() if part == "scales" else None, None,
                          torch.cuda.current_stream().cuda_stream)
    assert st == 0
    d_two = mx.gemm(ac, as_, bc, bs, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int32), d_two.view(torch.int32))
    assert torch.equal(buf, ac if part == "codes" else as_)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_random_product_within_the_accumulation_bound(mx, oracle_mod, cuda, shape):
    """D (fp32 out) against the fp64 product of the oracle's dequantized
    operands. Each product a_k b_k of two MXFP4 values is exact; fp32
    accumulation of K terms errs by at most K u sum |a_k b_k| in any order
    (u = 2^-24), a bound far below what a wrong code, scale or index costs."""
    M, N, K = shape
    a = inputs.outlier_act(M, K, seed=M + N)
    w = inputs.normal_weight(N, K, seed=K + 1)
    bc, bs = weights(mx, w, cuda)
    d = mx.quant_gemm(a.to(cuda), bc, bs, OAS, out_dtype=torch.float32)
    db = mx.quant_gemm(a.to(cuda), bc, bs, OAS)
    torch.cuda.synchronize()
    oc, os_, _ = oracle_mod.quantize(bits(a), E2M1, OAS)
    A = dequant64(oracle_mod, oc, os_, M, K)
    B = dequant64(oracle_mod, bc, untile(host(bs), N, K), N, K)
    ref = A @ B.T
    mag = np.abs(A) @ np.abs(B).T
    got = host(d).astype(np.float64)
    bound = K * 2.0 ** -24 * mag
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / np.maximum(bound, 1e-300))
    # bf16 output: the fp32 result rounded once to nearest even
    assert np.array_equal(bits(db), bits(d.to(torch.bfloat16)))


def test_shapes_empty_and_errors(mx, cuda):
    bc, bs = weights(mx, inputs.normal_weight(64, 512, seed=1), cuda)
    a = inputs.outlier_act(32, 512, seed=2).to(cuda)
    with pytest.raises(mx.MXError):
        mx.quant_gemm(a[:, :384].contiguous(), bc[:, :192].contiguous(), bs)   # K % 256
    with pytest.raises(mx.MXError):
        mx.quant_gemm(a, bc[:60].contiguous(), bs)                             # N % 8
    with pytest.raises(mx.MXError):
        mx.quant_gemm(a, bc, bs, scaling=16)                                   # MBS: no
    st = mx.mx_quant_gemm(a.data_ptr(), FLOOR, bc.data_ptr(), bs.data_ptr(), 0, 64, 512, 0, 0,
                          None, None, None, torch.cuda.current_stream().cuda_stream)
    assert st == 0                                                             # M == 0: nothing
    d = torch.full((32, 64), 7.0, dtype=torch.float32, device=cuda)
    st = mx.mx_gemm(0, 0, 0, 0, 32, 64, 0, 1, d.data_ptr(), None,
                    torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and bool((d == 0).all())                                    # K == 0: zeros
