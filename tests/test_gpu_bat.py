"""GPU parity of the BATQuant kernels ("BATQuant: Outlier-resilient MXFP4
Quantization via Learnable Block-wise Optimization", section 2) against the
oracle: the transformed bf16 rows and the fused quantizer's codes, scale bytes
and macro factors, bit for bit, through the C ABI.

The arithmetic order is fixed (fp32 fma chains, halves summed separately), so
the comparison with the oracle is exact, including the codes the rounding
decides. That order is a reading of the pages (they fix no precision), so the
GPU output is also checked against definitions that carry no summation order:
integer cases where every order gives the same bits (an int64 Kronecker
product), and random cases within the fp32 + bf16 rounding bound of an fp64
product; the fused quantizer's codes are then the oracle's quantization of the
GPU's own transformed rows.
"""

import numpy as np
import pytest
import torch

from fp8_quantization_mx_b200 import inputs

pytestmark = pytest.mark.gpu

E2M1, E4M3, E5M2, E3M2, E2M3, INT8 = 0, 1, 2, 3, 4, 5
FLOOR, CEIL, OAS_RULE, OAS, MBS_STATIC = 0, 1, 2, 3, 16
MMA = 1 << 8
A_DIMS = (1, 2, 4, 8, 16, 32)
# shapes: several warp tiles with a ragged last one; rows shorter than a
# 512-element tile (tiles wrap rows) and longer
SHAPES = [(37, 96), (9, 2048), (130, 1152), (5, 32), (1, 64), (3, 8192)]


def _np(t):
    return None if t is None else t.detach().cpu().numpy()


def run_both(mx, oracle_mod, x, params, fmt=None, scaling=None):
    A, B, bmin, bmax = params
    a = A.shape[0]
    xb = inputs.bf16_bits_numpy(x)
    if fmt is None:
        y = mx.bat_apply(x, A, B, bmin, bmax)
        torch.cuda.synchronize()
        want = oracle_mod.bat_apply(xb, a, _np(A), _np(B), _np(bmin), _np(bmax))
        return inputs.bf16_bits_numpy(y), want
    got = mx.bat_quantize(x, A, B, bmin, bmax, fmt, scaling)
    torch.cuda.synchronize()
    want = oracle_mod.bat_quantize(xb, a, _np(A), _np(B), _np(bmin), _np(bmax), fmt, scaling)
    return [_np(t) for t in got], list(want)


def assert_same(got, want):
    if isinstance(got, list):
        for g, w in zip(got, want):
            assert (g is None) == (w is None)
            if g is not None:
                assert np.array_equal(g, w), np.argwhere(g != w)[:5]
    else:
        assert np.array_equal(got, want), np.argwhere(got != want)[:5]


@pytest.mark.parametrize("a", A_DIMS)
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("clip", [False, True])
def test_apply_matches_oracle(mx, oracle_mod, cuda, a, shape, clip):
    rows, cols = shape
    x = inputs.outlier_act(rows, cols, seed=rows + cols).to(cuda)
    params = inputs.bat_params(a, cols // 32, seed=a + rows, device=cuda, spread=0.3, clip=clip)
    assert_same(*run_both(mx, oracle_mod, x, params))


@pytest.mark.parametrize("a", A_DIMS)
def test_quantize_fp4_floor_every_a(mx, oracle_mod, cuda, a):
    x = inputs.heavy_tail(67, 1152, seed=a).to(cuda)
    params = inputs.bat_params(a, 1152 // 32, seed=a, device=cuda)
    assert_same(*run_both(mx, oracle_mod, x, params, E2M1, FLOOR))


MODES = [(E2M1, FLOOR), (E2M1, CEIL), (E2M1, OAS_RULE), (E2M1, OAS), (E2M1, MBS_STATIC),
         (E2M1, OAS | MBS_STATIC), (E4M3, FLOOR), (E4M3, CEIL), (E4M3, OAS), (E5M2, OAS),
         (E3M2, FLOOR), (E3M2, OAS), (E2M3, CEIL), (E2M3, OAS), (INT8, FLOOR), (INT8, CEIL)]


@pytest.mark.parametrize("fm", MODES)
@pytest.mark.parametrize("a", [4, 8, 32])
def test_quantize_every_mode(mx, oracle_mod, cuda, fm, a):
    fmt, scaling = fm
    x = inputs.outlier_act(130, 1152, seed=fmt * 7 + scaling).to(cuda)
    params = inputs.bat_params(a, 1152 // 32, seed=11 + a, device=cuda)
    assert_same(*run_both(mx, oracle_mod, x, params, fmt, scaling))


@pytest.mark.parametrize("fm", [(E2M1, FLOOR), (E2M1, OAS | MBS_STATIC), (E4M3, OAS)])
def test_fused_equals_apply_then_quantize_with_tiled_scales(mx, cuda, fm):
    fmt, scaling = fm
    x = inputs.heavy_tail(300, 2048, seed=9).to(cuda)
    A, B, bmin, bmax = inputs.bat_params(8, 64, seed=9, device=cuda)
    y = mx.bat_apply(x, A, B, bmin, bmax)
    for flag in (0, MMA):
        want = mx.quantize(y, fmt, scaling | flag)
        got = mx.bat_quantize(x, A, B, bmin, bmax, fmt, scaling | flag)
        for g, w in zip(got, want):
            assert (g is None and w is None) or torch.equal(g, w)


def test_edge_blocks(mx, oracle_mod, cuda):
    """Zero blocks, NaN / Inf inputs, values that overflow fp32 and bf16 in
    the transform, subnormal results, thresholds 0 / NaN / > 1, negative
    zeros: bit-exact on both outputs."""
    rows, cols = 8, 512
    rng = np.random.default_rng(1)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[0, :32] = 0.0
    x[0, 32:64] = -0.0
    x[1, 5] = np.nan
    x[1, 40] = np.inf
    x[1, 70] = -np.inf
    x[2, :64] *= 2e37                     # fp32 overflow in the sums (some inputs Inf)
    x[3, :64] *= 1e-38                    # subnormal products
    x[4, 64:96] = 2.0 ** -126
    xb = torch.from_numpy(x).to(torch.bfloat16).to(cuda)
    nb = cols // 32
    for a in A_DIMS:
        A, B, _, _ = inputs.bat_params(a, nb, seed=a, device=cuda, spread=0.5, clip=False)
        bmin = torch.full((nb,), 0.9, device=cuda)
        bmax = torch.full((nb,), 0.9, device=cuda)
        bmin[0], bmax[0] = 0.0, 0.0
        bmin[1], bmax[1] = float("nan"), 0.5
        bmin[2], bmax[2] = 1.5, float("inf")
        bmin[3], bmax[3] = 0.0, 1.0
        for params in ((A, B, bmin, bmax), (A, B, None, None)):
            assert_same(*run_both(mx, oracle_mod, xb, params))
            assert_same(*run_both(mx, oracle_mod, xb, params, E2M1, OAS | MBS_STATIC))
            assert_same(*run_both(mx, oracle_mod, xb, params, E4M3, FLOOR))


@pytest.mark.parametrize("shape", [(3, 128), (17, 640), (2, 8192)])
def test_mbs_macro_blocks_across_chunks(mx, oracle_mod, cuda, shape):
    # one macro block per row; a partial 512-column chunk; 16 chunks per row
    rows, cols = shape
    x = inputs.heavy_tail(rows, cols, seed=cols).to(cuda)
    params = inputs.bat_params(4, cols // 32, seed=rows, device=cuda, spread=0.3)
    assert_same(*run_both(mx, oracle_mod, x, params, E2M1, OAS | MBS_STATIC))


def test_identity_parameters_are_plain_quantization(mx, cuda):
    x = inputs.heavy_tail(256, 4096, seed=4).to(cuda)
    for a in A_DIMS:
        A = torch.eye(a, device=cuda)
        B = torch.eye(32 // a, device=cuda).expand(4096 // 32, -1, -1).contiguous()
        got = mx.bat_quantize(x, A, B, format=E2M1, scaling=OAS)
        want = mx.quantize(x, E2M1, OAS)
        assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])


def test_full_moe_stack_sampled_rows(mx, oracle_mod, cuda):
    """The bench workload (MoE w13 [128, 1536, 2048], a = 8, clipping, MXFP4
    FLOOR) in the bench's launch configuration; 96 sampled rows against the
    oracle."""
    x = inputs.moe_w13(device=cuda).view(-1, 2048)
    params = inputs.bat_params(8, 64, device=cuda)
    A, B, bmin, bmax = params
    codes, scales, _ = mx.bat_quantize(x, A, B, bmin, bmax, E2M1, FLOOR)
    y = mx.bat_apply(x, A, B, bmin, bmax)
    torch.cuda.synchronize()
    idx = torch.randperm(x.shape[0], generator=torch.Generator().manual_seed(0))[:96]
    xs = inputs.bf16_bits_numpy(x[idx.to(cuda)])
    oc, os_, _ = oracle_mod.bat_quantize(xs, 8, _np(A), _np(B), _np(bmin), _np(bmax), E2M1, FLOOR)
    assert np.array_equal(codes[idx.to(cuda)].cpu().numpy(), oc)
    assert np.array_equal(scales[idx.to(cuda)].cpu().numpy(), os_)
    oy = oracle_mod.bat_apply(xs, 8, _np(A), _np(B), _np(bmin), _np(bmax))
    assert np.array_equal(inputs.bf16_bits_numpy(y[idx.to(cuda)]), oy)
    del x, y, codes, scales


def test_more_than_2_31_elements(mx, oracle_mod, cuda):
    """64-bit indexing: a tensor of 2^31 + 131072 elements (4.3 GB bf16); rows
    past the 2^31-th element against the oracle."""
    cols = 2048
    rows = (1 << 31) // cols + 64
    x = torch.empty(rows, cols, dtype=torch.bfloat16, device=cuda)
    x.copy_(inputs.outlier_act(64, cols, seed=77).to(cuda).repeat(rows // 64, 1))
    A, B, bmin, bmax = inputs.bat_params(8, cols // 32, seed=3, device=cuda)
    codes, scales, _ = mx.bat_quantize(x, A, B, bmin, bmax, E2M1, FLOOR)
    torch.cuda.synchronize()
    tail = slice(rows - 40, rows)
    xs = inputs.bf16_bits_numpy(x[tail])
    oc, os_, _ = oracle_mod.bat_quantize(xs, 8, _np(A), _np(B), _np(bmin), _np(bmax), E2M1, FLOOR)
    assert np.array_equal(codes[tail].cpu().numpy(), oc)
    assert np.array_equal(scales[tail].cpu().numpy(), os_)
    del x, codes, scales
    torch.cuda.empty_cache()


# ------------------------------------ structure-free definitions (fp64) ----

U = 2.0 ** -24


def _kron_product(xf, A, B):
    """x [rows, cols] times diag(B_j (x) A) over the 32-element blocks, in the
    dtype of the inputs (int64 or float64): numpy's Kronecker product, a
    plain matrix product, no chosen order."""
    rows, cols = xf.shape
    out = np.zeros_like(xf)
    for j in range(cols // 32):
        out[:, 32 * j:32 * j + 32] = xf[:, 32 * j:32 * j + 32] @ np.kron(B[j], A)
    return out


def _clip_blocks(y, bmin, bmax):
    """[beta_min_j min, beta_max_j max] of each row's block j, upper bound last."""
    rows, cols = y.shape
    yb = y.reshape(rows, cols // 32, 32)
    lo = bmin[None, :, None] * yb.min(axis=2, keepdims=True)
    hi = bmax[None, :, None] * yb.max(axis=2, keepdims=True)
    return np.minimum(np.maximum(yb, lo), hi).reshape(rows, cols)


def _bf16_bits_of_exact(v):
    """bf16 bits of exact values below 2^24 (float32 holds them; one RNE)."""
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _f64(bits16):
    return torch.from_numpy(np.ascontiguousarray(bits16).view(np.int16)).view(torch.bfloat16) \
        .double().numpy()


@pytest.mark.parametrize("a", A_DIMS)
@pytest.mark.parametrize("clip", [False, True])
def test_apply_integer_cases_equal_the_kronecker_product(mx, oracle_mod, cuda, a, clip):
    """Small integers: every fp32 partial sum is exact, so any summation order
    gives the exact product; the clip thresholds 0.5 and 0.75 keep the bounds
    exact. The GPU's bf16 output must be the one rounding of that exact value
    (a zero may carry either sign: which one depends on the order the zero
    terms are added in), and the fused codes the oracle's quantization of the
    GPU's rows."""
    b = 32 // a
    rng = np.random.default_rng(40 + a)
    rows, cols = 70, 1152
    xi = rng.integers(-8, 9, (rows, cols))
    Ai = rng.integers(-3, 4, (a, a))
    Bi = rng.integers(-3, 4, (cols // 32, b, b))
    exact = _kron_product(xi.astype(np.int64), Ai.astype(np.int64), Bi.astype(np.int64))
    assert np.abs(exact).max() < 2 ** 24
    bmin = bmax = None
    want = exact.astype(np.float64)
    if clip:
        bmin = np.where(np.arange(cols // 32) % 2, 0.5, 0.75).astype(np.float32)
        bmax = np.where(np.arange(cols // 32) % 3, 0.75, 0.5).astype(np.float32)
        want = _clip_blocks(want, bmin.astype(np.float64), bmax.astype(np.float64))
    want_bits = _bf16_bits_of_exact(want)
    dev = lambda t: None if t is None else torch.from_numpy(np.ascontiguousarray(t, np.float32)).to(cuda)
    x = torch.from_numpy(xi.astype(np.float32)).to(torch.bfloat16).to(cuda)
    y = mx.bat_apply(x, dev(Ai), dev(Bi), dev(bmin), dev(bmax))
    got = mx.bat_quantize(x, dev(Ai), dev(Bi), dev(bmin), dev(bmax), E2M1, OAS)
    torch.cuda.synchronize()
    yb = inputs.bf16_bits_numpy(y)
    unsigned_zero = lambda v: np.where(v == 0x8000, 0, v)
    assert np.array_equal(unsigned_zero(yb), want_bits)
    oc, os_, _ = oracle_mod.quantize(yb, E2M1, OAS)
    assert np.array_equal(_np(got[0]), oc) and np.array_equal(_np(got[1]), os_)


@pytest.mark.parametrize("a", A_DIMS)
@pytest.mark.parametrize("clip", [False, True])
@pytest.mark.parametrize("shape", [(37, 384), (130, 1152)])
def test_apply_within_the_rounding_bound_of_the_fp64_product(mx, oracle_mod, cuda, a, clip, shape):
    """Random data and parameters: |y_gpu - y| is bounded, per element, by
    the fp32 error of the transform and the thresholds, carried through the
    clip (1-Lipschitz in the value and in both bounds), plus the final bf16
    rounding (half an ulp, at most 2^-8 of the value). Chains of n products
    err by at most n u of their absolute sum, so 2 (a + b + 2) u of the
    absolute product bounds the transform (as for the oracle)."""
    rows, cols = shape
    b = 32 // a
    x = inputs.heavy_tail(rows, cols, seed=a * 31 + rows).to(cuda)
    A, B, bmin, bmax = inputs.bat_params(a, cols // 32, seed=a + cols, device=cuda, spread=0.3,
                                         clip=clip, lo=0.5)
    y = mx.bat_apply(x, A, B, bmin, bmax)
    fused = mx.bat_quantize(x, A, B, bmin, bmax, E2M1, OAS | MBS_STATIC)
    torch.cuda.synchronize()
    xf = _f64(inputs.bf16_bits_numpy(x))
    A64, B64 = _np(A).astype(np.float64), _np(B).astype(np.float64)
    ref = _kron_product(xf, A64, B64)
    mag = _kron_product(np.abs(xf), np.abs(A64), np.abs(B64))
    err_t = 2 * (a + b + 2) * U * mag                          # transform, per element
    if clip:
        bl, bh = _np(bmin).astype(np.float64), _np(bmax).astype(np.float64)
        ref = _clip_blocks(ref, bl, bh)
        eb = err_t.reshape(rows, cols // 32, 32).max(axis=2, keepdims=True)   # per block
        thr = np.maximum(bl, bh)[None, :, None]
        big = np.abs(ref).reshape(rows, cols // 32, 32).max(axis=2, keepdims=True)
        err_t = np.broadcast_to(np.maximum(1.0, thr) * eb + U * thr * big * (1 + 1e-6),
                                (rows, cols // 32, 32)).reshape(rows, cols)
    bound = err_t * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(ref)
    got = _f64(inputs.bf16_bits_numpy(y))
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / np.maximum(bound, 1e-300))
    # the transform really is evaluated (a wrong index moves values by O(1))
    assert np.abs(got - ref).max() > 0
    # the fused codes are exactly the oracle's quantization of the GPU's rows
    oc, os_, om = oracle_mod.quantize(inputs.bf16_bits_numpy(y), E2M1, OAS | MBS_STATIC)
    assert np.array_equal(_np(fused[0]), oc)
    assert np.array_equal(_np(fused[1]), os_)
    assert np.array_equal(_np(fused[2]), om)


def test_full_moe_stack_against_the_fp64_product(mx, cuda):
    """The bench workload (MoE w13 rows, a = 8, clipping) on 256 sampled rows:
    within the rounding bound of the fp64 product, in the bench's launch."""
    x = inputs.moe_w13(device=cuda).view(-1, 2048)
    A, B, bmin, bmax = inputs.bat_params(8, 64, device=cuda)
    y = mx.bat_apply(x, A, B, bmin, bmax)
    torch.cuda.synchronize()
    idx = torch.randperm(x.shape[0], generator=torch.Generator().manual_seed(1))[:256].to(cuda)
    xf = _f64(inputs.bf16_bits_numpy(x[idx]))
    got = _f64(inputs.bf16_bits_numpy(y[idx]))
    del x, y
    A64, B64 = _np(A).astype(np.float64), _np(B).astype(np.float64)
    bl, bh = _np(bmin).astype(np.float64), _np(bmax).astype(np.float64)
    ref = _clip_blocks(_kron_product(xf, A64, B64), bl, bh)
    mag = _kron_product(np.abs(xf), np.abs(A64), np.abs(B64))
    rows = len(xf)
    eb = (2 * (8 + 4 + 2) * U * mag).reshape(rows, 64, 32).max(axis=2, keepdims=True)
    big = np.abs(ref).reshape(rows, 64, 32).max(axis=2, keepdims=True)
    err = np.broadcast_to(eb + U * big * (1 + 1e-6), (rows, 64, 32)).reshape(rows, 2048)
    assert np.all(np.abs(got - ref) <= err * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(ref))
