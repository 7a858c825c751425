"""Pins of the oracle's BATQuant apply step ("BATQuant: Outlier-resilient MXFP4
Quantization via Learnable Block-wise Optimization", technical summary section
2: (a) block-diagonal affine transform with 32-element blocks, (b) GPK: each
block matrix is B_j (x) A, (c) block-wise learnable clipping).

The checks do not re-type the oracle's formula:
* exact small-integer cases against numpy's Kronecker product and an int64
  matrix product (pins the Kronecker convention and every index: a transposed
  factor or kron(A, B) fails);
* random data against an fp64 product within the fp32 rounding bound;
* hand-worked blocks for the summation-order reading (fma chains in index
  order, halves of the block summed separately where the index spans both)
  and for the clip;
* identity parameters reduce the whole step to plain MX quantization.
"""

import numpy as np
import pytest
import torch

import oracle

A_DIMS = (1, 2, 4, 8, 16, 32)
U = 2.0 ** -24


def bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b):
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).double().numpy()


def block_diag_product(xf, A, B):
    """x [rows, cols] @ diag(kron(B_j, A)) in float64 (or int64 for int inputs)."""
    rows, cols = xf.shape
    out = np.zeros_like(xf)
    for j in range(cols // 32):
        P = np.kron(B[j], A)
        out[:, 32 * j:32 * j + 32] = xf[:, 32 * j:32 * j + 32] @ P
    return out


@pytest.mark.parametrize("a", A_DIMS)
def test_identity_parameters_give_x(a):
    b = 32 // a
    x = bf16_bits(np.random.default_rng(a).standard_normal((8, 256)))
    A = np.eye(a, dtype=np.float32)
    B = np.broadcast_to(np.eye(b, dtype=np.float32), (8, b, b)).copy()
    assert np.array_equal(oracle.bat_apply(x, a, A, B), x)
    # and BATQuant with identity parameters is plain MX quantization
    for fmt, scaling in ((oracle.E2M1, oracle.FLOOR), (oracle.E2M1, oracle.OAS | oracle.MBS_STATIC),
                         (oracle.E4M3, oracle.FLOOR), (oracle.E2M3, oracle.OAS)):
        got = oracle.bat_quantize(x, a, A, B, fmt=fmt, scaling=scaling)
        want = oracle.quantize(x, fmt, scaling)
        for g, w in zip(got, want):
            assert (g is None and w is None) or np.array_equal(g, w)


@pytest.mark.parametrize("a", A_DIMS)
def test_exact_integer_case_matches_the_kronecker_product(a):
    # integers small enough that every fp32 partial sum is exact: the result
    # must be the exact matrix product, whatever the summation order
    b = 32 // a
    rng = np.random.default_rng(10 + a)
    rows, cols = 6, 128
    xi = rng.integers(-8, 9, (rows, cols))
    A = rng.integers(-3, 4, (a, a)).astype(np.float32)
    B = rng.integers(-3, 4, (cols // 32, b, b)).astype(np.float32)
    _, yf = oracle.bat_apply(bf16_bits(xi), a, A, B, want_f32=True)
    want = block_diag_product(xi.astype(np.int64), A.astype(np.int64), B.astype(np.int64))
    assert np.array_equal(yf.astype(np.int64), want)
    assert np.all(yf == want)
    if a not in (1, 32):
        # the other Kronecker order is a different map on these inputs
        other = np.zeros_like(want)
        for j in range(cols // 32):
            other[:, 32 * j:32 * j + 32] = xi[:, 32 * j:32 * j + 32] @ np.kron(A, B[j]).astype(np.int64)
        assert not np.array_equal(other, want)


@pytest.mark.parametrize("a", A_DIMS)
def test_random_case_within_the_fp32_rounding_bound(a):
    b = 32 // a
    rng = np.random.default_rng(20 + a)
    rows, cols = 16, 256
    x = bf16_bits(rng.standard_normal((rows, cols)) * np.exp(rng.standard_normal((rows, cols))))
    A = rng.standard_normal((a, a)).astype(np.float32)
    B = rng.standard_normal((cols // 32, b, b)).astype(np.float32)
    _, yf = oracle.bat_apply(x, a, A, B, want_f32=True)
    xf = bits_to_f64(x)
    exact = block_diag_product(xf, A.astype(np.float64), B.astype(np.float64))
    mag = block_diag_product(np.abs(xf), np.abs(A).astype(np.float64), np.abs(B).astype(np.float64))
    # stage 1: chains of a (or two of 16 plus an add), stage 2: two chains of
    # b/2 plus an add; each chain of n terms errs by at most n u of its
    # absolute sum, so 2 (a + b + 2) u of the absolute product is generous
    bound = 2 * (a + b + 2) * U * mag
    err = np.abs(yf.astype(np.float64) - exact)
    assert np.all(err <= bound)
    assert err.max() > 0   # the fp32 path really rounds (not a float64 copy)


def test_sum_order_hand_worked():
    """The summation-order reading on blocks where other orders differ.

    a = 4, A all ones: Z[0][s] = x0 + x1 + x2 + x3 as the chain
    ((1 + 2^-24) + 2^-24) - 1: each 1 + 2^-24 is a tie that rounds to 1, so
    the chain gives 0 (summing from the end would give 2^-23).
    a = 4, A = I, B column 0 all ones (b = 8): y[0] = (Z0 + .. + Z3) + (Z4 + ..
    + Z7) with Z0 = 1, Z1 = 2^-24, Z4 = Z5 = 2^-24: lower half 1 (a tie),
    upper half 2^-23, total 1 + 2^-23 (one chain over all eight would give 1).
    a = 32, A column 0 all ones: the same with x1 = 2^-24 in the lower half
    and x16 = x17 = 2^-24 in the upper half: 1 + 2^-23.
    """
    t = 2.0 ** -24
    x = np.zeros((1, 32))
    x[0, :4] = [1, t, t, -1]
    _, yf = oracle.bat_apply(bf16_bits(x), 4, np.ones((4, 4), np.float32),
                             np.eye(8, dtype=np.float32)[None], want_f32=True)
    assert np.all(yf[0, :4] == 0.0)

    x = np.zeros((1, 32))
    x[0, [0, 4, 16, 20]] = [1, t, t, t]
    B = np.zeros((1, 8, 8), np.float32)
    B[0, :, 0] = 1
    _, yf = oracle.bat_apply(bf16_bits(x), 4, np.eye(4, dtype=np.float32), B, want_f32=True)
    assert yf[0, 0] == np.float32(1 + 2 * t)

    x = np.zeros((1, 32))
    x[0, [0, 1, 16, 17]] = [1, t, t, t]
    A = np.zeros((32, 32), np.float32)
    A[:, 0] = 1
    _, yf = oracle.bat_apply(bf16_bits(x), 32, A, np.ones((1, 1, 1), np.float32), want_f32=True)
    assert yf[0, 0] == np.float32(1 + 2 * t)


def test_clip_hand_worked():
    eye = (np.eye(8, dtype=np.float32), np.eye(4, dtype=np.float32)[None])
    x = np.zeros((1, 32))
    x[0, :6] = [4, -8, -2, 1, 3, -1.5]
    # hi = 0.5 * 4 = 2, lo = 0.25 * -8 = -2
    y = bits_to_f64(oracle.bat_apply(bf16_bits(x), 8, *eye, np.float32([0.25]), np.float32([0.5])))
    assert list(y[0, :6]) == [2, -2, -2, 1, 2, -1.5]
    assert np.all(y[0, 6:] == 0)
    # all-positive block with lo > hi: lo = 1 * 1 = 1, hi = 0.1 * 4: the upper bound wins
    x = np.ones((1, 32))
    x[0, 0] = 4
    y = oracle.bat_apply(bf16_bits(x), 8, *eye, np.float32([1.0]), np.float32([0.1]), want_f32=True)[1]
    assert np.all(y == np.float32(0.1) * np.float32(4))
    # thresholds >= 1 leave the block alone; zero thresholds: lo = -0 / +0 -> 0
    x = np.random.default_rng(3).standard_normal((1, 32))
    xb = bf16_bits(x)
    assert np.array_equal(oracle.bat_apply(xb, 8, *eye, np.float32([1.0]), np.float32([1.5])), xb)
    y = bits_to_f64(oracle.bat_apply(xb, 8, *eye, np.float32([0.0]), np.float32([0.0])))
    assert np.all(y == 0)


def test_clip_all_negative_block_hand_worked():
    # max y = -1: hi = 0.5 * -1 = -0.5 lies above every value (no upper clip);
    # min y = -8: lo = 0.5 * -8 = -4, so -8 and -6 become -4
    eye = (np.eye(8, dtype=np.float32), np.eye(4, dtype=np.float32)[None])
    x = np.full((1, 32), -1.0)
    x[0, :3] = [-8, -6, -2]
    y = bits_to_f64(oracle.bat_apply(bf16_bits(x), 8, *eye, np.float32([0.5]), np.float32([0.5])))
    assert list(y[0, :3]) == [-4, -4, -2]
    assert np.all(y[0, 3:] == -1)


def test_nonfinite_blocks_are_not_clipped_and_nan_is_canonical():
    eye = (np.eye(8, dtype=np.float32), np.eye(4, dtype=np.float32)[None])
    x = np.full((1, 32), 2.0)
    x[0, 5] = np.inf
    y = oracle.bat_apply(bf16_bits(x), 8, *eye, np.float32([0.1]), np.float32([0.1]))
    # inf * 0 in the identity's zero entries: the rest of Z's row 0 is NaN,
    # and stage 2 carries 0 * NaN into every other output; only y[5] =
    # 1 * inf + 0 * 2 + ... stays infinite. Not clipped, NaN canonical.
    assert y[0, 5] == 0x7F80
    assert np.all(np.delete(y[0], 5) == 0x7FC0)
    q, s, _ = oracle.bat_quantize(bf16_bits(x), 8, *eye)
    assert s[0, 0] == 0xFF
