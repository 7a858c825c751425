"""Exhaustive pins of the oracle's element rounding.

Every finite bf16 value v, scaled by every E8M0 exponent E in [-127, 127], is
rounded by the oracle's nearest-grid search and compared with independent
library conversions: ml_dtypes' float4_e2m1fn cast (round to nearest even,
saturating, sign kept) and torch's float8_e4m3fn cast after clamping to
+-448 (torch's cast is round to nearest even but maps overflow to NaN, so the
clamp supplies the saturation the OCP rule asks for). v / 2^E is exact in
double and in float32 unless it under- or overflows float32, where both sides
agree on zero / saturation anyway.
"""

import ml_dtypes
import numpy as np
import pytest
import torch


def _finite_bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint16)
    v = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    return v[np.isfinite(v)]


VALUES = _finite_bf16_values()


def _e2m1_lib(q):
    with np.errstate(over="ignore"):
        return q.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8).astype(np.int32)


def _e4m3_lib(q):
    q32 = np.clip(q, -448.0, 448.0).astype(np.float32)
    return torch.from_numpy(q32).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int32)


@pytest.mark.parametrize("E", list(range(-127, 128)))
def test_e2m1_rounding_every_bf16_every_exponent(oracle_mod, E):
    X = 2.0 ** E
    got = oracle_mod.round_array(VALUES, X, oracle_mod.E2M1)
    ref = _e2m1_lib(VALUES / X)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("E", list(range(-127, 128, 3)) + [127])
def test_e4m3_rounding_every_bf16(oracle_mod, E):
    X = 2.0 ** E
    got = oracle_mod.round_array(VALUES, X, oracle_mod.E4M3)
    ref = _e4m3_lib(VALUES / X)
    # torch maps -0.0 to 0x80 and small negatives to 0x80 as well: signs kept
    assert np.array_equal(got, ref)


def test_e2m1_ties_go_to_even_codes(oracle_mod):
    # midpoints of the grid and where they go (code parity = mantissa LSB)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    expect = [0, 2, 2, 4, 4, 6, 6]
    for m, c in zip(mids, expect):
        assert oracle_mod.round_element(m, 1.0, oracle_mod.E2M1) == c
        assert oracle_mod.round_element(-m, 1.0, oracle_mod.E2M1) == c | 8


def test_saturation_and_signed_zero(oracle_mod):
    assert oracle_mod.round_element(1e30, 1.0, oracle_mod.E2M1) == 7
    assert oracle_mod.round_element(-1e30, 1.0, oracle_mod.E2M1) == 15
    assert oracle_mod.round_element(-0.1, 1.0, oracle_mod.E2M1) == 8
    assert oracle_mod.round_element(-0.0, 1.0, oracle_mod.E2M1) == 8
    assert oracle_mod.round_element(1e30, 1.0, oracle_mod.E4M3) == 0x7E
    assert oracle_mod.round_element(-1e-30, 1.0, oracle_mod.E4M3) == 0x80
