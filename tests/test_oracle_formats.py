"""Pins of the oracle's format definitions against independent library decoders.

The oracle decodes every format from its field definition; these tests compare
it with ml_dtypes (float4_e2m1fn, float8_e8m0fnu, bfloat16) and torch
(float8_e4m3fn, bfloat16), which share no code with it, and with the value set
the sources print (E2M1 {0, .5, 1, 1.5, 2, 3, 4, 6}: 2-bit exponent + 1-bit
mantissa, "[Axolotl] MXFP4 quantization support" section 2, maximum 6.0 in
"Unveiling the Potential of Quantization with MXFP4" 2.A; E8M0 = 2^k, same
paper, technical summary 1).
"""

import math

import ml_dtypes
import numpy as np
import torch


def test_e2m1_value_set(oracle_mod):
    vals = [oracle_mod.decode_e2m1(c) for c in range(16)]
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert vals == list(lib)
    assert sorted(set(abs(v) for v in vals)) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert max(vals) == 6.0
    # bit 3 is the sign: codes 8..15 mirror 0..7 (code 8 is -0)
    for c in range(8):
        assert vals[c + 8] == -vals[c] and math.copysign(1, vals[c + 8]) == -1


def test_e4m3_all_bytes(oracle_mod):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle_mod.decode_e4m3(b) for b in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}      # S.1111.111 only
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.nanmax(got) == 448.0


def test_e8m0_all_bytes(oracle_mod):
    ref = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = np.array([oracle_mod.decode_e8m0(b) for b in range(256)])
    assert np.isnan(got[255]) and np.isnan(ref[255])
    assert np.array_equal(got[:255], ref[:255])
    # every value is a power of two, 2^-127 .. 2^127
    assert np.array_equal(np.log2(got[:255]), np.arange(-127, 128))


def test_bf16_decode_all_patterns(oracle_mod):
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle_mod.decode_bf16(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_encode_matches_torch_rounding(oracle_mod):
    # float32 inputs (exact in double) so that torch's float32 -> bf16 cast is
    # a single round-to-nearest-even; cover normal, subnormal, ties, overflow
    rng = np.random.default_rng(7)
    u = rng.integers(0, 1 << 32, 20000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    extra = np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 2 ** -133, 2 ** -134,
                      3 * 2 ** -135, 3.3961e38, 3.4e38, -3.4e38, 1.5 * 2 ** -126], dtype=np.float32)
    f = np.concatenate([f, extra])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.encode_bf16_rne(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_encode_decode_roundtrip_all_finite_bf16(oracle_mod):
    for b in range(0, 1 << 16, 7):
        v = oracle_mod.decode_bf16(b)
        if math.isfinite(v):
            assert oracle_mod.encode_bf16_rne(v) == b
