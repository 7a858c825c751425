"""Brute-force and invariant pins of the oracle's scale selection.

* Every finite E8M0 exponent is scanned on seeded random blocks, with element
  codes from ml_dtypes' E2M1 cast (independent of the oracle) and exact
  rational SSEs where a comparison is close: the oracle's FLOOR / CEIL /
  OAS_RULE / OAS bytes must match what the definitions give, exponents >= e
  never beat e - 1, and OAS is the exact argmin over {e-2, e-1}.
* Invariants that the mathematics fixes: element-wise |err OAS_RULE| <=
  |err CEIL| (for a max significand in (1.5, 1.75] the finer grid contains the
  coarser one where it matters), hence the block SSE chain OAS <= OAS_RULE <=
  CEIL and OAS <= FLOOR; MBS-Dynamic <= MBS-Static and <= FLOOR (k = 0 is
  FLOOR); FLOOR fake-quantization is idempotent; grid-aligned input has zero
  error.
* MBS factors are re-derived by a vectorised numpy restatement (nearest-grid by
  distance in float64) and compared with the oracle's bytes.
"""

from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

FLOOR, CEIL, OAS_RULE, OAS = 0, 1, 2, 3
MBS_STATIC, MBS_DYNAMIC = 16, 32
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


def _to_bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _bits_to_f64(b):
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def random_blocks(n, seed):
    """Seeded blocks: Gaussian, heavy-tailed, amax on powers of two and on grid ties."""
    rng = np.random.default_rng(seed)
    kinds = rng.integers(0, 5, n)
    x = np.empty((n, 32))
    g = rng.standard_normal((n, 32))
    t = rng.standard_t(2, (n, 32))
    scale = 2.0 ** rng.integers(-20, 20, (n, 1))
    x[:] = g * scale
    x[kinds == 1] = (t * scale)[kinds == 1]
    # amax exactly a power of two
    m = kinds == 2
    x[m, 0] = scale[m, 0] * 4
    x[m, 1:] = np.clip(x[m, 1:], -3.9 * scale[m], 3.9 * scale[m])
    # every element on a grid point or a grid midpoint, random signs
    m = kinds == 3
    pts = np.array([0, .25, .5, .75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6, 7, 7.5])
    x[m] = rng.choice(pts, (m.sum(), 32)) * rng.choice([-1, 1], (m.sum(), 32)) * scale[m]
    # max significand in the OAS band (above 1.75) with a varied tail
    m = kinds == 4
    x[m, 0] = (7.0 + rng.random(m.sum())) * scale[m, 0]
    x[m, 1:] = rng.random((m.sum(), 31)) * rng.choice([0.3, 1.5, 3], (m.sum(), 1)) * scale[m]
    return _to_bf16_bits(x)


def e2m1_values_lib(xf, E):
    """Dequantized values with codes from ml_dtypes (independent of the oracle)."""
    with np.errstate(over="ignore"):
        q = (xf / 2.0 ** E).astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
    return q.astype(np.float64) * 2.0 ** E


def exact_sse(x, y):
    return sum((Fraction(float(a)) - Fraction(float(b))) ** 2 for a, b in zip(x, y))


def test_scale_bytes_by_definition(oracle_mod):
    bits = random_blocks(6000, 11)
    xf = _bits_to_f64(bits)
    amax = np.abs(xf).max(axis=1)
    _, e2 = np.frexp(amax)
    e = e2 - 1
    nz = amax > 0
    for rule in (FLOOR, CEIL, OAS_RULE, OAS):
        _, s, _ = oracle_mod.quantize(bits, 0, rule)
        s = s[:, 0].astype(int)
        if rule == FLOOR:
            exp = np.where(nz, np.clip(e - 2, -127, 127) + 127, 0)
            assert np.array_equal(s, exp)
        if rule == CEIL:
            E = np.where(amax <= 6 * 2.0 ** (e - 2), e - 2, e - 1)
            exp = np.where(nz, np.clip(E, -127, 127) + 127, 0)
            assert np.array_equal(s, exp)
        if rule == OAS_RULE:
            # the no-overflow max normalized into (3, 3.5] -> one step finer
            Ec = np.where(amax <= 6 * 2.0 ** (e - 2), e - 2, e - 1)
            nrm = amax / 2.0 ** Ec
            E = np.where((nrm > 3) & (nrm <= 3.5), Ec - 1, Ec)
            exp = np.where(nz, np.clip(E, -127, 127) + 127, 0)
            assert np.array_equal(s, exp)


def test_oas_is_exact_argmin_and_coarser_never_wins(oracle_mod):
    bits = random_blocks(3000, 12)
    xf = _bits_to_f64(bits)
    _, s_oas, _ = oracle_mod.quantize(bits, 0, OAS)
    amax = np.abs(xf).max(axis=1)
    e = np.frexp(amax)[1] - 1
    better_below = 0
    for i in range(len(xf)):
        if amax[i] == 0 or e[i] - 2 < -126 or e[i] + 3 > 127:
            continue
        x = xf[i]
        Es = np.arange(max(-127, e[i] - 12), min(127, e[i] + 4) + 1)
        sse = {int(E): float(((x - e2m1_values_lib(x, E)) ** 2).sum()) for E in Es}

        def exact(E):
            return exact_sse(x, e2m1_values_lib(x, E))

        s1, s2 = exact(e[i] - 2), exact(e[i] - 1)
        want = e[i] - 1 if s2 < s1 else e[i] - 2
        assert int(s_oas[i, 0]) == want + 127
        # exponents >= e never beat e - 1 (their grids restricted to the block
        # are subsets of e - 1's)
        for E in range(e[i], min(127, e[i] + 4) + 1):
            if sse[E] <= sse[e[i] - 1] * (1 + 1e-9):
                assert exact(E) >= s2
        # report only: how often a finer exponent than e - 2 would win
        best_below = min(sse[E] for E in Es if E <= e[i] - 3)
        if best_below < min(sse[e[i] - 2], sse[e[i] - 1]) * (1 - 1e-9):
            better_below += 1
    print(f"\nblocks where an exponent <= e-3 is strictly better: {better_below}")


def test_all_exponents_scan_small(oracle_mod):
    # every finite E8M0 exponent on a few hundred blocks; the minimum over the
    # full range is never at an exponent >= e
    bits = random_blocks(300, 13)
    xf = _bits_to_f64(bits)
    amax = np.abs(xf).max(axis=1)
    e = np.frexp(amax)[1] - 1
    for i in range(len(xf)):
        if amax[i] == 0:
            continue
        x = xf[i]
        sses = np.array([((x - e2m1_values_lib(x, E)) ** 2).sum() for E in range(-127, 128)])
        best = int(np.argmin(sses)) - 127
        assert best < e[i] or np.isclose(sses[best + 127], sses[e[i] - 1 + 127], rtol=1e-12)


def test_elementwise_oas_rule_no_worse_than_ceil(oracle_mod):
    bits = random_blocks(4000, 14)
    xf = _bits_to_f64(bits)
    y_rule = _bits_to_f64(oracle_mod.fake_quant_fwd(bits, 0, OAS_RULE))
    y_ceil = _bits_to_f64(oracle_mod.fake_quant_fwd(bits, 0, CEIL))
    # FP4 dequantized values are exact in bf16, and x - y is exact in double
    assert np.all(np.abs(xf - y_rule) <= np.abs(xf - y_ceil))


def test_sse_chain(oracle_mod):
    bits = random_blocks(1500, 15)
    xf = _bits_to_f64(bits)
    ys = {m: _bits_to_f64(oracle_mod.fake_quant_fwd(bits, 0, m)) for m in (FLOOR, CEIL, OAS_RULE, OAS)}
    for i in range(len(xf)):
        s = {m: exact_sse(xf[i], ys[m][i]) for m in ys}
        assert s[OAS] <= s[OAS_RULE] <= s[CEIL]
        assert s[OAS] <= s[FLOOR]


def _macro_sse_f64(x, y):
    """Normative MBS objective: sum of (x - y)^2 in double, element order."""
    s = 0.0
    for a, b in zip(x, y):
        d = a - b
        s = s + d * d
    return s


@pytest.mark.parametrize("rule", [FLOOR, OAS])
@pytest.mark.parametrize("fmt", [0, 6], ids=["block32", "block16"])
def test_mbs_dynamic_no_worse_than_static_and_plain(oracle_mod, rule, fmt):
    rng = np.random.default_rng(16)
    x = rng.standard_normal((6, 128 * 8)) * 2.0 ** rng.integers(-10, 10, (6, 1))
    x[:, rng.integers(0, 1024, 12)] *= 30
    bits = _to_bf16_bits(x)
    xf = _bits_to_f64(bits)
    ys = {}
    for m in (rule, rule | MBS_STATIC, rule | MBS_DYNAMIC):
        c, s, mac = oracle_mod.quantize(bits, fmt, m)
        ys[m] = oracle_mod.dequantize(c, s, mac, 6, 1024, fmt, out_fp32=True).view(np.float32).astype(np.float64)
    for r in range(6):
        for mb in range(8):
            sl = slice(128 * mb, 128 * mb + 128)
            sd = _macro_sse_f64(xf[r, sl], ys[rule | MBS_DYNAMIC][r, sl])
            ss = _macro_sse_f64(xf[r, sl], ys[rule | MBS_STATIC][r, sl])
            sp = _macro_sse_f64(xf[r, sl], ys[rule][r, sl])
            assert sd <= ss and sd <= sp


def _np_round_e2m1(a, X):
    """Vectorised nearest-grid rounding of magnitudes a / X (ties -> even code)."""
    cand = X[..., None] * GRID
    dist = np.abs(a[..., None] - cand)
    best = np.argmin(dist, axis=-1)
    # ties: argmin takes the lower code; move to the even one when tied
    lo = best
    hi = np.minimum(best + 1, 7)
    tie = (hi != lo) & (np.take_along_axis(dist, hi[..., None], -1)[..., 0] ==
                        np.take_along_axis(dist, lo[..., None], -1)[..., 0])
    best = np.where(tie & (lo % 2 == 1), hi, lo)
    return np.where(a >= 6 * X, 7, best)


def _np_floor_log2_over(a, f):
    e = np.frexp(a)[1] - 1
    return np.where(f * 2.0 ** e > a, e - 1, e)


def _np_mbs(xm, k, bs=32):
    """FLOOR sub-block bytes and the element-order SSE of a macro block for
    factor k, with sub-blocks of bs elements (32, or 16 for MXFP4 at block 16)."""
    f = 1 + k / 256
    blocks = np.abs(xm).reshape(128 // bs, bs)
    amax = blocks.max(axis=1)
    ep = np.where(amax > 0, _np_floor_log2_over(np.where(amax > 0, amax, 1), f), -200)
    E = np.clip(ep - 2, -127, 127)
    X = f * 2.0 ** E
    codes = _np_round_e2m1(blocks, np.repeat(X[:, None], bs, 1))
    y = GRID[codes] * X[:, None]
    return E + 127, _macro_sse_f64(blocks.ravel(), y.ravel())


@pytest.mark.parametrize("fmt,bs", [(0, 32), (6, 16)], ids=["block32", "block16"])
def test_mbs_factors_vs_numpy_restatement(oracle_mod, fmt, bs):
    rng = np.random.default_rng(17)
    x = rng.standard_normal((4, 128 * 6)) * 2.0 ** rng.integers(-6, 6, (4, 1))
    x[:, rng.integers(0, 768, 10)] *= 25
    bits = _to_bf16_bits(x)
    xf = _bits_to_f64(bits)
    nb = 128 // bs
    _, s_st, k_st = oracle_mod.quantize(bits, fmt, MBS_STATIC)
    _, s_dy, k_dy = oracle_mod.quantize(bits, fmt, MBS_DYNAMIC)
    for r in range(4):
        for mb in range(6):
            xm = xf[r, 128 * mb:128 * mb + 128]
            A = np.abs(xm).max()
            # static: smallest k with 6 (256 + k) 2^p >= 256 A, 6 * 2^p <= A < 12 * 2^p
            p = np.frexp(A / 6)[1] - 1
            while 6 * 2.0 ** p > A:
                p -= 1
            while 6 * 2.0 ** (p + 1) <= A:
                p += 1
            k = next((k for k in range(256) if 6 * (256 + k) * 2.0 ** p >= 256 * A), 0)
            assert int(k_st[r, mb]) == k
            bytes_st, _ = _np_mbs(xm, k, bs)
            assert np.array_equal(s_st[r, nb * mb:nb * mb + nb].astype(int), bytes_st)
            # dynamic: argmin over all 256 factors of the element-order SSE
            sses = [_np_mbs(xm, kk, bs)[1] for kk in range(256)]
            kd = int(np.argmin(sses))                  # first minimum = smallest k
            assert int(k_dy[r, mb]) == kd
            assert np.array_equal(s_dy[r, nb * mb:nb * mb + nb].astype(int), _np_mbs(xm, kd, bs)[0])


@pytest.mark.parametrize("fmt,rule", [(0, FLOOR), (1, FLOOR), (0, CEIL), (1, CEIL)])
def test_fake_quant_idempotent(oracle_mod, fmt, rule):
    bits = random_blocks(2000, 18)
    y1 = oracle_mod.fake_quant_fwd(bits, fmt, rule)
    y2 = oracle_mod.fake_quant_fwd(y1, fmt, rule)
    assert np.array_equal(y1, y2)


def test_grid_aligned_input_has_zero_error(oracle_mod):
    rng = np.random.default_rng(19)
    n = 512
    codes = rng.integers(0, 8, (n, 32))
    codes[:, 0] = rng.choice([6, 7], n)          # amax 4 or 6 -> FLOOR keeps E
    E = rng.integers(-100, 100, (n, 1))
    x = GRID[codes] * rng.choice([-1, 1], (n, 32)) * 2.0 ** E
    bits = _to_bf16_bits(x)
    _, sd, sx = oracle_mod.block_error(bits, 0, FLOOR, want_blocks=False)
    assert sd == 0.0 and sx > 0


def test_fake_quant_equals_dequantize_of_quantize(oracle_mod):
    bits = random_blocks(1000, 20).reshape(10, 3200)
    for fmt, modes in ((0, (FLOOR, CEIL, OAS_RULE, OAS, MBS_STATIC, OAS | MBS_STATIC)), (1, (FLOOR, CEIL))):
        for m in modes:
            c, s, mac = oracle_mod.quantize(bits, fmt, m)
            deq = oracle_mod.dequantize(c, s, mac, 10, 3200, fmt)
            assert np.array_equal(deq, oracle_mod.fake_quant_fwd(bits, fmt, m))


def test_ste_mask_is_the_unsaturated_set(oracle_mod):
    bits = random_blocks(2000, 21).reshape(500, 128)
    xf = _bits_to_f64(bits)
    ones = _to_bf16_bits(np.ones_like(xf))
    for fmt, maxv in ((0, 6.0), (1, 448.0)):
        for m in ((FLOOR, CEIL) if fmt else (FLOOR, CEIL, OAS_RULE, OAS, MBS_STATIC)):
            g = _bits_to_f64(oracle_mod.fake_quant_bwd(bits, ones, fmt, m))
            c, s, mac = oracle_mod.quantize(bits, fmt, m)
            X = 2.0 ** (s.astype(np.float64) - 127)
            if mac is not None:
                X = X * np.repeat(1 + mac.astype(np.float64) / 256, 4, axis=1)
            lim = np.repeat(maxv * X, 32, axis=1)
            assert lim.shape == xf.shape
            assert np.array_equal(g == 1.0, np.abs(xf) <= lim)


def test_block_error_consistent_with_dequantize(oracle_mod):
    bits = random_blocks(800, 22).reshape(25, 1024)
    xf = _bits_to_f64(bits)
    for fmt, m in ((0, FLOOR), (0, OAS), (1, FLOOR), (0, MBS_STATIC)):
        bs, sd, sx = oracle_mod.block_error(bits, fmt, m)
        c, s, mac = oracle_mod.quantize(bits, fmt, m)
        y = oracle_mod.dequantize(c, s, mac, 25, 1024, fmt, out_fp32=True).view(np.float32).astype(np.float64)
        d2 = ((xf - y) ** 2).reshape(25, 32, 32).sum(-1)
        assert np.allclose(bs, d2, rtol=1e-12, atol=0)
        assert np.isclose(sd, d2.sum(), rtol=1e-12) and np.isclose(sx, (xf ** 2).sum(), rtol=1e-12)


# ------------------------------------------------ 10^5 blocks, vectorised --

def _sse_at(xf, E):
    """Per-block SSE with codes from ml_dtypes at per-block exponents E (float64;
    each d and d^2 is exact, the 32-term sums round at most slightly)."""
    X = 2.0 ** E[:, None]
    with np.errstate(over="ignore"):
        q = (xf / X).astype(np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    return ((xf - q * X) ** 2).sum(axis=1)


def test_bruteforce_1e5_blocks(oracle_mod):
    """10^5 seeded blocks (Gaussian, heavy-tailed, amax on powers of two, on
    grid points and midpoints, in the OAS band): FLOOR/CEIL/OAS_RULE bytes by
    their closed forms; OAS is the exact argmin over {e-2, e-1}; exponents
    >= e never beat e-1; OAS <= OAS_RULE <= CEIL and OAS <= FLOOR. Exact
    rationals settle every comparison closer than 1e-9."""
    bits = random_blocks(100_000, 31)
    xf = _bits_to_f64(bits)
    amax = np.abs(xf).max(axis=1)
    e = np.frexp(amax)[1] - 1
    ok = (amax > 0) & (e - 2 >= -126) & (e + 3 <= 127)
    xf, bits, e, amax = xf[ok], bits[ok], e[ok], amax[ok]
    assert len(xf) > 90_000
    s = {m: oracle_mod.quantize(bits, 0, m)[1][:, 0].astype(int) - 127
         for m in (FLOOR, CEIL, OAS_RULE, OAS)}
    assert np.array_equal(s[FLOOR], e - 2)
    Ec = np.where(amax <= 6 * 2.0 ** (e - 2), e - 2, e - 1)
    assert np.array_equal(s[CEIL], Ec)
    nrm = amax / 2.0 ** Ec
    assert np.array_equal(s[OAS_RULE], np.where((nrm > 3) & (nrm <= 3.5), Ec - 1, Ec))

    s1, s2 = _sse_at(xf, e - 2), _sse_at(xf, e - 1)
    close = np.abs(s1 - s2) <= 1e-9 * np.maximum(s1, s2)
    want = np.where(s2 < s1, e - 1, e - 2)
    for i in np.nonzero(close)[0]:        # near ties: decide exactly
        a = exact_sse(xf[i], e2m1_values_lib(xf[i], e[i] - 2))
        b = exact_sse(xf[i], e2m1_values_lib(xf[i], e[i] - 1))
        want[i] = e[i] - 1 if b < a else e[i] - 2
    assert np.array_equal(s[OAS], want)

    for d in range(1, 6):                 # exponents e .. e+4 never beat e-1
        sd = _sse_at(xf, e - 1 + d)
        worse = sd < s2 * (1 - 1e-9)
        assert not worse.any()

    sse = {m: _sse_at(xf, s[m]) for m in s}
    tol = 1e-9 * sse[CEIL]
    assert np.all(sse[OAS] <= sse[OAS_RULE] + tol)
    assert np.all(sse[OAS_RULE] <= sse[CEIL] + tol)
    assert np.all(sse[OAS] <= sse[FLOOR] + tol)
