"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Codes, scale bytes, macro bytes, dequantized bf16/float bits and straight-
through gradients must be bit-identical; error statistics agree within a
relative 1e-6 (the kernel sums per-block squares in double and atomically adds
per-CTA double partials, the oracle sums sequentially in double). Inputs are
seeded and synthetic (fp8_quantization_mx_b200.inputs). The whole-tensor
comparisons at the workload sizes are in test_gpu_full_parity.py; here the
small and edge-case inputs, and a tensor past 2^31 elements.
"""

import numpy as np
import pytest
import torch

from fp8_quantization_mx_b200 import inputs

pytestmark = pytest.mark.gpu

E2M1, E4M3, E5M2, E3M2, E2M3, INT8, E2M1_B16, NVFP4 = 0, 1, 2, 3, 4, 5, 6, 7
FLOOR, CEIL, OAS_RULE, OAS = 0, 1, 2, 3
MBS_STATIC, MBS_DYNAMIC = 16, 32
FP4_MODES = [FLOOR, CEIL, OAS_RULE, OAS, MBS_STATIC, MBS_DYNAMIC, OAS | MBS_STATIC, OAS | MBS_DYNAMIC]
BYTE_FMTS = [E4M3, E5M2, E3M2, E2M3, INT8]
BYTE_MODES = {E4M3: [FLOOR, CEIL, OAS], E5M2: [FLOOR, CEIL, OAS], E3M2: [FLOOR, CEIL, OAS],
              E2M3: [FLOOR, CEIL, OAS], INT8: [FLOOR, CEIL]}
B16_MODES = [(E2M1_B16, FLOOR), (E2M1_B16, CEIL), (E2M1_B16, OAS_RULE), (E2M1_B16, OAS),
             (E2M1_B16, MBS_STATIC), (E2M1_B16, MBS_DYNAMIC), (E2M1_B16, OAS | MBS_STATIC),
             (E2M1_B16, OAS | MBS_DYNAMIC), (NVFP4, FLOOR)]
ALL = ([(E2M1, m) for m in FP4_MODES] + [(f, m) for f in BYTE_FMTS for m in BYTE_MODES[f]] +
       B16_MODES)
PACKED = (E2M1, E2M1_B16, NVFP4)
BLOCK = {f: (16 if f in (E2M1_B16, NVFP4) else 32) for f in range(8)}
EMAX = {E2M1: 2, E4M3: 8, E5M2: 15, E3M2: 4, E2M3: 2, INT8: 0}
FMT_NAMES = {E2M1: "fp4", E4M3: "e4m3", E5M2: "e5m2", E3M2: "e3m2", E2M3: "e2m3", INT8: "int8",
             E2M1_B16: "fp4b16", NVFP4: "nvfp4"}
REL = 1e-6


def ids(fm):
    fmt, m = fm
    names = {0: "FLOOR", 1: "CEIL", 2: "OAS_RULE", 3: "OAS"}
    s = names[m & 15]
    if m >> 4:
        s += "+MBS_" + ("STATIC" if m >> 4 == 1 else "DYNAMIC")
    return FMT_NAMES[fmt] + "-" + s


def bits(t):
    return inputs.bf16_bits_numpy(t)


def host_u8(t):
    return t.detach().cpu().numpy()


def from_bits(b, device):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(device)


# ------------------------------------------------------------ small inputs --

def special_blocks():
    """Blocks with zeros, signed zeros, NaN, Inf, subnormals, extremes and ties."""
    rows = []
    z = np.zeros(32, np.uint16)
    rows.append(z.copy())
    b = z.copy(); b[3] = 0x8000; rows.append(b)                       # -0
    b = z.copy(); b[0] = 0x7FC0; b[1] = 0x3F80; b[2] = 0xC000; rows.append(b)   # NaN
    b = z.copy(); b[5] = 0xFF80; b[6] = 0x4000; rows.append(b)         # -Inf
    b = z.copy(); b[0] = 0x7F80; rows.append(b)                        # +Inf
    b = np.arange(1, 33, dtype=np.uint16); rows.append(b)              # subnormals only
    b = (np.arange(32, dtype=np.uint16) + 0x8001); rows.append(b)      # negative subnormals
    b = z.copy(); b[0] = 0x7F7F; b[1:] = 0x0001; rows.append(b)        # max bf16 with tiny tail
    b = z.copy(); b[0] = 0x0080; b[1] = 0x0040; rows.append(b)         # smallest normal amax
    ties = np.array([4.0, .25, .75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.125, 7.0, 6.0, 3.0], np.float32)
    b = z.copy(); b[:12] = torch.from_numpy(ties).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    rows.append(b)
    for e in (-126, -100, -3, 0, 5, 60, 120, 125):
        v = np.full(32, 2.0 ** e, np.float32) * np.linspace(-7.5, 7.5, 32, dtype=np.float32)
        rows.append(torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    arr = np.stack(rows)
    # pad to a whole number of 128-element macro rows
    pad = (-len(arr)) % 4
    arr = np.concatenate([arr, np.zeros((pad, 32), np.uint16)])
    # a macro block made only of subnormals (its MBS factor comes from a
    # subnormal maximum), and one of mixed-sign subnormals and zeros
    sub = (np.arange(128, dtype=np.uint16) % 127 + 1)
    mixed = np.where(np.arange(128) % 3 == 0, 0, sub | np.where(np.arange(128) % 2, 0x8000, 0))
    # macro blocks whose MBS-Static factor is k = 64 (max 7.5) or k = 32 (max
    # 6.75), filled with the exact grid midpoints times f: every one of them is
    # a rounding tie under the macro factor
    ties_rows = []
    for amax, f in ((7.5, 1.25), (6.75, 1.125)):
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) * f
        vals = np.zeros(128, np.float32)
        for sb in range(4):
            blk = np.concatenate([[amax], mids, -mids, mids * 0.5, -mids * 0.5, [0.0, -0.0, amax - 0.25]])
            vals[32 * sb:32 * sb + len(blk)] = blk[:32]
        b16 = torch.from_numpy(vals).to(torch.bfloat16)
        assert torch.equal(b16.float(), torch.from_numpy(vals)), "tie values must be bf16-exact"
        ties_rows.append(b16.view(torch.int16).numpy().view(np.uint16))
    arr = np.concatenate([arr.reshape(-1, 128), sub[None], mixed.astype(np.uint16)[None],
                          np.stack(ties_rows)])
    return arr


def sweep_tie_blocks():
    """Macro blocks whose MBS-Dynamic SSE is smallest, with the same nonzero
    value, at two factors: constants exact on the grid under both k = 0 and
    k = 128 (6 -> 6 or 4; 3 -> 6 or 4 one binade down) or k = 64 and k = 224
    (7.5 -> 6 or 4), plus tiny elements that round to 0 under every factor.
    The smaller k must win; the search must not stop at the first of them."""
    rows = []
    for c, tiny in ((6.0, 2.0 ** -9), (3.0, -2.0 ** -10), (7.5, 2.0 ** -8), (-7.5, 2.0 ** -20),
                    (5.0, 2.0 ** -9)):
        v = np.full(128, c, np.float32)
        v[37], v[100] = tiny, -tiny
        rows.append(v)
    v = np.concatenate([np.full(32, 6.0), np.full(32, -3.0), np.full(32, 0.75),
                        np.full(32, 6.0 * 2 ** -10)]).astype(np.float32)
    v[5] = 2.0 ** -12
    rows.append(v)
    t = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.from_numpy(np.stack(rows)))
    return t


SMALL = {
    "outlier_act_256x4096": lambda: inputs.outlier_act(),
    "random_bits_3x160": lambda: inputs.random_bf16_bits((3, 160), seed=5),
    "random_bits_1x32": lambda: inputs.random_bf16_bits((1, 32), seed=6),
    "random_bits_5x96": lambda: inputs.random_bf16_bits((5, 96), seed=7),
    "random_bits_7x384": lambda: inputs.random_bf16_bits((7, 384), seed=8),
    "random_bits_33x1280": lambda: inputs.random_bf16_bits((33, 1280), seed=9),
    "heavy_tail_64x4096": lambda: inputs.heavy_tail(rows=64),
    "moe_4x1536x2048_head": lambda: inputs.moe_w13(experts=2, inter2=48),
    "special_blocks": lambda: torch.from_numpy(special_blocks().view(np.int16)).view(torch.bfloat16),
    "sweep_tie_blocks": sweep_tie_blocks,
}


def usable(name, fmt, m, x):
    cols = x.shape[-1]
    return not (m >> 4 and cols % 128)


@pytest.mark.parametrize("fm", ALL, ids=ids)
@pytest.mark.parametrize("name", list(SMALL))
def test_quantize_parity(mx, oracle_mod, cuda, name, fm):
    fmt, m = fm
    x = SMALL[name]()
    if not usable(name, fmt, m, x):
        pytest.skip("MBS needs cols % 128 == 0")
    c, s, mac = mx.quantize(x.to(cuda), fmt, m)
    torch.cuda.synchronize()
    oc, os_, omac = oracle_mod.quantize(bits(x), fmt, m)
    assert np.array_equal(host_u8(s), os_), "scale bytes"
    assert np.array_equal(host_u8(c), oc), "codes"
    if m >> 4:
        assert np.array_equal(host_u8(mac), omac), "macro factors"


@pytest.mark.parametrize("fm", ALL, ids=ids)
@pytest.mark.parametrize("name", ["outlier_act_256x4096", "random_bits_33x1280", "special_blocks",
                                  "heavy_tail_64x4096", "sweep_tie_blocks"])
def test_fake_quant_parity(mx, oracle_mod, cuda, name, fm):
    fmt, m = fm
    x = SMALL[name]()
    if not usable(name, fmt, m, x):
        pytest.skip("MBS needs cols % 128 == 0")
    xd = x.to(cuda)
    y, s = mx.fake_quant(xd, fmt, m, return_scales=True)
    g = inputs.qat_grad(*x.shape, seed=3).to(cuda)
    gx = mx.fake_quant_bwd(xd, g, fmt, m)
    torch.cuda.synchronize()
    oy, os_ = oracle_mod.fake_quant_fwd(bits(x), fmt, m, want_scales=True)
    assert np.array_equal(bits(y), oy), "fake-quant forward"
    assert np.array_equal(host_u8(s), os_), "scales_out"
    ogx = oracle_mod.fake_quant_bwd(bits(x), bits(g), fmt, m)
    assert np.array_equal(bits(gx), ogx), "straight-through backward"


@pytest.mark.parametrize("fm", ALL, ids=ids)
@pytest.mark.parametrize("name", ["outlier_act_256x4096", "heavy_tail_64x4096", "random_bits_7x384",
                                  "special_blocks", "sweep_tie_blocks"])
def test_block_error_parity(mx, oracle_mod, cuda, name, fm):
    fmt, m = fm
    x = SMALL[name]()
    if not usable(name, fmt, m, x):
        pytest.skip("MBS needs cols % 128 == 0")
    bs, tot = mx.block_error(x.to(cuda), fmt, m)
    torch.cuda.synchronize()
    obs, osd, osx = oracle_mod.block_error(bits(x), fmt, m)
    # the per-block output is a float: huge blocks overflow it on both sides
    obs = obs.astype(np.float32).astype(np.float64)
    gbs = bs.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isnan(obs), np.isnan(gbs))
    assert np.array_equal(np.isinf(obs), np.isinf(gbs))
    fin = np.isfinite(obs)
    assert np.allclose(gbs[fin], obs[fin], rtol=REL, atol=0)
    t = tot.cpu().numpy()
    for got, want in ((t[0], osd), (t[1], osx)):
        assert np.isnan(got) == np.isnan(want)
        if np.isfinite(want):
            assert np.isclose(got, want, rtol=REL, atol=0)


# ------------------------------------------------ exhaustive element values --

def test_every_scaled_value_at_several_exponents(mx, oracle_mod, cuda):
    """Each block: an anchor fixing E, then every bf16 pattern below it (both signs)."""
    rows = []
    allbits = np.arange(1 << 16, dtype=np.uint32)
    for E in (-127, -126, -90, -7, 0, 3, 64, 125):
        # anchor 7.9375 * 2^E (max significand below 8) -> FLOOR exponent E
        anchor_exp = E + 2 + 127
        if anchor_exp < 1:
            anchor = 0x0080                  # smallest normal: E clamps to -127
            lim = 0x0080
        else:
            anchor = (anchor_exp << 7) | 0x7F
            lim = anchor
        vals = allbits[(allbits & 0x7FFF) <= lim].astype(np.uint16)
        n = len(vals)
        per = 31
        nb = (n + per - 1) // per
        blk = np.zeros((nb, 32), np.uint16)
        blk[:, 0] = anchor
        flat = np.zeros(nb * per, np.uint16)
        flat[:n] = vals
        blk[:, 1:] = flat.reshape(nb, per)
        rows.append(blk)
    arr = np.concatenate(rows)
    arr = np.concatenate([arr, np.zeros(((-len(arr)) % 64, 32), np.uint16)]).reshape(-1, 2048)
    x = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16)
    for fmt in [E2M1] + BYTE_FMTS + [E2M1_B16, NVFP4]:
        c, s, _ = mx.quantize(x.to(cuda), fmt, FLOOR)
        y = mx.fake_quant(x.to(cuda), fmt, FLOOR)
        torch.cuda.synchronize()
        oc, os_, _ = oracle_mod.quantize(arr, fmt, FLOOR)
        assert np.array_equal(host_u8(s), os_)
        assert np.array_equal(host_u8(c), oc)
        assert np.array_equal(bits(y), oracle_mod.fake_quant_fwd(arr, fmt, FLOOR))


@pytest.mark.parametrize("fmt", [E2M1] + BYTE_FMTS + [E2M1_B16, NVFP4])
@pytest.mark.parametrize("out_fp32", [0, 1])
@pytest.mark.parametrize("with_macro", [False, True])
def test_dequantize_every_code_and_scale(mx, oracle_mod, cuda, fmt, out_fp32, with_macro):
    if fmt not in (E2M1, E2M1_B16) and with_macro:
        pytest.skip("macro factors are MXFP4 only")
    rng = np.random.default_rng(23)
    rows, cols = 256, 512
    # every scale byte in every row (NVFP4: every E4M3 byte, NaN and negative included)
    scales = np.tile(np.arange(256, dtype=np.uint8)[:, None], (1, cols // BLOCK[fmt]))
    rng.shuffle(scales, axis=1)
    if fmt in PACKED:
        codes = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
        codes[:, :8] = np.arange(0, 256, 17, dtype=np.uint8)[None, :8]
    else:
        codes = rng.integers(0, 256, (rows, cols), dtype=np.uint8)
        codes[0, :256] = np.arange(256, dtype=np.uint8)
        if fmt in (E3M2, E2M3):
            codes &= 0x3F          # an FP6 code occupies the low 6 bits of its byte
    macro = rng.integers(0, 256, (rows, cols // 128), dtype=np.uint8) if with_macro else None
    tdev = lambda a: None if a is None else torch.from_numpy(a).to(cuda)
    out = mx.dequantize(tdev(codes), tdev(scales), tdev(macro), fmt,
                        torch.float32 if out_fp32 else torch.bfloat16)
    torch.cuda.synchronize()
    ref = oracle_mod.dequantize(codes, scales, macro, rows, cols, fmt, out_fp32=bool(out_fp32))
    got = out.cpu().view(torch.int32 if out_fp32 else torch.int16).numpy()
    got = got.view(np.uint32 if out_fp32 else np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fm", ALL, ids=ids)
def test_dequantize_roundtrip(mx, oracle_mod, cuda, fm):
    fmt, m = fm
    x = SMALL["outlier_act_256x4096"]()
    c, s, mac = mx.quantize(x.to(cuda), fmt, m)
    y = mx.dequantize(c, s, mac, fmt)
    yf = mx.dequantize(c, s, mac, fmt, torch.float32)
    torch.cuda.synchronize()
    oc, os_, omac = oracle_mod.quantize(bits(x), fmt, m)
    assert np.array_equal(bits(y), oracle_mod.dequantize(oc, os_, omac, 256, 4096, fmt))
    assert np.array_equal(yf.cpu().view(torch.int32).numpy().view(np.uint32),
                          oracle_mod.dequantize(oc, os_, omac, 256, 4096, fmt, out_fp32=True))


# ------------------------------------------------------ edge behaviour --

def test_guard_bands(mx, cuda):
    """Outputs never write outside their extent (canary bytes on both sides)."""
    x = inputs.random_bf16_bits((3, 384), seed=11).to(cuda)
    for fmt, m in ((E2M1, FLOOR), (E2M1, OAS | MBS_DYNAMIC), (E4M3, CEIL), (E5M2, OAS),
                   (E2M3, OAS), (INT8, FLOOR), (E2M1_B16, OAS), (NVFP4, FLOOR)):
        ncode = 3 * 384 // (2 if fmt in PACKED else 1)
        nsc = 3 * 384 // BLOCK[fmt]
        pad = 256
        cbuf = torch.full((ncode + 2 * pad,), 0xA5, dtype=torch.uint8, device=cuda)
        sbuf = torch.full((nsc + 2 * pad,), 0x5A, dtype=torch.uint8, device=cuda)
        mbuf = torch.full((9 + 2 * pad,), 0x3C, dtype=torch.uint8, device=cuda)
        st = mx.mx_quantize(x.data_ptr(), 3, 384, fmt, m, cbuf[pad:].data_ptr(), sbuf[pad:].data_ptr(),
                            mbuf[pad:].data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0
        torch.cuda.synchronize()
        assert bool((cbuf[:pad] == 0xA5).all()) and bool((cbuf[pad + ncode:] == 0xA5).all())
        assert bool((sbuf[:pad] == 0x5A).all()) and bool((sbuf[pad + nsc:] == 0x5A).all())
        assert bool((mbuf[:pad] == 0x3C).all()) and bool((mbuf[pad + (9 if m >> 4 else 0):] == 0x3C).all())
    y = torch.full((3 * 384 + 512,), 7, dtype=torch.int16, device=cuda)
    st = mx.mx_fake_quant_fwd(x.data_ptr(), 3, 384, E2M1, OAS, y[256:].data_ptr(), None,
                              torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and bool((y[:256] == 7).all()) and bool((y[256 + 3 * 384:] == 7).all())


def test_empty_and_zero_rows(mx, cuda):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=cuda)
    c, s, _ = mx.quantize(x)
    assert c.shape == (0, 32) and s.shape == (0, 2)
    bs, tot = mx.block_error(x)
    torch.cuda.synchronize()
    assert tot.tolist() == [0.0, 0.0]


def test_side_stream_and_host_buffers(mx, oracle_mod, cuda):
    x = inputs.outlier_act()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        c, s, _ = mx.quantize(x.to(cuda, non_blocking=False))
    side.synchronize()
    hc, hs, _ = mx.quantize(x.pin_memory())
    torch.cuda.synchronize()
    oc, os_, _ = oracle_mod.quantize(bits(x))
    assert np.array_equal(host_u8(c), oc) and np.array_equal(hc.numpy(), oc)
    assert np.array_equal(hs.numpy(), os_)


def test_autograd_function(mx, oracle_mod, cuda):
    x = inputs.qat_act(rows=64, cols=256, device=cuda).requires_grad_(True)
    y = mx.MXFakeQuantize.apply(x, E2M1, FLOOR)
    g = inputs.qat_grad(64, 256, device=cuda)
    y.backward(g)
    torch.cuda.synchronize()
    xb = bits(x.detach())
    assert np.array_equal(bits(y.detach()), oracle_mod.fake_quant_fwd(xb))
    assert np.array_equal(bits(x.grad), oracle_mod.fake_quant_bwd(xb, bits(g)))


@pytest.mark.parametrize("fm", [(E2M1, FLOOR), (E2M1, OAS | MBS_STATIC), (NVFP4, FLOOR | (1 << 8))],
                         ids=["fp4-FLOOR", "fp4-OAS+MBS_STATIC", "nvfp4-mma-scales"])
def test_pinned_host_quantize_is_pipelined_and_identical(mx, cuda, fm):
    """A pinned host tensor above two chunks goes through the chunked
    upload / kernel / download pipeline (chunks of 512 and 488 rows here);
    the result must equal the all-device call bit for bit."""
    fmt, m = fm
    x = inputs.random_bf16_bits((1000, 65536), seed=31)
    xh = x.pin_memory()
    hc, hs, hm = mx.quantize(xh, fmt, m)
    torch.cuda.synchronize()
    dc, ds, dm = mx.quantize(x.to(cuda), fmt, m)
    torch.cuda.synchronize()
    assert hc.is_pinned() and hs.is_pinned()
    assert torch.equal(hc, dc.cpu()) and torch.equal(hs, ds.cpu())
    if dm is not None:
        assert torch.equal(hm, dm.cpu())


def test_more_than_2_31_elements(mx, oracle_mod, cuda):
    """A tensor past 2^31 elements (4.3 GB of bf16): slice, block and scale
    indices must not wrap. Rows around element 2^31 and the last rows are
    checked against the oracle; every block's FLOOR byte against its amax."""
    rows, cols = 1049088, 2048                       # 2,148,532,224 elements
    g = torch.Generator(device=cuda).manual_seed(77)
    x = torch.empty(rows, cols, dtype=torch.bfloat16, device=cuda)
    x.normal_(generator=g)
    c, s, _ = mx.quantize(x, E2M1, FLOOR)
    torch.cuda.synchronize()
    edge = (1 << 31) // cols                          # the row holding element 2^31
    r = np.array([0, edge - 1, edge, edge + 1, rows - 2, rows - 1])
    xs = bits(x[r])
    oc, os_, _ = oracle_mod.quantize(xs, E2M1, FLOOR)
    assert np.array_equal(host_u8(c[r]), oc)
    assert np.array_equal(host_u8(s[r]), os_)
    amax = x.view(-1, 32).abs().amax(dim=1).view(torch.int16).to(torch.int32)
    want = torch.clamp((amax >> 7) - 2, min=0).to(torch.uint8)
    assert torch.equal(s.view(-1), want)
    del amax, want
    y = mx.dequantize(c[-4:], s[-4:], None, E2M1)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y), oracle_mod.dequantize(host_u8(c[-4:]), host_u8(s[-4:]), None,
                                                         4, cols, E2M1))


def test_binding_rejects_bad_out_buffers(mx, cuda):
    """Caller buffers that do not fit what the kernels write raise ValueError
    before any launch: a host buffer for a device input, short or narrower
    buffers, a buffer on the wrong device."""
    x = inputs.random_bf16_bits((4, 256), seed=12).to(cuda)
    u8 = lambda n, dev=cuda: torch.empty(n, dtype=torch.uint8, device=dev)
    with pytest.raises(ValueError):
        mx.quantize(x, out=(u8(512, "cpu"), u8(32), None))           # host codes
    with pytest.raises(ValueError):
        mx.quantize(x, E2M1, FLOOR | (1 << 8), out=(u8(512), u8(32), None))   # tiled needs 1024
    with pytest.raises(ValueError):
        mx.quantize(x, E4M3, FLOOR, out=(u8(512), u8(32), None))     # FP8 codes: 1024
    c, s, _ = mx.quantize(x)
    with pytest.raises(ValueError):
        mx.dequantize(c, s, out_dtype=torch.float32,
                      out=torch.empty(4, 256, dtype=torch.bfloat16, device=cuda))
    with pytest.raises(ValueError):
        mx.dequantize(c, s[:, :4].contiguous())                          # short scales
    with pytest.raises(ValueError):
        mx.fake_quant(x, out=torch.empty(4, 255, dtype=torch.bfloat16, device=cuda))
    with pytest.raises(ValueError):
        mx.fake_quant_bwd(x, x.cpu())
    with pytest.raises(ValueError):
        mx.fake_quant_bwd(x, x, out=torch.empty(4, 256, dtype=torch.float32, device=cuda))
    torch.cuda.synchronize()


def _golden_macro_cases():
    import json
    import os
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                           "hand_blocks.json")) as f:
        g = json.load(f)
    modes = {"MBS_STATIC": MBS_STATIC, "MBS_DYNAMIC": MBS_DYNAMIC,
             "OAS|MBS_STATIC": OAS | MBS_STATIC, "OAS|MBS_DYNAMIC": OAS | MBS_DYNAMIC}
    return [(f"{b['id']}-{m}", b["values"], modes[m], e) for b in g["macro_blocks"]
            if "expect" in b for m, e in b["expect"].items()]


@pytest.mark.parametrize("case", _golden_macro_cases(), ids=[c[0] for c in _golden_macro_cases()])
def test_hand_macro_blocks_on_gpu(mx, cuda, case):
    """The hand-derived macro blocks (factor k, sub-block bytes, codes,
    dequantized values, SSE) straight against their written derivations, on
    the GPU; each block is repeated over 3 rows x 2 macro columns."""
    _, values, m, e = case
    v = np.zeros(128, np.float32)
    v[:len(values)] = values
    x = torch.from_numpy(np.tile(v, (3, 2))).to(torch.bfloat16).to(cuda)
    c, s, mac = mx.quantize(x, E2M1, m)
    yf = mx.dequantize(c, s, mac, E2M1, torch.float32)
    bs, tot = mx.block_error(x, E2M1, m)
    torch.cuda.synchronize()
    assert bool((mac == e["k"]).all())
    assert host_u8(s).tolist() == [e["bytes"] * 2] * 3
    nib = host_u8(c)[:, :len(e["codes"])]
    got_codes = np.stack([nib & 15, nib >> 4], axis=-1).reshape(3, -1)[:, :len(e["codes"])]
    assert got_codes.tolist() == [e["codes"]] * 3
    y = yf.cpu().numpy().reshape(3, 2, 128)
    assert np.all(y[:, :, :len(e["dequant"])] == np.array(e["dequant"], np.float32))
    assert np.all(y[:, :, len(e["dequant"]):] == 0)
    assert np.isclose(tot[0].item(), 6 * e["sse"], rtol=REL, atol=0)
