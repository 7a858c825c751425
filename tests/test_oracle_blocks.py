"""Hand-worked blocks (tests/golden/hand_blocks.json) through the oracle.

Each block's expected scale bytes and element codes are derived in the fixture
from what the sources fix (E2M1 grid and maximum 6.0, E8M0 = 2^k, block 32,
the OCP scale rule with round-to-nearest-even and saturation, and the OAS
statement of "Unveiling the Potential of Quantization with MXFP4" 2.A).
"""

import json
import os

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(HERE, "golden", "hand_blocks.json")) as f:
    GOLDEN = json.load(f)

MODES = {"FLOOR": 0, "CEIL": 1, "OAS_RULE": 2, "OAS": 3, "MBS_STATIC": 1 << 4,
         "MBS_DYNAMIC": 2 << 4, "OAS|MBS_STATIC": 3 | 1 << 4, "OAS|MBS_DYNAMIC": 3 | 2 << 4}
FMTS = {"E2M1": 0, "E4M3": 1, "E5M2": 2, "E3M2": 3, "E2M3": 4, "INT8": 5}


def _block(values, n=32):
    """bf16 bits of a block: floats must be bf16-exact; strings are raw bit patterns."""
    out = np.zeros(n, np.uint16)
    for i, v in enumerate(values):
        if isinstance(v, str):
            out[i] = int(v, 16)
            continue
        b = torch.tensor([float(v)], dtype=torch.float32).to(torch.bfloat16)
        assert b.to(torch.float32).item() == float(v), "fixture value not exact in bf16"
        out[i] = b.view(torch.int16).numpy().view(np.uint16)[0]
    return out


def _codes(codes_packed, fmt, n):
    if fmt == 0:
        out = []
        for byte in codes_packed.ravel():
            out += [int(byte) & 0xF, int(byte) >> 4]
        return out[:n]
    return [int(c) for c in codes_packed.ravel()[:n]]


@pytest.mark.parametrize("blk", GOLDEN["blocks"], ids=[b["id"] for b in GOLDEN["blocks"]])
def test_hand_block(oracle_mod, blk):
    fmt = FMTS[blk["format"]]
    x = _block(blk["values"])
    for mode, byte in blk["bytes"].items():
        codes, scales, _ = oracle_mod.quantize(x.reshape(1, 32), fmt, MODES[mode])
        assert int(scales[0, 0]) == byte, (mode, int(scales[0, 0]), byte)
        if mode in blk["codes"]:
            exp = blk["codes"][mode]
            assert _codes(codes, fmt, len(exp)) == exp, mode


def macro_cases():
    """(id, values, mode, expectation) of every hand-worked macro block."""
    out = []
    for blk in GOLDEN["macro_blocks"]:
        if "expect" in blk:
            out += [(f"{blk['id']}-{m}", blk["values"], m, e) for m, e in blk["expect"].items()]
    return out


@pytest.mark.parametrize("case", macro_cases(), ids=[c[0] for c in macro_cases()])
def test_hand_macro_block_modes(oracle_mod, case):
    """MBS-Static / Dynamic (with and without OAS) on hand-worked macro blocks:
    the factor, the sub-block bytes, the first codes, their dequantized
    values and the macro-block SSE, all derived by hand in the fixture."""
    _, values, mode, e = case
    x = _block(values, 128).reshape(1, 128)
    codes, scales, macro = oracle_mod.quantize(x, 0, MODES[mode])
    assert int(macro[0, 0]) == e["k"]
    assert [int(s) for s in scales[0]] == e["bytes"]
    assert _codes(codes, 0, len(e["codes"])) == e["codes"]
    y = oracle_mod.dequantize(codes, scales, macro, 1, 128, 0, out_fp32=True).view(np.float32)[0]
    assert [float(v) for v in y[:len(e["dequant"])]] == e["dequant"]
    assert np.all(y[len(e["dequant"]):] == 0)
    bs, sd, _ = oracle_mod.block_error(x, 0, MODES[mode])
    assert sd == e["sse"] and bs.sum() == e["sse"]


@pytest.mark.parametrize("blk", [b for b in GOLDEN["macro_blocks"] if "expect" not in b],
                         ids=[b["id"] for b in GOLDEN["macro_blocks"] if "expect" not in b])
def test_hand_macro_block(oracle_mod, blk):
    x = _block(blk["values"], 128)
    codes, scales, macro = oracle_mod.quantize(x.reshape(1, 128), 0, MODES[blk["scaling"]])
    assert int(macro[0, 0]) == blk["k"]
    assert [int(s) for s in scales[0]] == blk["bytes"]
    exp = blk["codes"]
    assert _codes(codes, 0, len(exp)) == exp
    # the dequantized maximum is 6 * (256 + k) / 256
    y = oracle_mod.dequantize(codes, scales, macro, 1, 128, 0, out_fp32=True)
    assert y.view(np.float32)[0, 0] == 6.0 * (256 + blk["k"]) / 256


def test_metadata_counts(oracle_mod):
    # one E8M0 byte per 32 elements, one factor byte per 128 (MBS); FP4 packs 2/byte
    # ("[vLLM] MXFP8/MXFP4" format table: 1 scale byte per 32 elements, ~3%)
    x = np.zeros((3, 256), np.uint16)
    c, s, m = oracle_mod.quantize(x, 0, 0)
    assert c.shape == (3, 128) and s.shape == (3, 8) and m is None
    c, s, m = oracle_mod.quantize(x, 0, 1 << 4)
    assert m.shape == (3, 2)
    c, s, m = oracle_mod.quantize(x, 1, 0)
    assert c.shape == (3, 256) and s.shape == (3, 8)
    # scale metadata per element: 1/32 byte = 3.125% of the 8-bit payload
    assert s.size / c.size == 1 / 32
