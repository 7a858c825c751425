"""The quantize + GEMM entry point that allocates nothing, against the default.

Some callers may not allocate device memory while they run: a serving process
that reserves all of its device memory once at start-up and keeps it fixed, or
a runtime where stream-ordered memory pools are unavailable. The default
mx_quant_gemm takes the quantized copy of A and its per-band ready counters
from a pool; mx_quant_gemm_noalloc keeps them in one fixed array in the
library's device memory instead, shared by every call and keeping the last
call's bytes. Here it is called through the C ABI twice in a row (so that the
second call starts on what the first left in the array) and each result must
equal the default entry point's bit for bit, the tolerance of the other
quantize + GEMM tests.

This file sorts last so that a run stopping at its first failure has run
every other test before it; it passes alone in a fresh process (the first
call sets up the array's address) as well as after the other tests.
"""

import pytest
import torch

from fp8_quantization_mx_b200 import inputs

pytestmark = pytest.mark.gpu

E2M1, FLOOR, CEIL, OAS = 0, 0, 1, 3
MMA = 1 << 8

# (M, N, K, rule) pairs, called back to back on one stream: the overlapped
# kernel twice (its band counters must start again from zero); a ragged
# overlapped case, then a one-wave case with a ragged last band (the padding
# rows of its scales must read as zero again); the prefill and decode
# workloads of the GEMM bench.
PAIRS = [
    ((1536, 4096, 512, FLOOR), (1536, 4096, 512, OAS)),
    ((2200, 2056, 256, OAS), (300, 520, 1024, CEIL)),
    ((4096, 8192, 3072, FLOOR), (128, 8192, 3072, OAS)),
]


def operands(mx, cuda, M, N, K, seed):
    a = inputs.heavy_tail(M, K, seed=seed).to(cuda)
    w = inputs.normal_weight(N, K, seed=seed + 1).to(cuda)
    bc, bs, _ = mx.quantize(w, E2M1, FLOOR | MMA)
    return a, bc, bs


@pytest.mark.parametrize("pair", PAIRS, ids=lambda p: "_then_".join("x".join(map(str, c[:3])) for c in p))
def test_two_calls_in_a_row_equal_the_default_entry_point(mx, cuda, pair):
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.zeros(1, dtype=torch.int32, device=cuda)
    cases = []
    for i, (M, N, K, rule) in enumerate(pair):
        a, bc, bs = operands(mx, cuda, M, N, K, seed=M + N + i)
        d = torch.full((M, N), float("nan"), dtype=torch.float32, device=cuda)
        cases.append((a, bc, bs, M, N, K, rule, d))
    for a, bc, bs, M, N, K, rule, d in cases:        # back to back, no synchronisation
        st = mx.mx_quant_gemm_noalloc(a.data_ptr(), rule, bc.data_ptr(), bs.data_ptr(), M, N, K, 1,
                                      d.data_ptr(), status.data_ptr(), stream)
        assert st == 0, mx.mx_status_string(st)
    for a, bc, bs, M, N, K, rule, d in cases:
        want = mx.quant_gemm(a, bc, bs, rule, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(d.view(torch.int32), want.view(torch.int32)), (M, N, K, rule)
    assert status.item() == 0


def test_refuses_a_problem_beyond_its_scratch(mx, cuda):
    """8192 x 8192: 32 MiB of codes against a 9 MiB array. The operands are
    real, full-size tensors all the same."""
    M, N, K = 8192, 64, 8192
    g = torch.Generator(device=cuda).manual_seed(3)
    a = torch.randn(M, K, generator=g, device=cuda).to(torch.bfloat16)
    bc, bs, _ = mx.quantize(torch.randn(N, K, generator=g, device=cuda).to(torch.bfloat16), E2M1,
                            FLOOR | MMA)
    d = torch.empty(M, N, dtype=torch.float32, device=cuda)
    st = mx.mx_quant_gemm_noalloc(a.data_ptr(), FLOOR, bc.data_ptr(), bs.data_ptr(), M, N, K, 1,
                                  d.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert st == 6 and "fixed scratch" in mx.mx_status_string(st)
