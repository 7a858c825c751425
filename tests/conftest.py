"""Shared fixtures. GPU tests carry the ``gpu`` marker; everything else runs on CPU."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build_oracle()
    oracle.set_threads(min(8, os.cpu_count() or 1))
    return oracle


@pytest.fixture(scope="session")
def mx():
    """The product binding with libmx.so built (nvcc cross-compiles without a GPU)."""
    from fp8_quantization_mx_b200 import build
    build.build()
    import fp8_quantization_mx_b200 as mx
    mx.load_library()
    return mx


@pytest.fixture(scope="session")
def cuda(mx):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)
