"""Seeded synthetic inputs for the MX quantization workloads.

This module only draws random numbers; it holds none of the quantization
arithmetic, so the CUDA path and the CPU oracle can both be fed from it.
Each generator draws in float32 from a seeded ``torch.Generator`` on the
requested device and rounds once to bf16 (``.to(torch.bfloat16)``). The same
seed on another device gives a different stream: a comparison always copies
the one generated tensor to wherever the second side runs.

Workloads (shapes and distributions of the sources' examples; no trained
weights or datasets are used anywhere):

* ``outlier_act``  256x4096, N(0,1), 0.1% of entries (distinct positions)
  multiplied by 50 with a random sign.
* ``mlp_weight``   8192x3072 N(0, 0.02^2): a Llama-3.2-3B MLP weight shape.
* ``qat_act``      16384x3072 Student-t (nu = 3) * 0.5, the t variate built as
  Z0 / sqrt((Z1^2 + Z2^2 + Z3^2) / 3) from four seeded normal draws.
* ``qat_weight``   8192x3072 N(0, 0.02^2); ``qat_grad`` N(0, 1) upstream grads.
* ``heavy_tail``   8192x4096 N(0,1), 16 distinct channels x100, then 0.05% of
  positions (distinct) x20.
* ``moe_w13``      [128, 1536, 2048] N(0, 0.02^2) times a per-expert factor
  drawn from U(0.5, 2).
* ``bat_params``   random stand-ins for BATQuant's learned parameters (none
  are available): A = I + s N(0,1) [a, a], B_j = I + s N(0,1) [cols/32, b, b]
  (s = 0.1 by default), clip thresholds U(0.8, 1), all float32.
"""

from __future__ import annotations

import hashlib

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_act(rows=256, cols=4096, seed=0, device="cpu", frac=0.001, factor=50.0):
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    n = rows * cols
    k = int(round(frac * n))
    idx = torch.randperm(n, generator=g, device=device)[:k]
    sign = torch.randint(0, 2, (k,), generator=g, device=device).to(torch.float32) * 2 - 1
    flat = x.view(-1)
    flat[idx] = flat[idx] * factor * sign
    return x.to(torch.bfloat16)


def normal_weight(rows=8192, cols=3072, seed=1, device="cpu", std=0.02):
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std
    return x.to(torch.bfloat16)


def mlp_weight(rows=8192, cols=3072, seed=1, device="cpu"):
    return normal_weight(rows, cols, seed, device)


def qat_act(rows=16384, cols=3072, seed=2, device="cpu", nu=3, scale=0.5):
    g = _gen(seed, device)
    z0 = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros_like(z0)
    for _ in range(nu):
        z = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
        chi2 += z * z
    t = z0 / torch.sqrt(chi2 / nu)
    return (t * scale).to(torch.bfloat16)


def qat_weight(rows=8192, cols=3072, seed=102, device="cpu"):
    return normal_weight(rows, cols, seed, device)


def qat_grad(rows, cols, seed=202, device="cpu"):
    g = _gen(seed, device)
    return torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def heavy_tail(rows=8192, cols=4096, seed=3, device="cpu", n_channels=16, channel_factor=100.0,
               spike_frac=0.0005, spike_factor=20.0):
    g = _gen(seed, device)
    x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    ch = torch.randperm(cols, generator=g, device=device)[:n_channels]
    x[:, ch] *= channel_factor
    n = rows * cols
    k = int(round(spike_frac * n))
    idx = torch.randperm(n, generator=g, device=device)[:k]
    flat = x.view(-1)
    flat[idx] = flat[idx] * spike_factor
    return x.to(torch.bfloat16)


def moe_w13(experts=128, inter2=1536, hidden=2048, seed=4, device="cpu", std=0.02):
    g = _gen(seed, device)
    x = torch.randn(experts, inter2, hidden, generator=g, device=device, dtype=torch.float32)
    s = torch.rand(experts, 1, 1, generator=g, device=device, dtype=torch.float32) * 1.5 + 0.5
    x.mul_(s).mul_(std)
    return x.to(torch.bfloat16)


def bat_params(a, n_blocks, seed=5, device="cpu", spread=0.1, clip=True, lo=0.8):
    """(A [a, a], B [n_blocks, b, b], beta_min, beta_max [n_blocks] or None) float32."""
    g = _gen(seed, device)
    b = 32 // a
    A = torch.eye(a, device=device) + spread * torch.randn(a, a, generator=g, device=device)
    B = torch.eye(b, device=device) + spread * torch.randn(n_blocks, b, b, generator=g, device=device)
    if not clip:
        return A.contiguous(), B.contiguous(), None, None
    bmin = lo + (1 - lo) * torch.rand(n_blocks, generator=g, device=device)
    bmax = lo + (1 - lo) * torch.rand(n_blocks, generator=g, device=device)
    return A.contiguous(), B.contiguous(), bmin, bmax


def random_bf16_bits(shape, seed=0, device="cpu", finite_only=True):
    """Uniformly random bf16 bit patterns (optionally without Inf/NaN)."""
    g = _gen(seed, device)
    bits = torch.randint(0, 1 << 16, shape, generator=g, device=device, dtype=torch.int32)
    if finite_only:
        exp = (bits >> 7) & 0xFF
        bits = torch.where(exp == 0xFF, bits & ~(1 << 14), bits)   # exponent 0xFF -> 0xBF
    return bits.to(torch.int16).view(torch.bfloat16)


def bf16_bits_numpy(x: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor's bit patterns."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def sha256(x: torch.Tensor) -> str:
    return hashlib.sha256(bf16_bits_numpy(x).tobytes()).hexdigest()


# name -> (generator, kwargs, description); shapes as in the module docstring
WORKLOADS = {
    "outlier_act_256x4096": (outlier_act, {}, "MXFP4 quantize+dequantize, 256x4096 N(0,1) with 0.1% x50 outliers"),
    "mlp_weight_8192x3072": (mlp_weight, {}, "MXFP8 quantize, Llama-3.2-3B MLP weight 8192x3072 N(0,0.02^2)"),
    "qat_act_16384x3072": (qat_act, {}, "MXFP4 fake-quant, Student-t(3)*0.5 activations 16384x3072"),
    "qat_weight_8192x3072": (qat_weight, {}, "MXFP4 fake-quant, weight 8192x3072 N(0,0.02^2)"),
    "heavy_tail_8192x4096": (heavy_tail, {}, "MXFP4 OAS/MBS vs plain, 8192x4096 with outlier channels and spikes"),
    "moe_w13_128x1536x2048": (moe_w13, {}, "MoE w13 expert stack 128x1536x2048 MXFP4 quantize+pack"),
}
