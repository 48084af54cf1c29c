"""Seeded synthetic inputs for KDA prefill and decode.

This module is shared by the tests, the benchmark and the smoke check.  It holds
no KDA arithmetic: it only draws random tensors with the distributions of the
long-context workloads (q, k ~ N(0,1) then L2-normalised per (token, head);
v ~ N(0,1); beta = sigmoid(N(0,1)); log_alpha = -softplus(N(0,1) + shift);
h0 ~ N(0, std)), seeded by a torch.Generator on the requested device.  It imports
nothing from the CUDA binding or from the oracle.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    gate_shift: float
    h0_std: float          # 0 -> zero initial state
    varlen_seqs: int = 0   # >0 -> packed varlen batch (B = 1) with this many sequences
    varlen_min: int = 0
    varlen_max: int = 0


@dataclass(frozen=True)
class DecodeShape:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    steps: int
    s0_std: float


# The five workloads, named by what they are.
TINY_FP32 = PrefillShape("tiny_fp32_B1_H2_T256_d64", 1, 256, 2, 64, 64, torch.float32, 0.0, 0.0)
TRAIN = PrefillShape("train_B4_H16_T4096_d128", 4, 4096, 16, 128, 128, torch.bfloat16, 2.0, 0.0)
LONG = PrefillShape("long_B1_H32_T131072_d128", 1, 131072, 32, 128, 128, torch.bfloat16, 2.0, 0.02)
VARLEN = PrefillShape("varlen_64seq_L512-16384_H32_d128", 1, 0, 32, 128, 128, torch.bfloat16, 2.0, 0.0,
                      varlen_seqs=64, varlen_min=512, varlen_max=16384)
DECODE = DecodeShape("decode_N256_H32_d128_1024steps", 256, 32, 128, 128, torch.bfloat16, 1024, 0.02)


def varlen_lengths(num_seqs: int, lo: int, hi: int, seed: int = 0) -> torch.Tensor:
    """Sequence lengths uniform in [lo, hi] (inclusive), drawn on the CPU."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randint(lo, hi + 1, (num_seqs,), generator=g, dtype=torch.int64)


def cu_seqlens_from_lengths(lengths: torch.Tensor) -> torch.Tensor:
    cu = torch.zeros(lengths.numel() + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lengths.to(torch.int64), 0).to(torch.int32)
    return cu


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_prefill(B: int, T: int, H: int, dk: int, dv: int, dtype: torch.dtype = torch.bfloat16,
                 gate_shift: float = 2.0, h0_std: float = 0.0, seed: int = 0,
                 device: str | torch.device = "cpu", cu_seqlens: torch.Tensor | None = None,
                 ) -> dict:
    """Draw one prefill batch.  Returns q, k, v (dtype), log_alpha, beta, h0 (fp32 or None),
    cu_seqlens (int32 on `device` or None) and num_seqs."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed)
    f32 = dict(device=device, dtype=torch.float32)
    q = _unit_rows(torch.randn(B, T, H, dk, generator=g, **f32)).to(dtype)
    k = _unit_rows(torch.randn(B, T, H, dk, generator=g, **f32)).to(dtype)
    v = torch.randn(B, T, H, dv, generator=g, **f32).to(dtype)
    log_alpha = -F.softplus(torch.randn(B, T, H, dk, generator=g, **f32) + gate_shift)
    beta = torch.sigmoid(torch.randn(B, T, H, generator=g, **f32))
    num_seqs = B if cu_seqlens is None else int(cu_seqlens.numel() - 1)
    h0 = None
    if h0_std > 0:
        h0 = torch.randn(num_seqs, H, dk, dv, generator=g, **f32) * h0_std
    cu = None if cu_seqlens is None else cu_seqlens.to(device=device, dtype=torch.int32)
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, h0=h0, cu_seqlens=cu,
                num_seqs=num_seqs)


def make_prefill_for(shape: PrefillShape, seed: int = 0, device="cpu") -> dict:
    cu = None
    T = shape.T
    if shape.varlen_seqs:
        lengths = varlen_lengths(shape.varlen_seqs, shape.varlen_min, shape.varlen_max, seed)
        cu = cu_seqlens_from_lengths(lengths)
        T = int(cu[-1])
    return make_prefill(shape.B, T, shape.H, shape.dk, shape.dv, shape.dtype, shape.gate_shift,
                        shape.h0_std, seed, device, cu)


def make_decode_state(N: int, H: int, dk: int, dv: int, std: float = 0.02, seed: int = 0,
                      device="cpu") -> torch.Tensor:
    g = torch.Generator(device=torch.device(device)).manual_seed(seed)
    return torch.randn(N, H, dk, dv, generator=g, device=device, dtype=torch.float32) * std


def make_decode_token(N: int, H: int, dk: int, dv: int, dtype=torch.bfloat16, gate_shift=2.0,
                      seed: int = 1000, device="cpu") -> dict:
    """Inputs of one decode step for N*H states (step s uses seed 1000 + s)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed)
    f32 = dict(device=device, dtype=torch.float32)
    q = _unit_rows(torch.randn(N, H, dk, generator=g, **f32)).to(dtype)
    k = _unit_rows(torch.randn(N, H, dk, generator=g, **f32)).to(dtype)
    v = torch.randn(N, H, dv, generator=g, **f32).to(dtype)
    log_alpha = -F.softplus(torch.randn(N, H, dk, generator=g, **f32) + gate_shift)
    beta = torch.sigmoid(torch.randn(N, H, generator=g, **f32))
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta)


def make_decode_tokens(N: int, Tq: int, H: int, dk: int, dv: int, dtype=torch.bfloat16, gate_shift=2.0,
                       seed: int = 2000, device="cpu") -> dict:
    """Inputs of Tq consecutive decode tokens for N sequences x H heads, token-major [N, Tq, H, ...]
    (the same distributions as make_decode_token)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(seed)
    f32 = dict(device=device, dtype=torch.float32)
    q = _unit_rows(torch.randn(N, Tq, H, dk, generator=g, **f32)).to(dtype)
    k = _unit_rows(torch.randn(N, Tq, H, dk, generator=g, **f32)).to(dtype)
    v = torch.randn(N, Tq, H, dv, generator=g, **f32).to(dtype)
    log_alpha = -F.softplus(torch.randn(N, Tq, H, dk, generator=g, **f32) + gate_shift)
    beta = torch.sigmoid(torch.randn(N, Tq, H, generator=g, **f32))
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta)
