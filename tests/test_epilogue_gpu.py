"""GPU parity of the output epilogue (kda_output_gate_norm, through the C ABI) against the fp64 oracle.

out[r, j] = o[r, j] / sqrt(mean_j o[r, j]^2 + eps) * weight[j] * sigmoid(g[r, j]) per (token, head) row.
The oracle runs on the same (bf16-rounded) values the GPU reads.  Tolerance, element by element:
|gpu - oracle| <= 2^-8 |oracle| + 1e-6 max|oracle| for bf16 (one final rounding to bf16, fp32
arithmetic before it), 4e-6 |oracle| + 1e-7 max|oracle| for fp32 (hardware rsqrt / exp2 approximations).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import kimi_delta_attention_29_b200 as kda
import oracle

pytestmark = pytest.mark.gpu

REL = {torch.bfloat16: 2.0 ** -8, torch.float32: 4e-6}
ABS = {torch.bfloat16: 1e-6, torch.float32: 1e-7}


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def make(n_tok, H, dv, dtype, seed, device, g_scale=2.0):
    gen = torch.Generator().manual_seed(seed)
    scale = torch.exp(torch.randn(n_tok, H, 1, generator=gen))          # rows of very different norms
    o = (torch.randn(n_tok, H, dv, generator=gen) * scale).to(dtype).to(device)
    g = (torch.randn(n_tok, H, dv, generator=gen) * g_scale).to(dtype).to(device)
    w = (0.5 + torch.rand(dv, generator=gen)).to(device)
    return o, g, w


def check(out, ref, dtype):
    got = np64(out)
    bound = REL[dtype] * np.abs(ref) + ABS[dtype] * np.abs(ref).max()
    assert np.isfinite(got).all()
    worst = float((np.abs(got - ref) - bound).max())
    assert worst <= 0.0, f"max excess over the bound {worst:.3e}"


@pytest.mark.parametrize("dtype,dv", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 128),
                                      (torch.float32, 64)])
@pytest.mark.parametrize("n_tok,H", [(1, 1), (37, 3), (1001, 4)])
def test_epilogue_matches_oracle(cuda_device, dtype, dv, n_tok, H):
    o, g, w = make(n_tok, H, dv, dtype, seed=n_tok + dv, device=cuda_device)
    out = kda.kda_output_gate_norm(o, g, w, eps=1e-6)
    torch.cuda.synchronize(cuda_device)
    check(out, oracle.output_gate_norm(np64(o), np64(g), np64(w), eps=1e-6), dtype)


def test_epilogue_in_place_and_unit_weight(cuda_device):
    o, g, _ = make(513, 2, 128, torch.bfloat16, seed=3, device=cuda_device)
    ref = oracle.output_gate_norm(np64(o), np64(g), None, eps=1e-5)
    res = kda.kda_output_gate_norm(o, g, None, eps=1e-5, out=o)
    torch.cuda.synchronize(cuda_device)
    assert res.data_ptr() == o.data_ptr()
    check(o, ref, torch.bfloat16)


def test_epilogue_saturated_gates(cuda_device):
    """g = +100 passes the normalised row through (times weight); g = -100 closes the gate exactly."""
    o, _, w = make(64, 2, 128, torch.float32, seed=4, device=cuda_device)
    g = torch.full_like(o, 100.0)
    g[:, 1] = -100.0
    out = kda.kda_output_gate_norm(o, g, w, eps=1e-6)
    torch.cuda.synchronize(cuda_device)
    assert torch.count_nonzero(out[:, 1]) == 0
    check(out, oracle.output_gate_norm(np64(o), np64(g), np64(w), eps=1e-6), torch.float32)


def test_epilogue_empty(cuda_device):
    o = torch.empty(0, 4, 128, dtype=torch.bfloat16, device=cuda_device)
    out = kda.kda_output_gate_norm(o, o, None)
    assert out.shape == o.shape


def test_epilogue_full_size_sampled(cuda_device):
    """The long-context output (131072 tokens x 32 heads x 128, bf16), 4,096 sampled rows checked."""
    T, H, dv = 131072, 32, 128
    gen = torch.Generator(device=cuda_device).manual_seed(9)
    o = torch.randn(T, H, dv, generator=gen, device=cuda_device).to(torch.bfloat16)
    g = (2.0 * torch.randn(T, H, dv, generator=gen, device=cuda_device)).to(torch.bfloat16)
    w = 0.5 + torch.rand(dv, generator=gen, device=cuda_device)
    out = kda.kda_output_gate_norm(o, g, w, eps=1e-6)
    torch.cuda.synchronize(cuda_device)
    rows = torch.from_numpy(np.random.default_rng(1).choice(T * H, size=4096, replace=False)).to(cuda_device)
    pick = lambda t: t.reshape(T * H, dv).index_select(0, rows)
    check(pick(out), oracle.output_gate_norm(np64(pick(o)), np64(pick(g)), np64(w), eps=1e-6), torch.bfloat16)
