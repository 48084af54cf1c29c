"""The layer prologue fused into the kernels (kda_chunk_fwd_ex / kda_decode_multi_ex): q and k
L2-normalised per (token, head), and the log decay taken from the gate projection g as
-exp(A_log[h]) * softplus(g + dt_bias[h, c]).  Reference: the fp64 oracle's prologue followed by its
token-by-token recurrence, on the same (bf16-rounded) raw inputs; tolerances as in the other parity
tests (bf16 2e-2, fp32 1e-4, relative to max |reference|)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import kimi_delta_attention_29_b200 as kda
import oracle
from kimi_delta_attention_29_b200 import _lib
from kimi_delta_attention_29_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
L2, GATE = _lib.KDA_PROLOGUE_L2NORM_QK, _lib.KDA_PROLOGUE_GATE


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(gpu, ref) -> float:
    g = np64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    return float(np.abs(g - ref).max() / max(np.abs(ref).max(), 1e-30))


def raw_layer_inputs(x, H, dk, dev, seed, flags=L2 | GATE):
    """Unnormalised q, k (rows scaled by e^N(0,1)); with the gate flag, log_alpha replaced by a gate
    projection g ~ 2 N(0,1) (without it, log_alpha stays a valid log decay <= 0); A_log, dt_bias."""
    g = torch.Generator().manual_seed(seed)
    for name in ("q", "k"):
        sc = torch.exp(torch.randn(*x[name].shape[:-1], 1, generator=g)).to(dev)
        x[name] = (x[name].float() * sc).to(x[name].dtype).contiguous()
    raw_g = torch.randn(*x["log_alpha"].shape, generator=g) * 2.0
    if flags & GATE:
        x["log_alpha"] = raw_g.to(dev)
    A_log = (torch.randn(H, generator=g) * 0.5).to(dev)
    dt_bias = (torch.randn(H, dk, generator=g) * 0.3).to(dev)
    return A_log, dt_bias


def oracle_with_prologue(x, flags, A_log, dt_bias, h0):
    q, k, la = oracle.prologue(np64(x["q"]), np64(x["k"]), np64(x["log_alpha"]), flags, A_log=np64(A_log),
                               dt_bias=np64(dt_bias))
    cu = None if x.get("cu_seqlens") is None else x["cu_seqlens"].cpu().numpy()
    return oracle.recurrent(q, k, np64(x["v"]), la, np64(x["beta"]), h0, cu)


@pytest.mark.parametrize("dtype,d,flags", [(torch.bfloat16, 128, L2), (torch.bfloat16, 128, GATE),
                                           (torch.bfloat16, 128, L2 | GATE), (torch.float32, 64, L2 | GATE),
                                           (torch.float32, 128, L2 | GATE)])
def test_prefill_prologue_matches_oracle(cuda_device, dtype, d, flags):
    H, T = 3, 200
    x = {kk: (vv.to(cuda_device) if isinstance(vv, torch.Tensor) else vv)
         for kk, vv in gen.make_prefill(2, T, H, d, d, dtype, h0_std=0.1, seed=21).items()}
    A_log, dt_bias = raw_layer_inputs(x, H, d, cuda_device, seed=5, flags=flags)
    o, hT = kda.kda_chunk_fwd_ex(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, flags=flags,
                                 A_log=A_log, dt_bias=dt_bias)
    o_ref, h_ref = oracle_with_prologue(x, flags, A_log, dt_bias, np64(x["h0"]))
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(hT, h_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_prefill_prologue_strong_gates(cuda_device, dtype, d):
    """Gate activations at the strong end of the layer's range: exp(A_log) up to 16 per head and
    gate projections ~ 3 N(0,1), so single steps reach log alpha of -100 and beyond."""
    H, T = 4, 260
    x = {kk: (vv.to(cuda_device) if isinstance(vv, torch.Tensor) else vv)
         for kk, vv in gen.make_prefill(1, T, H, d, d, dtype, h0_std=0.3, seed=31).items()}
    A_log, dt_bias = raw_layer_inputs(x, H, d, cuda_device, seed=7, flags=L2 | GATE)
    x["log_alpha"] = x["log_alpha"] * 1.5
    A_log = torch.log(torch.tensor([1.0, 4.0, 9.0, 16.0], device=cuda_device))
    o, hT = kda.kda_chunk_fwd_ex(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, flags=L2 | GATE,
                                 A_log=A_log, dt_bias=dt_bias)
    o_ref, h_ref = oracle_with_prologue(x, L2 | GATE, A_log, dt_bias, np64(x["h0"]))
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(hT, h_ref) <= TOL[dtype]


def test_prefill_prologue_varlen_and_no_bias(cuda_device):
    lens = torch.tensor([70, 0, 130, 5])
    cu = gen.cu_seqlens_from_lengths(lens)
    H, d = 2, 128
    x = {kk: (vv.to(cuda_device) if isinstance(vv, torch.Tensor) else vv)
         for kk, vv in gen.make_prefill(1, int(cu[-1]), H, d, d, torch.bfloat16, h0_std=0.2, seed=22,
                                        cu_seqlens=cu).items()}
    A_log, _ = raw_layer_inputs(x, H, d, cuda_device, seed=6)
    zero_bias = torch.zeros(H, d, device=cuda_device)
    o, hT = kda.kda_chunk_fwd_ex(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], x["cu_seqlens"],
                                 flags=L2 | GATE, A_log=A_log, dt_bias=None)
    o_ref, h_ref = oracle_with_prologue(x, L2 | GATE, A_log, zero_bias, np64(x["h0"]))
    assert rel_err(o, o_ref) <= 2e-2 and rel_err(hT, h_ref) <= 2e-2


def test_flags_zero_is_the_plain_entry_point(cuda_device):
    x = {kk: (vv.to(cuda_device) if isinstance(vv, torch.Tensor) else vv)
         for kk, vv in gen.make_prefill(1, 300, 2, 128, 128, torch.bfloat16, h0_std=0.1, seed=23).items()}
    o1, h1 = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None)
    o2, h2 = kda.kda_chunk_fwd_ex(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, flags=0)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_decode_multi_prologue_matches_oracle(cuda_device, dtype, d):
    N, Tq, H, P = 3, 11, 2, 5
    x = gen.make_decode_tokens(N, Tq, H, d, d, dtype=dtype, seed=24, device=cuda_device)
    A_log, dt_bias = raw_layer_inputs(x, H, d, cuda_device, seed=7)
    pool = gen.make_decode_state(P, H, d, d, std=0.3, seed=4, device=cuda_device)
    before = pool.clone()
    s_in, s_out = [4, 0, 2], [1, 3, 2]
    slot = lambda vals: torch.tensor(vals, dtype=torch.int32, device=cuda_device)
    o = kda.kda_decode_multi_ex(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, slot_in=slot(s_in),
                                slot_out=slot(s_out), flags=L2 | GATE, A_log=A_log, dt_bias=dt_bias)
    o_ref, S_ref = oracle_with_prologue(x, L2 | GATE, A_log, dt_bias, np64(before)[s_in])
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(pool[s_out], S_ref) <= TOL[dtype]
