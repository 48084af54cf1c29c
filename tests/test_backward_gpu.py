"""GPU parity of the chunkwise backward (kda_chunk_bwd, through the C ABI) against the fp64 oracle's
token-by-token adjoint (itself pinned by finite differences in test_oracle.py).

Inputs are the seeded prefill workloads' generators; the oracle runs on the same (bf16-rounded)
values the GPU reads.  Each gradient is compared as max |gpu - oracle| / max |oracle|: <= 1e-2 for
bf16 inputs (dq, dk, dv are rounded to bf16; fp32 arithmetic), <= 2e-4 for fp32 inputs.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import kimi_delta_attention_29_b200 as kda
import oracle
from kimi_delta_attention_29_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 1e-2, torch.float32: 2e-4}
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dh0")


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def upstream(x, N, dev, seed, with_dhT=True):
    g = torch.Generator().manual_seed(seed)
    do = torch.randn(x["v"].shape, generator=g).to(x["v"].dtype).to(dev)
    H, dk, dv = x["q"].shape[2], x["q"].shape[3], x["v"].shape[3]
    dhT = torch.randn(N, H, dk, dv, generator=g).to(dev) if with_dhT else None
    return do, dhT


def oracle_grads(x, do, dhT):
    cu = None if x.get("cu_seqlens") is None else x["cu_seqlens"].cpu().numpy()
    return oracle.recurrent_bwd(np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["log_alpha"]), np64(x["beta"]),
                                None if x["h0"] is None else np64(x["h0"]), cu, np64(do),
                                None if dhT is None else np64(dhT))


def check(got, ref, tol, names=NAMES):
    errs = {}
    for name in names:
        r = ref[name]
        den = float(np.abs(r).max())
        assert den > 0, name
        err = float(np.abs(np64(got[name]) - r).max() / den)
        assert np.isfinite(np64(got[name])).all(), name
        assert err <= tol, f"{name}: {err:.3e} > {tol:.1e}"
        errs[name] = err
    return errs


def run(x, do, dhT):
    return kda.kda_chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], x.get("cu_seqlens"), do=do,
                             dh_T=dhT)


@pytest.mark.parametrize("dtype,d,T", [(torch.bfloat16, 128, 200), (torch.bfloat16, 128, 64),
                                       (torch.float32, 64, 130), (torch.float32, 128, 97),
                                       (torch.bfloat16, 64, 1)])
def test_backward_matches_oracle(cuda_device, grad_log, dtype, d, T):
    x = gen.make_prefill(2, T, 2, d, d, dtype, gate_shift=1.0, h0_std=0.2, seed=50 + T, device=cuda_device)
    do, dhT = upstream(x, 2, cuda_device, seed=T)
    got = run(x, do, dhT)
    torch.cuda.synchronize(cuda_device)
    errs = check(got, oracle_grads(x, do, dhT), TOL[dtype])
    grad_log(f"backward {'bf16' if dtype == torch.bfloat16 else 'fp32'} d={d} B=2 H=2 T={T}", errs, TOL[dtype])


def test_backward_no_h0_no_dhT(cuda_device):
    x = gen.make_prefill(1, 150, 3, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.0, seed=61, device=cuda_device)
    x["h0"] = None
    do, _ = upstream(x, 1, cuda_device, seed=3, with_dhT=False)
    got = run(x, do, None)
    torch.cuda.synchronize(cuda_device)
    check(got, oracle_grads(x, do, None), TOL[torch.bfloat16])


def test_backward_varlen(cuda_device):
    lens = torch.tensor([70, 0, 130, 5])
    cu = gen.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    x = gen.make_prefill(1, T, 2, 128, 128, torch.bfloat16, gate_shift=1.0, h0_std=0.0, seed=62, device=cuda_device)
    x["h0"] = (0.2 * torch.randn(4, 2, 128, 128, generator=torch.Generator().manual_seed(1))).to(cuda_device)
    x["cu_seqlens"] = cu.to(torch.int32).to(cuda_device)
    do, dhT = upstream(x, 4, cuda_device, seed=4)
    got = run(x, do, dhT)
    torch.cuda.synchronize(cuda_device)
    ref = oracle_grads(x, do, dhT)
    check(got, ref, TOL[torch.bfloat16])
    # the empty sequence passes its state gradient straight through
    assert torch.equal(got["dh0"][1], dhT[1])


def test_backward_strong_decay_steps(cuda_device):
    """Steps at log alpha = -60 are applied as 2^-15 (as in the CUDA-core forward); everything else
    still matches the exact adjoint within the fp32 tolerance, and the clamped steps' dlog_alpha is 0."""
    x = gen.make_prefill(1, 160, 2, 64, 64, torch.float32, gate_shift=0.0, h0_std=0.3, seed=63)
    la = x["log_alpha"].clone()
    mask = torch.rand(la.shape, generator=torch.Generator().manual_seed(5)) < 0.03
    la[mask] = -60.0
    x["log_alpha"] = la
    x = {k_: (v_.to(cuda_device) if torch.is_tensor(v_) else v_) for k_, v_ in x.items()}
    do, dhT = upstream(x, 1, cuda_device, seed=6)
    got = run(x, do, dhT)
    torch.cuda.synchronize(cuda_device)
    check(got, oracle_grads(x, do, dhT), 1e-3)
    assert torch.count_nonzero(got["dlog_alpha"][mask.to(cuda_device)]) == 0


def test_backward_deterministic(cuda_device):
    x = gen.make_prefill(2, 300, 2, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.1, seed=64, device=cuda_device)
    do, dhT = upstream(x, 2, cuda_device, seed=7)
    a, b = run(x, do, dhT), run(x, do, dhT)
    torch.cuda.synchronize(cuda_device)
    for name in NAMES:
        assert torch.equal(a[name], b[name]), name


def test_backward_empty(cuda_device):
    x = gen.make_prefill(1, 0, 2, 128, 128, torch.bfloat16, h0_std=0.1, seed=65, device=cuda_device)
    do, dhT = upstream(x, 1, cuda_device, seed=8)
    got = run(x, do, dhT)
    torch.cuda.synchronize(cuda_device)
    assert torch.equal(got["dh0"], dhT)


def test_backward_train_shape_heads(cuda_device, grad_log):
    """The training workload's sequence length (T = 4096, d = 128, bf16), two heads, full comparison."""
    x = gen.make_prefill(1, 4096, 2, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.0, seed=66,
                         device=cuda_device)
    do, dhT = upstream(x, 1, cuda_device, seed=9)
    got = run(x, do, dhT)
    torch.cuda.synchronize(cuda_device)
    errs = check(got, oracle_grads(x, do, dhT), TOL[torch.bfloat16])
    grad_log("backward bf16 d=128 T=4096 (training length, 2 heads)", errs, TOL[torch.bfloat16])
