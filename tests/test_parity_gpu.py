"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Tolerance (the same for o and for the final state, each measured separately):
    max |gpu - oracle| / max |oracle|  <=  2e-2 for bf16 q/k/v/o  (fp32 gates, accumulation, state)
                                       <=  1e-4 for fp32 q/k/v/o
The oracle runs on the same bf16-rounded values the GPU reads, widened to float64.  Full-size
workloads are checked on sampled (sequence, head) units and sampled value columns: column j of
o and h_T depends only on column j of v and h0 (a pinned property of the oracle), so the oracle
can compute a few columns of a head cheaply.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import kimi_delta_attention_29_b200 as kda
import oracle
from kimi_delta_attention_29_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(gpu, ref) -> float:
    gpu = np64(gpu) if torch.is_tensor(gpu) else gpu
    den = float(np.abs(ref).max())
    assert den > 0, "reference is identically zero"
    return float(np.abs(gpu - ref).max() / den)


def to_dev(d, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in d.items()}


def run_fwd(x, **kw):
    return kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], x["cu_seqlens"], **kw)


def oracle_fwd(x, heads=None, cols=None):
    """Oracle on (optionally) a subset of heads and value columns."""
    sel = (lambda t, ax: t) if heads is None else (lambda t, ax: t.index_select(ax, torch.as_tensor(heads)))
    q, k, la = sel(x["q"].cpu(), 2), sel(x["k"].cpu(), 2), sel(x["log_alpha"].cpu(), 2)
    v, beta = sel(x["v"].cpu(), 2), sel(x["beta"].cpu(), 2)
    h0 = None if x["h0"] is None else sel(x["h0"].cpu(), 1)
    if cols is not None:
        v = v[..., cols]
        h0 = None if h0 is None else h0[..., cols]
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu().numpy()
    return oracle.recurrent(np64(q), np64(k), np64(v), np64(la), np64(beta),
                            None if h0 is None else np64(h0), cu_seqlens=cu)


# ------------------------------------------------------------------------------------------ decode
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.float32, 128),
                                     (torch.bfloat16, 64)])
def test_decode_matches_oracle(cuda_device, dtype, d):
    N, H, steps = 3, 2, 24
    S = gen.make_decode_state(N, H, d, d, std=0.5, seed=3, device=cuda_device)
    S_ref = np64(S)
    for s in range(steps):
        x = gen.make_decode_token(N, H, d, d, dtype=dtype, gate_shift=0.0, seed=100 + s, device=cuda_device)
        o = kda.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
        o_ref, S_ref = oracle.decode_step(np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["log_alpha"]),
                                          np64(x["beta"]), S_ref)
        assert rel_err(o, o_ref) <= TOL[dtype], f"step {s}"
    assert rel_err(S, S_ref) <= TOL[dtype]


def test_decode_full_size_sampled(cuda_device, parity_log):
    """256 x 32 states of 128 x 128, 1024 steps (the decode workload), sampled states checked."""
    shp = gen.DECODE
    S = gen.make_decode_state(shp.N, shp.H, shp.dk, shp.dv, std=shp.s0_std, seed=0, device=cuda_device)
    rng = np.random.default_rng(7)
    units = sorted(rng.choice(shp.N * shp.H, size=12, replace=False).tolist())
    idx = torch.as_tensor(units, device=cuda_device)
    flat = lambda t: t.reshape(shp.N * shp.H, *t.shape[2:])
    S_ref = np64(flat(S).index_select(0, idx))[:, None]              # [12, 1, dk, dv]
    worst = 0.0
    for s in range(shp.steps):
        x = gen.make_decode_token(shp.N, shp.H, shp.dk, shp.dv, dtype=shp.dtype, seed=1000 + s, device=cuda_device)
        o = kda.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
        pick = {kk: np64(flat(x[kk]).index_select(0, idx))[:, None] for kk in ("q", "k", "v", "log_alpha", "beta")}
        o_ref, S_ref = oracle.decode_step(pick["q"], pick["k"], pick["v"], pick["log_alpha"], pick["beta"], S_ref)
        if s % 64 == 0 or s == shp.steps - 1:
            worst = max(worst, rel_err(flat(o).index_select(0, idx)[:, None], o_ref))
    err_s = rel_err(flat(S).index_select(0, idx)[:, None], S_ref)
    parity_log("decode 256 x 32 states, 1024 steps (12 states; o every 64th step)", worst, err_s, TOL[shp.dtype])
    assert worst <= TOL[shp.dtype]
    assert err_s <= TOL[shp.dtype]


# ------------------------------------------------------------------------------------------ prefill
def test_prefill_tiny_fp32(cuda_device):
    """B=1, H=2, T=256, d=64, fp32 (the tiny fp32 workload), full comparison."""
    x = to_dev(gen.make_prefill_for(gen.TINY_FP32, seed=0), cuda_device)
    o, hT = run_fwd(x)
    o_ref, h_ref = oracle_fwd(x)
    assert rel_err(o, o_ref) <= 1e-4
    assert rel_err(hT, h_ref) <= 1e-4


@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200, 320])
def test_prefill_bf16_d128_lengths(cuda_device, T):
    x = to_dev(gen.make_prefill(2, T, 3, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.1, seed=T), cuda_device)
    o, hT = run_fwd(x)
    o_ref, h_ref = oracle_fwd(x)
    assert rel_err(o, o_ref) <= 2e-2
    assert rel_err(hT, h_ref) <= 2e-2


@pytest.mark.parametrize("gate_shift", [0.0, -1.0, 4.0])
def test_prefill_bf16_gate_ranges(cuda_device, gate_shift):
    """Weak decay (shift -1: alpha near 0.7) through strong decay (shift 4: G falls by ~270 per chunk)."""
    x = to_dev(gen.make_prefill(1, 256, 2, 128, 128, torch.bfloat16, gate_shift=gate_shift, h0_std=0.5, seed=11),
               cuda_device)
    o, hT = run_fwd(x)
    o_ref, h_ref = oracle_fwd(x)
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    assert rel_err(o, o_ref) <= 2e-2
    assert rel_err(hT, h_ref) <= 2e-2


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.float32, 128)])
def test_prefill_strong_decay_steps(cuda_device, dtype, d):
    """Steps whose decay leaves (almost) nothing: 3% of the log-gates at -60, one token with
    log alpha = -1e4 and one with -inf in every channel.  A block-split decay factor over such a step
    lies far outside the fp32 range; the chunked kernels apply these steps as a decay of 2^-15, so
    the result must stay finite and within the usual tolerance of the exact recurrence."""
    x = gen.make_prefill(2, 300, 2, d, d, dtype, gate_shift=0.0, h0_std=0.5, seed=41)
    g = torch.Generator().manual_seed(42)
    la = x["log_alpha"].clone()
    la[torch.rand(la.shape, generator=g) < 0.03] = -60.0
    la[0, 100] = -1e4
    la[1, 37] = float("-inf")
    x["log_alpha"] = la
    x = to_dev(x, cuda_device)
    o, hT = run_fwd(x)
    o_ref, h_ref = oracle_fwd(x)
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(hT, h_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,d", [(torch.float32, 128), (torch.bfloat16, 64)])
def test_prefill_cuda_core_path(cuda_device, dtype, d):
    x = to_dev(gen.make_prefill(2, 150, 2, d, d, dtype, gate_shift=1.0, h0_std=0.3, seed=5), cuda_device)
    o, hT = run_fwd(x)
    o_ref, h_ref = oracle_fwd(x)
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(hT, h_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_varlen_small(cuda_device, dtype, d):
    lens = torch.tensor([1, 0, 63, 64, 65, 130, 7])
    cu = gen.cu_seqlens_from_lengths(lens)
    x = to_dev(gen.make_prefill(1, int(cu[-1]), 2, d, d, dtype, gate_shift=2.0, h0_std=0.2, seed=9, cu_seqlens=cu),
               cuda_device)
    o, hT = run_fwd(x)
    o_ref, h_ref = oracle_fwd(x)
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(hT, h_ref) <= TOL[dtype]
    # packing changes nothing: each sequence run alone gives the same bits
    for n in range(len(lens)):
        a, b = int(cu[n]), int(cu[n + 1])
        if b == a:
            assert torch.equal(hT[n], x["h0"][n])
            continue
        xs = {kk: x[kk][:, a:b].clone() for kk in ("q", "k", "v", "log_alpha", "beta")}  # fresh, aligned
        on, hn = kda.kda_chunk_fwd(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"],
                                   x["h0"][n:n + 1].clone(), None)
        assert torch.equal(on, o[:, a:b]), f"sequence {n}"
        assert torch.equal(hn[0], hT[n]), f"sequence {n}"


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_empty_inputs_keep_the_state(cuda_device, dtype, d):
    """No tokens (T = 0; or varlen with every sequence empty): h_T = h0 exactly (zeros without h0)."""
    x = to_dev(gen.make_prefill(2, 0, 3, d, d, dtype, h0_std=0.3, seed=5), cuda_device)
    o, hT = run_fwd(x)
    assert o.numel() == 0 and torch.equal(hT, x["h0"])
    _, hz = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, None)
    assert torch.count_nonzero(hz) == 0
    cu = torch.zeros(4, dtype=torch.int32)
    y = to_dev(gen.make_prefill(1, 0, 3, d, d, dtype, h0_std=0.3, seed=6, cu_seqlens=cu), cuda_device)
    o, hT = run_fwd(y)
    assert o.numel() == 0 and torch.equal(hT, y["h0"])


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_zero_values_give_exact_zero(cuda_device, dtype, d):
    x = to_dev(gen.make_prefill(2, 200, 2, d, d, dtype, gate_shift=4.0, seed=1), cuda_device)
    x["v"] = torch.zeros_like(x["v"])
    o, hT = run_fwd(x)
    assert torch.count_nonzero(o) == 0
    assert torch.count_nonzero(hT) == 0


@pytest.mark.parametrize("split", [128, 100])
def test_continuity_in_place(cuda_device, split):
    """T tokens = first part, then the rest continuing from h_T (h_T aliased to h0, in place)."""
    x = to_dev(gen.make_prefill(1, 256, 2, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.1, seed=4), cuda_device)
    o, hT = run_fwd(x)
    part = lambda a, b: {kk: x[kk][:, a:b].clone() for kk in ("q", "k", "v", "log_alpha", "beta")}
    p1, p2 = part(0, split), part(split, 256)
    state = x["h0"].clone()
    o1, _ = kda.kda_chunk_fwd(p1["q"], p1["k"], p1["v"], p1["log_alpha"], p1["beta"], state, None, h_T=state)
    o2, _ = kda.kda_chunk_fwd(p2["q"], p2["k"], p2["v"], p2["log_alpha"], p2["beta"], state, None, h_T=state)
    o12 = torch.cat([o1, o2], 1)
    if split % 64 == 0:   # chunk boundaries line up: the same operations, the same bits
        assert torch.equal(o12, o) and torch.equal(state, hT)
    else:
        o_ref, h_ref = oracle_fwd(x)
        assert rel_err(o12, o_ref) <= 2e-2 and rel_err(state, h_ref) <= 2e-2


def test_deterministic(cuda_device):
    x = to_dev(gen.make_prefill(2, 300, 4, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.1, seed=8), cuda_device)
    o1, h1 = run_fwd(x)
    o2, h2 = run_fwd(x)
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_bad_seqlens_reported_on_device(cuda_device, dtype, d):
    cu = torch.tensor([0, 50, 40, 100], dtype=torch.int32)
    x = to_dev(gen.make_prefill(1, 100, 2, d, d, dtype, seed=2, cu_seqlens=cu), cuda_device)
    ws = kda.Workspace(cuda_device)
    run_fwd(x, workspace=ws)
    assert kda.kda_get_status(ws) == kda._lib.KDA_ERR_BAD_SEQLENS
    assert kda.kda_get_status(ws) == kda._lib.KDA_OK          # reading clears it
    x["cu_seqlens"] = torch.tensor([0, 40, 50, 100], dtype=torch.int32, device=cuda_device)
    run_fwd(x, workspace=ws)
    assert kda.kda_get_status(ws) == kda._lib.KDA_OK


# --------------------------------------------------------------------------- full-size workloads
def _sampled_check(x, o, hT, units, cols, tol, label, log):
    """units: list of (sequence n, head h); compares the o rows of that sequence and h_T[n, h] on the
    value columns `cols`.  The heads of one sequence go to the oracle in one call (one unit per
    thread).  Records the largest error of each kind for the terminal summary."""
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu()
    B, T = x["q"].shape[:2]
    by_seq = {}
    for n, h in units:
        by_seq.setdefault(n, []).append(h)
    worst_o = worst_h = 0.0
    for n, heads in sorted(by_seq.items()):
        if cu is None:
            b, a, e = n, 0, T
        else:
            b, a, e = 0, int(cu[n]), int(cu[n + 1])
        hs = torch.as_tensor(sorted(heads))
        xs = {kk: x[kk][b:b + 1, a:e].index_select(2, hs.to(x[kk].device)) for kk in ("q", "k", "v", "log_alpha", "beta")}
        xs["h0"] = None if x["h0"] is None else x["h0"][n:n + 1].index_select(1, hs.to(x["h0"].device))
        xs["cu_seqlens"] = None
        o_ref, h_ref = oracle_fwd(xs, cols=cols)
        og = o[b:b + 1, a:e].index_select(2, hs.to(o.device))[..., cols]
        hg = hT[n:n + 1].index_select(1, hs.to(hT.device))[..., cols]
        eo, eh = rel_err(og, o_ref), rel_err(hg, h_ref)
        assert eo <= tol and eh <= tol, (n, heads, eo, eh)
        worst_o, worst_h = max(worst_o, eo), max(worst_h, eh)
    log(label, worst_o, worst_h, tol)


# value columns spread over the four TMEM lane quadrants of the state kernel (32 channels each)
COLS16 = [0, 9, 18, 31, 32, 45, 58, 63, 64, 77, 90, 95, 96, 109, 122, 127]


def test_train_shape_sampled(cuda_device, parity_log):
    """B=4, H=16, T=4096, d=128, bf16, h0 = 0."""
    x = gen.make_prefill_for(gen.TRAIN, seed=0, device=cuda_device)
    o, hT = run_fwd(x)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    _sampled_check(x, o, hT, units=[(0, 0), (1, 7), (2, 15), (3, 3), (0, 9), (2, 4)], cols=COLS16, tol=2e-2,
                   label="training shape B=4 H=16 T=4096 (6 heads x 16 columns)", log=parity_log)


def test_train_shape_full(cuda_device, parity_log):
    """B=4, H=16, T=4096, d=128, bf16: every output element and every final state against the
    oracle (4 x 16 units, all 128 value columns; about a second of oracle time on 16 threads)."""
    x = gen.make_prefill_for(gen.TRAIN, seed=1, device=cuda_device)
    o, hT = run_fwd(x)
    torch.cuda.synchronize()
    o_ref, h_ref = oracle_fwd(x)
    eo, eh = rel_err(o, o_ref), rel_err(hT, h_ref)
    parity_log("training shape B=4 H=16 T=4096, every element (all 64 units x 128 columns)", eo, eh, 2e-2)
    assert eo <= 2e-2 and eh <= 2e-2, (eo, eh)


def test_long_context_sampled(cuda_device, parity_log):
    """B=1, H=32, T=131072, d=128, bf16, h0 ~ N(0, 0.02): the prefill the benchmark times."""
    x = gen.make_prefill_for(gen.LONG, seed=0, device=cuda_device)
    ws = kda.Workspace(cuda_device)
    o, hT = run_fwd(x, workspace=ws)
    assert kda.kda_get_status(ws) == kda._lib.KDA_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    _sampled_check(x, o, hT, units=[(0, h) for h in (0, 4, 9, 13, 18, 22, 27, 31)], cols=COLS16, tol=2e-2,
                   label="long context B=1 H=32 T=131072 (8 heads x 16 columns)", log=parity_log)


def test_varlen_batch_sampled(cuda_device, parity_log):
    """64 packed sequences, lengths uniform in [512, 16384], H=32, d=128, bf16."""
    x = gen.make_prefill_for(gen.VARLEN, seed=0, device=cuda_device)
    ws = kda.Workspace(cuda_device)
    o, hT = run_fwd(x, workspace=ws)
    assert kda.kda_get_status(ws) == kda._lib.KDA_OK
    _sampled_check(x, o, hT, units=[(0, 0), (17, 9), (40, 31), (63, 20), (5, 3), (29, 16), (52, 27), (11, 12)],
                   cols=COLS16, tol=2e-2, label="packed varlen 64 sequences H=32 (8 units x 16 columns)", log=parity_log)
