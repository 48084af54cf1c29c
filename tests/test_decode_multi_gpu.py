"""kda_decode_multi: Tq recurrent steps per sequence on a slot-indexed state pool.

Reference: the fp64 token-by-token oracle (the definition of the recurrence), started from the
state each sequence reads from the pool; the result must equal Tq calls of the one-token decode and
a prefill of the same tokens.  Tolerances are those of the other parity tests (bf16 2e-2, fp32 1e-4,
relative to max |reference|)."""
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


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(gpu, ref) -> float:
    g = np64(gpu) if isinstance(gpu, torch.Tensor) else gpu
    return float(np.abs(g - ref).max() / max(np.abs(ref).max(), 1e-30))


def _slots(vals, dev):
    return torch.tensor(vals, dtype=torch.int32, device=dev)


@pytest.mark.parametrize("dtype,d,Tq", [(torch.bfloat16, 128, 4), (torch.bfloat16, 64, 7), (torch.float32, 128, 3),
                                        (torch.float32, 64, 16)])
def test_pool_slots_match_oracle(cuda_device, dtype, d, Tq):
    N, H, P = 5, 3, 12
    pool = gen.make_decode_state(P, H, d, d, std=0.5, seed=5, device=cuda_device)
    before = pool.clone()
    s_in, s_out = [7, 2, 9, 0, 4], [1, 3, 5, 6, 8]           # outputs to other slots: inputs kept
    x = gen.make_decode_tokens(N, Tq, H, d, d, dtype=dtype, gate_shift=0.0, seed=11, device=cuda_device)
    o = kda.kda_decode_multi(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool,
                             slot_in=_slots(s_in, cuda_device), slot_out=_slots(s_out, cuda_device))
    h0 = np64(before)[s_in]
    o_ref, S_ref = oracle.recurrent(np64(x["q"]), np64(x["k"]), np64(x["v"]), np64(x["log_alpha"]),
                                    np64(x["beta"]), h0)
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(pool[s_out], S_ref) <= TOL[dtype]
    untouched = [p for p in range(P) if p not in s_out]
    assert torch.equal(pool[untouched], before[untouched])   # read slots and idle slots unchanged


def test_in_place_commit_equals_repeated_single_steps(cuda_device):
    """slot_out = slot_in (commit): equals Tq calls of kda_decode_step on the same states."""
    N, Tq, H, d = 4, 6, 2, 128
    pool = gen.make_decode_state(N, H, d, d, std=0.3, seed=8, device=cuda_device)
    S = pool.clone()
    x = gen.make_decode_tokens(N, Tq, H, d, d, dtype=torch.bfloat16, seed=12, device=cuda_device)
    o = kda.kda_decode_multi(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool)  # slots NULL: slot n
    for t in range(Tq):
        step = {kk: x[kk][:, t].contiguous() for kk in ("q", "k", "v", "log_alpha", "beta")}
        o_t = kda.kda_decode_step(step["q"], step["k"], step["v"], step["log_alpha"], step["beta"], S)
        assert rel_err(o[:, t], np64(o_t)) <= 1e-2, f"token {t}"
    assert rel_err(pool, np64(S)) <= 1e-4


def test_equals_prefill_of_the_same_tokens(cuda_device):
    """Tq decode tokens from h0 = Tq-token prefill from h0 (fp32, both within 1e-4 of the oracle)."""
    N, Tq, H, d = 2, 40, 2, 64
    x = gen.make_decode_tokens(N, Tq, H, d, d, dtype=torch.float32, gate_shift=0.0, seed=13, device=cuda_device)
    pool = gen.make_decode_state(N, H, d, d, std=0.2, seed=9, device=cuda_device)
    h0 = pool.clone()
    o = kda.kda_decode_multi(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool)
    o_p, hT = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], h0)
    assert rel_err(o, np64(o_p)) <= 1e-4
    assert rel_err(pool, np64(hT)) <= 1e-4


def test_bad_slot_is_skipped_and_reported(cuda_device):
    N, Tq, H, d, P = 3, 2, 2, 64, 4
    pool = gen.make_decode_state(P, H, d, d, std=0.5, seed=6, device=cuda_device)
    before = pool.clone()
    x = gen.make_decode_tokens(N, Tq, H, d, d, dtype=torch.float32, seed=14, device=cuda_device)
    o = torch.full((N, Tq, H, d), 7.0, device=cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    kda.kda_decode_multi(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool,
                         slot_in=_slots([0, 5, 2], cuda_device), slot_out=_slots([1, 3, -1], cuda_device),
                         o=o, status=status)
    assert kda.kda_get_status(status) == _lib.KDA_ERR_BAD_SLOT
    assert kda.kda_get_status(status) == _lib.KDA_OK          # read-and-clear
    assert torch.equal(o[1:], torch.full_like(o[1:], 7.0))    # skipped sequences: nothing written
    assert torch.equal(pool[[0, 2, 3]], before[[0, 2, 3]])    # only sequence 0's output slot (1) changes
    o_ref, S_ref = oracle.recurrent(np64(x["q"][:1]), np64(x["k"][:1]), np64(x["v"][:1]),
                                    np64(x["log_alpha"][:1]), np64(x["beta"][:1]), np64(before)[[0]])
    assert rel_err(o[:1], o_ref) <= 1e-4
    assert rel_err(pool[[1]], S_ref) <= 1e-4


def test_full_size_pool_sampled(cuda_device):
    """The decode workload's pool (256 x 32 states of 128 x 128, bf16 tokens), 8 tokens per call, a
    random permutation of slots; sampled (sequence, head) states checked against the oracle."""
    shp = gen.DECODE
    N, H, d, Tq = shp.N, shp.H, shp.dk, 8
    pool = gen.make_decode_state(N, H, d, d, std=shp.s0_std, seed=0, device=cuda_device)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(3)).to(torch.int32)
    sel = [0, 17, 101, 255]
    h0 = np64(pool[perm[sel].long()])
    x = gen.make_decode_tokens(N, Tq, H, d, d, dtype=shp.dtype, seed=15, device=cuda_device)
    o = kda.kda_decode_multi(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool,
                             slot_in=perm.to(cuda_device), slot_out=perm.to(cuda_device))
    pick = {kk: np64(x[kk][sel]) for kk in ("q", "k", "v", "log_alpha", "beta")}
    o_ref, S_ref = oracle.recurrent(pick["q"], pick["k"], pick["v"], pick["log_alpha"], pick["beta"], h0)
    assert rel_err(o[sel], o_ref) <= TOL[shp.dtype]
    assert rel_err(pool[perm[sel].long()], S_ref) <= TOL[shp.dtype]
