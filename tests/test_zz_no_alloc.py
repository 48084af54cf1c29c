"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (a plugin that only receives its input and output buffers, an
engine that has reserved all free device memory for its own pool), so they cannot pass the
workspace kda_chunk_fwd needs.  kda_chunk_fwd_noalloc runs the same kernels on a fixed 64 MiB
scratch array the library keeps in device memory.  This test calls it through the C ABI twice in
a row, on different inputs, and checks each result against kda_chunk_fwd with a caller workspace,
within the parity tolerance of the other GPU tests (bf16: 2e-2 relative to max |reference|).
It sits in its own file so that it is collected last.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import kimi_delta_attention_29_b200 as kda
from kimi_delta_attention_29_b200 import _lib
from kimi_delta_attention_29_b200 import inputs as gen

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _noalloc_fn():
    lib = _lib.load()
    fn = lib.kda_chunk_fwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp, vp]
    fn.restype = i
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_noalloc(fn, x, o, hT, stream):
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    N = x["num_seqs"]
    return fn(_p(x["q"]), _p(x["k"]), _p(x["v"]), _p(x["log_alpha"]), _p(x["beta"]), _p(x["h0"]),
              _p(x["cu_seqlens"]), N, B, T, H, dk, dv, 64, _lib.KDA_BF16, _p(o), _p(hT),
              ctypes.c_void_p(stream.cuda_stream))


def _rel(a, b):
    return float((a.float() - b.float()).abs().max() / b.float().abs().max())


def test_noalloc_matches_workspace_entry_point(cuda_device):
    fn = _noalloc_fn()
    stream = torch.cuda.current_stream(cuda_device)
    cases = [
        gen.make_prefill(2, 700, 8, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.1, seed=21, device=cuda_device),
        gen.make_prefill(1, 1000, 12, 128, 128, torch.bfloat16, gate_shift=1.0, h0_std=0.3, seed=22,
                         device=cuda_device),
    ]
    for n, x in enumerate(cases):   # two calls in a row: the second must not see the first's scratch
        o_ref, h_ref = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None)
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(h_ref, float("nan"))
        assert _call_noalloc(fn, x, o, hT, stream) == _lib.KDA_OK, f"call {n}"
        torch.cuda.synchronize(cuda_device)
        assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
        assert _rel(o, o_ref) <= TOL, f"call {n}: o"
        assert _rel(hT, h_ref) <= TOL, f"call {n}: h_T"


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    fn = _noalloc_fn()
    stream = torch.cuda.current_stream(cuda_device)
    x = gen.make_prefill(1, 1792, 32, 128, 128, torch.bfloat16, seed=23, device=cuda_device)  # needs > 64 MiB
    o = torch.empty_like(x["v"])
    hT = torch.empty(1, 32, 128, 128, device=cuda_device)
    assert _call_noalloc(fn, x, o, hT, stream) == _lib.KDA_ERR_WORKSPACE_TOO_SMALL


def test_noalloc_varlen_matches_workspace_entry_point(cuda_device):
    """Packed sequences (cu_seqlens) through the no-alloc entry point: the chunk table, the
    longest-first layout and the ready words all live in the shared scratch."""
    fn = _noalloc_fn()
    stream = torch.cuda.current_stream(cuda_device)
    lengths = torch.tensor([64, 1, 300, 127, 65, 129], dtype=torch.int64)  # full, ragged and 1-token chunks
    cu = gen.cu_seqlens_from_lengths(lengths)
    x = gen.make_prefill(1, int(cu[-1]), 8, 128, 128, torch.bfloat16, gate_shift=1.5, h0_std=0.2, seed=24,
                         device=cuda_device, cu_seqlens=cu)
    assert kda.kda_chunk_fwd_workspace_size(1, int(cu[-1]), 8, 128, 128, x["num_seqs"]) <= 64 << 20
    o_ref, h_ref = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], x["cu_seqlens"])
    o = torch.full_like(o_ref, float("nan"))
    hT = torch.full_like(h_ref, float("nan"))
    assert _call_noalloc(fn, x, o, hT, stream) == _lib.KDA_OK
    torch.cuda.synchronize(cuda_device)
    assert torch.isfinite(o.float()).all() and torch.isfinite(hT).all()
    assert _rel(o, o_ref) <= TOL
    assert _rel(hT, h_ref) <= TOL


def test_noalloc_repeat_call_allocates_nothing(cuda_device):
    """After the first call on the device (which loads the library's device code and scratch), a call
    leaves the device's free memory exactly where it was: nothing is allocated, not even by CUDA."""
    fn = _noalloc_fn()
    stream = torch.cuda.current_stream(cuda_device)
    x = gen.make_prefill(1, 640, 8, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.1, seed=25, device=cuda_device)
    o = torch.empty_like(x["v"])
    hT = torch.empty(1, 8, 128, 128, device=cuda_device)
    assert _call_noalloc(fn, x, o, hT, stream) == _lib.KDA_OK  # first call of this test (others ran before)
    torch.cuda.synchronize(cuda_device)
    free0 = torch.cuda.mem_get_info(cuda_device)[0]
    for _ in range(3):
        assert _call_noalloc(fn, x, o, hT, stream) == _lib.KDA_OK
    torch.cuda.synchronize(cuda_device)
    assert torch.cuda.mem_get_info(cuda_device)[0] == free0
