"""Guard bands around output buffers: every entry point writes inside its outputs and nowhere else.

(compute-sanitizer is not available on the test machines; this checks the same property for the
outputs.)  Each output is a view into the middle of a larger buffer filled with a sentinel; after
the call the bands before and after the view must still hold the sentinel, bit for bit.  Shapes are
ragged (a partial last chunk, odd row counts) so that tail handling is exercised.
"""
from __future__ import annotations

import pytest
import torch

import kimi_delta_attention_29_b200 as kda
from kimi_delta_attention_29_b200 import inputs as gen

pytestmark = pytest.mark.gpu

PAD = 4096          # elements on each side (16-byte aligned for every dtype used)
SENTINEL = 1024.0   # exact in bf16 and fp32


def guarded(shape, dtype, device):
    n = 1
    for s in shape:
        n *= s
    full = torch.full((n + 2 * PAD,), SENTINEL, dtype=dtype, device=device)
    return full, full[PAD:PAD + n].view(shape)


def intact(full) -> bool:
    torch.cuda.synchronize(full.device)
    return bool((full[:PAD] == SENTINEL).all()) and bool((full[-PAD:] == SENTINEL).all())


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_prefill_writes_only_its_outputs(cuda_device, dtype, d):
    B, T, H = 2, 200, 3
    x = gen.make_prefill(B, T, H, d, d, dtype, gate_shift=1.0, h0_std=0.1, seed=91, device=cuda_device)
    of, o = guarded((B, T, H, d), dtype, cuda_device)
    hf, hT = guarded((B, H, d, d), torch.float32, cuda_device)
    kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None, o=o, h_T=hT)
    assert intact(of) and intact(hf)
    assert not bool((o == SENTINEL).all()) and not bool((hT == SENTINEL).all())


def test_decode_writes_only_its_state_and_output(cuda_device):
    N, H, d = 3, 2, 128
    sf, S = guarded((N, H, d, d), torch.float32, cuda_device)
    S.copy_(gen.make_decode_state(N, H, d, d, std=0.1, seed=92, device=cuda_device))
    of, o = guarded((N, H, d), torch.bfloat16, cuda_device)
    t = gen.make_decode_token(N, H, d, d, seed=93, device=cuda_device)
    kda.kda_decode_step(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], S, o=o)
    assert intact(sf) and intact(of)


def test_epilogue_writes_only_its_output(cuda_device):
    rows, H, d = 37, 3, 128
    g = torch.Generator(device=cuda_device).manual_seed(94)
    o = torch.randn(rows, H, d, generator=g, device=cuda_device).to(torch.bfloat16)
    gg = torch.randn(rows, H, d, generator=g, device=cuda_device).to(torch.bfloat16)
    yf, y = guarded((rows, H, d), torch.bfloat16, cuda_device)
    kda.kda_output_gate_norm(o, gg, None, out=y)
    assert intact(yf)
