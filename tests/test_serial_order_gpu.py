"""The tensor-core prefill's two launch orders give the same bits.

Concurrently (the default), the state kernel runs on a side stream while the intra-chunk kernel
produces the records it waits for; with KDA_PREFILL_SERIAL=1 (read once per process, for profilers
that serialise kernels) the intra-chunk kernel runs to completion first.  The arithmetic is the same
in both orders, so o and h_T must match bit for bit.  The serial run happens in a child process.
"""
from __future__ import annotations

import os
import subprocess
import sys
import tempfile

import pytest
import torch

import kimi_delta_attention_29_b200 as kda
from kimi_delta_attention_29_b200 import inputs as gen

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import kimi_delta_attention_29_b200 as kda
from kimi_delta_attention_29_b200 import inputs as gen
dev = torch.device("cuda:0")
for (B, T, H, seed) in [(1, 4100, 8, 7), (2, 333, 4, 8)]:
    x = gen.make_prefill(B, T, H, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.05, seed=seed, device=dev)
    o, h = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None)
    torch.save({"o": o.cpu(), "h": h.cpu()}, f"{sys.argv[2]}/serial_{seed}.pt")
"""


def test_serial_launch_order_is_bit_identical(cuda_device):
    with tempfile.TemporaryDirectory() as d:
        env = dict(os.environ, KDA_PREFILL_SERIAL="1")
        r = subprocess.run([sys.executable, "-c", CHILD, ROOT, d], env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        for (B, T, H, seed) in [(1, 4100, 8, 7), (2, 333, 4, 8)]:
            x = gen.make_prefill(B, T, H, 128, 128, torch.bfloat16, gate_shift=2.0, h0_std=0.05, seed=seed,
                                 device=cuda_device)
            o, h = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["h0"], None)
            ref = torch.load(f"{d}/serial_{seed}.pt")
            assert torch.equal(o.cpu(), ref["o"]), f"o differs (seed {seed})"
            assert torch.equal(h.cpu(), ref["h"]), f"h_T differs (seed {seed})"
