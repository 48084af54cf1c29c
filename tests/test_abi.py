"""C-ABI checks that need no GPU: the library loads, exports every entry point include/kda.h
declares, and rejects invalid arguments on the host before anything is launched."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from kimi_delta_attention_29_b200 import _lib
from kimi_delta_attention_29_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return _lib.load()


def declared_functions() -> list[str]:
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(kda_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(_lib.EXPORTED) <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported by libkda.so"


def test_status_strings_and_version(lib):
    assert lib.kda_version() >= 100
    for code in range(0, -13, -1):
        s = _lib.status_string(code)
        assert s.startswith("KDA_")
    assert "unknown" in _lib.status_string(-999)


def test_workspace_size_queries(lib):
    ws = lib.kda_chunk_fwd_workspace_size
    assert ws(1, 131072, 32, 128, 128, 1, 64, _lib.KDA_BF16) > 4 * 2**30       # WY records for 2048 chunks
    assert ws(1, 256, 2, 64, 64, 1, 64, _lib.KDA_F32) == 256                     # CUDA-core path: status only
    assert ws(1, 256, 2, 64, 64, 1, 32, _lib.KDA_F32) == 0                       # chunk 32 unsupported
    assert ws(1, 256, 2, 96, 96, 1, 64, _lib.KDA_BF16) == 0                      # head dim 96 unsupported
    assert ws(1, 256, 2, 128, 128, 1, 64, 7) == 0                                # bad dtype
    assert ws(2, 256, 2, 128, 128, 3, 64, _lib.KDA_BF16) == 0                    # N != B without varlen


# Fake, 256-byte aligned device addresses: every call below must fail validation before it touches them.
A = 1 << 20


def _fwd(lib, **kw):
    args = dict(q=A, k=2 * A, v=3 * A, la=4 * A, beta=5 * A, h0=None, cu=None, N=1, B=1, T=128, H=2, dk=128,
                dv=128, chunk=64, dtype=_lib.KDA_BF16, o=6 * A, hT=7 * A, ws=8 * A, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    c = ctypes.c_void_p
    return lib.kda_chunk_fwd(c(args["q"]), c(args["k"]), c(args["v"]), c(args["la"]), c(args["beta"]),
                             c(args["h0"]), c(args["cu"]), args["N"], args["B"], args["T"], args["H"],
                             args["dk"], args["dv"], args["chunk"], args["dtype"], c(args["o"]), c(args["hT"]),
                             c(args["ws"]), args["ws_bytes"], c(args["stream"]))


def test_chunk_fwd_rejects_on_host(lib):
    assert _fwd(lib, dtype=5) == _lib.KDA_ERR_BAD_DTYPE
    assert _fwd(lib, q=None) == _lib.KDA_ERR_NULL_ARG
    assert _fwd(lib, ws=None) == _lib.KDA_ERR_NULL_ARG
    assert _fwd(lib, B=0) == _lib.KDA_ERR_BAD_SHAPE
    assert _fwd(lib, T=-1) == _lib.KDA_ERR_BAD_SHAPE
    assert _fwd(lib, N=2) == _lib.KDA_ERR_BAD_SHAPE                      # N != B without cu_seqlens
    assert _fwd(lib, B=2, N=2, cu=9 * A) == _lib.KDA_ERR_BAD_SHAPE      # varlen needs B = 1
    assert _fwd(lib, chunk=32) == _lib.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, dk=128, dv=64) == _lib.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, dk=96, dv=96) == _lib.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, v=3 * A + 8) == _lib.KDA_ERR_MISALIGNED
    assert _fwd(lib, ws=8 * A + 16) == _lib.KDA_ERR_MISALIGNED          # workspace needs 256-byte alignment
    assert _fwd(lib, o=A) == _lib.KDA_ERR_ALIASING                       # o on top of q
    assert _fwd(lib, hT=3 * A) == _lib.KDA_ERR_ALIASING                  # h_T on top of v
    assert _fwd(lib, h0=7 * A + 1024, hT=7 * A) == _lib.KDA_ERR_ALIASING  # partial h0 / h_T overlap
    assert _fwd(lib, ws_bytes=1024) == _lib.KDA_ERR_WORKSPACE_TOO_SMALL


def test_decode_rejects_on_host(lib):
    c = ctypes.c_void_p

    def dec(q=A, k=2 * A, v=3 * A, la=4 * A, beta=5 * A, S=6 * A, N=4, H=2, dk=128, dv=128,
            dtype=_lib.KDA_BF16, o=8 * A):
        return lib.kda_decode_step(c(q), c(k), c(v), c(la), c(beta), c(S), N, H, dk, dv, dtype, c(o), c(None))

    assert dec(dtype=3) == _lib.KDA_ERR_BAD_DTYPE
    assert dec(S=None) == _lib.KDA_ERR_NULL_ARG
    assert dec(N=0) == _lib.KDA_ERR_BAD_SHAPE
    assert dec(dk=32, dv=32) == _lib.KDA_ERR_UNSUPPORTED
    assert dec(o=8 * A + 4) == _lib.KDA_ERR_MISALIGNED
    assert dec(o=6 * A) == _lib.KDA_ERR_ALIASING                         # o inside S
    assert dec(S=A) == _lib.KDA_ERR_ALIASING                             # S on top of q


def test_binding_refuses_noncontiguous():
    import torch
    import kimi_delta_attention_29_b200 as kda
    x = torch.zeros(4, 8)[:, ::2]
    with pytest.raises(ValueError):
        kda._ptr(x)


def _multi(lib, **kw):
    args = dict(q=A, k=2 * A, v=3 * A, la=4 * A, beta=5 * A, pool=6 * A, P=8, si=None, so=None, N=4, Tq=3, H=2,
                dk=128, dv=128, dtype=_lib.KDA_BF16, o=7 * A, status=None, stream=None)
    args.update(kw)
    c = ctypes.c_void_p
    return lib.kda_decode_multi(c(args["q"]), c(args["k"]), c(args["v"]), c(args["la"]), c(args["beta"]),
                                c(args["pool"]), args["P"], c(args["si"]), c(args["so"]), args["N"], args["Tq"],
                                args["H"], args["dk"], args["dv"], args["dtype"], c(args["o"]), c(args["status"]),
                                c(args["stream"]))


def test_decode_multi_rejects_on_host(lib):
    assert _multi(lib, dtype=9) == _lib.KDA_ERR_BAD_DTYPE
    assert _multi(lib, pool=None) == _lib.KDA_ERR_NULL_ARG
    assert _multi(lib, o=None) == _lib.KDA_ERR_NULL_ARG
    assert _multi(lib, Tq=0) == _lib.KDA_ERR_BAD_SHAPE
    assert _multi(lib, P=0) == _lib.KDA_ERR_BAD_SHAPE
    assert _multi(lib, N=9) == _lib.KDA_ERR_BAD_SHAPE                  # slot n must exist without slot arrays
    assert _multi(lib, dk=96, dv=96) == _lib.KDA_ERR_UNSUPPORTED
    assert _multi(lib, q=A + 8) == _lib.KDA_ERR_MISALIGNED
    assert _multi(lib, si=9 * A + 2) == _lib.KDA_ERR_MISALIGNED         # int32 slot array
    assert _multi(lib, o=A) == _lib.KDA_ERR_ALIASING                    # o overlaps q
    assert _multi(lib, pool=5 * A) == _lib.KDA_ERR_ALIASING             # pool overlaps beta
    assert _multi(lib, status=6 * A) == _lib.KDA_ERR_ALIASING           # status inside the pool


def _fwd_ex(lib, flags=0, A_log=None, dt_bias=None, **kw):
    args = dict(q=A, k=2 * A, v=3 * A, la=4 * A, beta=5 * A, h0=None, cu=None, N=1, B=1, T=128, H=2, dk=128,
                dv=128, chunk=64, dtype=_lib.KDA_BF16, o=6 * A, hT=7 * A, ws=8 * A, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    c = ctypes.c_void_p
    return lib.kda_chunk_fwd_ex(c(args["q"]), c(args["k"]), c(args["v"]), c(args["la"]), c(args["beta"]),
                                c(args["h0"]), c(args["cu"]), args["N"], args["B"], args["T"], args["H"], args["dk"],
                                args["dv"], args["chunk"], args["dtype"], c(args["o"]), c(args["hT"]), c(args["ws"]),
                                args["ws_bytes"], flags, c(A_log), c(dt_bias), c(args["stream"]))


def test_prologue_arguments_rejected_on_host(lib):
    assert _fwd_ex(lib, flags=4) == _lib.KDA_ERR_UNSUPPORTED                        # unknown flag bit
    assert _fwd_ex(lib, flags=_lib.KDA_PROLOGUE_GATE) == _lib.KDA_ERR_NULL_ARG       # gate needs A_log
    assert _fwd_ex(lib, flags=_lib.KDA_PROLOGUE_GATE, A_log=9 * A + 4) == _lib.KDA_ERR_MISALIGNED
    assert _fwd_ex(lib, flags=_lib.KDA_PROLOGUE_GATE, A_log=9 * A, dt_bias=10 * A + 8) == _lib.KDA_ERR_MISALIGNED
    assert _fwd_ex(lib, flags=_lib.KDA_PROLOGUE_GATE, A_log=6 * A) == _lib.KDA_ERR_ALIASING     # inside o
    assert _fwd_ex(lib, flags=3, A_log=9 * A, dt_bias=7 * A) == _lib.KDA_ERR_ALIASING           # inside h_T
    c = ctypes.c_void_p
    rc = lib.kda_decode_multi_ex(c(A), c(2 * A), c(3 * A), c(4 * A), c(5 * A), c(6 * A), 8, None, None, 4, 3, 2, 128,
                                 128, _lib.KDA_BF16, c(7 * A), None, 8, None, None, None)
    assert rc == _lib.KDA_ERR_UNSUPPORTED


def test_output_gate_norm_rejects_on_host(lib):
    """Every rejection returns before a launch; no call here reaches the kernel."""
    c, f = ctypes.c_void_p, ctypes.c_float
    fn = lib.kda_output_gate_norm

    def call(o=A, g=2 * A, w=None, eps=1e-6, n_tok=4, H=2, dv=128, dtype=_lib.KDA_BF16, out=3 * A):
        return fn(c(o) if o else None, c(g) if g else None, c(w) if w else None, f(eps), n_tok, H, dv, dtype,
                  c(out) if out else None, None)

    assert call(dtype=7) == _lib.KDA_ERR_BAD_DTYPE
    assert call(n_tok=-1) == _lib.KDA_ERR_BAD_SHAPE
    assert call(H=0) == _lib.KDA_ERR_BAD_SHAPE
    assert call(dv=96) == _lib.KDA_ERR_UNSUPPORTED
    assert call(eps=-1e-3) == _lib.KDA_ERR_BAD_VALUE
    assert call(eps=float("nan")) == _lib.KDA_ERR_BAD_VALUE
    assert call(eps=float("inf")) == _lib.KDA_ERR_BAD_VALUE
    assert call(n_tok=0, o=None, g=None, out=None) == _lib.KDA_OK           # empty: nothing enqueued
    assert call(o=None) == _lib.KDA_ERR_NULL_ARG
    assert call(g=None) == _lib.KDA_ERR_NULL_ARG
    assert call(out=None) == _lib.KDA_ERR_NULL_ARG
    assert call(o=A + 8) == _lib.KDA_ERR_MISALIGNED
    assert call(w=5 * A + 4) == _lib.KDA_ERR_MISALIGNED
    assert call(out=A + 256) == _lib.KDA_ERR_ALIASING                        # partial overlap with o
    assert call(out=2 * A) == _lib.KDA_ERR_ALIASING                          # out is g
    assert call(w=3 * A + 64) == _lib.KDA_ERR_ALIASING                       # weight inside out


def test_chunk_bwd_rejects_on_host(lib):
    """Every rejection returns before a launch; no call here reaches a kernel."""
    c = ctypes.c_void_p
    B, T, H, d = 1, 128, 2, 128
    need = lib.kda_chunk_bwd_workspace_size(B, T, H, d, d, B, 64, _lib.KDA_BF16)
    assert need > 0
    assert lib.kda_chunk_bwd_workspace_size(B, T, H, 96, 96, B, 64, _lib.KDA_BF16) == 0
    assert lib.kda_chunk_bwd_workspace_size(B, T, H, d, d, B, 32, _lib.KDA_BF16) == 0

    def call(dtype=_lib.KDA_BF16, q=A, ws=64 * A, ws_bytes=None, dq=20 * A, chunk=64, dk=d, dv=d, do=7 * A):
        return lib.kda_chunk_bwd(c(q) if q else None, c(2 * A), c(3 * A), c(4 * A), c(5 * A), None, None, B, B, T, H,
                                 dk, dv, chunk, dtype, c(do) if do else None, None, c(dq), c(21 * A), c(22 * A),
                                 c(23 * A), c(24 * A), None, c(ws) if ws else None,
                                 need if ws_bytes is None else ws_bytes, None)

    assert call(dtype=9) == _lib.KDA_ERR_BAD_DTYPE
    assert call(ws=0) == _lib.KDA_ERR_NULL_ARG
    assert call(chunk=32) == _lib.KDA_ERR_UNSUPPORTED
    assert call(dk=64) == _lib.KDA_ERR_UNSUPPORTED
    assert call(q=0) == _lib.KDA_ERR_NULL_ARG
    assert call(do=0) == _lib.KDA_ERR_NULL_ARG
    assert call(q=A + 4) == _lib.KDA_ERR_MISALIGNED
    assert call(ws=64 * A + 16) == _lib.KDA_ERR_MISALIGNED
    assert call(ws_bytes=need - 1) == _lib.KDA_ERR_WORKSPACE_TOO_SMALL
    assert call(dq=A + 1024) == _lib.KDA_ERR_ALIASING          # dq inside q
    assert call(dq=21 * A + 256) == _lib.KDA_ERR_ALIASING      # dq overlaps dk


def test_state_compose_rejects_on_host(lib):
    c = ctypes.c_void_p
    f = lib.kda_state_compose

    def call(Mb=A, h0=None, R=2, H=2, dk=128, dv=128, S_in=None, S_out=8 * A):
        return f(c(Mb) if Mb else None, c(h0) if h0 else None, R, H, dk, dv, c(S_in) if S_in else None,
                 c(S_out) if S_out else None, None)

    assert call(Mb=0) == _lib.KDA_ERR_NULL_ARG
    assert call(S_out=0) == _lib.KDA_ERR_NULL_ARG
    assert call(R=0) == _lib.KDA_ERR_BAD_SHAPE
    assert call(dk=96) == _lib.KDA_ERR_UNSUPPORTED
    assert call(S_out=8 * A + 4) == _lib.KDA_ERR_MISALIGNED
    assert call(S_out=A + 4096) == _lib.KDA_ERR_ALIASING                     # output inside Mb
    assert call(S_in=A + 1024) == _lib.KDA_ERR_ALIASING


def test_segment_map_rejects_on_host(lib):
    c = ctypes.c_void_p
    f = lib.kda_segment_map
    W = 1 << 30  # a workspace address no argument below reaches

    def call(T=100, H=2, dk=128, dv=128, dtype=_lib.KDA_BF16, o0=None, Mb=8 * A, ws=W, ws_bytes=1 << 30, x=A):
        ptr = lambda p: c(p) if p else None
        return f(ptr(x), ptr(x + A // 4), ptr(x + A // 2), ptr(x + 3 * A // 4), ptr(x + A - 4096), T, H, dk, dv, 64,
                 dtype, ptr(o0), ptr(Mb), ptr(ws), ws_bytes, None)

    assert call(Mb=0) == _lib.KDA_ERR_NULL_ARG
    assert call(ws=0) == _lib.KDA_ERR_NULL_ARG
    assert call(x=0) == _lib.KDA_ERR_NULL_ARG
    assert call(dtype=7) == _lib.KDA_ERR_BAD_DTYPE
    assert call(T=-1) == _lib.KDA_ERR_BAD_SHAPE
    assert call(dk=64, dv=64) == _lib.KDA_ERR_UNSUPPORTED          # CUDA-core sizes: two prefills instead
    assert call(dtype=_lib.KDA_F32) == _lib.KDA_ERR_UNSUPPORTED
    assert call(Mb=8 * A + 4) == _lib.KDA_ERR_MISALIGNED
    assert call(ws=W + 16) == _lib.KDA_ERR_MISALIGNED
    assert call(ws_bytes=1024) == _lib.KDA_ERR_WORKSPACE_TOO_SMALL
    assert call(Mb=A + 4096) == _lib.KDA_ERR_ALIASING                 # map inside q
    assert call(o0=8 * A + 4096) == _lib.KDA_ERR_ALIASING             # outputs inside the map
    assert call(Mb=W + 4096) == _lib.KDA_ERR_ALIASING                 # map inside the workspace


def test_binding_constants_match_the_header():
    """The binding's status codes and prologue flags are the header's, and its trace names cover
    every kernel id the library reports."""
    header = open(os.path.join(ROOT, "include", "kda.h")).read()
    codes = dict((name, int(val)) for name, val in re.findall(r"\b(KDA_(?:OK|ERR_\w+))\s*=\s*(-?\d+)", header))
    assert codes, "no status codes found in include/kda.h"
    for name, val in codes.items():
        assert getattr(_lib, name) == val, name
    flags = dict((name, int(val)) for name, val in re.findall(r"\b(KDA_PROLOGUE_\w+)\s*=\s*(\d+)", header))
    assert flags and all(getattr(_lib, n) == v for n, v in flags.items())
    common = open(os.path.join(ROOT, "kimi_delta_attention_29_b200", "csrc", "kda_common.cuh")).read()
    enum = re.search(r"enum KernelId \{(.*?)\};", common, re.S).group(1)
    ids = [int(v) for v in re.findall(r"=\s*(\d+)", enum)]
    assert sorted(ids) == sorted(_lib.KERNEL_NAMES), (ids, sorted(_lib.KERNEL_NAMES))
