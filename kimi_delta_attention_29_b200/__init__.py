"""B200 (sm_100a) Kimi Delta Attention: chunkwise prefill and recurrent decode.

The Python functions below share their names with the C ABI in include/kda.h and only
marshal arguments (tensor pointers, sizes, the current CUDA stream) into libkda.so.  torch is
used for device memory and streams; every step of the method runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import KdaError, status_string  # noqa: F401
from ._lib import KDA_PROLOGUE_GATE, KDA_PROLOGUE_L2NORM_QK  # noqa: F401

__all__ = ["kda_chunk_fwd", "kda_chunk_fwd_ex", "kda_chunk_fwd_workspace_size", "kda_chunk_bwd",
           "kda_chunk_bwd_workspace_size", "kda_decode_step", "kda_decode_multi", "kda_decode_multi_ex",
           "kda_output_gate_norm", "kda_state_compose", "kda_segment_map", "kda_get_status", "kda_status_string",
           "kda_trace_begin", "kda_trace_end", "KdaError", "Workspace", "KDA_PROLOGUE_GATE",
           "KDA_PROLOGUE_L2NORM_QK"]


def _torch():
    import torch
    return torch


def _dtype_code(dt) -> int:
    torch = _torch()
    if dt == torch.bfloat16:
        return _lib.KDA_BF16
    if dt == torch.float32:
        return _lib.KDA_F32
    return 99  # rejected by the library as KDA_ERR_BAD_DTYPE


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("KDA tensors must be contiguous (dense row-major layout)")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def kda_status_string(code: int) -> str:
    return status_string(code)


def kda_chunk_fwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                                 chunk_size: int = 64, dtype=None) -> int:
    torch = _torch()
    code = _dtype_code(dtype if dtype is not None else torch.bfloat16)
    return int(_lib.load().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, code))


def kda_chunk_bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int, num_seqs: int,
                                 chunk_size: int = 64, dtype=None) -> int:
    """Bytes of device workspace kda_chunk_bwd needs (0 for unsupported sizes)."""
    torch = _torch()
    code = _dtype_code(dtype if dtype is not None else torch.bfloat16)
    return int(_lib.load().kda_chunk_bwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, code))


class Workspace:
    """A reusable device workspace for kda_chunk_fwd (grows on demand, never shrinks)."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        torch = _torch()
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


def kda_chunk_fwd(q, k, v, log_alpha, beta, h0=None, cu_seqlens=None, chunk_size: int = 64, o=None,
                  h_T=None, output_final_state: bool = True, workspace=None, stream=None):
    """Chunkwise KDA forward.  q, k [B,T,H,dk], v [B,T,H,dv] (bf16 or fp32), log_alpha [B,T,H,dk]
    fp32, beta [B,T,H] fp32, h0 [N,H,dk,dv] fp32 or None, cu_seqlens int32 [N+1] (device) or None.
    Returns (o, h_T); h_T is None when output_final_state is False and none was passed."""
    torch = _torch()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if h_T is None and output_final_state:
        h_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    code = _dtype_code(q.dtype)
    need = int(_lib.load().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, N, chunk_size, code))
    if isinstance(workspace, Workspace):
        ws = workspace.get(need)
    elif workspace is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    else:
        ws = workspace
    rc = _lib.load().kda_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(h0), _ptr(cu_seqlens), N, B, T, H,
        dk, dv, chunk_size, code, _ptr(o), _ptr(h_T), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream, q.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd")
    return o, h_T


def kda_chunk_fwd_ex(q, k, v, log_alpha, beta, h0=None, cu_seqlens=None, flags: int = 0, A_log=None,
                     dt_bias=None, chunk_size: int = 64, o=None, h_T=None, output_final_state: bool = True,
                     workspace=None, stream=None):
    """kda_chunk_fwd with the layer prologue fused in: flags KDA_PROLOGUE_L2NORM_QK (L2-normalise q and
    k rows) and / or KDA_PROLOGUE_GATE (log_alpha holds the gate projection g; the decay used is
    -exp(A_log[h]) * softplus(g + dt_bias[h, c])).  A_log [H] fp32, dt_bias [H, dk] fp32 or None."""
    torch = _torch()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if h_T is None and output_final_state:
        h_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    code = _dtype_code(q.dtype)
    need = int(_lib.load().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, N, chunk_size, code))
    if isinstance(workspace, Workspace):
        ws = workspace.get(need)
    elif workspace is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    else:
        ws = workspace
    rc = _lib.load().kda_chunk_fwd_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(h0), _ptr(cu_seqlens), N, B, T, H,
        dk, dv, chunk_size, code, _ptr(o), _ptr(h_T), _ptr(ws), ws.numel() * ws.element_size(), int(flags),
        _ptr(A_log), _ptr(dt_bias), _stream(stream, q.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_ex")
    return o, h_T


def kda_decode_multi_ex(q, k, v, log_alpha, beta, S_pool, slot_in=None, slot_out=None, flags: int = 0, A_log=None,
                        dt_bias=None, o=None, status=None, stream=None):
    """kda_decode_multi with the layer prologue fused in (see kda_chunk_fwd_ex)."""
    torch = _torch()
    N, Tq, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((N, Tq, H, dv), dtype=q.dtype, device=q.device)
    rc = _lib.load().kda_decode_multi_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S_pool),
                                         S_pool.shape[0], _ptr(slot_in), _ptr(slot_out), N, Tq, H, dk, dv,
                                         _dtype_code(q.dtype), _ptr(o), _ptr(status), int(flags), _ptr(A_log),
                                         _ptr(dt_bias), _stream(stream, q.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_decode_multi_ex")
    return o


def kda_decode_multi(q, k, v, log_alpha, beta, S_pool, slot_in=None, slot_out=None, o=None, status=None,
                     stream=None):
    """Tq recurrent steps per sequence on a slot-indexed state pool.  q, k [N,Tq,H,dk], v [N,Tq,H,dv]
    (bf16 or fp32), log_alpha [N,Tq,H,dk] fp32, beta [N,Tq,H] fp32, S_pool [P,H,dk,dv] fp32 (read at
    slot_in, written at slot_out), slot_in / slot_out int32 [N] on the device or None (slot n),
    status: int32 device tensor receiving KDA_ERR_BAD_SLOT, or None.  Returns o [N,Tq,H,dv]."""
    torch = _torch()
    N, Tq, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((N, Tq, H, dv), dtype=q.dtype, device=q.device)
    rc = _lib.load().kda_decode_multi(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S_pool),
                                      S_pool.shape[0], _ptr(slot_in), _ptr(slot_out), N, Tq, H, dk, dv,
                                      _dtype_code(q.dtype), _ptr(o), _ptr(status), _stream(stream, q.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_decode_multi")
    return o


def kda_chunk_bwd(q, k, v, log_alpha, beta, h0=None, cu_seqlens=None, do=None, dh_T=None, want_dh0: bool = True,
                  chunk_size: int = 64, workspace=None, stream=None):
    """Gradients of kda_chunk_fwd for upstream do [B,T,H,dv] (input dtype) and dh_T [N,H,dk,dv] fp32 (None:
    zero).  Returns a dict: dq, dk [B,T,H,dk] and dv [B,T,H,dv] in the input dtype, dlog_alpha [B,T,H,dk]
    and dbeta [B,T,H] fp32, dh0 [N,H,dk,dv] fp32 (None unless want_dh0)."""
    torch = _torch()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    code = _dtype_code(q.dtype)
    lib = _lib.load()
    need = kda_chunk_bwd_workspace_size(B, T, H, dk, dv, N, chunk_size, q.dtype)
    if need == 0:
        raise KdaError(_lib.KDA_ERR_UNSUPPORTED, "kda_chunk_bwd_workspace_size")
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=q.device)
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dlog_alpha": torch.empty_like(log_alpha), "dbeta": torch.empty_like(beta),
         "dh0": torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device) if want_dh0 else None}
    rc = lib.kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(h0), _ptr(cu_seqlens), N, B, T,
                           H, dk, dv, chunk_size, code, _ptr(do), _ptr(dh_T), _ptr(g["dq"]), _ptr(g["dk"]),
                           _ptr(g["dv"]), _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dh0"]), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream, q.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_chunk_bwd")
    return g


def kda_state_compose(Mb, h0=None, want_S_in: bool = True, stream=None):
    """Composition of R segment maps: Mb [R, H, dk, dk + dv] fp32 (rows [M_r | b_r]), h0 [H, dk, dv] fp32 or
    None.  Returns (S_in [R, H, dk, dv] or None, S_out [H, dk, dv]): the state entering each segment and
    the state after the last."""
    torch = _torch()
    R, H, dk, w = Mb.shape
    dv = w - dk
    S_in = torch.empty((R, H, dk, dv), dtype=torch.float32, device=Mb.device) if want_S_in else None
    S_out = torch.empty((H, dk, dv), dtype=torch.float32, device=Mb.device)
    rc = _lib.load().kda_state_compose(_ptr(Mb), _ptr(h0), R, H, dk, dv, _ptr(S_in), _ptr(S_out),
                                       _stream(stream, Mb.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_state_compose")
    return S_in, S_out


def kda_segment_map(q, k, v, log_alpha, beta, want_o: bool = True, chunk_size: int = 64, workspace=None,
                    stream=None):
    """One segment's map for kda_state_compose in one pass: q, k [1,T,H,dk], v [1,T,H,dv] bf16 with
    dk = dv = 128, log_alpha [1,T,H,dk] fp32, beta [1,T,H] fp32.  Returns (o0 [1,T,H,dv] or None, Mb
    [H, dk, dk + dv] fp32): the outputs from a zero incoming state and the rows [M | b]."""
    torch = _torch()
    _, T, H, dk = q.shape
    dv = v.shape[-1]
    o0 = torch.empty((1, T, H, dv), dtype=q.dtype, device=q.device) if want_o else None
    Mb = torch.empty((H, dk, dk + dv), dtype=torch.float32, device=q.device)
    code = _dtype_code(q.dtype)
    need = int(_lib.load().kda_chunk_fwd_workspace_size(1, T, H, dk, dv, 1, chunk_size, code))
    if isinstance(workspace, Workspace):
        ws = workspace.get(need)
    elif workspace is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    else:
        ws = workspace
    rc = _lib.load().kda_segment_map(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), T, H, dk, dv,
                                     chunk_size, code, _ptr(o0), _ptr(Mb), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream, q.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_segment_map")
    return o0, Mb


def kda_output_gate_norm(o, g, weight=None, eps: float = 1e-6, out=None, stream=None):
    """The layer's output epilogue: out = RMSNorm(o) over the head dim (dv) x weight[dv] x sigmoid(g),
    per (token, head) row.  o, g [..., H, dv] contiguous, bf16 or fp32 (same dtype); weight [dv] fp32 or
    None; out=o runs in place.  Returns out."""
    torch = _torch()
    H, dv = o.shape[-2], o.shape[-1]
    n_tok = o.numel() // (H * dv) if H * dv else 0
    if out is None:
        out = torch.empty_like(o)
    rc = _lib.load().kda_output_gate_norm(_ptr(o), _ptr(g), _ptr(weight), float(eps), n_tok, H, dv,
                                          _dtype_code(o.dtype), _ptr(out), _stream(stream, o.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_output_gate_norm")
    return out


def kda_get_status(workspace, stream=None) -> int:
    buf = workspace.buf if isinstance(workspace, Workspace) else workspace
    return int(_lib.load().kda_get_status(_ptr(buf), _stream(stream, buf.device)))


def kda_decode_step(q, k, v, log_alpha, beta, S, o=None, stream=None):
    """One recurrent step on S [N,H,dk,dv] fp32 (updated in place).  q, k [N,H,dk], v [N,H,dv],
    log_alpha [N,H,dk] fp32, beta [N,H] fp32.  Returns o [N,H,dv]."""
    torch = _torch()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    rc = _lib.load().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), N, H,
                                     dk, dv, _dtype_code(q.dtype), _ptr(o), _stream(stream, q.device))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_decode_step")
    return o


def kda_trace_begin(max_kernels: int) -> None:
    """Start per-kernel device timing for the next `max_kernels` library kernels (diagnostics)."""
    rc = _lib.load().kda_trace_begin(int(max_kernels))
    if rc != _lib.KDA_OK:
        raise KdaError(rc, "kda_trace_begin")


def kda_trace_end(capacity: int = 4096) -> list[tuple[str, float]]:
    """Synchronize, stop tracing and return [(kernel name, milliseconds), ...] in launch order."""
    ids = (ctypes.c_int * capacity)()
    ms = (ctypes.c_float * capacity)()
    n = _lib.load().kda_trace_end(ids, ms, capacity)
    if n < 0:
        raise KdaError(n, "kda_trace_end")
    return [(_lib.KERNEL_NAMES.get(ids[i], str(ids[i])), float(ms[i])) for i in range(min(n, capacity))]
