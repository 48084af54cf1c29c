"""KDA oracle: double-precision CPU reference for Kimi Delta Attention.

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product path (the CUDA library and
its Python binding) never does, and this package imports nothing from it.

Source: the Kimi Linear summary page (th.news.hada.io, topic 31936), sections
"From linear attention to Gated DeltaNet", "Fine-grained memory control of KDA",
"Chunkwise parallel algorithm" and "Reduced computation vs general DPLR".  Per
(sequence, head):

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t

with alpha_t = exp(log_alpha_t) channel-wise.  Functions take numpy arrays (any
float dtype; they are widened to float64) in token-major layout
q, k, log_alpha [B,T,H,dk], v [B,T,H,dv], beta [B,T,H], state [N,H,dk,dv].
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

def _bind(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    i = ctypes.c_int
    lib.kda_oracle_recurrent.argtypes = [dp, dp, dp, dp, dp, dp, ip, i, i, i, i, i, i, dp, dp]
    lib.kda_oracle_recurrent.restype = i
    lib.kda_oracle_chunkwise.argtypes = [dp, dp, dp, dp, dp, dp, ip, i, i, i, i, i, i, i, dp, dp]
    lib.kda_oracle_chunkwise.restype = i
    lib.kda_oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, dp, i, i, i, i, dp]
    lib.kda_oracle_decode_step.restype = i
    lib.kda_oracle_prologue.argtypes = [dp, dp, dp, ctypes.c_int64, i, i, ctypes.c_uint, ctypes.c_double, dp, dp]
    lib.kda_oracle_prologue.restype = i
    lib.kda_oracle_recurrent_bwd.argtypes = [dp, dp, dp, dp, dp, dp, ip, i, i, i, i, i, i, dp, dp, dp, dp, dp, dp,
                                             dp, dp]
    lib.kda_oracle_recurrent_bwd.restype = i
    lib.kda_oracle_output_gate_norm.argtypes = [dp, dp, dp, ctypes.c_int64, i, ctypes.c_double, dp]
    lib.kda_oracle_output_gate_norm.restype = i
    lib.kda_oracle_num_threads.restype = i
    lib.kda_oracle_set_num_threads.argtypes = [i]
    return lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shapes(q, v, cu_seqlens):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
    else:
        cu = None
        N = B
    return B, T, H, dk, dv, N, cu


class Oracle:
    """One loaded build of the oracle library (the trusted one, or a planted-mistake
    variant used only to show that the pins catch mistakes)."""

    def __init__(self, path: str):
        self.path = path
        self.lib = _bind(path)

    def recurrent(self, q, k, v, log_alpha, beta, h0=None, cu_seqlens=None):
        """Token-by-token reference.  Returns (o [B,T,H,dv], h_T [N,H,dk,dv]) as float64."""
        q, k, v, la, bt = (_f64(x) for x in (q, k, v, log_alpha, beta))
        B, T, H, dk, dv, N, cu = _shapes(q, v, cu_seqlens)
        h0a = None if h0 is None else _f64(h0)
        o = np.zeros((B, T, H, dv), np.float64)
        hT = np.zeros((N, H, dk, dv), np.float64)
        rc = self.lib.kda_oracle_recurrent(
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bt), _ptr(h0a),
            None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            N, B, T, H, dk, dv, _ptr(o), _ptr(hT))
        if rc != 0:
            raise ValueError(f"kda_oracle_recurrent rejected its arguments (rc={rc})")
        return o, hT

    def recurrent_bwd(self, q, k, v, log_alpha, beta, h0=None, cu_seqlens=None, do=None, dhT=None):
        """Gradients of the token-by-token map for upstream gradients do [B,T,H,dv] (dL/do) and dhT
        [N,H,dk,dv] (dL/dh_T, None = 0).  Returns a dict of float64 arrays: dq, dk, dv, dlog_alpha,
        dbeta and dh0 (the gradient for the initial states, zero states when h0 is None)."""
        q, k, v, la, bt, dout = (_f64(x) for x in (q, k, v, log_alpha, beta, do))
        B, T, H, dk, dv, N, cu = _shapes(q, v, cu_seqlens)
        h0a = None if h0 is None else _f64(h0)
        dhTa = None if dhT is None else _f64(dhT)
        g = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v), "dlog_alpha": np.zeros_like(la),
             "dbeta": np.zeros_like(bt), "dh0": np.zeros((N, H, dk, dv), np.float64)}
        rc = self.lib.kda_oracle_recurrent_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bt), _ptr(h0a),
            None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            N, B, T, H, dk, dv, _ptr(dout), _ptr(dhTa), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
            _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dh0"]))
        if rc != 0:
            raise ValueError(f"kda_oracle_recurrent_bwd rejected its arguments (rc={rc})")
        return g

    def chunkwise(self, q, k, v, log_alpha, beta, h0=None, cu_seqlens=None, chunk=64):
        """Chunkwise WY / UT-transform restatement of the same map (float64)."""
        q, k, v, la, bt = (_f64(x) for x in (q, k, v, log_alpha, beta))
        B, T, H, dk, dv, N, cu = _shapes(q, v, cu_seqlens)
        h0a = None if h0 is None else _f64(h0)
        o = np.zeros((B, T, H, dv), np.float64)
        hT = np.zeros((N, H, dk, dv), np.float64)
        rc = self.lib.kda_oracle_chunkwise(
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bt), _ptr(h0a),
            None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            N, B, T, H, dk, dv, int(chunk), _ptr(o), _ptr(hT))
        if rc != 0:
            raise ValueError(f"kda_oracle_chunkwise rejected its arguments (rc={rc})")
        return o, hT

    def decode_step(self, q, k, v, log_alpha, beta, S):
        """One recurrent step on S [N,H,dk,dv].  Returns (o [N,H,dv], S_new) as float64."""
        q, k, v, la, bt = (_f64(x) for x in (q, k, v, log_alpha, beta))
        S = np.array(S, dtype=np.float64, copy=True, order="C")
        N, H, dk = q.shape
        dv = v.shape[-1]
        o = np.zeros((N, H, dv), np.float64)
        rc = self.lib.kda_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bt),
                                             _ptr(S), N, H, dk, dv, _ptr(o))
        if rc != 0:
            raise ValueError(f"kda_oracle_decode_step rejected its arguments (rc={rc})")
        return o, S

    def prologue(self, q, k, log_alpha, flags, A_log=None, dt_bias=None, eps=1e-6):
        """The layer's prologue on token-major q, k, log_alpha [..., H, dk] (float64 copies are
        returned): flags & 1 L2-normalises q and k rows; flags & 2 turns the gate pre-activation in
        log_alpha into -exp(A_log[h]) * softplus(g + dt_bias[h, c])."""
        q, k, la = (np.array(x, dtype=np.float64, copy=True, order="C") for x in (q, k, log_alpha))
        H, dk = q.shape[-2], q.shape[-1]
        n_tok = q.size // (H * dk)
        al = None if A_log is None else _f64(A_log)
        db = None if dt_bias is None else _f64(dt_bias)
        rc = self.lib.kda_oracle_prologue(_ptr(q), _ptr(k), _ptr(la), n_tok, H, dk, int(flags), float(eps),
                                          _ptr(al), _ptr(db))
        if rc != 0:
            raise ValueError(f"kda_oracle_prologue rejected its arguments (rc={rc})")
        return q, k, la

    def output_gate_norm(self, o, g, weight=None, eps=1e-6):
        """The layer's output epilogue on rows of length dv (the last axis of o and g): per-row RMSNorm
        times weight[dv] times sigmoid(g).  Returns a float64 array shaped like o."""
        o, g = _f64(o), _f64(g)
        if o.shape != g.shape or o.ndim < 1:
            raise ValueError("o and g must have the same shape")
        dv = o.shape[-1]
        w = None if weight is None else _f64(weight)
        if w is not None and w.shape != (dv,):
            raise ValueError("weight must have shape [dv]")
        out = np.empty_like(o)
        rc = self.lib.kda_oracle_output_gate_norm(_ptr(o), _ptr(g), _ptr(w), o.size // dv, dv, float(eps), _ptr(out))
        if rc != 0:
            raise ValueError(f"kda_oracle_output_gate_norm rejected its arguments (rc={rc})")
        return out

    def num_threads(self) -> int:
        return int(self.lib.kda_oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.kda_oracle_set_num_threads(int(n))


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def recurrent(*args, **kw):
    return default().recurrent(*args, **kw)


def chunkwise(*args, **kw):
    return default().chunkwise(*args, **kw)


def prologue(*args, **kw):
    return default().prologue(*args, **kw)


def recurrent_bwd(*args, **kw):
    return default().recurrent_bwd(*args, **kw)


def output_gate_norm(*args, **kw):
    return default().output_gate_norm(*args, **kw)


def decode_step(*args, **kw):
    return default().decode_step(*args, **kw)


def num_threads() -> int:
    return default().num_threads()


def set_num_threads(n: int) -> None:
    default().set_num_threads(n)
