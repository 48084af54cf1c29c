"""Pins for the fp64 CPU oracle (no GPU).

The pages (Kimi Linear summary, th.news.hada.io topic 31936) print no worked
numbers, so the oracle is pinned by what they and the mathematics fix:

  * exact rational arithmetic on a hand-sized case, in the DPLR matrix form
    (section "Fine-grained memory control of KDA": a diagonal gate inside a
    transition tied to the key, section "Reduced computation vs general DPLR");
  * the dense transition product (I - b k k^T) Diag(a) applied matrix by matrix;
  * the delta rule as one step of online gradient descent on 1/2||S^T k - v||^2,
    differentiated by autograd (section "From linear attention to Gated DeltaNet");
  * reductions to DeltaNet (a = 1) and to scalar-gated Gated DeltaNet (a constant
    over channels) written as separate loops (same section);
  * the chunkwise WY / UT-transform form equal to the recurrence, and continuity
    across a split (section "Chunkwise parallel algorithm": each chunk's final
    state is the next chunk's initial state);
  * closed forms (beta = 0, one token, orthonormal-key recall), v = 0 => o = 0,
    linearity in (V, h0), column separability, the contraction bound for unit
    keys, varlen packing = separate runs, and decode steps = the recurrence.

Each pin is a function of an Oracle build so that the planted-mistake test can
show every variant in oracle/kda_oracle.c (KDA_ORACLE_MUTANT) fails at least one.
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))


def _inputs(rng, B, T, H, dk, dv, gate_shift=0.0, unit_keys=True, h0_scale=1.0, state=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk)) + gate_shift))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    h0 = rng.standard_normal((B, H, dk, dv)) * h0_scale if state else None
    return q, k, v, la, beta, h0


def _rel(a, b):
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / den)


# --------------------------------------------------------------------------- pins
def pin_exact_rational(orc) -> float:
    """d_k = d_v = 2, T = 3: the transition (I - b k k^T) Diag(a) S + b k v^T evaluated in
    exact rational arithmetic (Fractions); the oracle sees log(a) and must agree to rounding."""
    F = Fraction
    ks = [(F(1), F(0)), (F(3, 5), F(4, 5)), (F(0), F(1))]
    qs = [(F(1, 2), F(-1)), (F(2), F(1, 3)), (F(-3, 4), F(5, 4))]
    vs = [(F(1), F(2)), (F(-1, 2), F(3)), (F(7, 4), F(-2))]
    als = [(F(1, 2), F(1, 4)), (F(3, 4), F(1)), (F(1, 8), F(5, 8))]
    bs = [F(1, 2), F(1, 3), F(3, 4)]
    S = [[F(1, 3), F(-2)], [F(1, 5), F(1, 7)]]
    exp_o = []
    for t in range(3):
        k, q, v, a, b = ks[t], qs[t], vs[t], als[t], bs[t]
        D = [[a[i] * S[i][j] for j in range(2)] for i in range(2)]                # Diag(a) S
        KtD = [sum(k[i] * D[i][j] for i in range(2)) for j in range(2)]           # k^T D
        S = [[D[i][j] - b * k[i] * KtD[j] + b * k[i] * v[j] for j in range(2)] for i in range(2)]
        exp_o.append([sum(S[i][j] * q[i] for i in range(2)) for j in range(2)])
    f = lambda x: np.array(x, dtype=np.float64)
    q = f([[qs[t]] for t in range(3)])[None]          # [1,3,1,2]
    k = f([[ks[t]] for t in range(3)])[None]
    v = f([[vs[t]] for t in range(3)])[None]
    la = np.log(f([[als[t]] for t in range(3)]))[None]
    beta = f([[bs[t]] for t in range(3)])[None]
    h0 = f([[[F(1, 3), F(-2)], [F(1, 5), F(1, 7)]]])[None]   # [1,1,2,2]
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    err_o = np.abs(o[0, :, 0, :] - f(exp_o)).max()
    err_h = np.abs(hT[0, 0] - f(S)).max()
    return float(max(err_o, err_h))


def pin_dense_transition(orc) -> float:
    """S_t = (I - b k k^T) Diag(a) S_{t-1} + b k v^T, o_t = S_t^T q_t, as explicit dense matrices."""
    rng = np.random.default_rng(11)
    q, k, v, la, beta, h0 = _inputs(rng, 2, 12, 2, 4, 3)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    err = 0.0
    for b in range(2):
        for h in range(2):
            S = h0[b, h].copy()
            for t in range(12):
                kk = k[b, t, h][:, None]
                M = (np.eye(4) - beta[b, t, h] * kk @ kk.T) @ np.diag(np.exp(la[b, t, h]))
                S = M @ S + beta[b, t, h] * kk @ v[b, t, h][None, :]
                err = max(err, np.abs(S.T @ q[b, t, h] - o[b, t, h]).max())
            err = max(err, np.abs(S - hT[b, h]).max())
    return float(err)


def pin_gradient_step(orc) -> float:
    """Decay by Diag(a), then one gradient-descent step of size b on 1/2||S^T k - v||^2 (autograd)."""
    rng = np.random.default_rng(12)
    q, k, v, la, beta, h0 = _inputs(rng, 1, 10, 1, 5, 4)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    S = torch.tensor(h0[0, 0])
    err = 0.0
    for t in range(10):
        Sd = (torch.exp(torch.tensor(la[0, t, 0]))[:, None] * S).requires_grad_(True)
        kt, vt = torch.tensor(k[0, t, 0]), torch.tensor(v[0, t, 0])
        loss = 0.5 * ((Sd.T @ kt - vt) ** 2).sum()
        (g,) = torch.autograd.grad(loss, Sd)
        S = (Sd - float(beta[0, t, 0]) * g).detach()
        err = max(err, float((S.T @ torch.tensor(q[0, t, 0]) - torch.tensor(o[0, t, 0])).abs().max()))
    return max(err, float((S - torch.tensor(hT[0, 0])).abs().max()))


def pin_deltanet(orc) -> float:
    """alpha = 1: the classical delta rule S <- S + b k (v - S^T k)^T."""
    rng = np.random.default_rng(13)
    q, k, v, la, beta, h0 = _inputs(rng, 1, 20, 2, 6, 5)
    la = np.zeros_like(la)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    err = 0.0
    for h in range(2):
        S = h0[0, h].copy()
        for t in range(20):
            kt = k[0, t, h]
            S = S + beta[0, t, h] * np.outer(kt, v[0, t, h] - S.T @ kt)
            err = max(err, np.abs(S.T @ q[0, t, h] - o[0, t, h]).max())
        err = max(err, np.abs(S - hT[0, h]).max())
    return float(err)


def pin_gated_deltanet(orc) -> float:
    """alpha constant over channels: Gated DeltaNet S <- a (I - b k k^T) S + b k v^T."""
    rng = np.random.default_rng(14)
    q, k, v, la, beta, h0 = _inputs(rng, 1, 20, 2, 6, 5)
    la = np.repeat(la[..., :1], 6, axis=-1)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    err = 0.0
    for h in range(2):
        S = h0[0, h].copy()
        for t in range(20):
            kt = k[0, t, h]
            a = np.exp(la[0, t, h, 0])
            S = a * (S - beta[0, t, h] * np.outer(kt, kt @ S)) + beta[0, t, h] * np.outer(kt, v[0, t, h])
            err = max(err, np.abs(S.T @ q[0, t, h] - o[0, t, h]).max())
        err = max(err, np.abs(S - hT[0, h]).max())
    return float(err)


def pin_chunkwise(orc) -> float:
    """WY / UT-transform chunkwise form equals the recurrence for several chunk sizes and a ragged tail."""
    rng = np.random.default_rng(15)
    q, k, v, la, beta, h0 = _inputs(rng, 2, 150, 2, 8, 6, gate_shift=1.0)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    err = 0.0
    for C in (1, 2, 4, 16, 64):
        oc, hc = orc.chunkwise(q, k, v, la, beta, h0, chunk=C)
        err = max(err, _rel(oc, o), _rel(hc, hT))
    return err


def pin_zero_values(orc) -> float:
    rng = np.random.default_rng(16)
    q, k, v, la, beta, _ = _inputs(rng, 1, 40, 2, 8, 8)
    o, hT = orc.recurrent(q, k, np.zeros_like(v), la, beta, None)
    return float(max(np.abs(o).max(), np.abs(hT).max()))


def pin_continuity(orc) -> float:
    """Running T tokens equals running T/2, then T/2 more from the carried state."""
    rng = np.random.default_rng(17)
    q, k, v, la, beta, h0 = _inputs(rng, 2, 64, 2, 8, 8)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    s = slice(0, 32), slice(32, 64)
    o1, h1 = orc.recurrent(q[:, s[0]], k[:, s[0]], v[:, s[0]], la[:, s[0]], beta[:, s[0]], h0)
    o2, h2 = orc.recurrent(q[:, s[1]], k[:, s[1]], v[:, s[1]], la[:, s[1]], beta[:, s[1]], h1)
    return max(_rel(np.concatenate([o1, o2], 1), o), _rel(h2, hT))


def pin_linearity(orc) -> float:
    """(V, h0) -> (O, h_T) is linear for fixed q, k, alpha, beta."""
    rng = np.random.default_rng(18)
    q, k, v1, la, beta, h01 = _inputs(rng, 1, 30, 2, 6, 5)
    v2 = rng.standard_normal(v1.shape)
    h02 = rng.standard_normal(h01.shape)
    a, b = 0.7, -1.9
    o1, s1 = orc.recurrent(q, k, v1, la, beta, h01)
    o2, s2 = orc.recurrent(q, k, v2, la, beta, h02)
    o3, s3 = orc.recurrent(q, k, a * v1 + b * v2, la, beta, a * h01 + b * h02)
    return max(_rel(a * o1 + b * o2, o3), _rel(a * s1 + b * s2, s3))


def pin_column_separability(orc) -> float:
    """Column j of o and h_T depends only on column j of V and h0."""
    rng = np.random.default_rng(19)
    q, k, v, la, beta, h0 = _inputs(rng, 1, 40, 2, 6, 7)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    cols = [1, 4, 6]
    oc, hc = orc.recurrent(q, k, v[..., cols], la, beta, h0[..., cols])
    return max(_rel(oc, o[..., cols]), _rel(hc, hT[..., cols]))


def pin_beta_zero(orc) -> float:
    """beta = 0: S_t = Diag(exp(sum_{s<=t} log_alpha_s)) h0 and o_t = S_t^T q_t."""
    rng = np.random.default_rng(20)
    q, k, v, la, beta, h0 = _inputs(rng, 1, 25, 2, 6, 4)
    o, hT = orc.recurrent(q, k, v, la, np.zeros_like(beta), h0)
    G = np.cumsum(la, axis=1)                                     # [1,T,H,dk]
    St = np.exp(G)[0][:, :, :, None] * h0[0][None]                # [T,H,dk,dv]
    o_ref = np.einsum("thij,thi->thj", St, q[0])
    return max(_rel(o[0], o_ref), _rel(hT[0], St[-1]))


def pin_single_token(orc) -> float:
    """T = 1: S_1 = (I - b k k^T) Diag(a) h0 + b k v^T, written with numpy.linalg products."""
    rng = np.random.default_rng(21)
    q, k, v, la, beta, h0 = _inputs(rng, 3, 1, 2, 5, 5)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    err = 0.0
    for b in range(3):
        for h in range(2):
            kk = k[b, 0, h]
            S1 = np.linalg.multi_dot([np.eye(5) - beta[b, 0, h] * np.outer(kk, kk),
                                      np.diag(np.exp(la[b, 0, h])), h0[b, h]]) \
                + beta[b, 0, h] * np.outer(kk, v[b, 0, h])
            err = max(err, _rel(hT[b, h], S1), _rel(o[b, 0, h], S1.T @ q[b, 0, h]))
    return err


def pin_orthonormal_recall(orc) -> float:
    """alpha = 1, beta = 1, k_t = e_t, h0 = 0: querying e_j returns v_j exactly; writing key
    e_j again with beta = 1 replaces its value (the delta rule overwrites, it does not add)."""
    d, T = 6, 8
    rng = np.random.default_rng(22)
    keys = [t % d for t in range(T)]                  # keys 0..5, then 0 and 1 again
    k = np.zeros((1, T, 1, d))
    for t, j in enumerate(keys):
        k[0, t, 0, j] = 1.0
    v = rng.standard_normal((1, T, 1, d))
    q = np.zeros((1, T, 1, d))
    for t in range(T):
        q[0, t, 0, keys[t]] = 1.0
    o, hT = orc.recurrent(q, k, v, np.zeros((1, T, 1, d)), np.ones((1, T, 1)), None)
    err = float(np.abs(o[0, :, 0] - v[0, :, 0]).max())                  # query the key just written
    last = {j: t for t, j in enumerate(keys)}
    expect = np.zeros((d, d))
    for j, t in last.items():
        expect[j] = v[0, t, 0]
    return max(err, float(np.abs(hT[0, 0] - expect).max()))


def pin_contraction(orc) -> float:
    """Unit keys, beta in (0,1), alpha in (0,1]: ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t||.
    Returns the largest violation (<= 0 when the bound holds)."""
    rng = np.random.default_rng(23)
    q, k, v, la, beta, h0 = _inputs(rng, 1, 40, 1, 6, 6)
    S = h0[:, :]                                   # [1,1,dk,dv] as the decode state
    worst = -np.inf
    for t in range(40):
        _, S_new = orc.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], beta[:, t], S)
        bound = np.linalg.norm(S) + beta[0, t, 0] * np.linalg.norm(v[0, t, 0])
        worst = max(worst, np.linalg.norm(S_new) - bound)
        S = S_new
    return float(max(worst, 0.0))


def pin_varlen(orc) -> float:
    """A packed varlen batch equals separate runs of each sequence."""
    rng = np.random.default_rng(24)
    lens = [5, 1, 37, 64, 70]
    T = sum(lens)
    q, k, v, la, beta, _ = _inputs(rng, 1, T, 2, 6, 5, state=False)
    h0 = rng.standard_normal((len(lens), 2, 6, 5))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, hT = orc.recurrent(q, k, v, la, beta, h0, cu_seqlens=cu)
    err = 0.0
    for n in range(len(lens)):
        s = slice(cu[n], cu[n + 1])
        on, hn = orc.recurrent(q[:, s], k[:, s], v[:, s], la[:, s], beta[:, s], h0[n:n + 1])
        err = max(err, float(np.abs(on - o[:, s]).max()), float(np.abs(hn[0] - hT[n]).max()))
    oc, hc = orc.chunkwise(q, k, v, la, beta, h0, cu_seqlens=cu, chunk=16)
    return max(err, _rel(oc, o), _rel(hc, hT))


def pin_decode_matches_prefill(orc) -> float:
    """Decode steps applied token by token reproduce the prefill recurrence."""
    rng = np.random.default_rng(25)
    q, k, v, la, beta, h0 = _inputs(rng, 3, 9, 2, 5, 4)
    o, hT = orc.recurrent(q, k, v, la, beta, h0)
    S = h0.copy()
    err = 0.0
    for t in range(9):
        ot, S = orc.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], beta[:, t], S)
        err = max(err, float(np.abs(ot - o[:, t]).max()))
    return max(err, float(np.abs(S - hT).max()))


# ------------------------------------------------------------------------------------- output epilogue
# out = o / sqrt(mean(o^2) + eps) * weight * sigmoid(g) per row (Kimi Linear page, section "Kimi
# Linear model composition": per-head RMSNorm and a data-dependent output gate; sigmoid reading).
def _epi_inputs(rows=5, dv=16, seed=60):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((rows, dv)), rng.standard_normal((rows, dv)), 0.5 + rng.random(dv)


def pin_epilogue_constant_rows(orc):
    """Rows of one repeated value c have RMS |c|: with eps = 0 and g = 0 the output is sign(c) w / 2."""
    rows, dv = 4, 16
    c = np.array([3.0, -0.25, 1e-3, -7.5])
    o = np.repeat(c[:, None], dv, axis=1)
    w = 0.5 + np.arange(dv) / dv
    out = orc.output_gate_norm(o, np.zeros((rows, dv)), w, eps=0.0)
    return float(np.abs(out - np.sign(c)[:, None] * w[None] * 0.5).max())


def pin_epilogue_unit_rms(orc):
    """With weight 1, a saturated gate (g = 40: sigmoid = 1 - 4e-18) and eps = 0, every output row has
    mean square 1, and scaling o by any positive constant changes nothing."""
    o, _, _ = _epi_inputs()
    g = np.full_like(o, 40.0)
    out = orc.output_gate_norm(o, g, None, eps=0.0)
    out3 = orc.output_gate_norm(3.7 * o, g, None, eps=0.0)
    return max(float(np.abs((out ** 2).mean(axis=1) - 1.0).max()), float(np.abs(out3 - out).max()))


def pin_epilogue_eps_inside_root(orc):
    """eps equal to a row's mean square halves it under the root: the output shrinks by 1 / sqrt(2)."""
    o, g, w = _epi_inputs(rows=1)
    ms = float((o ** 2).mean())
    a = orc.output_gate_norm(o, g, w, eps=0.0)
    b = orc.output_gate_norm(o, g, w, eps=ms)
    return float(np.abs(b - a / np.sqrt(2.0)).max())


def pin_epilogue_gate(orc):
    """sigmoid(ln 3) = 3/4 and sigmoid(-ln 3) = 1/4 against the saturated gate; g = -800 closes it to 0;
    the gate of channel j scales only channel j."""
    o, _, w = _epi_inputs(rows=2)
    ref = orc.output_gate_norm(o, np.full_like(o, 40.0), w, eps=1e-6)
    up = orc.output_gate_norm(o, np.full_like(o, np.log(3.0)), w, eps=1e-6)
    dn = orc.output_gate_norm(o, np.full_like(o, -np.log(3.0)), w, eps=1e-6)
    shut = orc.output_gate_norm(o, np.full_like(o, -800.0), w, eps=1e-6)
    g1 = np.full_like(o, 40.0)
    g1[1, 5] = np.log(3.0)
    one = orc.output_gate_norm(o, g1, w, eps=1e-6)
    mask = np.ones_like(o, dtype=bool)
    mask[1, 5] = False
    return max(float(np.abs(up - 0.75 * ref).max()), float(np.abs(dn - 0.25 * ref).max()),
               float(np.abs(shut).max()), float(np.abs(one[mask] - ref[mask]).max()),
               float(abs(one[1, 5] - 0.75 * ref[1, 5])))


# ------------------------------------------------------------------------------------- backward
def _fd_check(orc, cu_seqlens, use_h0, use_dhT, seed):
    """Central finite differences of L = <o, W_o> + <h_T, W_h> on a tiny case against the backward
    oracle's gradients for every input element (step 1e-5: truncation ~1e-10, rounding ~1e-11)."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 7, 2, 3, 4
    x = {"q": rng.standard_normal((B, T, H, dk)), "k": 0.5 * rng.standard_normal((B, T, H, dk)),
         "v": rng.standard_normal((B, T, H, dv)), "log_alpha": -rng.random((B, T, H, dk)),
         "beta": rng.random((B, T, H))}
    N = 1 if cu_seqlens is None else len(cu_seqlens) - 1
    if use_h0:
        x["h0"] = rng.standard_normal((N, H, dk, dv))
    W_o = rng.standard_normal((B, T, H, dv))
    W_h = rng.standard_normal((N, H, dk, dv)) if use_dhT else None

    def loss(**kw):
        o, hT = orc.recurrent(kw["q"], kw["k"], kw["v"], kw["log_alpha"], kw["beta"], kw.get("h0"), cu_seqlens)
        return float((o * W_o).sum() + (0.0 if W_h is None else (hT * W_h).sum()))

    g = orc.recurrent_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x.get("h0"), cu_seqlens, W_o, W_h)
    names = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta", "h0": "dh0"}
    err = 0.0
    for name, a in x.items():
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            kw = dict(x)
            ap, am = a.copy(), a.copy()
            ap[idx] += 1e-5
            am[idx] -= 1e-5
            kw[name] = ap
            lp = loss(**kw)
            kw[name] = am
            fd[idx] = (lp - loss(**kw)) / 2e-5
        err = max(err, float(np.abs(fd - g[names[name]]).max() / max(np.abs(fd).max(), 1e-300)))
    if not use_h0:  # dL/dh0 at zero initial states, by differences in h0 around zero
        h0z = np.zeros((N, H, dk, dv))
        fd = np.zeros_like(h0z)
        for idx in np.ndindex(h0z.shape):
            ap, am = h0z.copy(), h0z.copy()
            ap[idx] += 1e-5
            am[idx] -= 1e-5
            fd[idx] = (loss(**dict(x, h0=ap)) - loss(**dict(x, h0=am))) / 2e-5
        err = max(err, float(np.abs(fd - g["dh0"]).max() / max(np.abs(fd).max(), 1e-300)))
    return err


def pin_backward_finite_differences(orc):
    return _fd_check(orc, None, use_h0=True, use_dhT=True, seed=70)


def pin_backward_varlen_zero_start(orc):
    return _fd_check(orc, np.array([0, 3, 3, 7]), use_h0=False, use_dhT=False, seed=71)


PINS = {
    "exact_rational": (pin_exact_rational, 1e-13),
    "dense_transition": (pin_dense_transition, 1e-12),
    "gradient_step": (pin_gradient_step, 1e-12),
    "deltanet": (pin_deltanet, 1e-12),
    "gated_deltanet": (pin_gated_deltanet, 1e-12),
    "chunkwise": (pin_chunkwise, 1e-11),
    "zero_values": (pin_zero_values, 0.0),
    "continuity": (pin_continuity, 1e-13),
    "linearity": (pin_linearity, 1e-12),
    "column_separability": (pin_column_separability, 0.0),
    "beta_zero": (pin_beta_zero, 1e-13),
    "single_token": (pin_single_token, 1e-13),
    "orthonormal_recall": (pin_orthonormal_recall, 1e-15),
    "contraction": (pin_contraction, 1e-12),
    "varlen": (pin_varlen, 1e-12),
    "decode_matches_prefill": (pin_decode_matches_prefill, 1e-13),
    "epilogue_constant_rows": (pin_epilogue_constant_rows, 1e-15),
    "epilogue_unit_rms": (pin_epilogue_unit_rms, 1e-14),
    "epilogue_eps_inside_root": (pin_epilogue_eps_inside_root, 1e-15),
    "epilogue_gate": (pin_epilogue_gate, 1e-15),
    "backward_finite_differences": (pin_backward_finite_differences, 1e-8),
    "backward_varlen_zero_start": (pin_backward_varlen_zero_start, 1e-8),
}


@pytest.mark.parametrize("name", sorted(PINS))
def test_oracle_pin(name):
    fn, tol = PINS[name]
    err = fn(oracle.default())
    assert err <= tol, f"pin {name}: error {err:.3e} > {tol:.1e}"


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11])
def test_pins_catch_planted_mistakes(mutant, tmp_path):
    """Every planted mistake in the oracle's token update (1-5), output epilogue (6-8) or backward
    recurrence (9-11) fails at least one pin."""
    orc = oracle.Oracle(oracle_build.build_mutant(mutant, str(tmp_path)))
    failed = []
    for name, (fn, tol) in PINS.items():
        try:
            err = fn(orc)
        except Exception:          # a wrong variant may also break an exact identity
            err = np.inf
        if not err <= tol:
            failed.append(name)
    assert failed, f"mutant {mutant} passed every pin"


def test_golden_regression():
    """The oracle reproduces its stored output on a tiny seeded case (guards unintended edits)."""
    with open(os.path.join(HERE, "golden", "oracle_tiny_d4_T10.json")) as f:
        g = json.load(f)
    arr = {k: np.array(v, dtype=np.float64) for k, v in g["inputs"].items()}
    o, hT = oracle.recurrent(arr["q"], arr["k"], arr["v"], arr["log_alpha"], arr["beta"], arr["h0"])
    assert np.abs(o - np.array(g["o"])).max() <= 1e-14
    assert np.abs(hT - np.array(g["h_T"])).max() <= 1e-14


def test_oracle_rejects_bad_seqlens():
    rng = np.random.default_rng(0)
    q, k, v, la, beta, _ = _inputs(rng, 1, 10, 1, 4, 4, state=False)
    with pytest.raises(ValueError):
        oracle.recurrent(q, k, v, la, beta, None, cu_seqlens=np.array([0, 6, 5, 10]))
    with pytest.raises(ValueError):
        oracle.recurrent(q, k, v, la, beta, None, cu_seqlens=np.array([0, 6, 9]))


# ------------------------------------------------------------------------------------- layer prologue
# Page, section "Kimi Linear model composition": q and k are L2-normalised per head; the channel-wise
# decay comes from a gate projection through a GDN / Mamba-style decay function, read here as
# log alpha = -exp(A_log[h]) * softplus(g + dt_bias[h, c]).  These pins fix each part by a property
# or a closed-form limit, not by re-evaluating the formula.
def test_prologue_l2_normalisation_pins():
    rng = np.random.default_rng(31)
    q, k = rng.normal(size=(5, 3, 8)), rng.normal(size=(5, 3, 8)) * 7.0
    g = rng.normal(size=(5, 3, 8))
    qn, kn, la = oracle.prologue(q, k, g, 1, eps=0.0)
    assert np.allclose(np.linalg.norm(qn, axis=-1), 1.0, atol=1e-14)            # unit rows
    assert np.allclose(np.linalg.norm(kn, axis=-1), 1.0, atol=1e-14)
    assert np.allclose(np.sum(qn * q, -1), np.linalg.norm(q, axis=-1), rtol=1e-14)  # same direction
    q3, k3, _ = oracle.prologue(3.5 * q, 0.25 * k, g, 1, eps=0.0)                 # scale invariance
    assert np.allclose(q3, qn, rtol=1e-14, atol=0) and np.allclose(k3, kn, rtol=1e-14, atol=0)
    assert np.array_equal(la, g)                                                  # gate untouched
    qe, _, _ = oracle.prologue(q, k, g, 1, eps=1e-6)                              # eps inside the root
    ss = np.sum(q * q, -1, keepdims=True)
    assert np.allclose(qe * np.sqrt(ss + 1e-6), q, rtol=1e-14)


def test_prologue_gate_pins():
    H, dk = 2, 6
    A_log = np.array([0.7, -1.3])
    dt_bias = np.linspace(-0.5, 0.5, H * dk).reshape(H, dk)
    a = np.exp(A_log)[:, None]
    z = np.zeros((1, H, dk))
    # softplus(0) = log 2: g = -dt_bias gives log alpha = -exp(A_log) log 2 on every channel
    _, _, la0 = oracle.prologue(z, z, -dt_bias[None], 2, A_log=A_log, dt_bias=dt_bias)
    assert np.allclose(la0[0], -a * np.log(2.0), rtol=1e-15)
    # large argument: softplus(x) = x + log(1 + e^-x) -> x (linear regime), per head and per channel
    g = 60.0 + np.arange(H * dk, dtype=np.float64).reshape(1, H, dk)
    _, _, la1 = oracle.prologue(z, z, g, 2, A_log=A_log, dt_bias=dt_bias)
    assert np.allclose(la1[0], -a * (g[0] + dt_bias), rtol=1e-15)
    # very negative argument: softplus(x) -> e^x
    gn = -40.0 - np.arange(H * dk, dtype=np.float64).reshape(1, H, dk)
    _, _, la2 = oracle.prologue(z, z, gn, 2, A_log=A_log, dt_bias=dt_bias)
    assert np.allclose(la2[0], -a * np.exp(gn[0] + dt_bias), rtol=1e-12)
    # A_log -> -inf: no decay at all (alpha = 1); without dt_bias the bias is zero
    _, _, la3 = oracle.prologue(z, z, np.ones((1, H, dk)), 2, A_log=np.full(H, -800.0))
    assert np.all(la3 == 0.0)
    _, _, la4 = oracle.prologue(z, z, -np.zeros((1, H, dk)), 2, A_log=A_log)
    assert np.allclose(la4[0], -a * np.log(2.0) * np.ones((H, dk)), rtol=1e-15)
    # every decay is <= 0 (alpha in (0, 1])
    _, _, la5 = oracle.prologue(z, z, np.random.default_rng(3).normal(size=(1, H, dk)) * 10, 2, A_log=A_log,
                                dt_bias=dt_bias)
    assert np.all(la5 <= 0.0)


# ----------------------------------------------------------------- chunkwise form of the backward
def test_chunkwise_backward_matches_the_adjoint():
    """The chunk-by-chunk reverse pass (the algebra of the GPU backward, oracle/chunkwise_bwd.py)
    equals the token-by-token adjoint, which the finite-difference pins fix: 3 chunks with a ragged
    last one, h0 and dh_T, two sequences."""
    from oracle.chunkwise_bwd import chunkwise_bwd
    rng = np.random.default_rng(80)
    B, T, H, dk, dv = 2, 150, 2, 8, 6
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk)) / np.sqrt(dk)
    v = rng.standard_normal((B, T, H, dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk)) + 1.0))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    h0 = 0.3 * rng.standard_normal((B, H, dk, dv))
    do = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    ref = oracle.recurrent_bwd(q, k, v, la, beta, h0, None, do, dhT)
    got = chunkwise_bwd(q, k, v, la, beta, h0, do, dhT, chunk=64)
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dh0"):
        err = np.abs(got[name] - ref[name]).max() / np.abs(ref[name]).max()
        assert err <= 1e-12, f"{name}: {err:.3e}"
