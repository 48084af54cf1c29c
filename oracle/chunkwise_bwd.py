"""KDA oracle, second form of the backward: the reverse-mode derivative taken chunk by chunk.

TEST INFRASTRUCTURE ONLY (like the rest of this package): it restates in float64 numpy the
chunkwise reverse pass that the GPU backward is built on, so that its algebra can be checked
against the token-by-token adjoint (kda_oracle_recurrent_bwd), which is itself pinned by finite
differences.

Source: the Kimi Linear summary page (th.news.hada.io, topic 31936), section "Chunkwise parallel
algorithm" (chunks passing their final state on; the rank-1 updates packed through the UT
transform T = (I + A)^-1; an output mixing the state term with the intra-chunk term) and section
"Reduced computation vs general DPLR" (two decayed Gram matrices, A from k-k and P from q-k).  Per
chunk with incoming state S, running log-gate G (G_r = sum_{s<=r} log_alpha_s per channel) and
last row L:

    Abar[r][i] = sum_c k_rc k_ic e^{G_rc - G_ic} (i < r),   P[r][i] = sum_c q_rc k_ic e^{...} (i <= r)
    T = (I + Diag(beta) Abar)^-1,   X1 = V - K~ S,   Delta = T Diag(beta) X1
    O = Q~ S + P Delta,   S' = e^{G_L} o S + K^^T Delta
    K~ = K o e^G,  Q~ = Q o e^G,  K^ = K o e^{G_L - G}

and its reverse for upstream dO and dS' is written out step by step below, each step the
derivative of one line above.  Plain matrix products; no blocking beyond the chunk itself.
"""
from __future__ import annotations

import numpy as np


def _chunk_forward(K, Q, V, la, bt, S):
    L = K.shape[0]
    G = np.cumsum(la, axis=0)
    E = np.exp(G[:, None, :] - G[None, :, :])  # [r, i, c]: e^{G_rc - G_ic}
    strict, incl = np.tril(np.ones((L, L)), -1), np.tril(np.ones((L, L)))
    Abar = np.einsum("rc,ic,ric->ri", K, K, E) * strict
    P = np.einsum("rc,ic,ric->ri", Q, K, E) * incl
    T = np.linalg.inv(np.eye(L) + bt[:, None] * Abar)
    Kt, Qt, Kh = K * np.exp(G), Q * np.exp(G), K * np.exp(G[-1] - G)
    X1 = V - Kt @ S
    Delta = T @ (bt[:, None] * X1)
    return dict(G=G, E=E, Abar=Abar, P=P, T=T, Kt=Kt, Qt=Qt, Kh=Kh, X1=X1, Delta=Delta,
                O=Qt @ S + P @ Delta, S_next=np.exp(G[-1])[:, None] * S + Kh.T @ Delta)


def _chunk_backward(K, Q, V, la, bt, S, dS_next, dO):
    f = _chunk_forward(K, Q, V, la, bt, S)
    L = K.shape[0]
    G, E, T, P, Kt, Qt, Kh, X1, Delta = (f[n] for n in ("G", "E", "T", "P", "Kt", "Qt", "Kh", "X1", "Delta"))
    strict, incl = np.tril(np.ones((L, L)), -1), np.tril(np.ones((L, L)))
    # O = Q~ S + P Delta  and  S' = e^{G_L} o S + K^^T Delta
    dDelta = Kh @ dS_next + P.T @ dO
    dQt = dO @ S.T
    dP = (dO @ Delta.T) * incl
    dKh = Delta @ dS_next.T
    dS = np.exp(G[-1])[:, None] * dS_next + Qt.T @ dO
    # Delta = T Diag(beta) X1
    Z = T.T @ dDelta
    dX1 = bt[:, None] * Z
    dT = dDelta @ (bt[:, None] * X1).T
    dbeta = (Z * X1).sum(axis=1)
    # X1 = V - K~ S
    dV = dX1
    dKt = -dX1 @ S.T
    dS = dS - Kt.T @ dX1
    # T = (I + A)^-1 with A = Diag(beta) Abar (strictly lower)
    dA = -(T.T @ dT @ T.T) * strict
    dbeta += (dA * f["Abar"]).sum(axis=1)
    dAbar = bt[:, None] * dA
    # Abar and P: decayed Gram products, channel by channel
    WA, WP = dAbar[:, :, None] * E, dP[:, :, None] * E  # [r, i, c]
    dK = np.einsum("ric,ic->rc", WA, K) + np.einsum("ric,rc->ic", WA, K) + np.einsum("ric,rc->ic", WP, Q)
    dQ = np.einsum("ric,ic->rc", WP, K)
    dG = (np.einsum("ric,rc,ic->rc", WA, K, K) + np.einsum("ric,rc,ic->rc", WP, Q, K)
          - np.einsum("ric,rc,ic->ic", WA, K, K) - np.einsum("ric,rc,ic->ic", WP, Q, K))
    # K~, Q~, K^ and the state decay e^{G_L}
    dK += dKt * np.exp(G) + dKh * np.exp(G[-1] - G)
    dQ += dQt * np.exp(G)
    dG += dKt * Kt + dQt * Qt - dKh * Kh
    dG[-1] += (dKh * Kh).sum(axis=0) + np.exp(G[-1]) * (S * dS_next).sum(axis=1)
    # G = running sum of log_alpha
    dla = np.cumsum(dG[::-1], axis=0)[::-1]
    return dict(dq=dQ, dk=dK, dv=dV, dlog_alpha=dla, dbeta=dbeta, dS=dS)


def chunkwise_bwd(q, k, v, log_alpha, beta, h0=None, do=None, dhT=None, chunk=64):
    """Gradients of the chunkwise forward for one batch of sequences (no varlen): q, k, log_alpha
    [B,T,H,dk], v [B,T,H,dv], beta [B,T,H], h0 [B,H,dk,dv] or None, do [B,T,H,dv], dhT [B,H,dk,dv]
    or None.  Returns float64 arrays dq, dk, dv, dlog_alpha, dbeta, dh0 (shapes as the inputs)."""
    q, k, v, la, bt, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta, do))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dlog_alpha": np.zeros_like(la), "dbeta": np.zeros_like(bt), "dh0": np.zeros((B, H, dk, dv))}
    starts = list(range(0, T, chunk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if h0 is None else np.asarray(h0, dtype=np.float64)[b, h].copy()
            states = []
            for c0 in starts:  # forward: the state entering each chunk
                states.append(S)
                sl = slice(c0, c0 + chunk)
                S = _chunk_forward(k[b, sl, h], q[b, sl, h], v[b, sl, h], la[b, sl, h], bt[b, sl, h], S)["S_next"]
            dS = np.zeros((dk, dv)) if dhT is None else np.asarray(dhT, dtype=np.float64)[b, h].copy()
            for n in reversed(range(len(starts))):  # reverse: chunks in reverse order, carrying dS
                sl = slice(starts[n], starts[n] + chunk)
                g = _chunk_backward(k[b, sl, h], q[b, sl, h], v[b, sl, h], la[b, sl, h], bt[b, sl, h], states[n],
                                    dS, do[b, sl, h])
                for name in ("dq", "dk", "dv", "dlog_alpha"):
                    out[name][b, sl, h] = g[name]
                out["dbeta"][b, sl, h] = g["dbeta"]
                dS = g["dS"]
            out["dh0"][b, h] = dS
    return out
