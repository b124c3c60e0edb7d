"""Separately written NumPy fp64 forms that pin the C token oracle.

TEST INFRASTRUCTURE (see the package header).  None of these shares code with
``gdn2_ref.c``; each is written from its own definition:

* ``kda_recurrence``      S_t = (I - beta_t k k^T) Diag(alpha_t) S_{t-1} + beta_t k v^T,
                          o_t = S_t^T q_t.  Kimi Delta Attention, the special case the
                          aiexpert.news article names (both gates collapse to one scalar).
* ``gated_deltanet_recurrence``  same with a scalar decay alpha_t (needhelp.icu
                          "Generalisierungshierarchie": Gated DeltaNet = KDA with
                          collapsed decay).
* ``deltanet_recurrence`` no decay, no gates beyond beta (the original DeltaNet).
* ``gla_closed_form``     b = 0: gated additive linear attention written as a direct
                          O(T^2) sum over the global log-decay prefix sums.
* ``chunked_fwd``         the chunkwise form the aiexpert.news article names ("chunkwise
                          WY algorithm with the decay absorbed into asymmetric erase
                          factors"), with the auxiliary matrices of the aixai.ru post's
                          "Как это реализуется на практике" section (gate-weighted keys E,
                          gate-weighted delta values, A and T = (I + A)^{-1}).
* ``chunked_bwd``         reverse-mode of ``chunked_fwd`` derived by hand; the gates sit
                          inside the products E~ = (b.k) e^G and X = w.v, as the aixai.ru
                          post requires ("gates inside the products, not scalar
                          post-scaling").

All inputs are [B,T,H,D] arrays (S0 [B,H,Dk,Dv]); outputs fp64.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _np(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _s0(S0, B, H, Dk, Dv):
    return np.zeros((B, H, Dk, Dv)) if S0 is None else _np(S0)


def kda_recurrence(q, k, v, g, beta, S0=None):
    """KDA: beta [B,T,H] scalar per token, g [B,T,H,Dk] channel-wise log decay."""
    q, k, v, g, beta = map(_np, (q, k, v, g, beta))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S0 = _s0(S0, B, H, Dk, Dv)
    o = np.zeros((B, T, H, Dv))
    ST = np.zeros((B, H, Dk, Dv))
    I = np.eye(Dk)
    for bb in range(B):
        for hh in range(H):
            S = S0[bb, hh].copy()
            for t in range(T):
                kt = k[bb, t, hh][:, None]
                bt = beta[bb, t, hh]
                S = (I - bt * kt @ kt.T) @ np.diag(np.exp(g[bb, t, hh])) @ S + bt * kt @ v[bb, t, hh][None, :]
                o[bb, t, hh] = S.T @ q[bb, t, hh]
            ST[bb, hh] = S
    return o, ST


def gated_deltanet_recurrence(q, k, v, gs, beta, S0=None):
    """Gated DeltaNet: scalar log decay gs [B,T,H] and scalar beta [B,T,H]."""
    q, k, v, gs, beta = map(_np, (q, k, v, gs, beta))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S0 = _s0(S0, B, H, Dk, Dv)
    o = np.zeros((B, T, H, Dv))
    ST = np.zeros((B, H, Dk, Dv))
    I = np.eye(Dk)
    for bb in range(B):
        for hh in range(H):
            S = S0[bb, hh].copy()
            for t in range(T):
                kt = k[bb, t, hh][:, None]
                bt = beta[bb, t, hh]
                S = np.exp(gs[bb, t, hh]) * ((I - bt * kt @ kt.T) @ S) + bt * kt @ v[bb, t, hh][None, :]
                o[bb, t, hh] = S.T @ q[bb, t, hh]
            ST[bb, hh] = S
    return o, ST


def deltanet_recurrence(q, k, v, beta, S0=None):
    """DeltaNet: S_t = (I - beta k k^T) S_{t-1} + beta k v^T."""
    q, k, v, beta = map(_np, (q, k, v, beta))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S0 = _s0(S0, B, H, Dk, Dv)
    o = np.zeros((B, T, H, Dv))
    ST = np.zeros((B, H, Dk, Dv))
    for bb in range(B):
        for hh in range(H):
            S = S0[bb, hh].copy()
            for t in range(T):
                kt = k[bb, t, hh]
                S = S - beta[bb, t, hh] * np.outer(kt, kt @ S) + beta[bb, t, hh] * np.outer(kt, v[bb, t, hh])
                o[bb, t, hh] = S.T @ q[bb, t, hh]
            ST[bb, hh] = S
    return o, ST


def gla_closed_form(q, k, v, g, w, S0=None):
    """b = 0: o_t = S0^T (e^{G_t} q_t) + sum_{i<=t} <q_t e^{G_t - G_i}, k_i> (w_i v_i),
    S_T = Diag(e^{G_T}) S0 + sum_i Diag(e^{G_T - G_i}) k_i (w_i v_i)^T, G the global cumsum."""
    q, k, v, g, w = map(_np, (q, k, v, g, w))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S0 = _s0(S0, B, H, Dk, Dv)
    G = np.cumsum(g, axis=1)
    o = np.zeros((B, T, H, Dv))
    ST = np.zeros((B, H, Dk, Dv))
    for bb in range(B):
        for hh in range(H):
            x = w[bb, :, hh] * v[bb, :, hh]                  # [T, Dv]
            Gh = G[bb, :, hh]                                 # [T, Dk]
            for t in range(T):
                acc = S0[bb, hh].T @ (np.exp(Gh[t]) * q[bb, t, hh])
                for i in range(t + 1):
                    coef = np.sum(q[bb, t, hh] * k[bb, i, hh] * np.exp(Gh[t] - Gh[i]))
                    acc = acc + coef * x[i]
                o[bb, t, hh] = acc
            S = np.exp(Gh[T - 1])[:, None] * S0[bb, hh]
            for i in range(T):
                S = S + np.outer(np.exp(Gh[T - 1] - Gh[i]) * k[bb, i, hh], x[i])
            ST[bb, hh] = S
    return o, ST


def _chunk_factors(qc, kc, vc, gc, bc, wc):
    G = np.cumsum(gc, axis=0)              # inclusive within the chunk
    GL = G[-1]
    Qt = qc * np.exp(G)
    Et = bc * kc * np.exp(G)
    Kt = kc * np.exp(-G)
    Kh = kc * np.exp(GL - G)
    gam = np.exp(GL)
    L = qc.shape[0]
    A = np.tril(Et @ Kt.T, -1)
    Tm = solve_triangular(np.eye(L) + A, np.eye(L), lower=True, unit_diagonal=True)
    X = wc * vc
    W = Tm @ Et
    U = Tm @ X
    P = np.tril(Qt @ Kt.T)
    return dict(G=G, GL=GL, Qt=Qt, Et=Et, Kt=Kt, Kh=Kh, gam=gam, A=A, Tm=Tm, X=X, W=W, U=U, P=P)


def chunked_fwd(q, k, v, g, b, w, S0=None, C=64):
    """Chunkwise form: per chunk, with S the chunk-start state,
    U~ = T (w.V) - T E~ S;  O = Q~ S + tril(Q~ K~^T) U~;  S <- Diag(gamma) S + K^^T U~."""
    q, k, v, g, b, w = map(_np, (q, k, v, g, b, w))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S0 = _s0(S0, B, H, Dk, Dv)
    o = np.zeros((B, T, H, Dv))
    ST = np.zeros((B, H, Dk, Dv))
    for bb in range(B):
        for hh in range(H):
            S = S0[bb, hh].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, min(T, c0 + C))
                f = _chunk_factors(q[bb, sl, hh], k[bb, sl, hh], v[bb, sl, hh], g[bb, sl, hh],
                                   b[bb, sl, hh], w[bb, sl, hh])
                Ub = f["U"] - f["W"] @ S
                o[bb, sl, hh] = f["Qt"] @ S + f["P"] @ Ub
                S = f["gam"][:, None] * S + f["Kh"].T @ Ub
            ST[bb, hh] = S
    return o, ST


def chunked_bwd(q, k, v, g, b, w, S0, do, dST=None, C=64):
    """Hand-derived reverse mode of ``chunked_fwd``.  Returns dq, dk, dv, dg, db, dw, dS0."""
    q, k, v, g, b, w, do = map(_np, (q, k, v, g, b, w, do))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    S0 = _s0(S0, B, H, Dk, Dv)
    dST = np.zeros((B, H, Dk, Dv)) if dST is None else _np(dST)
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g),
                                            ("db", b), ("dw", w))}
    out["dS0"] = np.zeros((B, H, Dk, Dv))
    for bb in range(B):
        for hh in range(H):
            starts = list(range(0, T, C))
            states, facts = [], []
            S = S0[bb, hh].copy()
            for c0 in starts:
                sl = slice(c0, min(T, c0 + C))
                f = _chunk_factors(q[bb, sl, hh], k[bb, sl, hh], v[bb, sl, hh], g[bb, sl, hh],
                                   b[bb, sl, hh], w[bb, sl, hh])
                f["Ub"] = f["U"] - f["W"] @ S
                states.append(S)
                facts.append(f)
                S = f["gam"][:, None] * S + f["Kh"].T @ f["Ub"]
            dSn = dST[bb, hh].copy()
            for ci in range(len(starts) - 1, -1, -1):
                c0 = starts[ci]
                sl = slice(c0, min(T, c0 + C))
                f, S = facts[ci], states[ci]
                dO = do[bb, sl, hh]
                kc, vc, bc, wc = k[bb, sl, hh], v[bb, sl, hh], b[bb, sl, hh], w[bb, sl, hh]
                Ub, P, Qt, Kt, Kh, Et, W, Tm, X = (f[n] for n in ("Ub", "P", "Qt", "Kt", "Kh", "Et", "W", "Tm", "X"))
                G, GL, gam = f["G"], f["GL"], f["gam"]
                # O = Q~ S + P U~ ;  S_next = Diag(gam) S + K^^T U~
                dP = np.tril(dO @ Ub.T)
                dUb = P.T @ dO + Kh @ dSn
                dQt = dO @ S.T + dP @ Kt
                dKt = dP.T @ Qt
                dS = Qt.T @ dO + gam[:, None] * dSn - W.T @ dUb
                dgam = np.sum(dSn * S, axis=1)
                dKh = Ub @ dSn.T
                # U~ = T X - W S with W = T E~ and U = T X
                dW = -dUb @ S.T
                dX = Tm.T @ dUb
                dEt = Tm.T @ dW
                dTm = dUb @ X.T + dW @ Et.T
                # T = (I + A)^{-1}, A = strict_lower(E~ K~^T)
                dA = np.tril(-Tm.T @ dTm @ Tm.T, -1)
                dEt = dEt + dA @ Kt
                dKt = dKt + dA.T @ Et
                # factors -> inputs
                eG, emG, eLG = np.exp(G), np.exp(-G), np.exp(GL - G)
                out["dq"][bb, sl, hh] = dQt * eG
                d_e = dEt * eG                      # gradient w.r.t. e = b.k
                out["db"][bb, sl, hh] = d_e * kc
                out["dk"][bb, sl, hh] = d_e * bc + dKt * emG + dKh * eLG
                out["dw"][bb, sl, hh] = dX * vc
                out["dv"][bb, sl, hh] = dX * wc
                dG = dQt * Qt + dEt * Et - dKt * Kt - dKh * Kh
                dG[-1] += np.sum(dKh * Kh, axis=0) + dgam * gam
                out["dg"][bb, sl, hh] = np.cumsum(dG[::-1], axis=0)[::-1]
                dSn = dS
            out["dS0"][bb, hh] = dSn
    return out
