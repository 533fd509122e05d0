"""Independent fp64 formulations of KDA used to pin the oracle.

Nothing here is shared with the oracle (C) or with the CUDA path; it is a
second, differently structured derivation of the same mathematics, written
with numpy so that a reader can check it against the equations by eye.

1. ``chunked``: the chunk-parallel closed form.  Per chunk of C tokens with
   incoming state S0, log-decay cumsum G_r = sum_{s<=r} g_s and
   Gamma_r = exp(G_r):
       Akk[r,s] = beta_r sum_c k_r[c] k_s[c] exp(G_r[c]-G_s[c])   (s < r)
       Aqk[r,s] = sum_c q_r[c] k_s[c] exp(G_r[c]-G_s[c])          (s <= r)
       U  = (I + Akk)^{-1} Diag(beta) (V - (K*Gamma) S0)
       O  = (Q*Gamma) S0 + Aqk U
       S' = Diag(Gamma_L) S0 + (K*exp(G_L - G))^T U
   Derived by unrolling the recurrence inside one chunk: the pseudo-value
   u_r = beta_r (v_r - (decayed state)^T k_r) satisfies the unit
   lower-triangular system above.  The linear solve is numpy's.

2. ``product_form``: the recurrence exactly as written, with dense matrices:
       S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
       o_t = S_t^T q_t.
"""
from __future__ import annotations

import numpy as np


def _clamp(g):
    return np.maximum(g, -5.0)


def chunked_unit(q, k, v, g, beta, S0, C):
    """One (sequence, head): q, k, g [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv]."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.array(S0, dtype=np.float64, copy=True)
    O = np.zeros((T, dv))
    for t0 in range(0, T, C):
        t1 = min(T, t0 + C)
        L = t1 - t0
        Q, K, V, b = q[t0:t1], k[t0:t1], v[t0:t1], beta[t0:t1]
        G = np.cumsum(_clamp(g[t0:t1]), axis=0)           # [L, dk]
        D = np.exp(G[:, None, :] - G[None, :, :])          # [L, L, dk], r, s
        Akk = np.einsum("rc,sc,rsc->rs", K, K, D) * b[:, None]
        Aqk = np.einsum("rc,sc,rsc->rs", Q, K, D)
        Akk = np.tril(Akk, -1)
        Aqk = np.tril(Aqk, 0)
        Gam = np.exp(G)
        rhs = b[:, None] * (V - (K * Gam) @ S)
        U = np.linalg.solve(np.eye(L) + Akk, rhs)
        O[t0:t1] = (Q * Gam) @ S + Aqk @ U
        S = np.exp(G[-1])[:, None] * S + (K * np.exp(G[-1][None, :] - G)).T @ U
    return O, S


def chunked(q, k, v, g, beta, state_in, cu_seqlens, C):
    """Packed batch: q [rows, H, dk] ...; returns (o [rows, H, dv], S [N, H, dk, dv])."""
    rows, H, dk = q.shape
    dv = v.shape[-1]
    N = len(cu_seqlens) - 1
    o = np.zeros((rows, H, dv))
    S_out = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, e = int(cu_seqlens[n]), int(cu_seqlens[n + 1])
        for h in range(H):
            S0 = np.zeros((dk, dv)) if state_in is None else state_in[n, h]
            if e > a:
                O, S = chunked_unit(q[a:e, h], k[a:e, h], v[a:e, h], g[a:e, h],
                                    beta[a:e, h], S0, C)
                o[a:e, h] = O
            else:
                S = np.array(S0, dtype=np.float64)
            S_out[n, h] = S
    return o, S_out


def product_form_unit(q, k, v, g, beta, S0):
    T, dk = q.shape
    S = np.array(S0, dtype=np.float64, copy=True)
    O = np.zeros((T, v.shape[1]))
    I = np.eye(dk)
    for t in range(T):
        kt = k[t][:, None]
        S = (I - beta[t] * kt @ kt.T) @ np.diag(np.exp(_clamp(g[t]))) @ S \
            + beta[t] * kt @ v[t][None, :]
        O[t] = S.T @ q[t]
    return O, S
