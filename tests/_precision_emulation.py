"""Numerical emulation of the bf16 prefill's precision scheme (test evidence only).

This is not the oracle and nothing here checks a kernel.  It evaluates the
chunked (WY) form of the recurrence in fp64, written out from its algebra,
with a rounding applied to every operand at the point where a tensor-core
implementation has to store it in a narrow type.  Comparing its result with
the oracle's shows what each precision choice costs in the parity metric
max|delta| / rms(reference), independently of any GPU code.

Chunked form, per chunk of C = 64 tokens (L valid rows), with the chunk-local
cumsum G_r = sum_{s<=r} max(g_s, -5) and Gamma = exp(G):
    Aqk[r,s] = sum_c q_r[c] k_s[c] exp(G_r[c] - G_s[c])          (s <= r)
    Akk[r,s] = beta_r sum_c k_r[c] k_s[c] exp(G_r[c] - G_s[c])   (s <  r)
    T = (I + Akk)^{-1} Diag(beta),  R = Aqk T
    W = T (K * Gamma),  P = Q * Gamma - R (K * Gamma),  Khat = K * exp(G_L - G)
    U = T V - W S,  O = R V + P S,  S <- Diag(exp(G_L)) S + Khat^T U
The decay-rescaled products split exp(G_r - G_s) as exp(G_r - R_a) exp(R_a - G_s)
with R_a the cumsum at the end of the 16-row block before row r's block a; the
operands rounded are q_r exp(G_r - R_a), k_r exp(G_r - R_a) and k_s exp(R_a - G_s).
"""
from __future__ import annotations

import numpy as np


def round_tf32(x):
    """Round to tf32 (10 explicit significand bits), nearest, ties away from zero."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x1000) & 0xFFFFE000).astype(np.uint32)
    return u.view(np.float32).astype(np.float64)


def round_bf16(x):
    """Round to bf16 (7 explicit significand bits), nearest even."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return u.view(np.float32).astype(np.float64)


def round_fp16(x):
    """Round to fp16 (10 explicit significand bits, max 65504), nearest even."""
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)


def round_fp32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


ROUND = {"tf32": round_tf32, "bf16": round_bf16, "fp16": round_fp16, "fp32": round_fp32,
         "none": lambda x: np.asarray(x, np.float64)}


def chunk_factors(qc, kc, gc, bc, akk="tf32", store="fp16"):
    """The per-chunk factors of one chunk (L <= 64 rows): dict of T, R, W, P, Khat
    (each rounded to `store`) and Gamma_L (fp32), with Akk / Aqk built from operands
    rounded to `akk` and accumulated in fp32."""
    ra, rs, f32 = ROUND[akk], ROUND[store], round_fp32
    L, dk = qc.shape
    G = np.cumsum(np.maximum(gc, -5.0), axis=0)
    blk = np.arange(L) // 16
    Rref = np.zeros((4, dk))
    for a in range(1, 4):
        if 16 * a - 1 < L:
            Rref[a] = G[16 * a - 1]
    Aqk = np.zeros((L, L))
    Akk = np.zeros((L, L))
    for a in range(4):
        rows = np.nonzero(blk == a)[0]
        if rows.size == 0:
            continue
        cols = np.arange(0, rows[-1] + 1)
        e_r = np.exp(G[rows] - Rref[a])
        Bq = ra(qc[rows] * e_r)
        Bk = ra(kc[rows] * e_r)
        As = ra(kc[cols] * np.exp(Rref[a] - G[cols]))
        Aqk[np.ix_(rows, cols)] = f32(Bq @ As.T)
        Akk[np.ix_(rows, cols)] = f32(Bk @ As.T) * bc[rows, None]
    Aqk = np.tril(Aqk)
    Akk = np.tril(Akk, -1)
    X = f32(np.linalg.inv(np.eye(L) + Akk))
    Tm = rs(X * bc[None, :])
    R = rs(f32(rs(Aqk) @ Tm))
    Gam = np.exp(G)
    KG = rs(kc * Gam)
    QG = rs(qc * Gam)
    return {"T": Tm, "R": R, "W": rs(f32(Tm @ KG)), "P": rs(f32(QG - R @ KG)),
            "Khat": rs(kc * np.exp(G[L - 1] - G)), "Gamma_L": f32(np.exp(G[L - 1]))}


def prefill_unit(q, k, v, g, beta, S0, akk="tf32", store="fp16", out="fp32", C=64):
    """One (sequence, head): q, k, g [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv] (fp64).

    akk:   type of the decay-rescaled operands of Akk / Aqk
    store: type of every other stored matrix operand (T, R, W, P, Khat, V, and the
           copies of U and S that feed products); accumulation is fp32
    out:   type o is written in
    Returns (o [T, dv], S_T [dk, dv]).
    """
    rs, ro, f32 = ROUND[store], ROUND[out], round_fp32
    T_len = q.shape[0]
    S = np.array(S0, np.float64)
    o = np.zeros((T_len, v.shape[1]))
    for t0 in range(0, T_len, C):
        sl = slice(t0, min(T_len, t0 + C))
        f = chunk_factors(q[sl], k[sl], g[sl], beta[sl], akk=akk, store=store)
        Vs = rs(v[sl])
        Ss = rs(S)
        U = f32(f["T"] @ Vs - f["W"] @ Ss)
        o[sl] = ro(f32(f["R"] @ Vs + f["P"] @ Ss))
        S = f32(f["Gamma_L"][:, None] * S + f["Khat"].T @ rs(U))
    return o, S


def prefill_heads(inp, heads, T_len, **scheme):
    """The emulation on sequence 0 of an equal-length batch, for the given heads and
    the first T_len tokens; returns o [T_len, len(heads), dv], S [len(heads), dk, dv]."""
    f = lambda x: x.detach().to("cpu").double().numpy()
    os_, ss = [], []
    for h in heads:
        S0 = np.zeros((inp.dk, inp.dv)) if inp.state_in is None else f(inp.state_in[0, h])
        o, S = prefill_unit(f(inp.q[0, :T_len, h]), f(inp.k[0, :T_len, h]), f(inp.v[0, :T_len, h]),
                            f(inp.g[0, :T_len, h]), f(inp.beta[0, :T_len, h]), S0, **scheme)
        os_.append(o)
        ss.append(S)
    return np.stack(os_, 1), np.stack(ss, 0)
