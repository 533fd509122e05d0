"""The backward of the chunked (WY) form, written out in fp64 numpy (test code only).

This is the per-chunk adjoint a tensor-core backward evaluates: given the chunk's
start state S, the gradient dS' of its end state and dO of its outputs, it
returns the gradients of the chunk's q, k, v, g, beta and of S.  It is not the
oracle (oracle.backward differentiates the token recurrence by autograd); the
CPU test pins it to the oracle so that the algebra a kernel will follow is
known to be exact before it is written.

Forward, per chunk of L rows (G = cumsum(max(g, -5)), Gamma = exp(G), rows
indexed r, s, channels c):
    M[r,s]   = sum_c k_r k_s exp(G_r - G_s)   (s < r),    Akk = Diag(beta) M
    Aqk[r,s] = sum_c q_r k_s exp(G_r - G_s)   (s <= r)
    X = (I + Akk)^-1,  T = X Diag(beta)
    Ut = V - (K*Gamma) S,  U = T Ut,  O = (Q*Gamma) S + Aqk U
    S' = Diag(Gamma_L) S + (K*Gamma_L/Gamma)^T U
Backward:
    dU = Aqk^T dO + Khat dS',  dUt = T^T dU,  dV = dUt,  dT = dU Ut^T
    dAqk = tril(dO U^T),  dQt = dO S^T,  dKt = -dUt S^T,  dKhat = U dS'^T
    dbeta += colsum(X * dT);  dAkk = strict_tril(-X^T (dT Diag(beta)) X^T)
    dbeta += rowsum(dAkk * M);  dM = Diag(beta) dAkk
    a decayed form F[r,s] = sum_c a_r b_s exp(G_r - G_s) with upstream dF gives
    da_r = sum_s dF[r,s] b_s exp(G_r - G_s),  db_s = sum_r dF[r,s] a_r exp(G_r - G_s),
    dG_r += a_r da_r,  dG_s -= b_s db_s
    dq = dQt Gamma + da(Aqk);  dk = dKt Gamma + dKhat Gamma_L/Gamma + db(Aqk) + da(M) + db(M)
    dG_{L-1} += sum_r Khat_r dKhat_r + Gamma_L rowsum(dS' * S)
    dg = reverse cumsum of dG over the rows, zero where g < -5
    dS = Diag(Gamma_L) dS' + (Q*Gamma)^T dO - (K*Gamma)^T dUt
"""
from __future__ import annotations

import numpy as np


def chunk_forward(q, k, v, g, beta, S):
    L = q.shape[0]
    G = np.cumsum(np.maximum(g, -5.0), 0)
    gam = np.exp(G)
    gam_l = np.exp(G[L - 1])
    E = np.exp(G[:, None, :] - G[None, :, :])
    M = np.tril(np.einsum("rc,sc,rsc->rs", k, k, E), -1)
    Aqk = np.tril(np.einsum("rc,sc,rsc->rs", q, k, E))
    X = np.linalg.inv(np.eye(L) + beta[:, None] * M)
    T = X * beta[None, :]
    Kt, Qt, Kh = k * gam, q * gam, k * np.exp(G[L - 1][None, :] - G)
    Ut = v - Kt @ S
    U = T @ Ut
    return dict(gam=gam, gam_l=gam_l, E=E, M=M, Aqk=Aqk, X=X, T=T, Kt=Kt, Qt=Qt, Kh=Kh, Ut=Ut,
                U=U, O=Qt @ S + Aqk @ U, S_end=gam_l[:, None] * S + Kh.T @ U)


def chunk_backward(q, k, v, g, beta, S, dO, dS_end, f):
    L = q.shape[0]
    E, gam, gam_l = f["E"], f["gam"], f["gam_l"]
    dU = f["Aqk"].T @ dO + f["Kh"] @ dS_end
    dUt = f["T"].T @ dU
    dT = dU @ f["Ut"].T
    dAqk = np.tril(dO @ f["U"].T)
    dQt, dKt, dKh = dO @ S.T, -dUt @ S.T, f["U"] @ dS_end.T
    dbeta = np.sum(f["X"] * dT, axis=0)
    dAkk = np.tril(-f["X"].T @ (dT * beta[None, :]) @ f["X"].T, -1)
    dbeta = dbeta + np.sum(dAkk * f["M"], axis=1)
    dM = beta[:, None] * dAkk

    def decayed(a, b, dF):
        return (np.einsum("rs,sc,rsc->rc", dF, b, E), np.einsum("rs,rc,rsc->sc", dF, a, E))

    da_q, db_qk = decayed(q, k, dAqk)
    da_k, db_kk = decayed(k, k, dM)
    dq = dQt * gam + da_q
    dk = dKt * gam + dKh * (gam_l[None, :] / gam) + db_qk + da_k + db_kk
    dG = (f["Qt"] * dQt + f["Kt"] * dKt - f["Kh"] * dKh + q * da_q - k * db_qk + k * da_k
          - k * db_kk)
    dG[L - 1] += np.sum(f["Kh"] * dKh, axis=0) + gam_l * np.sum(dS_end * S, axis=1)
    dg = np.cumsum(dG[::-1], axis=0)[::-1] * (g >= -5.0)
    dS = gam_l[:, None] * dS_end + f["Qt"].T @ dO - f["Kt"].T @ dUt
    return dq, dk, dUt, dg, dbeta, dS


def backward(q, k, v, g, beta, S0, dout, dS_final, C=64):
    """One (sequence, head): q, k, g [T, dk]; v, dout [T, dv]; beta [T]; S0, dS_final
    [dk, dv].  Forward chunk by chunk keeping each chunk's start state, then the
    chunks in reverse.  Returns (dq, dk, dv, dg, dbeta, dS0)."""
    T_len = q.shape[0]
    starts = list(range(0, T_len, C))
    states, fwd = [np.array(S0, np.float64)], []
    for t0 in starts:
        sl = slice(t0, min(T_len, t0 + C))
        f = chunk_forward(q[sl], k[sl], v[sl], g[sl], beta[sl], states[-1])
        fwd.append(f)
        states.append(f["S_end"])
    grads = [np.zeros_like(x, dtype=np.float64) for x in (q, k, v, g, beta)]
    dS = np.array(dS_final, np.float64)
    for ci in reversed(range(len(starts))):
        sl = slice(starts[ci], min(T_len, starts[ci] + C))
        *gr, dS = chunk_backward(q[sl], k[sl], v[sl], g[sl], beta[sl], states[ci], dout[sl], dS,
                                 fwd[ci])
        for acc, x in zip(grads, gr):
            acc[sl] = x
    return (*grads, dS)


# ---------------------------------------------------------------- the WY-slot form
# The same adjoint split the way a chunk-parallel implementation on top of the
# forward's workspace would run it: the chunk-to-chunk chain needs only the
# forward's per-chunk factors (T, R, W, P, Khat, Gamma_L), and the gradients of
# those factors are then pulled back to q, k, g, beta without the state.

def wy_factors(q, k, g, beta):
    L = q.shape[0]
    G = np.cumsum(np.maximum(g, -5.0), 0)
    gam = np.exp(G)
    E = np.exp(G[:, None, :] - G[None, :, :])
    M = np.tril(np.einsum("rc,sc,rsc->rs", k, k, E), -1)
    Aqk = np.tril(np.einsum("rc,sc,rsc->rs", q, k, E))
    X = np.linalg.inv(np.eye(L) + beta[:, None] * M)
    T = X * beta[None, :]
    Kt, Qt = k * gam, q * gam
    R = Aqk @ T
    return dict(gam=gam, gam_l=np.exp(G[L - 1]), E=E, M=M, Aqk=Aqk, X=X, T=T, Kt=Kt, Qt=Qt,
                Kh=k * np.exp(G[L - 1][None, :] - G), R=R, W=T @ Kt, P=Qt - R @ Kt)


def wy_state_part(f, v, S, dO, dS_end):
    """The chain step and the factor gradients: only f's T, R, W, P, Khat, Gamma_L,
    the chunk's V, its start state S, dO and dS' are used."""
    U = f["T"] @ v - f["W"] @ S
    dU = f["Kh"] @ dS_end
    dS = f["gam_l"][:, None] * dS_end + f["P"].T @ dO - f["W"].T @ dU
    dV = f["T"].T @ dU + f["R"].T @ dO
    grads = dict(dT=dU @ v.T, dR=dO @ v.T, dW=-dU @ S.T, dP=dO @ S.T, dKh=U @ dS_end.T,
                 dGl=np.sum(dS_end * S, axis=1))
    return dS, dV, grads


def wy_input_part(q, k, g, beta, f, gr, upper=None):
    """Pull the factor gradients back to q, k, g, beta (no state involved).
    upper(shape), when given, is added to the strictly upper triangles of dR' and
    dT' as they are formed: no output may depend on those entries."""
    L = q.shape[0]
    E, gam, gam_l = f["E"], f["gam"], f["gam_l"]
    dP = gr["dP"]
    dR = gr["dR"] - dP @ f["Kt"].T
    if upper is not None:
        dR = dR + np.triu(upper(dR.shape), 1)
    dKt = f["T"].T @ gr["dW"] - f["R"].T @ dP
    dT = gr["dT"] + f["Aqk"].T @ dR + gr["dW"] @ f["Kt"].T
    if upper is not None:
        dT = dT + np.triu(upper(dT.shape), 1)
    dAqk = np.tril(dR @ f["T"].T)
    dbeta = np.sum(f["X"] * dT, axis=0)
    dAkk = np.tril(-f["X"].T @ (dT * beta[None, :]) @ f["X"].T, -1)
    dbeta = dbeta + np.sum(dAkk * f["M"], axis=1)
    dM = beta[:, None] * dAkk

    def decayed(a, b, dF):
        return (np.einsum("rs,sc,rsc->rc", dF, b, E), np.einsum("rs,rc,rsc->sc", dF, a, E))

    da_q, db_qk = decayed(q, k, dAqk)
    da_k, db_kk = decayed(k, k, dM)
    dKh = gr["dKh"]
    dq = dP * gam + da_q
    dk = dKt * gam + dKh * (gam_l[None, :] / gam) + db_qk + da_k + db_kk
    dG = (f["Qt"] * dP + f["Kt"] * dKt - f["Kh"] * dKh + q * da_q - k * db_qk + k * da_k
          - k * db_kk)
    dG[L - 1] += np.sum(f["Kh"] * dKh, axis=0) + gam_l * gr["dGl"]
    dg = np.cumsum(dG[::-1], axis=0)[::-1] * (g >= -5.0)
    return dq, dk, dg, dbeta


def wy_backward(q, k, v, g, beta, S0, dout, dS_final, C=64, upper=None):
    """As backward(), through the WY-slot split (upper: see wy_input_part)."""
    T_len = q.shape[0]
    starts = list(range(0, T_len, C))
    states, facs = [np.array(S0, np.float64)], []
    for t0 in starts:
        sl = slice(t0, min(T_len, t0 + C))
        f = wy_factors(q[sl], k[sl], g[sl], beta[sl])
        facs.append(f)
        U = f["T"] @ v[sl] - f["W"] @ states[-1]
        states.append(f["gam_l"][:, None] * states[-1] + f["Kh"].T @ U)
    dq, dk, dv, dg, db = (np.zeros_like(x, dtype=np.float64) for x in (q, k, v, g, beta))
    dS = np.array(dS_final, np.float64)
    for ci in reversed(range(len(starts))):
        sl = slice(starts[ci], min(T_len, starts[ci] + C))
        dS_prev, dv[sl], gr = wy_state_part(facs[ci], v[sl], states[ci], dout[sl], dS)
        dq[sl], dk[sl], dg[sl], db[sl] = wy_input_part(q[sl], k[sl], g[sl], beta[sl], facs[ci], gr, upper)
        dS = dS_prev
    return dq, dk, dv, dg, db, dS

