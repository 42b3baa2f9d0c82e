"""Chunkwise restatement of KDA in fp64 -- TEST INFRASTRUCTURE ONLY.

This is a second, independent evaluation of the same operator that follows
the chunk algorithm named on "Kimi Linear ... 深度解读报告" (zako-mio knowledge
base), section 3.1 "DPLR 特化：硬件高效 chunkwise 算法": with both low-rank
vectors of the DPLR transition bound to k, a chunk needs only two C x C
matrices (one from K K^T, one from Q K^T), and the rest follows from a WY
representation, a UT transform and a forward-substitution triangular inverse.
The pages print no chunk formulas; the ones below are derived from the token
recurrence

    S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = scale * S_t^T q_t.

For a chunk of L tokens with entry state S0 and G_r = sum_{i<=r} g_i:

    Kt = K * e^G,  Kh = K * e^-G,  Qt = Q * e^G,  Kend = K * e^(G_L - G)
    A  = strict_lower(Diag(beta) Kt Kh^T)           (decayed beta K K^T)
    T  = (I + A)^-1 Diag(beta)                      (forward substitution)
    W  = T Kt,  U' = T V                            (WY / UT transform)
    P  = lower_incl(Qt Kh^T)                        (decayed Q K^T)
    U  = U' - W S0
    O  = scale * (Qt S0 + P U)
    S_L = Diag(e^{G_L}) S0 + Kend^T U

Derivation: unrolling the recurrence inside the chunk gives
(I + A) U = Diag(beta) (V - Kt S0) for the rows u_r = beta_r (v_r - S_bar_r^T k_r),
and the state/output are sums of decayed rank-one terms k_i u_i^T.  With C = 1
this reduces to the token form.  Nothing here is blocked or fused beyond what
these formulas state; every matrix is formed explicitly.
"""
from __future__ import annotations

import numpy as np


def forward_substitution(A: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """T = (I + A)^-1 Diag(beta) for strictly lower-triangular A, one row at a
    time: T_r = beta_r e_r - sum_{i<r} A_{r,i} T_i."""
    L = A.shape[0]
    T = np.zeros((L, L), dtype=np.float64)
    for r in range(L):
        row = np.zeros(L, dtype=np.float64)
        row[r] = beta[r]
        for i in range(r):
            row -= A[r, i] * T[i]
        T[r] = row
    return T


def chunk_step(q, k, v, g, beta, S0, scale):
    """One chunk (L tokens) of one head.  q, k, g: [L, dk]; v: [L, dv];
    beta: [L]; S0: [dk, dv].  Returns a dict with the output O [L, dv], the
    exit state S [dk, dv] and every intermediate of the algorithm."""
    q, k, v, g, beta, S0 = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta, S0))
    L = q.shape[0]
    G = np.cumsum(g, axis=0)
    eG, emG = np.exp(G), np.exp(-G)
    Kt, Kh, Qt = k * eG, k * emG, q * eG
    Kend = k * np.exp(G[L - 1][None, :] - G)
    A = np.tril(beta[:, None] * (Kt @ Kh.T), -1)
    T = forward_substitution(A, beta)
    W = T @ Kt
    Up = T @ v
    P = np.tril(Qt @ Kh.T)
    U = Up - W @ S0
    O = scale * (Qt @ S0 + P @ U)
    S = np.exp(G[L - 1])[:, None] * S0 + Kend.T @ U
    return dict(G=G, Kt=Kt, Kh=Kh, Qt=Qt, Kend=Kend, A=A, T=T, W=W, Up=Up,
                P=P, U=U, O=O, S=S)


def chunked_forward(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
                    scale=None, chunk: int = 64):
    """Chunkwise fp64 KDA forward with the same interface and layouts as
    ``oracle.kda_forward``: chunks restart at every sequence start; the last
    chunk of a sequence may be partial; a zero-length sequence passes its
    state through."""
    from . import _f64
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    if cu_seqlens is None:
        bounds = [(n * T, (n + 1) * T) for n in range(B)]
    else:
        cu = np.asarray(cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                        dtype=np.int64)
        bounds = [(int(cu[n]), int(cu[n + 1])) for n in range(cu.shape[0] - 1)]
    N = len(bounds)
    s0 = _f64(initial_state)
    qf, kf, vf, gf = (x.reshape(B * T, H, -1) for x in (q, k, v, g))
    bf = b.reshape(B * T, H)
    out = np.zeros((B * T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    for n, (t0, t1) in enumerate(bounds):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else s0[n, h].copy()
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                r = chunk_step(qf[c0:c1, h], kf[c0:c1, h], vf[c0:c1, h], gf[c0:c1, h],
                               bf[c0:c1, h], S, scale)
                out[c0:c1, h] = r["O"]
                S = r["S"]
            fs[n, h] = S
    return out.reshape(B, T, H, dv), fs


# ---------------------------------------------------------------- backward
#
# The adjoint of chunk_step, for training with the operator ("深度解读报告"
# 3.4: the layer is trained end to end).  Given dO (adjoint of the chunk's output) and dS (adjoint of its exit
# state S_L), each line of chunk_step is differentiated in reverse order:
#
#   O   = scale (Qt S0 + P U)     dQt = scale dO S0^T ; dS0 += scale Qt^T dO
#                                 dP = lower_incl(scale dO U^T) ; dU = scale P^T dO
#   S_L = Diag(Gam) S0 + Kend^T U dS0 += Diag(Gam) dS ; dGam = rowsum(dS * S0)
#                                 dKend = U dS^T ; dU += Kend dS
#   U   = T R, R = V - Kt S0      dT = dU R^T ; dR = T^T dU ; dV = dR
#                                 dKt = -dR S0^T ; dS0 -= Kt^T dR
#   T   = M Diag(beta)            dM = dT Diag(beta) ; dbeta_i = sum_r dT_ri M_ri
#   M   = (I + A)^-1              dA = strict_lower(-M^T dM M^T)
#   A   = strict_lower(Diag(beta) Kt Kh^T)
#                                 dbeta_r += sum_i dA_ri (Kt Kh^T)_ri
#                                 dKt += Diag(beta) dA Kh ; dKh = (Diag(beta) dA)^T Kt
#   P   = lower_incl(Qt Kh^T)     dQt += dP Kh ; dKh += dP^T Qt
#
# and through the decay factors of Kt, Kh, Qt, Kend, Gam (all functions of
# G = cumsum(g)), dg = the reverse cumulative sum of dG.  Every matrix is
# formed explicitly; M is the explicit inverse of I + A.

def chunk_step_backward(q, k, v, g, beta, S0, scale, dO, dS):
    """Adjoint of ``chunk_step``: returns (dq, dk, dv, dg, dbeta, dS0)."""
    q, k, v, g, beta, S0, dO, dS = (np.asarray(x, dtype=np.float64)
                                    for x in (q, k, v, g, beta, S0, dO, dS))
    L = q.shape[0]
    G = np.cumsum(g, axis=0)
    eG, emG = np.exp(G), np.exp(-G)
    Kt, Kh, Qt = k * eG, k * emG, q * eG
    Eend = np.exp(G[L - 1][None, :] - G)
    Kend = k * Eend
    Gam = np.exp(G[L - 1])
    KK = Kt @ Kh.T
    A = np.tril(beta[:, None] * KK, -1)
    M = np.linalg.inv(np.eye(L) + A)
    T = M * beta[None, :]
    P = np.tril(Qt @ Kh.T)
    R = v - Kt @ S0
    U = T @ R
    # output
    dQt = scale * dO @ S0.T
    dS0 = scale * Qt.T @ dO
    dP = np.tril(scale * dO @ U.T)
    dU = scale * P.T @ dO
    # exit state
    dS0 = dS0 + Gam[:, None] * dS
    dGam = np.sum(dS * S0, axis=1)
    dKend = U @ dS.T
    dU = dU + Kend @ dS
    # U = T R, R = V - Kt S0
    dT = dU @ R.T
    dR = T.T @ dU
    dv = dR
    dKt = -dR @ S0.T
    dS0 = dS0 - Kt.T @ dR
    # T = M Diag(beta), M = (I + A)^-1
    dM = dT * beta[None, :]
    dbeta = np.sum(dT * M, axis=0)
    dA = np.tril(-M.T @ dM @ M.T, -1)
    # A = strict_lower(Diag(beta) Kt Kh^T)
    dbeta = dbeta + np.sum(dA * KK, axis=1)
    dB = beta[:, None] * dA
    dKt = dKt + dB @ Kh
    dKh = dB.T @ Kt
    # P = lower_incl(Qt Kh^T)
    dQt = dQt + dP @ Kh
    dKh = dKh + dP.T @ Qt
    # the decay factors
    dq = dQt * eG
    dk = dKt * eG + dKh * emG + dKend * Eend
    dG = dQt * Qt + dKt * Kt - dKh * Kh - dKend * Kend
    dG[L - 1] += np.sum(dKend * Kend, axis=0) + dGam * Gam
    dg = np.cumsum(dG[::-1], axis=0)[::-1]
    return dq, dk, dv, dg, dbeta, dS0


def chunked_backward(q, k, v, log_alpha, beta, d_out, initial_state=None, d_final_state=None,
                     cu_seqlens=None, scale=None, chunk: int = 64):
    """Chunkwise fp64 backward with the interface of ``oracle.kda_backward``:
    the forward chunk by chunk keeping every entry state, then the chunks in
    reverse carrying the state adjoint."""
    from . import _f64
    q, k, v, g, b, do = (_f64(x) for x in (q, k, v, log_alpha, beta, d_out))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if scale is None:
        scale = dk ** -0.5
    if cu_seqlens is None:
        bounds = [(n * T, (n + 1) * T) for n in range(B)]
    else:
        cu = np.asarray(cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                        dtype=np.int64)
        bounds = [(int(cu[n]), int(cu[n + 1])) for n in range(cu.shape[0] - 1)]
    N = len(bounds)
    s0 = _f64(initial_state)
    dfs = _f64(d_final_state)
    flat = [x.reshape(B * T, H, -1) for x in (q, k, v, g, do)]
    qf, kf, vf, gf, dof = flat
    bf = b.reshape(B * T, H)
    grads = [np.zeros_like(x) for x in (qf, kf, vf, gf)]
    dbeta = np.zeros((B * T, H), dtype=np.float64)
    ds0 = np.zeros((N, H, dk, dv), dtype=np.float64)
    for n, (t0, t1) in enumerate(bounds):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else s0[n, h].copy()
            starts, entry = list(range(t0, t1, chunk)), []
            for c0 in starts:
                c1 = min(c0 + chunk, t1)
                entry.append(S)
                S = chunk_step(qf[c0:c1, h], kf[c0:c1, h], vf[c0:c1, h], gf[c0:c1, h],
                               bf[c0:c1, h], S, scale)["S"]
            dS = np.zeros((dk, dv)) if dfs is None else dfs[n, h].copy()
            for c0, S0 in zip(starts[::-1], entry[::-1]):
                c1 = min(c0 + chunk, t1)
                r = chunk_step_backward(qf[c0:c1, h], kf[c0:c1, h], vf[c0:c1, h], gf[c0:c1, h],
                                        bf[c0:c1, h], S0, scale, dof[c0:c1, h], dS)
                for gr, part in zip(grads, r[:4]):
                    gr[c0:c1, h] = part
                dbeta[c0:c1, h] = r[4]
                dS = r[5]
            ds0[n, h] = dS
    shapes = [(B, T, H, dk), (B, T, H, dk), (B, T, H, dv), (B, T, H, dk)]
    dq, dkk, dvv, dg = (x.reshape(s) for x, s in zip(grads, shapes))
    return dq, dkk, dvv, dg, dbeta.reshape(B, T, H), ds0
