"""Chunked backward pass of the gated delta rule — TEST INFRASTRUCTURE ONLY.

The same gradients as oracle/backward.py, but derived through the chunked (WY / UT)
re-association of "論文解説: Qwen3.8-Next の設計", section "GDNの中身", Eq. (1), chunk by chunk
in reverse.  It is the reference a chunked tensor-core backward is checked against, step
by step: every intermediate below (dU, dW, dT, dA, dG) is a quantity such a kernel forms.

Per chunk of L tokens with incoming state S0 (the forward, as in the chunked oracle):
    G_i = sum_{m<=i} g_m,  gam_i = exp(G_i),  M_ij = exp(G_i - G_j) for j <= i
    A = strictly lower (beta_i M_ij k_i.k_j),  T = (I + A)^-1
    Kb = diag(beta gam) K,  Vb = diag(beta) V,  W = T Kb,  Ut = T Vb,  U = Ut - W S0
    P = lower incl. diagonal (M_ij q_i.k_j)
    O = scale (diag(gam) Q S0 + P U)
    Kd = diag(exp(G_{L-1} - G_j)) K,  S1 = gam_{L-1} S0 + Kd^T U
Reverse, given dO and dS1 (the gradient of the state after the chunk), with dO' = scale dO:
    dU  = P^T dO' + Kd dS1
    dS0 = (diag(gam) Q)^T dO' + gam_{L-1} dS1 - W^T dU
    dP  = lower(dO' U^T);   dKd = U dS1^T;   d(gam_i) from O: dO'_i . (S0^T q_i)
    dW  = -dU S0^T;  dUt = dU;  dT = dW Kb^T + dUt Vb^T;  dKb = T^T dW;  dVb = T^T dUt
    dA  = strictly lower(-T^T dT T^T)
then the products P, A, Kb, Vb, Kd and the decays gam, M pass their gradients to q, k, v,
beta and G, and dg is the reverse cumulative sum of dG inside the chunk.  Plain numpy in
fp64; pinned against oracle/backward.py (itself pinned by finite differences) in
tests/test_oracle_backward_chunked.py.
"""
from __future__ import annotations

import numpy as np

from .backward import _f64


def _chunk_forward(q, k, v, g, beta, S0):
    L = q.shape[0]
    G = np.cumsum(g)
    gam = np.exp(G)
    idx = np.arange(L)
    low_incl = idx[:, None] >= idx[None, :]
    low_strict = idx[:, None] > idx[None, :]
    M = np.where(low_incl, np.exp(G[:, None] - G[None, :]), 0.0)
    KK = k @ k.T
    A = np.where(low_strict, beta[:, None] * M * KK, 0.0)
    T = np.linalg.inv(np.eye(L) + A)
    Kb = (beta * gam)[:, None] * k
    Vb = beta[:, None] * v
    W = T @ Kb
    Ut = T @ Vb
    U = Ut - W @ S0
    QK = q @ k.T
    P = np.where(low_incl, M * QK, 0.0)
    dec = np.exp(G[-1] - G)
    Kd = dec[:, None] * k
    S1 = gam[-1] * S0 + Kd.T @ U
    return dict(G=G, gam=gam, M=M, KK=KK, A=A, T=T, Kb=Kb, Vb=Vb, W=W, U=U, QK=QK, P=P,
                dec=dec, Kd=Kd, S1=S1, low_incl=low_incl, low_strict=low_strict)


def _chunk_backward(q, k, v, g, beta, S0, dO, dS1, scale):
    f = _chunk_forward(q, k, v, g, beta, S0)
    gam, M, T, W, U, P = f["gam"], f["M"], f["T"], f["W"], f["U"], f["P"]
    Kb, Vb, Kd, dec = f["Kb"], f["Vb"], f["Kd"], f["dec"]
    dOs = scale * dO
    # O = diag(gam) Q S0 + P U;  S1 = gam_end S0 + Kd^T U
    dU = P.T @ dOs + Kd @ dS1
    dS0 = (gam[:, None] * q).T @ dOs + gam[-1] * dS1 - W.T @ dU
    dq = gam[:, None] * (dOs @ S0.T)
    dG = gam * np.einsum("id,id->i", dOs, (S0.T @ q.T).T)
    dG[-1] += gam[-1] * np.sum(dS1 * S0)
    # P_ij = M_ij q_i.k_j (j <= i)
    dP = np.where(f["low_incl"], dOs @ U.T, 0.0)
    dq += (dP * M) @ k
    dk = (dP * M).T @ q
    dM = dP * f["QK"]
    # Kd_j = dec_j k_j, dec_j = exp(G_end - G_j)
    dKd = U @ dS1.T
    dk += dec[:, None] * dKd
    ddec = dec * np.einsum("jd,jd->j", dKd, k)
    dG[-1] += ddec.sum()
    dG -= ddec
    # U = Ut - W S0;  W = T Kb;  Ut = T Vb
    dW = -dU @ S0.T
    dT = dW @ Kb.T + dU @ Vb.T
    dKb = T.T @ dW
    dVb = T.T @ dU
    # Kb_i = beta_i gam_i k_i;  Vb_i = beta_i v_i
    dk += (beta * gam)[:, None] * dKb
    kb_dot = np.einsum("id,id->i", dKb, k)
    dbeta = gam * kb_dot
    dG += beta * gam * kb_dot
    dv = beta[:, None] * dVb
    dbeta += np.einsum("id,id->i", dVb, v)
    # T = (I + A)^-1;  A_ij = beta_i M_ij k_i.k_j (j < i)
    dA = np.where(f["low_strict"], -T.T @ dT @ T.T, 0.0)
    dbeta += np.sum(dA * M * f["KK"], axis=1)
    dM += dA * beta[:, None] * f["KK"]
    dKK = dA * beta[:, None] * M
    dk += dKK @ k + dKK.T @ k
    # M_ij = exp(G_i - G_j)
    dMM = dM * M
    dG += dMM.sum(axis=1) - dMM.sum(axis=0)
    # G_i = sum_{m <= i} g_m
    dg = np.cumsum(dG[::-1])[::-1]
    return dq, dk, dv, dg, dbeta, dS0, f["S1"]


def backward_chunked(q, k, v, g, beta, S0, d_out, dS_final=None, cu_seqlens=None,
                     scale: float = 1.0, chunk: int = 64):
    """Same arguments and results as oracle.backward.backward, computed chunk by chunk."""
    q, k, v, g, beta, d_out = (_f64(x) for x in (q, k, v, g, beta, d_out))
    Ttot, H_qk, dk = q.shape
    H_v, dv = v.shape[1:]
    group = H_v // H_qk
    cu = (np.array([0, Ttot]) if cu_seqlens is None else
          np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = len(cu) - 1
    S0 = np.zeros((N, H_v, dk, dv)) if S0 is None else _f64(S0)
    dSf = np.zeros((N, H_v, dk, dv)) if dS_final is None else _f64(dS_final)
    dq = np.zeros((Ttot, H_qk, dk)); dkk = np.zeros((Ttot, H_qk, dk))
    dvv = np.zeros((Ttot, H_v, dv)); dg = np.zeros((Ttot, H_v)); db = np.zeros((Ttot, H_v))
    dS0 = np.zeros((N, H_v, dk, dv))
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        bounds = [(c, min(c + chunk, t1)) for c in range(t0, t1, chunk)]
        for h in range(H_v):
            hq = h // group
            # forward over the chunks: the state entering each chunk
            starts, S = [], S0[n, h].copy()
            for a, b in bounds:
                starts.append(S)
                S = _chunk_forward(q[a:b, hq], k[a:b, hq], v[a:b, h], g[a:b, h],
                                   beta[a:b, h], S)["S1"]
            # reverse over the chunks
            dS = dSf[n, h].copy()
            for (a, b), Sc in zip(reversed(bounds), reversed(starts)):
                r = _chunk_backward(q[a:b, hq], k[a:b, hq], v[a:b, h], g[a:b, h],
                                    beta[a:b, h], Sc, d_out[a:b, h], dS, scale)
                dq[a:b, hq] += r[0]; dkk[a:b, hq] += r[1]; dvv[a:b, h] = r[2]
                dg[a:b, h] = r[3]; db[a:b, h] = r[4]
                dS = r[5]
            dS0[n, h] = dS
    return dq, dkk, dvv, dg, db, dS0
