"""Backward pass of the gated delta rule — TEST INFRASTRUCTURE ONLY (see oracle/__init__).

The gradients of L with respect to the inputs and S0, given dL/do_t and dL/dS_final,
for the recurrence of "論文解説: Qwen3.8-Next の設計", section "GDNの中身", Eq. (1):

    alpha_t = exp(g_t),  a_t = S_{t-1}^T k_t,  u_t = beta_t (v_t - alpha_t a_t),
    S_t = alpha_t S_{t-1} + k_t u_t^T,   o_t = scale * S_t^T q_t.

Reverse-mode differentiation of those four lines, token by token from the last to the
first, with dS the gradient of the state after token t:

    dS    += scale * q_t do_t^T                 (o_t reads S_t)
    dq_t   = scale * S_t do_t
    du     = dS^T k_t                           (S_t = alpha S_{t-1} + k u^T)
    dk_t   = dS u_t
    dalpha = <dS, S_{t-1}>
    dbeta  = <du, v_t - alpha a_t>              (u = beta (v - alpha a))
    dv_t   = beta du
    da     = -alpha beta du
    dalpha += -beta <du, a_t>
    dk_t  += S_{t-1} da                         (a = S_{t-1}^T k)
    dS     = alpha dS + k_t da^T                (the gradient of S_{t-1})
    dg_t   = alpha * dalpha

and dS0 is dS after the first token.  Plain numpy in fp64, one (sequence, value head) at
a time; the states are recomputed forward first and kept.  q/k gradients of value heads
that share a q/k head are summed.  Pinned by central finite differences of the forward
oracle (tests/test_oracle.py).
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def backward(q, k, v, g, beta, S0, d_out, dS_final=None, cu_seqlens=None, scale: float = 1.0):
    """q,k [T,H_qk,dk]; v, d_out [T,H_v,dv]; g, beta [T,H_v]; S0, dS_final [N,H_v,dk,dv] or None.

    Returns dq, dk [T,H_qk,dk], dv [T,H_v,dv], dg, dbeta [T,H_v], dS0 [N,H_v,dk,dv] (fp64).
    """
    q, k, v, g, beta, d_out = (_f64(x) for x in (q, k, v, g, beta, d_out))
    T, H_qk, dk = q.shape
    H_v, dv = v.shape[1:]
    group = H_v // H_qk
    cu = (np.array([0, T]) if cu_seqlens is None else
          np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = len(cu) - 1
    S0 = np.zeros((N, H_v, dk, dv)) if S0 is None else _f64(S0)
    dSf = np.zeros((N, H_v, dk, dv)) if dS_final is None else _f64(dS_final)
    dq = np.zeros((T, H_qk, dk)); dkk = np.zeros((T, H_qk, dk)); dvv = np.zeros((T, H_v, dv))
    dg = np.zeros((T, H_v)); db = np.zeros((T, H_v)); dS0 = np.zeros((N, H_v, dk, dv))
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        for h in range(H_v):
            hq = h // group
            # forward: the states before and after every token
            S = S0[n, h].copy()
            states, avec, uvec = [S.copy()], [], []
            for t in range(t0, t1):
                al = np.exp(g[t, h])
                a = S.T @ k[t, hq]
                u = beta[t, h] * (v[t, h] - al * a)
                S = al * S + np.outer(k[t, hq], u)
                states.append(S.copy()); avec.append(a); uvec.append(u)
            # reverse
            dS = dSf[n, h].copy()
            for i in range(t1 - t0 - 1, -1, -1):
                t = t0 + i
                al, bt = np.exp(g[t, h]), beta[t, h]
                S_t, S_p, a, u = states[i + 1], states[i], avec[i], uvec[i]
                kt, qt = k[t, hq], q[t, hq]
                dS = dS + scale * np.outer(qt, d_out[t, h])
                dq[t, hq] += scale * S_t @ d_out[t, h]
                du = dS.T @ kt
                dk_t = dS @ u
                dal = np.sum(dS * S_p)
                db[t, h] = du @ (v[t, h] - al * a)
                dvv[t, h] = bt * du
                da = -al * bt * du
                dal += -bt * (du @ a)
                dk_t = dk_t + S_p @ da
                dkk[t, hq] += dk_t
                dS = al * dS + np.outer(kt, da)
                dg[t, h] = al * dal
            dS0[n, h] = dS
    return dq, dkk, dvv, dg, db, dS0
