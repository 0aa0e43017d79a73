"""Sequence-parallel (segmented) form of the gated delta rule — TEST INFRASTRUCTURE ONLY.

Only tests/ may import this module.  It shares no code with the CUDA library.

What it computes.  Eq. (1) of "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section
"GDNの中身", makes every step affine in the state:

    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = scale S_t^T q_t.

So over a run of tokens (a segment) that starts from a state S_in,

    S_end = M S_in + B,        o_t = o_t^local + S_in^T psi_t,

where B and o^local are the run started from S_in = 0, M (dk x dk) is the run started
from S_in = I with every v_t = 0 (the product of the per-token factors
alpha_t (I - beta_t k_t k_t^T)), and psi_t (a dk-vector) is that same run's output at t:
from S_in = I the state at t is the transfer Phi_t, and scale Phi_t^T q_t = psi_t, so
scale (Phi_t S_in)^T q_t = S_in^T psi_t.  A sequence cut into segments is then the local
and transfer runs of every segment (independent of one another), the scan
S_in(p + 1) = M_p S_in(p) + B_p, and the output correction.  This is the decomposition the
library's long-sequence schedule computes; here every piece is a call of the pinned
token-by-token oracle, in fp64.
"""
from __future__ import annotations

import numpy as np

from . import recurrent


def segment_runs(q, k, v, g, beta, S_in, scale=1.0):
    """One segment of one sequence (q, k [T, H_qk, dk]; v [T, H_v, dv]; g, beta [T, H_v];
    S_in [H_v, dk, dv] or None for zero).  Returns (o_local, B, psi, M) with o_local
    [T, H_v, dv], B [H_v, dk, dv], psi [T, H_v, dk], M [H_v, dk, dk]."""
    T, H_qk, dk = q.shape
    H_v = v.shape[1]
    S0 = None if S_in is None else np.asarray(S_in, dtype=np.float64)[None]
    o_local, B = recurrent(q, k, v, g, beta, S0, None, scale=scale)
    eye = np.broadcast_to(np.eye(dk), (1, H_v, dk, dk)).copy()
    psi, M = recurrent(q, k, np.zeros((T, H_v, dk)), g, beta, eye, None, scale=scale)
    return o_local, B[0], psi, M[0]


def segmented(q, k, v, g, beta, S0=None, seg_tokens=64, scale=1.0):
    """The whole sequence (shapes as in segment_runs, S0 [H_v, dk, dv] or None) cut into
    segments of seg_tokens tokens.  Returns (out [T, H_v, dv], S_final [H_v, dk, dv])."""
    T = q.shape[0]
    H_v, dv = v.shape[1:]
    dk = q.shape[2]
    bounds = list(range(0, T, seg_tokens)) + [T]
    runs = []
    for p, (a, b) in enumerate(zip(bounds[:-1], bounds[1:])):
        # the first segment starts from S0 and is exact; the others start from zero
        runs.append(segment_runs(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b],
                                 S0 if p == 0 else None, scale))
    out = np.zeros((T, H_v, dv))
    S_in = np.zeros((H_v, dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    for p, (a, b) in enumerate(zip(bounds[:-1], bounds[1:])):
        o_local, B, psi, M = runs[p]
        if p == 0:
            out[a:b] = o_local
            S_in = B
            continue
        # o_t += S_in^T psi_t per value head; S_end = M S_in + B
        out[a:b] = o_local + np.einsum("hdv,thd->thv", S_in, psi)
        S_in = np.einsum("hde,hev->hdv", M, S_in) + B
    return out, S_in
