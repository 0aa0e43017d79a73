"""Exact rational brute force for the gated delta rule, independent of the oracle.

Two formulations of "論文解説: Qwen3.8-Next の設計", section "GDNの中身", Eq. (1),
both in exact ``fractions.Fraction`` arithmetic on tiny inputs:

* ``step_matrices``: build the dk x dk matrix M_t = alpha_t (I - beta_t k_t k_t^T)
  explicitly and apply S_t = M_t S_{t-1} + beta_t k_t v_t^T;
* ``unrolled``: the closed form obtained by unrolling Eq. (1),
      S_T = (M_T ... M_1) S_0 + sum_j (M_T ... M_{j+1}) beta_j k_j v_j^T.

The output is read after the update, o_t = scale * S_t^T q_t (the one-token
concept code in the same section).  Neither function shares code with oracle/.
"""
from __future__ import annotations

from fractions import Fraction as F


def _eye(n):
    return [[F(int(i == j)) for j in range(n)] for i in range(n)]


def _matmul(A, B):
    return [[sum((A[i][m] * B[m][j] for m in range(len(B))), F(0)) for j in range(len(B[0]))]
            for i in range(len(A))]


def _add(A, B):
    return [[A[i][j] + B[i][j] for j in range(len(A[0]))] for i in range(len(A))]


def _outer(x, y, c=F(1)):
    return [[c * xi * yj for yj in y] for xi in x]


def _M(alpha, beta, k):
    n = len(k)
    I = _eye(n)
    kk = _outer(k, k, beta)
    return [[alpha * (I[i][j] - kk[i][j]) for j in range(n)] for i in range(n)]


def _readout(S, q, scale):
    dv = len(S[0])
    return [scale * sum((S[i][j] * q[i] for i in range(len(q))), F(0)) for j in range(dv)]


def step_matrices(q, k, v, alpha, beta, S0, scale=F(1)):
    """Returns ([o_1..o_T], [S_1..S_T]) for one head; all arguments are Fractions."""
    S = [row[:] for row in S0]
    outs, states = [], []
    for t in range(len(k)):
        S = _add(_matmul(_M(alpha[t], beta[t], k[t]), S), _outer(k[t], v[t], beta[t]))
        states.append(S)
        outs.append(_readout(S, q[t], scale))
    return outs, states


def unrolled(k, v, alpha, beta, S0):
    """S_T by the unrolled closed form of Eq. (1)."""
    T = len(k)
    dk = len(S0)
    Ms = [_M(alpha[t], beta[t], k[t]) for t in range(T)]

    def prod(lo, hi):            # M_hi ... M_lo (1-based, inclusive), identity if empty
        P = _eye(dk)
        for t in range(lo, hi + 1):
            P = _matmul(Ms[t - 1], P)
        return P

    S = _matmul(prod(1, T), S0)
    for j in range(1, T + 1):
        S = _add(S, _matmul(prod(j + 1, T), _outer(k[j - 1], v[j - 1], beta[j - 1])))
    return S
