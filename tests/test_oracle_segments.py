"""The segmented form of the recurrence (oracle/segments.py) against the sequential oracle.

Cutting a sequence into segments is exact (Eq. (1) of "論文解説: Qwen3.8-Next の設計",
section "GDNの中身", is affine in the state), so outputs and the final state must equal the
token-by-token run up to fp64 rounding, for any segment length, with ragged tails, grouped
heads, an initial state, strong decay and a read-out scale.  Planted mistakes in the
composition each break that equality."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import segments


def _draw(T, H_qk, H_v, dk, dv, seed, g_mult=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H_qk, dk))
    k = rng.standard_normal((T, H_qk, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H_v, dv))
    g = -g_mult * np.log1p(np.exp(rng.standard_normal((T, H_v))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H_v))))
    S0 = 0.3 * rng.standard_normal((H_v, dk, dv))
    return q, k, v, g, beta, S0


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


@pytest.mark.parametrize("seg", [1, 5, 16, 37, 64])
@pytest.mark.parametrize("with_s0", [False, True])
def test_segmented_equals_sequential(seg, with_s0):
    q, k, v, g, beta, S0 = _draw(150, 2, 4, 6, 5, 7 + seg)
    S0 = S0 if with_s0 else None
    ref_o, ref_S = oracle.recurrent(q, k, v, g, beta, None if S0 is None else S0[None],
                                    scale=0.7)
    o, S = segments.segmented(q, k, v, g, beta, S0, seg, scale=0.7)
    assert _rel(o, ref_o) < 1e-11
    assert _rel(S, ref_S[0]) < 1e-11


def test_segmented_strong_decay():
    q, k, v, g, beta, S0 = _draw(200, 1, 2, 8, 8, 3, g_mult=3.0)
    ref_o, ref_S = oracle.recurrent(q, k, v, g, beta, S0[None])
    o, S = segments.segmented(q, k, v, g, beta, S0, 48)
    assert _rel(o, ref_o) < 1e-11 and _rel(S, ref_S[0]) < 1e-11


def test_transfer_is_product_of_step_factors():
    """M of one segment equals the product of alpha_t (I - beta_t k_t k_t^T), formed here
    by explicit matrix products (a route that does not run the recurrence)."""
    q, k, v, g, beta, _ = _draw(12, 1, 1, 4, 3, 11)
    _, _, _, M = segments.segment_runs(q, k, v, g, beta, None)
    P = np.eye(4)
    for t in range(12):
        kt = k[t, 0]
        P = np.exp(g[t, 0]) * (np.eye(4) - beta[t, 0] * np.outer(kt, kt)) @ P
    assert _rel(M[0], P) < 1e-13


def _mutant_composition(q, k, v, g, beta, S0, seg, which):
    """A copy of segments.segmented with one planted mistake."""
    T = q.shape[0]
    H_v, dv = v.shape[1:]
    bounds = list(range(0, T, seg)) + [T]
    out = np.zeros((T, H_v, dv))
    S_in = S0
    for p, (a, b) in enumerate(zip(bounds[:-1], bounds[1:])):
        start = S0 if (p == 0 and which != "drop_s0") else None
        o_local, B, psi, M = segments.segment_runs(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], start)
        if p == 0:
            out[a:b] = o_local
            S_in = B
            continue
        if which == "no_correction":
            out[a:b] = o_local
        elif which == "psi_transposed_use":      # S_in psi in place of S_in^T psi (dk = dv)
            out[a:b] = o_local + np.einsum("hvd,thd->thv", S_in, psi)
        else:
            out[a:b] = o_local + np.einsum("hdv,thd->thv", S_in, psi)
        if which == "M_transposed":
            S_in = np.einsum("hed,hev->hdv", M, S_in) + B
        elif which == "B_dropped":
            S_in = np.einsum("hde,hev->hdv", M, S_in)
        else:
            S_in = np.einsum("hde,hev->hdv", M, S_in) + B
    return out, S_in


@pytest.mark.parametrize("which", ["drop_s0", "no_correction", "psi_transposed_use",
                                   "M_transposed", "B_dropped"])
def test_planted_mistakes_break_equality(which):
    # slow decay, so the transfer of a 40-token segment is far from zero
    q, k, v, g, beta, S0 = _draw(120, 2, 2, 5, 5, 19, g_mult=0.01)
    ref_o, ref_S = oracle.recurrent(q, k, v, g, beta, S0[None])
    o, S = _mutant_composition(q, k, v, g, beta, S0, 40, which)
    assert max(_rel(o, ref_o), _rel(S, ref_S[0])) > 1e-3
