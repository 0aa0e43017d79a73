"""Pins for the CPU oracle, each against something other than the oracle itself.

Rule under test: "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "GDNの中身",
Eq. (1) S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, the ranges
alpha, beta in (0, 1) stated under it, and the concept code's read-out after the
update (o_t = S_t^T q_t).  Pins used:
  * a hand-worked example (tests/golden/handworked_dk2_dv2_t2.txt);
  * exact rational brute force with explicit dk x dk step matrices, and the
    unrolled closed form (tests/brute.py);
  * closed forms: beta = 0 (pure decay, one numpy matmul per token); alpha = beta = 1
    with unit keys (S_t^T k_t = v_t); orthonormal keys (S = sum k_j v_j^T);
  * invariants: zero in -> zero out, reset by alpha -> 0, the Frobenius-norm bound,
    scale linearity, GVA == repeated heads, varlen == separate runs, split runs;
  * the chunked re-association equals the sequential form for C in {1, 16, 64}.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction as F

import numpy as np
import pytest

import brute
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel_err(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.max(np.abs(ref))
    num = np.max(np.abs(x - ref)) if x.size else 0.0
    return num / den if den > 0 else num


def rand_case(rng, T, H_qk, H_v, dk, dv, unit_k=True, s0=True, N=None, lens=None):
    if lens is None:
        lens = [T] if N is None else list(rng.integers(0, T + 1, size=N))
    Tt = int(sum(lens))
    q = rng.standard_normal((Tt, H_qk, dk))
    k = rng.standard_normal((Tt, H_qk, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((Tt, H_v, dv))
    g = -np.log1p(np.exp(rng.standard_normal((Tt, H_v))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((Tt, H_v))))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    S0 = rng.standard_normal((len(lens), H_v, dk, dv)) * 0.3 if s0 else None
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0, cu_seqlens=cu)


# --------------------------------------------------------------------------- golden
def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(":", 1)
            rows = [r.split() for r in rest.split(";")]
            vals[key.strip()] = [[F(x) for x in r] for r in rows]
    return vals


def test_golden_handworked_brute():
    G = _read_golden("handworked_dk2_dv2_t2.txt")
    k, v, q = G["k"], G["v"], G["q"]
    alpha, beta = G["alpha"][0], G["beta"][0]
    outs, states = brute.step_matrices(q, k, v, alpha, beta, [[F(0)] * 2 for _ in range(2)])
    flat = lambda S: [x for r in S for x in r]
    assert flat(states[0]) == G["S_1"][0]
    assert outs[0] == G["o_1"][0]
    assert flat(states[1]) == G["S_2"][0]
    assert outs[1] == G["o_2"][0]


@pytest.mark.parametrize("precision,tol", [("f64", 1e-14), ("f32", 2e-6)])
def test_golden_handworked_oracle(precision, tol):
    G = _read_golden("handworked_dk2_dv2_t2.txt")
    fl = lambda rows: np.array([[float(x) for x in r] for r in rows])
    k, v, q = fl(G["k"])[:, None, :], fl(G["v"])[:, None, :], fl(G["q"])[:, None, :]
    g = np.log(fl(G["alpha"]))[0][:, None]
    beta = fl(G["beta"])[0][:, None]
    # full sequence: outputs at both tokens and the final state
    out, S = oracle.recurrent(q, k, v, g, beta, precision=precision)
    assert np.allclose(out[0, 0], fl(G["o_1"])[0], rtol=0, atol=tol)
    assert np.allclose(out[1, 0], fl(G["o_2"])[0], rtol=0, atol=tol)
    assert np.allclose(S[0, 0].ravel(), fl(G["S_2"])[0], rtol=0, atol=tol)
    # prefix of one token gives S_1
    out1, S1 = oracle.recurrent(q[:1], k[:1], v[:1], g[:1], beta[:1], precision=precision)
    assert np.allclose(S1[0, 0].ravel(), fl(G["S_1"])[0], rtol=0, atol=tol)
    # and the fixture separates Eq. (1) from the concept code's alpha-free erase term
    assert not np.allclose(S[0, 0].ravel(), fl(G["S_2_concept_code_variant"])[0], atol=1e-3)


# ----------------------------------------------------------------------- brute force
def _rand_frac(rng, lo, hi, den=8):
    return F(int(rng.integers(lo * den, hi * den + 1)), den)


@pytest.mark.parametrize("seed,T,dk,dv", [(0, 1, 1, 1), (1, 5, 2, 3), (2, 9, 4, 4),
                                          (3, 16, 6, 5), (4, 12, 3, 6), (5, 16, 5, 2)])
def test_bruteforce_exact(seed, T, dk, dv):
    rng = np.random.default_rng(seed)
    k = [[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(T)]
    v = [[_rand_frac(rng, -2, 2) for _ in range(dv)] for _ in range(T)]
    q = [[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(T)]
    alpha = [F(int(rng.integers(1, 16)), 16) for _ in range(T)]     # in (0, 1)
    beta = [F(int(rng.integers(1, 16)), 16) for _ in range(T)]      # in (0, 1)
    S0 = [[_rand_frac(rng, -1, 1) for _ in range(dv)] for _ in range(dk)]
    scale = F(3, 4)
    outs, states = brute.step_matrices(q, k, v, alpha, beta, S0, scale)
    assert brute.unrolled(k, v, alpha, beta, S0) == states[-1]   # two exact formulations agree

    fl = lambda x: np.array(x, dtype=np.float64)
    out, S = oracle.recurrent(fl(q)[:, None], fl(k)[:, None], fl(v)[:, None],
                              np.log(fl(alpha))[:, None], fl(beta)[:, None],
                              S0=fl(S0)[None, None], scale=float(scale))
    ref_o = np.array([[float(x) for x in o] for o in outs])
    ref_S = np.array([[float(x) for x in r] for r in states[-1]])
    assert rel_err(out[:, 0], ref_o) < 1e-12
    assert rel_err(S[0, 0], ref_S) < 1e-12


def test_bruteforce_exact_multihead_varlen():
    """GVA (2 q/k heads for 4 value heads) and three ragged sequences, against brute force."""
    rng = np.random.default_rng(11)
    H_qk, H_v, dk, dv = 2, 4, 3, 2
    lens = [4, 0, 7]
    Tt = sum(lens)
    k = [[[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(H_qk)] for _ in range(Tt)]
    q = [[[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(H_qk)] for _ in range(Tt)]
    v = [[[_rand_frac(rng, -2, 2) for _ in range(dv)] for _ in range(H_v)] for _ in range(Tt)]
    al = [[F(int(rng.integers(1, 16)), 16) for _ in range(H_v)] for _ in range(Tt)]
    be = [[F(int(rng.integers(1, 16)), 16) for _ in range(H_v)] for _ in range(Tt)]
    S0 = [[[[_rand_frac(rng, -1, 1) for _ in range(dv)] for _ in range(dk)] for _ in range(H_v)]
          for _ in range(len(lens))]
    fl = lambda x: np.array(x, dtype=np.float64)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    out, S = oracle.recurrent(fl(q), fl(k), fl(v), np.log(fl(al)), fl(be), S0=fl(S0), cu_seqlens=cu)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        for h in range(H_v):
            hq = h // (H_v // H_qk)
            outs, states = brute.step_matrices(
                [q[t][hq] for t in range(a, b)], [k[t][hq] for t in range(a, b)],
                [v[t][h] for t in range(a, b)], [al[t][h] for t in range(a, b)],
                [be[t][h] for t in range(a, b)], S0[n][h])
            final = states[-1] if states else S0[n][h]
            assert rel_err(S[n, h], np.array(final, dtype=float)) < 1e-12
            if outs:
                assert rel_err(out[a:b, h], np.array(outs, dtype=float)) < 1e-12


# ------------------------------------------------------------------ closed forms
def test_zero_write_zero_state_gives_zero():
    c = rand_case(np.random.default_rng(1), 50, 2, 2, 8, 5, s0=False)
    c["beta"][:] = 0.0
    out, S = oracle.recurrent(**c)
    assert np.all(out == 0) and np.all(S == 0)


def test_pure_decay_closed_form():
    """beta = 0: S_t = gamma_t S0 with gamma_t = exp(sum_{s<=t} g_s); o_t = scale gamma_t S0^T q_t."""
    rng = np.random.default_rng(2)
    c = rand_case(rng, 40, 2, 4, 6, 7)
    c["beta"][:] = 0.0
    out, S = oracle.recurrent(**c, scale=1.5)
    hq = np.arange(4) // 2
    gamma = np.exp(np.cumsum(c["g"], axis=0))                        # [T, H_v]
    for h in range(4):
        ref = 1.5 * gamma[:, h:h + 1] * np.matmul(c["q"][:, hq[h]], c["S0"][0, h])
        assert rel_err(out[:, h], ref) < 1e-13
        assert rel_err(S[0, h], gamma[-1, h] * c["S0"][0, h]) < 1e-13


def _chain(c, lo, hi, S):
    """Run tokens [lo, hi) of a single-sequence case starting from state S."""
    sl = slice(lo, hi)
    return oracle.recurrent(c["q"][sl], c["k"][sl], c["v"][sl], c["g"][sl], c["beta"][sl], S0=S)


def test_unit_write_recalls_value():
    """alpha = beta = 1 and |k| = 1: the written key reads back its value, S_t^T k_t = v_t."""
    rng = np.random.default_rng(3)
    c = rand_case(rng, 12, 1, 1, 8, 5)
    c["g"][:] = 0.0
    c["beta"][:] = 1.0
    S = c["S0"]
    for t in range(12):
        _, S = _chain(c, t, t + 1, S)
        assert rel_err(S[0, 0].T @ c["k"][t, 0], c["v"][t, 0]) < 1e-13


def test_orthonormal_keys_store_all_pairs():
    """alpha = beta = 1, S0 = 0, orthonormal keys: S = sum_j k_j v_j^T and q = k_j reads v_j."""
    rng = np.random.default_rng(4)
    dk, dv = 8, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:, None, :]                              # row j is the j-th orthonormal key
    v = rng.standard_normal((dk, 1, dv))
    q = k.copy()
    out, S = oracle.recurrent(q, k, v, np.zeros((dk, 1)), np.ones((dk, 1)))
    assert rel_err(S[0, 0], sum(np.outer(k[j, 0], v[j, 0]) for j in range(dk))) < 1e-13
    # query every key after all writes: each returns its own value
    out2, _ = oracle.recurrent(k, k, np.zeros_like(v), np.zeros((dk, 1)), np.zeros((dk, 1)), S0=S)
    assert rel_err(out2[:, 0], v[:, 0]) < 1e-13


def test_reset_when_alpha_vanishes():
    """alpha_r ~ 1.8e-35 (g = -80) erases the past: later outputs equal a fresh run from r."""
    rng = np.random.default_rng(5)
    c = rand_case(rng, 60, 1, 2, 7, 4)
    r = 23
    c["g"][r, :] = -80.0
    out, S = oracle.recurrent(**c)
    sl = slice(r, 60)
    out2, S2 = oracle.recurrent(c["q"][sl], c["k"][sl], c["v"][sl], c["g"][sl], c["beta"][sl])
    assert rel_err(out[r:], out2) < 1e-12
    assert rel_err(S, S2) < 1e-12


def test_frobenius_bound():
    """Unit k: I - beta k k^T has spectral norm <= 1, so |S_t|_F <= alpha |S_{t-1}|_F + beta |v_t|."""
    rng = np.random.default_rng(6)
    c = rand_case(rng, 40, 1, 1, 9, 5)
    S = c["S0"]
    for t in range(40):
        prev = np.linalg.norm(S[0, 0])
        _, S = _chain(c, t, t + 1, S)
        bound = math.exp(c["g"][t, 0]) * prev + c["beta"][t, 0] * np.linalg.norm(c["v"][t, 0])
        assert np.linalg.norm(S[0, 0]) <= bound * (1 + 1e-12)


# -------------------------------------------------------------------- invariants
def test_scale_is_linear():
    c = rand_case(np.random.default_rng(7), 30, 2, 2, 5, 5)
    o1, S1 = oracle.recurrent(**c)
    o2, S2 = oracle.recurrent(**c, scale=-2.5)
    assert rel_err(o2, -2.5 * o1) < 1e-14 and np.array_equal(S1, S2)


def test_gva_equals_repeated_heads():
    rng = np.random.default_rng(8)
    c = rand_case(rng, 33, 2, 6, 6, 4)
    o, S = oracle.recurrent(**c)
    rep = dict(c, q=np.repeat(c["q"], 3, axis=1), k=np.repeat(c["k"], 3, axis=1))
    o2, S2 = oracle.recurrent(**rep)
    assert np.array_equal(o, o2) and np.array_equal(S, S2)


def test_varlen_equals_separate_runs():
    rng = np.random.default_rng(9)
    c = rand_case(rng, 40, 2, 2, 5, 6, lens=[13, 0, 40, 1, 27])
    o, S = oracle.recurrent(**c)
    cu = c["cu_seqlens"]
    for n in range(5):
        sl = slice(cu[n], cu[n + 1])
        o2, S2 = oracle.recurrent(c["q"][sl], c["k"][sl], c["v"][sl], c["g"][sl], c["beta"][sl],
                                  S0=c["S0"][n:n + 1])
        assert np.array_equal(o[sl], o2) and np.array_equal(S[n], S2[0])


def test_split_run_resumes_from_state():
    c = rand_case(np.random.default_rng(10), 70, 1, 2, 6, 6)
    o, S = oracle.recurrent(**c)
    o1, S1 = _chain(c, 0, 31, c["S0"])
    o2, S2 = _chain(c, 31, 70, S1)
    assert np.array_equal(np.concatenate([o1, o2]), o) and np.array_equal(S2, S)


def test_l2norm_flag_matches_prenormalised_inputs():
    rng = np.random.default_rng(12)
    c = rand_case(rng, 25, 2, 2, 6, 3, unit_k=False)
    o, S = oracle.recurrent(**c, l2norm=True)
    nq = c["q"] / np.sqrt((c["q"] ** 2).sum(-1, keepdims=True) + 1e-6)
    nk = c["k"] / np.sqrt((c["k"] ** 2).sum(-1, keepdims=True) + 1e-6)
    o2, S2 = oracle.recurrent(**dict(c, q=nq, k=nk))
    assert rel_err(o, o2) < 1e-13 and rel_err(S, S2) < 1e-13


def test_alpha_inside_erase_term():
    """Eq. (1) keeps alpha on the erase term; the concept code's variant drops it.

    The two agree when alpha = 1 and differ otherwise, so the oracle follows Eq. (1).
    """
    rng = np.random.default_rng(13)
    c = rand_case(rng, 20, 1, 1, 5, 4)

    def concept_code(c):
        S = c["S0"][0, 0].copy()
        for t in range(len(c["k"])):
            k, v = c["k"][t, 0], c["v"][t, 0]
            e = v - S.T @ k
            S = math.exp(c["g"][t, 0]) * S + c["beta"][t, 0] * np.outer(k, e)
        return S

    _, S = oracle.recurrent(**c)
    assert rel_err(S[0, 0], concept_code(c)) > 1e-3
    c1 = dict(c, g=np.zeros_like(c["g"]))
    _, S1 = oracle.recurrent(**c1)
    assert rel_err(S1[0, 0], concept_code(c1)) < 1e-13


# ------------------------------------------------------------------ chunk algebra
@pytest.mark.parametrize("C", [1, 16, 64])
def test_chunked_equals_sequential(C):
    rng = np.random.default_rng(20 + C)
    c = rand_case(rng, 150, 2, 4, 16, 12, lens=[150, 64, 1, 65, 0, 129])
    o, S = oracle.recurrent(**c, scale=0.7)
    o2, S2 = oracle.chunked(**c, scale=0.7, chunk=C)
    assert rel_err(o2, o) < 1e-10 and rel_err(S2, S) < 1e-10


def test_chunked_handles_strong_decay():
    """In-chunk cumulative decay near -50 (g ~ -softplus(N(0,1)) over 64 tokens) stays finite."""
    rng = np.random.default_rng(30)
    c = rand_case(rng, 256, 1, 1, 32, 32)
    c["g"] = c["g"] * 1.5
    o, S = oracle.recurrent(**c)
    o2, S2 = oracle.chunked(**c, chunk=64)
    assert np.isfinite(o2).all() and rel_err(o2, o) < 1e-10 and rel_err(S2, S) < 1e-10


# ------------------------------------------------------------------ precision variants
def test_f32_variant_tracks_f64():
    c = rand_case(np.random.default_rng(40), 300, 2, 2, 32, 32)
    o, S = oracle.recurrent(**c)
    o32, S32 = oracle.recurrent(**c, precision="f32")
    assert rel_err(o32, o) < 2e-5 and rel_err(S32, S) < 2e-5


def test_decode_step_is_one_token_recurrence():
    rng = np.random.default_rng(41)
    c = rand_case(rng, 6, 2, 4, 5, 3, lens=[1] * 6)
    o, S = oracle.recurrent(**c)
    o2, S2 = oracle.decode_step(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S0"])
    assert np.array_equal(o, o2) and np.array_equal(S, S2)


def test_decode_multi_against_brute_force():
    """Multi-token decode: outputs over all T tokens and the state committed after c of
    them, against the exact brute force (two sequences, one head, c = 2 and c = 0)."""
    rng = np.random.default_rng(43)
    T, dk, dv = 4, 3, 2
    seqs, commits = [], [2, 0]
    for _ in range(2):
        k = [[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(T)]
        v = [[_rand_frac(rng, -2, 2) for _ in range(dv)] for _ in range(T)]
        q = [[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(T)]
        alpha = [F(int(rng.integers(1, 16)), 16) for _ in range(T)]
        beta = [F(int(rng.integers(1, 16)), 16) for _ in range(T)]
        S0 = [[_rand_frac(rng, -1, 1) for _ in range(dv)] for _ in range(dk)]
        seqs.append((q, k, v, alpha, beta, S0))
    fl = lambda x: np.array(x, dtype=np.float64)
    Q = np.stack([fl(s[0]) for s in seqs])[:, :, None]          # [N, T, 1, dk]
    K = np.stack([fl(s[1]) for s in seqs])[:, :, None]
    V = np.stack([fl(s[2]) for s in seqs])[:, :, None]
    G = np.log(np.stack([fl(s[3]) for s in seqs]))[:, :, None]
    B = np.stack([fl(s[4]) for s in seqs])[:, :, None]
    S0 = np.stack([fl(s[5]) for s in seqs])[:, None]            # [N, 1, dk, dv]
    out, S = oracle.decode_multi(Q, K, V, G, B, S0, n_commit=np.array(commits))
    for n, (q, k, v, alpha, beta, s0) in enumerate(seqs):
        outs, states = brute.step_matrices(q, k, v, alpha, beta, s0)
        ref_o = np.array([[float(x) for x in o] for o in outs])
        assert rel_err(out[n, :, 0], ref_o) < 1e-12
        ref_S = states[commits[n] - 1] if commits[n] > 0 else s0
        assert rel_err(S[n, 0], np.array([[float(x) for x in r] for r in ref_S])) < 1e-12


def test_gates_from_logits_closed_forms():
    """softplus(0) = ln 2 and sigmoid(0) = 1/2; softplus(a) -> a for large a and -> e^a
    for very negative a (no overflow, no loss of the small value); both gates inside
    (0, 1) over the whole range."""
    a = np.array([0.0, 40.0, -40.0, 800.0, -800.0, 1.5])
    g, beta = oracle.gates_from_logits(a, a)
    assert g[0] == -np.log(2.0) and beta[0] == 0.5
    assert abs(g[1] + 40.0) < 1e-15 and abs(g[2] + np.exp(-40.0)) < 1e-30
    assert g[3] == -800.0 and abs(g[4]) < 1e-300
    assert abs(g[5] + np.log1p(np.exp(1.5))) < 1e-15
    assert abs(beta[5] - 1.0 / (1.0 + np.exp(-1.5))) < 1e-15
    alpha = np.exp(g)
    assert np.all((alpha > 0) | (g < -700)) and np.all(alpha <= 1) and np.all((beta >= 0) & (beta <= 1))


def test_gate_logits_zero_is_half_against_brute_force():
    """Zero logits give alpha = beta = 1/2 exactly; the recurrence fed through the gate
    prologue then matches the exact brute force with alpha = beta = 1/2."""
    rng = np.random.default_rng(47)
    T, dk, dv = 6, 3, 2
    k = [[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(T)]
    v = [[_rand_frac(rng, -2, 2) for _ in range(dv)] for _ in range(T)]
    q = [[_rand_frac(rng, -1, 1) for _ in range(dk)] for _ in range(T)]
    S0 = [[_rand_frac(rng, -1, 1) for _ in range(dv)] for _ in range(dk)]
    half = [F(1, 2)] * T
    outs, states = brute.step_matrices(q, k, v, half, half, S0)
    g, beta = oracle.gates_from_logits(np.zeros((T, 1)), np.zeros((T, 1)))
    fl = lambda x: np.array(x, dtype=np.float64)
    out, S = oracle.recurrent(fl(q)[:, None], fl(k)[:, None], fl(v)[:, None], g, beta,
                              S0=fl(S0)[None, None])
    assert rel_err(out[:, 0], np.array([[float(x) for x in o] for o in outs])) < 1e-12
    assert rel_err(S[0, 0], np.array([[float(x) for x in r] for r in states[-1]])) < 1e-12


def _fd_case(seed):
    rng = np.random.default_rng(seed)
    T, Hq, Hv, dk, dv = 7, 1, 2, 3, 2
    c = dict(q=rng.normal(size=(T, Hq, dk)), k=rng.normal(size=(T, Hq, dk)) * 0.5,
             v=rng.normal(size=(T, Hv, dv)), g=-np.abs(rng.normal(size=(T, Hv))) * 0.5,
             beta=1 / (1 + np.exp(-rng.normal(size=(T, Hv)))),
             S0=rng.normal(size=(2, Hv, dk, dv)) * 0.3)
    dO = rng.normal(size=(T, Hv, dv))
    dSf = rng.normal(size=(2, Hv, dk, dv))
    return c, dO, dSf, np.array([0, 3, 7])


def _fd_errors(backward_fn, seed=0, scale=0.7):
    """Worst relative gap, per gradient, between backward_fn and central differences of
    L = <out, dO> + <S_final, dS_final> through the forward oracle."""
    c, dO, dSf, cu = _fd_case(seed)
    names = ["q", "k", "v", "g", "beta", "S0"]

    def L(vals):
        o, S = oracle.recurrent(vals["q"], vals["k"], vals["v"], vals["g"], vals["beta"],
                                S0=vals["S0"], cu_seqlens=cu, scale=scale)
        return np.sum(o * dO) + np.sum(S * dSf)

    grads = backward_fn(c["q"], c["k"], c["v"], c["g"], c["beta"], c["S0"], dO, dSf, cu,
                        scale=scale)
    out = []
    for name, G in zip(names, grads):
        A = c[name]
        num = np.zeros_like(A)
        for idx in np.ndindex(A.shape):
            hi = dict(c); lo = dict(c)
            hi[name] = A.copy(); hi[name][idx] += 1e-6
            lo[name] = A.copy(); lo[name][idx] -= 1e-6
            num[idx] = (L(hi) - L(lo)) / 2e-6
        out.append(np.abs(num - G).max() / max(np.abs(num).max(), 1e-12))
    return out


def test_backward_matches_finite_differences():
    """Every gradient of the backward oracle (q, k, v, g, beta, S0; two ragged sequences,
    two value heads on one q/k head, a given S0 and dS_final) against central
    differences of the forward oracle."""
    from oracle.backward import backward
    assert max(_fd_errors(backward)) < 1e-7


@pytest.mark.parametrize("old,new", [
    ("dal += -bt * (du @ a)", "dal += bt * (du @ a)"),            # sign of the erase term
    ("da = -al * bt * du", "da = -bt * du"),                      # alpha dropped in da
    ("dq[t, hq] += scale * S_t @ d_out[t, h]", "dq[t, hq] += scale * S_p @ d_out[t, h]"),
    ("dS = dS + scale * np.outer(qt, d_out[t, h])", "dS = dS + np.outer(qt, d_out[t, h])"),
])
def test_backward_pins_catch_plausible_mistakes(old, new):
    """The finite-difference pin fails for each planted mistake in the backward oracle."""
    import inspect
    import oracle.backward as ob
    src = inspect.getsource(ob)
    assert old in src
    ns = {}
    exec(compile(src.replace(old, new), "mutant", "exec"), ns)
    assert max(_fd_errors(ns["backward"])) > 1e-3


def test_rejects_bad_sizes():
    c = rand_case(np.random.default_rng(42), 5, 2, 3, 4, 4)      # H_v not a multiple of H_qk
    with pytest.raises(ValueError):
        oracle.recurrent(**c)
