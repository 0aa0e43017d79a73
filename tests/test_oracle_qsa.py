"""Pins for the QSA indexer oracle, each against something other than the oracle.

Operation: "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "部品②: QSA":
keys mean-pooled over r = 4 tokens before positional encoding, one position (the
block's first) per pooled key, partial RoPE on 64 of 128 dims, 4 query heads sharing
one key head, a budget of 2048 tokens (512 blocks), kept blocks expanded to tokens.

Pins used:
  * hand-worked rotary values (unit vectors at chosen dims, frequencies 1, 1/10, 1/100);
  * the rotary map as multiplication by a unit complex number, and its
    relative-position identity;
  * exact rational brute force (fractions) of pooling, scoring, ranking, ties,
    eligibility and expansion with the rotation switched off;
  * with the rotation on: the score written in the relative-position form from the
    raw (unpooled) keys, which fixes "pool, then rotate at the block start";
  * edge cases: empty and short sequences, a budget above the eligible count, the
    causality boundary, all-equal scores.
Every check takes the oracle module as an argument so tests/test_oracle_qsa_mutants.py
can run the same battery against planted mistakes.
"""
from __future__ import annotations

from fractions import Fraction as F

import numpy as np
import pytest

from oracle import qsa as Q0

ROPE_64_FREQ = {0: 1.0, 8: 0.1, 16: 0.01, 24: 0.001}   # base 10000, 64 rotary dims


# ----------------------------------------------------------------------- rotary pins
def check_rope_hand_values(Q):
    """Unit vector e_i at position p turns into cos(p w_i) e_i + sin(p w_i) e_{i+32}, and
    e_{i+32} into -sin e_i + cos e_{i+32}, with w_0 = 1, w_8 = 1/10, w_16 = 1/100,
    w_24 = 1/1000 (base 10000 over 64 rotary dims); dims 64.. are untouched."""
    p = 3
    for i, w in ROPE_64_FREQ.items():
        e = np.zeros(128); e[i] = 1.0
        y = Q.rope_partial(e, p)
        want = np.zeros(128); want[i] = np.cos(p * w); want[i + 32] = np.sin(p * w)
        assert np.allclose(y, want, atol=1e-15), i
        e2 = np.zeros(128); e2[i + 32] = 1.0
        y2 = Q.rope_partial(e2, p)
        want2 = np.zeros(128); want2[i] = -np.sin(p * w); want2[i + 32] = np.cos(p * w)
        assert np.allclose(y2, want2, atol=1e-15), i
    for i in (64, 100, 127):
        e = np.zeros(128); e[i] = 1.0
        assert np.array_equal(Q.rope_partial(e, 12345), e)


def _rope_complex(x, pos, rope_dims=64, base=10000.0):
    """Rotary map as z_i -> z_i exp(j pos w_i) with z_i = x_i + j x_{i+half}."""
    half = rope_dims // 2
    w = np.array([base ** (-(i / half)) for i in range(half)])
    z = x[..., :half] + 1j * x[..., half:rope_dims]
    z = z * np.exp(1j * np.asarray(pos, np.float64)[..., None] * w)
    out = np.array(x, np.float64, copy=True)
    out[..., :half], out[..., half:rope_dims] = z.real, z.imag
    return out


def check_rope_complex_form(Q):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 128))
    pos = np.array([0, 1, 4, 77, 4096, 262143, 1048572])
    # the two forms round w differently in the last bit: at position 1e6 the angles then
    # differ by about 1e6 * 1.1e-16 rad, hence the absolute tolerance
    assert np.allclose(Q.rope_partial(x, pos), _rope_complex(x, pos), rtol=0, atol=1e-8)


def check_rope_relative_position(Q):
    """<R(m) x, R(n) y> = <R(m - n) x, y>, norms kept."""
    rng = np.random.default_rng(2)
    x, y = rng.standard_normal(128), rng.standard_normal(128)
    for m, n in [(5, 2), (1000, 996), (300000, 12)]:
        lhs = Q.rope_partial(x, m) @ Q.rope_partial(y, n)
        rhs = Q.rope_partial(x, m - n) @ y
        assert abs(lhs - rhs) < 1e-9 * np.abs(x).sum() * np.abs(y).sum()
        assert abs(np.linalg.norm(Q.rope_partial(x, m)) - np.linalg.norm(x)) < 1e-12


# ------------------------------------------------------------ exact brute force (no RoPE)
def _rand_int_case(rng, lens, D, H, lo=-3, hi=4):
    T = int(sum(lens))
    k = rng.integers(lo, hi, size=(T, D)).astype(np.float64)
    q = rng.integers(lo, hi, size=(len(lens), H, D)).astype(np.float64)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return k, q, cu


def _brute_index(k, q, cu, q_pos, budget, r=4):
    """Fractions throughout; ranking by Python's sort on (-score, block)."""
    N = len(cu) - 1
    res = []
    for n in range(N):
        toks = [[F(int(x)) for x in row] for row in k[cu[n]:cu[n + 1]]]
        nb = len(toks) // r
        pooled = [[sum(toks[r * b + j][d] for j in range(r)) / r for d in range(k.shape[1])]
                  for b in range(nb)]
        elig = [b for b in range(nb) if r * b + r - 1 <= q_pos[n]]
        scores = {b: sum(F(int(q[n, h, d])) * pooled[b][d]
                         for h in range(q.shape[1]) for d in range(k.shape[1])) for b in elig}
        ranked = sorted(elig, key=lambda b: (-scores[b], b))[:budget]
        kept = sorted(ranked)
        res.append((pooled, kept, [scores[b] for b in kept]))
    return res


def check_bruteforce_exact(Q, seed=3, lens=(0, 3, 4, 17, 41, 64), D=6, H=4, budget=5):
    rng = np.random.default_rng(seed)
    k, q, cu = _rand_int_case(rng, lens, D, H)
    q_pos = np.array([max(0, L - 1) + (7 if i == 3 else 0) for i, L in enumerate(lens)])
    q_pos[-1] = 30        # a query partway into the cache: causality cuts the tail
    k_hat, cu_b = Q.compress_keys(k, cu, rope_dims=0)
    bi, bs, ti = Q.index_decode(q, q_pos, k_hat, cu_b, budget_blocks=budget, rope_dims=0)
    want = _brute_index(k, q, cu, q_pos, budget)
    for n, (pooled, kept, sc) in enumerate(want):
        assert list(cu_b[n + 1] - cu_b[n:n + 1]) == [len(pooled)]
        assert np.array_equal(k_hat[cu_b[n]:cu_b[n + 1]], np.array(pooled, np.float64).reshape(-1, D))
        assert list(bi[n, :len(kept)]) == kept and np.all(bi[n, len(kept):] == -1)
        assert np.array_equal(bs[n, :len(kept)], np.array([float(s) for s in sc]))
        assert np.all(np.isneginf(bs[n, len(kept):]))
        toks = [4 * b + j for b in kept for j in range(4)]
        assert list(ti[n, :len(toks)]) == toks and np.all(ti[n, len(toks):] == -1)


def check_ties_go_to_earlier_block(Q):
    """All-equal keys give all-equal scores: the earliest blocks are kept."""
    D, H, nb = 4, 4, 40
    k = np.ones((4 * nb, D))
    q = np.ones((1, H, D))
    k_hat, cu_b = Q.compress_keys(k, [0, 4 * nb], rope_dims=0)
    bi, bs, _ = Q.index_decode(q, [4 * nb - 1], k_hat, cu_b, budget_blocks=7, rope_dims=0)
    assert list(bi[0]) == list(range(7))
    # two tiers: odd blocks score higher; ties within a tier go to the earlier block
    k2 = np.ones((4 * nb, D)); k2[[t for t in range(4 * nb) if (t // 4) % 2 == 1]] *= 2
    k_hat2, _ = Q.compress_keys(k2, [0, 4 * nb], rope_dims=0)
    bi2, _, _ = Q.index_decode(q, [4 * nb - 1], k_hat2, cu_b, budget_blocks=nb // 2 + 3,
                               rope_dims=0)
    assert list(bi2[0]) == sorted(list(range(1, nb, 2)) + [0, 2, 4])


def check_causality_boundary(Q):
    """Block b enters at q_pos = 4 b + 3 (its last token), not at 4 b + 2."""
    D, H, nb = 4, 4, 10
    rng = np.random.default_rng(4)
    k = rng.standard_normal((4 * nb, D))
    q = rng.standard_normal((1, H, D))
    k_hat, cu_b = Q.compress_keys(k, [0, 4 * nb], rope_dims=0)
    for b in range(nb):
        bi_in, _, _ = Q.index_decode(q, [4 * b + 3], k_hat, cu_b, budget_blocks=nb, rope_dims=0)
        bi_out, _, _ = Q.index_decode(q, [4 * b + 2], k_hat, cu_b, budget_blocks=nb, rope_dims=0)
        assert list(bi_in[0, :b + 1]) == list(range(b + 1)) and bi_in[0, b + 1:].max(initial=-1) == -1
        assert list(bi_out[0, :b]) == list(range(b)) and bi_out[0, b:].max(initial=-1) == -1


# ------------------------------------------------------------- with RoPE: relative form
def _relative_scores(k_tok, q, q_pos, r=4, rope_dims=64, base=10000.0):
    """Score of block b from the raw tokens: pool in the complex rotary pairs and the
    pass-through dims, then Re(sum_h z_q conj(z_k) exp(j (q_pos - r b) w)) + plain dot."""
    half = rope_dims // 2
    w = np.array([base ** (-(i / half)) for i in range(half)])
    nb = k_tok.shape[0] // r
    out = []
    for b in range(nb):
        blk = k_tok[r * b:r * b + r]
        zk = (blk[:, :half] + 1j * blk[:, half:rope_dims]).sum(axis=0) / r
        rest_k = blk[:, rope_dims:].sum(axis=0) / r
        s = 0.0
        for h in range(q.shape[0]):
            zq = q[h, :half] + 1j * q[h, half:rope_dims]
            s += np.real(np.sum(zq * np.conj(zk) * np.exp(1j * (q_pos - r * b) * w)))
            s += q[h, rope_dims:] @ rest_k
        out.append(s)
    return np.array(out)


def check_scores_relative_form(Q):
    rng = np.random.default_rng(5)
    for T, q_pos, p0 in [(64, 63, 0), (400, 399, 0), (400, 1_000_003, 999_604)]:
        k = rng.standard_normal((T, 128))
        q = rng.standard_normal((1, 4, 128))
        k_hat, cu_b = Q.compress_keys(k, [0, T], pos0=[p0])
        s = Q.block_scores(q[0], q_pos, k_hat)
        want = _relative_scores(k, q[0], q_pos - p0)
        assert np.allclose(s, want, rtol=0, atol=1e-9 * np.abs(want).max()), (T, q_pos)


def check_heads_sum(Q):
    rng = np.random.default_rng(6)
    k = rng.standard_normal((80, 128))
    q = rng.standard_normal((4, 128))
    k_hat, _ = Q.compress_keys(k, [0, 80])
    s = Q.block_scores(q, 90, k_hat)
    parts = sum(Q.block_scores(q[h:h + 1], 90, k_hat) for h in range(4))
    assert np.allclose(s, parts, rtol=0, atol=1e-12 * np.abs(s).max())


def check_equal_rows_score_equal(Q):
    """Ties are decided by block order only if equal rows score exactly equal, wherever
    they sit in the cache."""
    rng = np.random.default_rng(7)
    v = rng.standard_normal(128)
    kh = rng.standard_normal((5003, 128))
    pos = rng.choice(5003, 700, replace=False)
    kh[pos] = v
    s = Q.block_scores(rng.standard_normal((4, 128)), 123457, kh)
    assert np.unique(s[pos]).size == 1


BATTERY = [
    ("rope_hand", check_rope_hand_values),
    ("rope_complex", check_rope_complex_form),
    ("rope_relative", check_rope_relative_position),
    ("brute", check_bruteforce_exact),
    ("ties", check_ties_go_to_earlier_block),
    ("causality", check_causality_boundary),
    ("relative_scores", check_scores_relative_form),
    ("heads_sum", check_heads_sum),
    ("equal_rows", check_equal_rows_score_equal),
]


@pytest.mark.parametrize("name,fn", BATTERY, ids=[b[0] for b in BATTERY])
def test_qsa_oracle_pin(name, fn):
    fn(Q0)


@pytest.mark.parametrize("seed,lens,budget", [(7, (5, 8, 12), 1), (8, (40, 0, 33), 100),
                                              (9, (128,), 32)])
def test_qsa_bruteforce_more(seed, lens, budget):
    check_bruteforce_exact(Q0, seed=seed, lens=lens, budget=budget)


def test_qsa_constants_from_the_pages():
    """r = 4, 4 query heads over 1 key head, partial RoPE on 64 of 128 dims, a budget of
    2048 tokens = 512 blocks."""
    assert (Q0.R, Q0.HEADS, Q0.ROPE_DIMS, Q0.D) == (4, 4, 64, 128)
    assert Q0.TOKEN_BUDGET == 2048 and Q0.BLOCK_BUDGET == 512


def test_qsa_multi_query_is_per_query_indexing():
    """T queries per sequence: query j equals a single query at q_pos + j (with its own
    causal cut), checked exactly with the rotation off against the fraction brute force."""
    rng = np.random.default_rng(12)
    lens = (0, 17, 41, 64)
    k, _, cu = _rand_int_case(rng, lens, 6, 4)
    q = rng.integers(-3, 4, size=(len(lens), 3, 4, 6)).astype(np.float64)
    q_pos = np.array([0, 12, 30, 61])
    k_hat, cu_b = Q0.compress_keys(k, cu, rope_dims=0)
    bi, bs, ti = Q0.index_multi(q, q_pos, k_hat, cu_b, budget_blocks=5, rope_dims=0)
    assert bi.shape == (4, 3, 5) and ti.shape == (4, 3, 20)
    for j in range(3):
        want = _brute_index(k, q[:, j], cu, q_pos + j, 5)
        for n, (_, kept, sc) in enumerate(want):
            assert list(bi[n, j, :len(kept)]) == kept and np.all(bi[n, j, len(kept):] == -1)
            assert np.array_equal(bs[n, j, :len(kept)], np.array([float(x) for x in sc]))
