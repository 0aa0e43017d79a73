"""GPU parity of the QSA indexer (libgdn through the C ABI) against the CPU oracle.

Operation: "論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "部品②: QSA".

Block cache (gdn_qsa_compress): each written row must equal the oracle's float64 row to
within the bf16 rounding of the kernel's fp32 value.  bf16 keeps 8 significant bits, so
rounding to nearest moves a value by at most 2^-8 of itself: |gpu - ref| <= 2^-8 |ref| +
1e-5 (the last term covers the fp32 pooling and rotation).

Indexer (gdn_qsa_index_decode): the kernel ranks fp32 scores, the oracle float64 ones,
so the kept set is compared where it is unique and checked for validity elsewhere:
  * per block, t_b = 8e-6 * sum_d (sum_h |RoPE(q_h)_d|) |k_hat_b,d| bounds |s32 - s64|
    (fp32 rotation and head sum, then a 128-term fp32 dot: about 25 roundings of
    2^-24 on that sum of magnitudes, taken with a factor 4 of margin);
  * kept scores agree with the oracle's to t_b;
  * no dropped block beats a kept one by more than their tolerances;
  * the kept set equals the oracle's except for blocks whose score lies within
    2 max(t) of the oracle's budget-th score;
  * where scores tie exactly on both sides (repeated cache rows), the kept set must equal
    the oracle's exactly (ties to the earlier block);
  * tokens are the kept blocks expanded (4 per block), padding -1 / -inf.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import linear_attention_token_b200 as gdn
from linear_attention_token_b200 import inputs
from oracle import qsa as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


# ------------------------------------------------------------------- compress
def _compress_case(lens, pos0=None, slack=None, seed=11):
    N = len(lens)
    k = inputs.qsa_keys(int(sum(lens)), seed, DEV)
    cu = inputs.qsa_offsets(lens, DEV)
    blocks = [L // 4 for L in lens]
    if slack is not None:                            # rows the kernel must leave alone
        blocks = [b + s for b, s in zip(blocks, slack)]
    cub = inputs.qsa_offsets(blocks, DEV)
    sentinel = torch.full((int(sum(blocks)), 128), 7.0, dtype=torch.bfloat16, device=DEV)
    k_hat = sentinel.clone()
    p0 = None if pos0 is None else torch.tensor(pos0, dtype=torch.int32, device=DEV)
    gdn.gdn_qsa_compress(k, cu, cub, k_hat=k_hat, pos0=p0)
    torch.cuda.synchronize()
    ref, ref_cub = O.compress_keys(k.float().cpu().numpy(), cu.cpu().numpy(),
                                   None if pos0 is None else np.array(pos0))
    got = k_hat.float().cpu().numpy()
    cub_h = cub.cpu().numpy()
    for n in range(N):
        nb = lens[n] // 4
        g = got[cub_h[n]:cub_h[n] + nb]
        r = ref[ref_cub[n]:ref_cub[n] + nb]
        assert np.all(np.abs(g - r) <= 2.0 ** -8 * np.abs(r) + 1e-5), n
        assert np.all(got[cub_h[n] + nb:cub_h[n + 1]] == 7.0), n


@pytest.mark.parametrize("lens,pos0,slack", [
    ((256,), None, None),
    ((0, 3, 4, 37, 1000, 4099), None, None),
    ((64, 200, 8), [0, 5, 1_000_000], None),
    ((40, 13, 9), [2_000_000_000, 7, 0], [3, 0, 2]),      # rows past the tokens stay as they were
])
def test_qsa_compress_matches_oracle(lens, pos0, slack):
    _compress_case(lens, pos0, slack)


def test_qsa_compress_full_size_sampled():
    """Two sequences of 1,048,576 tokens (262,144 blocks each); 2,000 sampled blocks."""
    lens = (1 << 20, 1 << 20)
    k = inputs.qsa_keys(sum(lens), 12, DEV)
    cu = inputs.qsa_offsets(lens, DEV)
    cub = inputs.qsa_offsets([L // 4 for L in lens], DEV)
    k_hat = torch.empty(sum(lens) // 4, 128, dtype=torch.bfloat16, device=DEV)
    gdn.gdn_qsa_compress(k, cu, cub, k_hat=k_hat)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(sum(lens) // 4, 2000, replace=False))
    kc = k.view(-1, 4, 128)[torch.as_tensor(rows, device=DEV)].float().cpu().numpy()
    got = k_hat[torch.as_tensor(rows, device=DEV)].float().cpu().numpy()
    for i, row in enumerate(rows):
        b = row % ((1 << 20) // 4)
        ref, _ = O.compress_keys(kc[i], [0, 4], pos0=[4 * b])
        assert np.all(np.abs(got[i] - ref[0]) <= 2.0 ** -8 * np.abs(ref[0]) + 1e-5), row


# -------------------------------------------------------------------- indexer
def _tol(q, q_pos, k_hat_rows, scale=8e-6):
    qh = O.rope_partial(q, np.full(q.shape[0], q_pos))
    return scale * (np.abs(k_hat_rows) @ np.abs(qh).sum(axis=0))


def _check_index(q, q_pos, k_hat, cu_blocks, budget, out, exact_ties=False, ref_rows=None,
                 tol_scale=8e-6):
    """ref_rows: the oracle's own cache (float64, from raw keys) when k_hat was written by
    the kernel under test; tol_scale then also covers the cache's bf16 rounding."""
    bi, bs, ti = (t.cpu().numpy() for t in out)
    qn = q.float().cpu().numpy()
    qp = q_pos.cpu().numpy()
    kh = k_hat.float().cpu().numpy() if ref_rows is None else np.asarray(ref_rows, np.float64)
    cb = cu_blocks.cpu().numpy()
    for n in range(qn.shape[0]):
        e = O.eligible_blocks(cb[n + 1] - cb[n], int(qp[n]))
        rows = kh[cb[n]:cb[n] + e]
        s = O.block_scores(qn[n], int(qp[n]), rows)
        t = _tol(qn[n], int(qp[n]), rows, tol_scale)
        keep = min(e, budget)
        G = bi[n, :keep]
        assert np.all(bi[n, keep:] == -1) and np.all(np.isneginf(bs[n, keep:]))
        assert np.all(np.diff(G) > 0) and (keep == 0 or (G[0] >= 0 and G[-1] < e))
        toks = (4 * G[:, None] + np.arange(4)[None, :]).reshape(-1)
        assert np.array_equal(ti[n, :4 * keep], toks) and np.all(ti[n, 4 * keep:] == -1)
        if keep == 0:
            continue
        assert np.all(np.abs(bs[n, :keep] - s[G]) <= t[G]), n
        Oset = O.select_blocks(s, budget)
        if exact_ties:
            assert np.array_equal(G, Oset), n
            continue
        out_mask = np.ones(e, bool); out_mask[G] = False
        if out_mask.any():
            assert (s[G] + t[G]).min() >= (s[out_mask] - t[out_mask]).max(), n
        sigma = np.sort(s)[::-1][keep - 1]
        band = np.abs(s - sigma) <= 2 * t.max()
        diff = np.setxor1d(G, Oset)
        assert np.all(band[diff]), (n, diff[~band[diff]])


def _run_index(q, q_pos, k_hat, cu_blocks, budget, ws=None):
    out = gdn.gdn_qsa_index_decode(q, q_pos, k_hat, cu_blocks, budget, workspace=ws)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("budget", [512, 64, 1, 4096])
def test_qsa_index_ragged(budget):
    w = inputs.qsa_workloads()[1]
    x = inputs.qsa_decode_inputs(w, DEV)
    out = _run_index(x["q"], x["q_pos"], x["k_hat"], x["cu_blocks"], budget)
    _check_index(x["q"], x["q_pos"], x["k_hat"], x["cu_blocks"], budget, out)


def test_qsa_index_causal_cut_and_empty():
    """Queries before the cache end (only blocks wholly at or before them count), a query
    at position 2 (no whole block yet) and an empty cache."""
    blocks = [5000, 5000, 0, 3000, 7]
    cub = inputs.qsa_offsets(blocks, DEV)
    k_hat = inputs.qsa_cache(sum(blocks), 21, DEV)
    q = inputs.qsa_queries(len(blocks), 22, DEV)
    q_pos = torch.tensor([19999, 4098, 100, 2, 1_000_000], dtype=torch.int32, device=DEV)
    for budget in (512, 2000):
        out = _run_index(q, q_pos, k_hat, cub, budget)
        _check_index(q, q_pos, k_hat, cub, budget, out)


def test_qsa_index_exact_ties_listed_and_overflowed():
    """Repeated rows tie exactly on both sides; the earlier blocks must win.  The threshold
    bin holds 3,000 blocks in one sequence (candidate list) and 40,000 in the other (past
    the list: the exact selection then reads the scores themselves)."""
    blocks = [9000, 40000]
    cub = inputs.qsa_offsets(blocks, DEV)
    k_hat = torch.cat([inputs.qsa_palette_cache(9000, 3, 31, DEV),
                       inputs.qsa_palette_cache(40000, 1, 32, DEV)])
    q = inputs.qsa_queries(2, 33, DEV)
    q_pos = torch.tensor([4 * 9000 - 1, 4 * 40000 - 1], dtype=torch.int32, device=DEV)
    for budget in (512, 4096, 1):
        out = _run_index(q, q_pos, k_hat, cub, budget)
        _check_index(q, q_pos, k_hat, cub, budget, out, exact_ties=True)


def test_qsa_index_many_sequences():
    rng = np.random.default_rng(5)
    blocks = [int(x) for x in rng.integers(0, 3000, size=300)]
    cub = inputs.qsa_offsets(blocks, DEV)
    k_hat = inputs.qsa_cache(sum(blocks), 41, DEV)
    q = inputs.qsa_queries(len(blocks), 42, DEV)
    q_pos = torch.tensor([4 * b + 3 for b in blocks], dtype=torch.int32, device=DEV)
    out = _run_index(q, q_pos, k_hat, cub, 512)
    _check_index(q, q_pos, k_hat, cub, 512, out)


def test_qsa_index_workspace_is_left_clean():
    """Two calls on one workspace give identical results, and a third call on other
    inputs still matches the oracle."""
    w = inputs.qsa_workloads()[1]
    x = inputs.qsa_decode_inputs(w, DEV)
    ws = gdn.qsa_index_workspace(w.num_seqs, x["k_hat"].shape[0])
    a = _run_index(x["q"], x["q_pos"], x["k_hat"], x["cu_blocks"], 512, ws)
    a = [t.clone() for t in a]
    b = _run_index(x["q"], x["q_pos"], x["k_hat"], x["cu_blocks"], 512, ws)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    x2 = inputs.qsa_decode_inputs(w, DEV, seed=999)
    c = _run_index(x2["q"], x2["q_pos"], x2["k_hat"], x2["cu_blocks"], 300, ws)
    _check_index(x2["q"], x2["q_pos"], x2["k_hat"], x2["cu_blocks"], 300, c)


def test_qsa_index_full_size():
    """The benchmark workload: 8 sequences with 1,048,576 cached tokens each (262,144
    blocks), budget 512 blocks; two sequences are checked block by block."""
    w = inputs.qsa_workloads()[0]
    x = inputs.qsa_decode_inputs(w, DEV)
    out = _run_index(x["q"], x["q_pos"], x["k_hat"], x["cu_blocks"], w.budget_blocks)
    nb = w.blocks[0]
    sub = [0, 5]
    rows = torch.cat([x["k_hat"][i * nb:(i + 1) * nb] for i in sub])
    cub = inputs.qsa_offsets([nb] * len(sub), DEV)
    _check_index(x["q"][sub], x["q_pos"][sub], rows, cub, w.budget_blocks,
                 tuple(t[sub] for t in out))


@pytest.mark.parametrize("budget", [512, 4096])
def test_qsa_index_cache_past_the_bitmap(budget):
    """300,000 eligible blocks (past the 262,144-block bitmap of the finish kernel, so the
    kept list is sorted instead: by rank for <= 1024 kept blocks, bitonic above)."""
    blocks = [300_000, 1000]
    cub = inputs.qsa_offsets(blocks, DEV)
    k_hat = inputs.qsa_cache(sum(blocks), 51, DEV)
    q = inputs.qsa_queries(2, 52, DEV)
    q_pos = torch.tensor([4 * b - 1 for b in blocks], dtype=torch.int32, device=DEV)
    out = _run_index(q, q_pos, k_hat, cub, budget)
    _check_index(q, q_pos, k_hat, cub, budget, out)


# ------------------------------------------------------- T queries per sequence
def _check_multi(q, q_pos, k_hat, cub, budget, out, exact_ties=False):
    """Query j of every sequence against the oracle's single query at q_pos + j."""
    bi, bs, ti = out
    for j in range(q.shape[1]):
        _check_index(q[:, j], q_pos + j, k_hat, cub, budget, (bi[:, j], bs[:, j], ti[:, j]),
                     exact_ties)


def _run_multi(q, q_pos, k_hat, cub, budget, ws=None):
    out = gdn.gdn_qsa_index_multi(q, q_pos, k_hat, cub, budget, workspace=ws)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_qsa_multi_ragged(T):
    w = inputs.qsa_workloads()[1]
    x = inputs.qsa_decode_inputs(w, DEV)
    q = inputs.qsa_multi_queries(w.num_seqs, T, 61, DEV)
    q_pos = torch.tensor([max(0, L - T) for L in w.ctx_lens], dtype=torch.int32, device=DEV)
    out = _run_multi(q, q_pos, x["k_hat"], x["cu_blocks"], 512)
    _check_multi(q, q_pos, x["k_hat"], x["cu_blocks"], 512, out)


def test_qsa_multi_one_query_equals_decode():
    w = inputs.qsa_workloads()[1]
    x = inputs.qsa_decode_inputs(w, DEV)
    a = _run_multi(x["q"][:, None].contiguous(), x["q_pos"], x["k_hat"], x["cu_blocks"], 300)
    b = _run_index(x["q"], x["q_pos"], x["k_hat"], x["cu_blocks"], 300)
    for u, v in zip(a, b):
        assert torch.equal(u[:, 0], v)


def test_qsa_multi_queries_cross_block_boundaries():
    """Queries at 4b + 1 .. 4b + 4: block b becomes eligible at the third query, block b + 1
    at none; and a sequence whose first queries see no whole block yet."""
    blocks = [3000, 700, 5]
    cub = inputs.qsa_offsets(blocks, DEV)
    k_hat = inputs.qsa_cache(sum(blocks), 62, DEV)
    q = inputs.qsa_multi_queries(3, 4, 63, DEV)
    q_pos = torch.tensor([4 * 1999 + 1, 4 * 699 + 1, 0], dtype=torch.int32, device=DEV)
    for budget in (512, 2000):
        out = _run_multi(q, q_pos, k_hat, cub, budget)
        _check_multi(q, q_pos, k_hat, cub, budget, out)


def test_qsa_multi_exact_ties():
    blocks = [9000, 30000]
    cub = inputs.qsa_offsets(blocks, DEV)
    k_hat = torch.cat([inputs.qsa_palette_cache(9000, 3, 64, DEV),
                       inputs.qsa_palette_cache(30000, 1, 65, DEV)])
    q = inputs.qsa_multi_queries(2, 3, 66, DEV)
    q_pos = torch.tensor([4 * 9000 - 3, 4 * 30000 - 3], dtype=torch.int32, device=DEV)
    out = _run_multi(q, q_pos, k_hat, cub, 512)
    _check_multi(q, q_pos, k_hat, cub, 512, out, exact_ties=True)


def test_qsa_multi_full_size():
    """8 sequences x 262,144 blocks, 4 queries each (the multi-query bench workload);
    sequences 0 and 5 checked block by block for all 4 queries."""
    w = inputs.qsa_workloads()[0]
    x = inputs.qsa_decode_inputs(w, DEV)
    q = inputs.qsa_multi_queries(w.num_seqs, 4, 67, DEV)
    q_pos = torch.tensor([L - 4 for L in w.ctx_lens], dtype=torch.int32, device=DEV)
    out = _run_multi(q, q_pos, x["k_hat"], x["cu_blocks"], w.budget_blocks)
    nb = w.blocks[0]
    sub = [0, 5]
    rows = torch.cat([x["k_hat"][i * nb:(i + 1) * nb] for i in sub])
    cub = inputs.qsa_offsets([nb] * len(sub), DEV)
    _check_multi(q[sub], q_pos[sub], rows, cub, w.budget_blocks, tuple(t[sub] for t in out))


# ------------------------------------------------------------- as a decode loop uses it
def test_qsa_compress_incremental_equals_full():
    """Compressing only the newest blocks (pos0 = their first token's position, rows at
    their place in the cache) gives the rows of one full compression, bit for bit."""
    L = 4 * 1000 + 3
    k = inputs.qsa_keys(L, 81, DEV)
    full = torch.empty(L // 4, 128, dtype=torch.bfloat16, device=DEV)
    gdn.gdn_qsa_compress(k, inputs.qsa_offsets([L], DEV), inputs.qsa_offsets([L // 4], DEV),
                         k_hat=full)
    inc = torch.full_like(full, 3.0)
    done = 0
    for upto in (400, 1, 0, 599):                  # blocks compressed by each call
        t0 = 4 * done
        part = k[t0:t0 + 4 * upto]
        view = inc[done:done + upto]
        gdn.gdn_qsa_compress(part, inputs.qsa_offsets([4 * upto], DEV),
                             inputs.qsa_offsets([upto], DEV), k_hat=view,
                             pos0=torch.tensor([t0], dtype=torch.int32, device=DEV))
        done += upto
    torch.cuda.synchronize()
    assert done == L // 4 and torch.equal(inc, full)


def test_qsa_decode_loop_against_oracle():
    """Eight decode steps of one sequence: append a key each step, compress a block when its
    4th token arrives, index the new token's query; every step matches the oracle run on
    the keys so far."""
    T0 = 4 * 3000 + 1
    steps = 8
    keys = inputs.qsa_keys(T0 + steps, 82, DEV)
    qs = inputs.qsa_queries(steps, 83, DEV)
    cap = (T0 + steps) // 4
    k_hat = torch.zeros(cap, 128, dtype=torch.bfloat16, device=DEV)
    nb = T0 // 4
    gdn.gdn_qsa_compress(keys[:4 * nb], inputs.qsa_offsets([4 * nb], DEV),
                         inputs.qsa_offsets([nb], DEV), k_hat=k_hat[:nb])
    ws = gdn.qsa_index_workspace(1, cap)
    for s in range(steps):
        t = T0 + s                                 # position of this step's token
        if (t + 1) % 4 == 0:                       # its block is complete: compress it
            b = t // 4
            gdn.gdn_qsa_compress(keys[4 * b:4 * b + 4], inputs.qsa_offsets([4], DEV),
                                 inputs.qsa_offsets([1], DEV), k_hat=k_hat[b:b + 1],
                                 pos0=torch.tensor([4 * b], dtype=torch.int32, device=DEV))
            nb = b + 1
        cub = inputs.qsa_offsets([nb], DEV)
        q_pos = torch.tensor([t], dtype=torch.int32, device=DEV)
        out = _run_index(qs[s:s + 1], q_pos, k_hat[:nb], cub, 512, ws)
        # the oracle builds its own cache from the raw keys of tokens 0..t (float64); the
        # kernel's cache rounds each element to bf16 (at most 2^-8 of it), which the score
        # tolerance covers on top of the fp32 arithmetic
        ref_rows, _ = O.compress_keys(keys[:4 * nb].float().cpu().numpy(), [0, 4 * nb])
        assert np.all(np.abs(k_hat[:nb].float().cpu().numpy() - ref_rows)
                      <= 2.0 ** -8 * np.abs(ref_rows) + 1e-5)
        _check_index(qs[s:s + 1], q_pos, k_hat[:nb], cub, 512, out, ref_rows=ref_rows,
                     tol_scale=2.0 ** -8 + 8e-6)
