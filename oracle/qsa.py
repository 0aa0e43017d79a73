"""CPU oracle for the QSA compressed indexer — TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py may
import this module; the CUDA library never calls it and shares no code with it.

What it computes ("論文解説: Qwen3.8-Next の設計" (ta-paperlens), section
"部品②: QSA — 「どこを見るか」を決める係のコストを下げる"; the budget in blocks is from
"一个176B模型，每个Token只激活6B：Qwen3.8-Flash-Next正在重新定义“大模型有多大”", section
"GDN + QSA：长上下文开始从“完整注意力”转向分工架构"):

  1. the indexer's key sequence is cut into blocks of r = 4 tokens and each block is
     mean-pooled, BEFORE any positional encoding;
  2. each pooled block key then gets partial RoPE (64 of its 128 dimensions) at ONE
     position, the block's first token;
  3. the indexer is multi-query: 4 query heads share the one key head; a query token
     scores every block it may see, one score per block;
  4. the best blocks are kept within the token budget K = 2048 tokens = 512 blocks;
  5. the kept blocks are expanded back to their tokens.

Readings where the section is silent (each one is also pinned by a test):
  * RoPE pairs dimension i with i + rope_dims/2 (rotate-half) over the FIRST rope_dims
    dimensions, angle = position * base^(-2i/rope_dims), base = 10000; the remaining
    dimensions pass through.  The query heads get RoPE at the query's own position.
  * The four heads' logits are summed (plain multi-query logits, no weights and no
    nonlinearity; the pages give none).  Any positive scale leaves the choice unchanged,
    so none is applied.
  * Causality: a block may be scored by the query at position t only when all r of its
    tokens are at or before t (r b + r - 1 <= t), since its pooled key mixes all r.
  * Ties between equal scores go to the earlier block.  Kept blocks are reported in
    ascending block order, each with its score; tokens in ascending order.

Everything is float64 numpy; positions are integers.  Functions take the
indexer key sequence per token ``k`` [T_total, D] (one key head), sequence offsets
``cu_seqlens`` [N+1], and for the decode indexer one query per sequence ``q``
[N, H, D] at absolute position ``q_pos`` [N].
"""
from __future__ import annotations

import numpy as np

R = 4                  # tokens per compressed block (compression ratio r)
D = 128                # indexer head dimension
ROPE_DIMS = 64         # dimensions that get rotary position encoding
HEADS = 4              # indexer query heads sharing one key head
TOKEN_BUDGET = 2048    # tokens kept per query (K)
BLOCK_BUDGET = TOKEN_BUDGET // R
ROPE_BASE = 10000.0


def rope_partial(x, pos, rope_dims: int = ROPE_DIMS, base: float = ROPE_BASE):
    """Rotary encoding of the first ``rope_dims`` dims of x [..., D] at integer positions
    ``pos`` (broadcast against x's leading dims); dims >= rope_dims pass through."""
    x = np.asarray(x, np.float64)
    out = x.copy()
    if rope_dims == 0:
        return out
    half = rope_dims // 2
    inv_freq = base ** (-2.0 * np.arange(half, dtype=np.float64) / rope_dims)
    ang = np.asarray(pos, np.float64)[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:rope_dims]
    out[..., :half] = x1 * c - x2 * s
    out[..., half:rope_dims] = x2 * c + x1 * s
    return out


def blocks_of(seq_len: int, r: int = R) -> int:
    """Whole blocks in a sequence of ``seq_len`` tokens (a trailing partial block is not
    compressed yet)."""
    return int(seq_len) // r


def compress_keys(k, cu_seqlens, pos0=None, r: int = R, rope_dims: int = ROPE_DIMS,
                  base: float = ROPE_BASE):
    """Step 1-2: mean-pool r tokens per block, then RoPE at the block's first position.

    k [T_total, D]; sequence n spans tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 and its
    first token sits at absolute position pos0[n] (0 when pos0 is None).  Returns
    (k_hat [total_blocks, D] float64, cu_blocks [N+1] int64), block b of sequence n at
    row cu_blocks[n] + b, pooled from tokens cu_seqlens[n] + r b .. + r - 1 and placed
    at position pos0[n] + r b."""
    k = np.asarray(k, np.float64)
    cu = np.asarray(cu_seqlens, np.int64)
    N = len(cu) - 1
    p0 = np.zeros(N, np.int64) if pos0 is None else np.asarray(pos0, np.int64)
    nbs = [blocks_of(cu[n + 1] - cu[n], r) for n in range(N)]
    cu_blocks = np.concatenate([[0], np.cumsum(nbs)]).astype(np.int64)
    out = np.zeros((int(cu_blocks[-1]), k.shape[1]), np.float64)
    for n in range(N):
        for b in range(nbs[n]):
            t0 = cu[n] + r * b
            pooled = k[t0:t0 + r].mean(axis=0)
            out[cu_blocks[n] + b] = rope_partial(pooled, p0[n] + r * b, rope_dims, base)
    return out, cu_blocks


def eligible_blocks(n_blocks: int, q_pos: int, r: int = R) -> int:
    """Blocks 0 .. e-1 of a cache of n_blocks may be scored by a query at q_pos."""
    return max(0, min(int(n_blocks), (int(q_pos) + 1) // r))


def block_scores(q, q_pos: int, k_hat, rope_dims: int = ROPE_DIMS, base: float = ROPE_BASE):
    """Step 3 for one query token: q [H, D] (before RoPE), k_hat [nb, D] (encoded).
    Score of block b = sum over heads h of RoPE(q_h, q_pos) . k_hat_b."""
    qh = rope_partial(q, np.full(q.shape[0], q_pos), rope_dims, base)
    k_hat = np.asarray(k_hat, np.float64)
    s = np.zeros(k_hat.shape[0], np.float64)
    for h in range(qh.shape[0]):
        # each row's dot product by the same elementwise reduction, so that equal rows
        # score exactly equal (a matrix-vector library call may round rows differently by
        # position, which would break exact ties by noise)
        s += (k_hat * qh[h]).sum(axis=1)
    return s


def select_blocks(scores, budget: int):
    """Step 4: the ``budget`` best blocks (ties to the earlier block), ascending."""
    scores = np.asarray(scores, np.float64)
    order = sorted(range(len(scores)), key=lambda b: (-scores[b], b))
    return np.array(sorted(order[:budget]), np.int64)


def expand_tokens(blocks, r: int = R):
    """Step 5: block b -> tokens r b .. r b + r - 1, ascending."""
    return np.array([r * int(b) + j for b in blocks for j in range(r)], np.int64)


def index_decode(q, q_pos, k_hat, cu_blocks, budget_blocks: int = BLOCK_BUDGET,
                 r: int = R, rope_dims: int = ROPE_DIMS, base: float = ROPE_BASE):
    """The indexer for one new token per sequence.

    q [N, H, D]; q_pos [N] absolute position of each query; k_hat [total_blocks, D] the
    compressed cache, sequence n in rows cu_blocks[n] .. cu_blocks[n+1]-1 (block b of a
    sequence covers its tokens r b .. r b + r - 1).  Returns
      block_idx [N, budget]      kept blocks ascending, -1 after the last;
      block_score [N, budget]    their scores, -inf after the last;
      token_idx [N, r budget]    their tokens ascending, -1 after the last."""
    q = np.asarray(q, np.float64)
    cb = np.asarray(cu_blocks, np.int64)
    N = q.shape[0]
    bi = np.full((N, budget_blocks), -1, np.int64)
    bs = np.full((N, budget_blocks), -np.inf, np.float64)
    ti = np.full((N, r * budget_blocks), -1, np.int64)
    for n in range(N):
        e = eligible_blocks(cb[n + 1] - cb[n], int(q_pos[n]), r)
        s = block_scores(q[n], int(q_pos[n]), np.asarray(k_hat)[cb[n]:cb[n] + e], rope_dims, base)
        kept = select_blocks(s, budget_blocks)
        bi[n, :len(kept)] = kept
        bs[n, :len(kept)] = s[kept]
        tok = expand_tokens(kept, r)
        ti[n, :len(tok)] = tok
    return bi, bs, ti


def index_multi(q, q_pos, k_hat, cu_blocks, budget_blocks: int = BLOCK_BUDGET, r: int = R,
                rope_dims: int = ROPE_DIMS, base: float = ROPE_BASE):
    """T consecutive query tokens per sequence against one cache (drafted tokens checked
    together): q [N, T, H, D]; query j of sequence n sits at position q_pos[n] + j and is
    indexed exactly as a single query there (index_decode), with its own causal cut.
    Returns block_idx [N, T, budget], block_score [N, T, budget], token_idx [N, T, r budget]."""
    q = np.asarray(q, np.float64)
    N, T = q.shape[0], q.shape[1]
    outs = [index_decode(q[:, j], np.asarray(q_pos, np.int64) + j, k_hat, cu_blocks,
                         budget_blocks, r, rope_dims, base) for j in range(T)]
    return tuple(np.stack([o[i] for o in outs], axis=1) for i in range(3))
