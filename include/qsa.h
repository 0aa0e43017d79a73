/* libgdn: the QSA compressed indexer (C ABI).
 *
 * Operation ("論文解説: Qwen3.8-Next の設計" (ta-paperlens), section "部品②: QSA — 「どこを
 * 見るか」を決める係のコストを下げる"; the budget in blocks from "一个176B模型，每个Token只
 * 激活6B：Qwen3.8-Flash-Next正在重新定义“大模型有多大”", section "GDN + QSA"):
 *
 *   1. the indexer's keys (one key head, 128 dims) are cut into blocks of r = 4 tokens and
 *      each block is averaged, before any positional encoding;
 *   2. the averaged key gets rotary position encoding on its first 64 dims at one
 *      position, the block's first token (pairs (i, i + 32), angle = p * base^(-i/32));
 *      dims 64..127 pass through;
 *   3. a query token's 4 indexer heads (sharing that key head) each get the rotation at
 *      the query's position; the score of a block is the sum over the 4 heads of
 *      query . key;
 *   4. a query keeps its budget of best blocks (2048 tokens = 512 blocks in the paper's
 *      setting), ties to the earlier block; only blocks whose 4 tokens all lie at or
 *      before the query are scored;
 *   5. the kept blocks are expanded to their tokens.
 *
 * Ownership and errors follow gdn.h: the caller owns every buffer (device memory unless
 * stated); nothing allocates, frees or synchronises; argument checks run on the host
 * and return before anything is enqueued.  Inputs must be finite.
 */
#ifndef LIBGDN_QSA_H
#define LIBGDN_QSA_H

#include "gdn.h"

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_QSA_R 4              /* tokens per compressed block                        */
#define GDN_QSA_DIM 128          /* indexer head dimension                             */
#define GDN_QSA_ROPE_DIMS 64     /* dims with rotary encoding (the first 64)           */
#define GDN_QSA_HEADS 4          /* indexer query heads per token                      */
#define GDN_QSA_MAX_BUDGET 4096  /* largest budget_blocks accepted                     */
#define GDN_QSA_MAX_SEQS 4096    /* largest num_seqs x n_queries accepted by the indexer */
#define GDN_QSA_MAX_QUERIES 4    /* largest n_queries of gdn_qsa_index_multi            */

/* Steps 1-2: compress keys into the block cache.
 *   k          : [T_total, 128] bf16, the indexer key of every token (before rotation).
 *   cu_seqlens : DEVICE int32[num_seqs + 1] token offsets (non-decreasing, from 0).
 *   cu_blocks  : DEVICE int32[num_seqs + 1] row offsets of each sequence in k_hat
 *                (non-decreasing, from 0, cu_blocks[num_seqs] == total_blocks).
 *   pos0       : DEVICE int32[num_seqs] absolute position of each sequence's first token,
 *                or NULL for 0 (lets a caller compress only the newest tokens).
 *   k_hat      : [total_blocks, 128] bf16, written: row cu_blocks[n] + b holds block b of
 *                sequence n, pooled from its tokens 4b..4b+3 and rotated at position
 *                pos0[n] + 4b.  Only b < min(cu_blocks[n+1] - cu_blocks[n], len_n / 4) is
 *                written; other rows are left as they are.
 *   rope_base  : rotary base (10000 in the usual setting).
 * k and k_hat 16-byte aligned, the offsets 4-byte aligned.  total_blocks == 0 is a no-op. */
gdn_status gdn_qsa_compress(const void *k, const int32_t *cu_seqlens, const int32_t *cu_blocks,
                            const int32_t *pos0, void *k_hat, int32_t num_seqs,
                            int64_t total_blocks, float rope_base, cudaStream_t stream);

/* Bytes of device workspace gdn_qsa_index_decode needs.  It must be zero-filled before its
 * first use; each call leaves it zeroed again for the next one (zero-fill it again after a
 * call that returned an error). */
size_t gdn_qsa_index_workspace_size(int32_t num_seqs, int64_t total_blocks);

/* Steps 3-5 for one new token per sequence (decode).
 *   q            : [num_seqs, 4, 128] bf16, the indexer query heads (before rotation).
 *   q_pos        : DEVICE int32[num_seqs], absolute position of each query (>= 0); blocks
 *                  b < min(cu_blocks[n+1] - cu_blocks[n], (q_pos[n] + 1) / 4) are scored.
 *   k_hat        : [total_blocks, 128] bf16 block cache laid out as gdn_qsa_compress writes.
 *   cu_blocks    : DEVICE int32[num_seqs + 1] row offsets, as above.
 *   budget_blocks: blocks kept per query, 1..GDN_QSA_MAX_BUDGET.
 *   block_idx    : [num_seqs, budget_blocks] int32, written: kept blocks (indices within
 *                  the sequence) in ascending order, then -1.
 *   block_score  : [num_seqs, budget_blocks] fp32 or NULL: their scores, then -inf.
 *   token_idx    : [num_seqs, 4 * budget_blocks] int32 or NULL: the kept blocks' tokens in
 *                  ascending order, then -1.
 *   workspace    : device scratch of gdn_qsa_index_workspace_size bytes (see there).
 * q and k_hat 16-byte aligned; the rest 4-byte aligned.  num_seqs == 0 is a no-op.
 * Scores are accumulated in fp32; ranking uses those fp32 values. */
gdn_status gdn_qsa_index_decode(const void *q, const int32_t *q_pos, const void *k_hat,
                                const int32_t *cu_blocks, int32_t num_seqs,
                                int64_t total_blocks, int32_t budget_blocks, float rope_base,
                                int32_t *block_idx, float *block_score, int32_t *token_idx,
                                void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Bytes of device workspace gdn_qsa_index_multi needs for n_queries queries per sequence
 * (same zero-fill rule as gdn_qsa_index_workspace_size); 0 for n_queries outside
 * 1..GDN_QSA_MAX_QUERIES. */
size_t gdn_qsa_index_multi_workspace_size(int32_t num_seqs, int64_t total_blocks,
                                          int32_t n_queries);

/* Steps 3-5 for n_queries consecutive tokens per sequence (for instance drafted tokens
 * checked together): query j of sequence n sits at position q_pos[n] + j and is indexed
 * exactly as gdn_qsa_index_decode indexes a single query there, with its own causal cut.
 * Each cache row is read once for all of a sequence's queries.
 *   q          : [num_seqs, n_queries, 4, 128] bf16.
 *   block_idx  : [num_seqs, n_queries, budget_blocks] int32, written.
 *   block_score: [num_seqs, n_queries, budget_blocks] fp32 or NULL.
 *   token_idx  : [num_seqs, n_queries, 4 * budget_blocks] int32 or NULL.
 *   workspace  : gdn_qsa_index_multi_workspace_size bytes.
 * The other arguments are those of gdn_qsa_index_decode.  GDN_ERR_UNSUPPORTED for
 * n_queries outside 1..GDN_QSA_MAX_QUERIES or num_seqs x n_queries > GDN_QSA_MAX_SEQS. */
gdn_status gdn_qsa_index_multi(const void *q, const int32_t *q_pos, const void *k_hat,
                               const int32_t *cu_blocks, int32_t num_seqs, int64_t total_blocks,
                               int32_t n_queries, int32_t budget_blocks, float rope_base,
                               int32_t *block_idx, float *block_score, int32_t *token_idx,
                               void *workspace, size_t workspace_bytes, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBGDN_QSA_H */
