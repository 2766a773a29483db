/*
 * msa.h - C ABI of libmsa.so: MiniMax Sparse Attention (MSA) on B200 (sm_100a).
 *
 * MSA is two-stage block-sparse GQA attention:
 *   stage 1, the index branch: one index query per GQA group is scored against a
 *     single-head index key shared by all heads; token scores are max-pooled into
 *     per-block scores under the causal mask, and a top-k picks the KV blocks of
 *     each (query, group).  Sources: "MiniMax goes sparse" (atlascloud.ai),
 *     section 1, step 1; "MiniMax M3 的 MSA 与阶跃 Step 3.7 Flash 的 MFA"
 *     (ai.air7.fun), section "MSA：稀疏注意力的一种极简实现", first layer.
 *   stage 2, the sparse branch: exact softmax attention over the raw K/V of only
 *     the selected blocks; all query heads of a group share the group's
 *     selection.  Sources: the same sections, step 2 / second layer.
 *
 * Shapes and notation
 *   batch         number of sequences b
 *   n_q           query tokens per sequence (n_q = 1 is one decode step)
 *   max_kv        token capacity of the K/V buffers (allocated length)
 *   seq_lens[b]   KV length L_b of sequence b (device int32; NULL: all = max_kv)
 *   H, h          query heads and KV heads; h is also the number of index groups;
 *                 G = H / h heads per group, head hq belongs to group hq / G
 *   d, d_idx      head dim of q/k/v and of q_idx/k_idx
 *   block         tokens per KV block B; nblk = ceil(max_kv / B)
 *   topk          blocks kept per (query, group)
 *   Query t of sequence b sits at absolute position p = L_b - n_q + t.
 *
 * Tensor layouts (element strides given in msa_params_t; the innermost axis is
 * always contiguous):
 *   q      bf16 [batch, n_q, H, d]          k, v   bf16 [batch, max_kv, h, d]
 *   q_idx  bf16 [batch, n_q, h, d_idx]      k_idx  bf16 [batch, max_kv, d_idx]
 *   out    bf16 [batch, n_q, H, d]
 *   block_ids    int32 [batch, n_q, h, topk]   dense, row-major
 *   block_scores fp32  [batch, n_q, h, nblk]   dense, row-major
 *   lse          fp32  [batch, n_q, H]         dense, row-major (natural log)
 *
 * Paged KV cache (optional; block_table != NULL): k, v and k_idx are pools of
 * pages of `block` tokens each,
 *   k, v   bf16 [num_pages, block, h, d]    k_idx  bf16 [num_pages, block, d_idx]
 * with k/v_strides = [page, token in page, kv head] and ki_strides = [page, token
 * in page], and block_table (device int32 [batch, table_stride]) gives the page of
 * each logical block: block_table[b * table_stride + beta] holds tokens
 * [beta * block, (beta + 1) * block) of sequence b.  Only rows beta <
 * ceil(L_b / block) are read, so table_stride >= ceil(max_kv / block).  A page
 * id outside [0, num_pages) is recorded as MSA_ERR_DEVICE_ASSERT and that block
 * reads as zeros.  Results are the same as with the contiguous layout.
 *
 * Supported sizes: d in {64, 128}; d_idx in {32, 64, 128}; block in {16, 32, 64,
 * 128}; 1 <= G <= 16; 1 <= topk <= 4096; h <= 16; n_q <= max_kv; all base pointers
 * 16-byte aligned and every outer stride a multiple of 8 elements.  Anything else
 * returns MSA_ERR_UNSUPPORTED (or MSA_ERR_INVALID_ARG for inconsistent input).
 * There is no CPU fallback.
 *
 * Ownership and execution
 *   The caller owns every buffer, the workspace included; the library allocates
 *   no memory and keeps no state between calls (one exception:
 *   msa_sparse_attn_noalloc below uses a fixed array in the library's own device
 *   memory and remembers that array's address per device).  All pointers except `params`
 *   are device pointers.  Calls are asynchronous on `stream`: argument errors
 *   return before anything is launched, launch failures return MSA_ERR_CUDA, and
 *   errors found on the device (a bounded wait that ran out, an id out of range)
 *   are recorded in a sticky word at the start of the workspace that
 *   msa_get_device_status() reads.  Calls that share a workspace must be ordered
 *   on one stream.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

typedef uint16_t msa_bf16_t;          /* raw bf16 bits */
typedef struct CUstream_st* msa_stream_t; /* same handle as cudaStream_t; NULL = legacy default */

typedef enum msa_status {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,   /* null pointer, inconsistent shape, bad stride */
  MSA_ERR_UNSUPPORTED = 2,   /* a size outside the supported set above */
  MSA_ERR_WORKSPACE = 3,     /* workspace null, misaligned or smaller than msa_workspace_size() */
  MSA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  MSA_ERR_TIMEOUT = 5,       /* device: a bounded wait in a kernel ran out */
  MSA_ERR_DEVICE_ASSERT = 6  /* device: an input broke a precondition (e.g. block id >= nblk) */
} msa_status_t;

typedef enum msa_op {
  MSA_OP_INDEX_SELECT = 0,
  MSA_OP_SPARSE_ATTN = 1,
  MSA_OP_FORWARD = 2,
  MSA_OP_APPEND_KV = 3,
  MSA_OP_BLOCK_SCORES = 4,
  MSA_OP_INDEX_CANDIDATES = 5,
  MSA_OP_SELECT_CANDIDATES = 6,
  MSA_OP_SHARD_LENGTHS = 7,
  MSA_OP_INDEX_TOPK = 8
} msa_op_t;

typedef struct msa_params {
  int32_t batch, n_q, max_kv, H, h, d, d_idx, block, topk;
  int32_t causal;          /* 1: query at p sees tokens j <= p; 0: all j < L_b */
  int32_t force_own_block; /* 1: the block holding p is always selected */
  float softmax_scale;     /* <= 0 selects 1/sqrt(d) */
  const int32_t* seq_lens; /* device [batch]; NULL means every L_b = max_kv */
  int64_t q_strides[3];    /* q:     [b, t, head]  strides in elements */
  int64_t k_strides[3];    /* k:     [b, token, kv head] */
  int64_t v_strides[3];    /* v:     [b, token, kv head] */
  int64_t qi_strides[3];   /* q_idx: [b, t, group] */
  int64_t ki_strides[2];   /* k_idx: [b, token] */
  int64_t o_strides[3];    /* out:   [b, t, head] */
  /* paged K/V/K_idx (see above); block_table NULL means contiguous tensors */
  const int32_t* block_table; /* device [batch, table_stride] */
  int64_t table_stride;       /* entries per sequence row of block_table */
  int64_t num_pages;          /* pages in each of the k, v and k_idx pools */
} msa_params_t;

/* Bytes of workspace `op` needs for these shapes (0 on invalid params).  The
 * workspace must be 256-byte aligned.  It starts with a 4096-byte status region
 * (the sticky device status word and the decode attention's per-row merge
 * counters, which are zero between calls) and holds, when the caller does not
 * supply them, block scores and block ids, plus the split-KV partial results of
 * the attention. */
MSA_API size_t msa_workspace_size(const msa_params_t* params, msa_op_t op);

/* Stage 1 (index branch).  For every (b, t, g):
 *   S[beta] = max over visible tokens j of block beta of <q_idx[b,t,g,:], k_idx[b,j,:]>
 *   (unscaled fp32 dot products of bf16 inputs; visible = j < L_b and, when causal,
 *   j <= p; blocks with no visible token score -inf), then the top-k blocks by
 *   (score descending, block id ascending), the own block first when forced.
 *   block_ids receives min(topk, F) ids in ascending order followed by -1 padding,
 *   F being the number of blocks with a visible token.
 *   block_scores (nullable) receives S for every block (-inf past the frontier).
 * Sources: "MiniMax goes sparse" section 1 step 1; "MiniMax M3 的 MSA ..." first layer. */
MSA_API msa_status_t msa_index_select(const msa_params_t* params, const msa_bf16_t* q_idx,
                              const msa_bf16_t* k_idx, int32_t* block_ids,
                              float* block_scores, void* workspace, size_t workspace_bytes,
                              msa_stream_t stream);

/* Stage 2 (sparse branch).  For every (b, t, hq) with g = hq / G:
 *   keys J = tokens j of the blocks in block_ids[b,t,g,:] (entries < 0 are empty
 *   slots, any order, no repeats) with j < L_b and, when causal, j <= p;
 *   out = softmax(scale * q . k_J^T) v_J  (fp32 softmax and accumulation, bf16 out),
 *   lse (nullable) = log sum_j exp(scale * q . k_j); rows with no key get out = 0,
 *   lse = -inf.  Ids >= nblk are skipped and flagged MSA_ERR_DEVICE_ASSERT.
 * Works for prefill (n_q > 1) and decode (n_q = 1).
 * Sources: "MiniMax goes sparse" section 1 step 2; "MiniMax M3 的 MSA ..." second layer. */
MSA_API msa_status_t msa_sparse_attn(const msa_params_t* params, const msa_bf16_t* q,
                             const msa_bf16_t* k, const msa_bf16_t* v,
                             const int32_t* block_ids, msa_bf16_t* out, float* lse,
                             void* workspace, size_t workspace_bytes, msa_stream_t stream);

/* Both stages in one call: msa_index_select followed by msa_sparse_attn on its ids.
 * block_ids, block_scores and lse are optional outputs (nullable). */
MSA_API msa_status_t msa_forward(const msa_params_t* params, const msa_bf16_t* q, const msa_bf16_t* k,
                         const msa_bf16_t* v, const msa_bf16_t* q_idx, const msa_bf16_t* k_idx,
                         msa_bf16_t* out, int32_t* block_ids, float* block_scores, float* lse,
                         void* workspace, size_t workspace_bytes, msa_stream_t stream);

/* Decode-step cache write, so that a step needs no per-row copies: for every
 * sequence b and new token t < n_q (params->n_q new tokens per sequence, already
 * counted in seq_lens), at position pos = L_b - n_q + t:
 *   k[b, pos, g, :] = k_new[b, t, g, :]   v[b, pos, g, :] = v_new[b, t, g, :]
 *   k_idx[b, pos, :] = k_idx_new[b, t, :]
 * k_new, v_new: bf16 [batch, n_q, h, d] and k_idx_new: bf16 [batch, n_q, d_idx],
 * dense row-major and 16-byte aligned; any of the three may be NULL (that cache
 * is not written, and its cache pointer may then be NULL).  k, v, k_idx and their
 * strides (k_strides, v_strides, ki_strides) are those the other calls take,
 * paged caches included (row pos % block of page block_table[b, pos / block]).
 * A position < 0 or a page id outside the pool is recorded as
 * MSA_ERR_DEVICE_ASSERT and that token is not written.  The workspace holds the
 * status region only (msa_workspace_size(params, MSA_OP_APPEND_KV) bytes).
 * The cache keeps the plain GQA layout ("MiniMax M3 的 MSA ...", section
 * "三条有意为之的减法", first item), one block per physical block ("深度解析M3多模态
 * 模型与Token Plan", list of MSA's innovations, first item). */
MSA_API msa_status_t msa_append_kv(const msa_params_t* params, const msa_bf16_t* k_new,
                                   const msa_bf16_t* v_new, const msa_bf16_t* k_idx_new,
                                   msa_bf16_t* k, msa_bf16_t* v, msa_bf16_t* k_idx,
                                   void* workspace, size_t workspace_bytes, msa_stream_t stream);

/* Stage 1, first half: the block scores alone (the index scan with its fused
 * causal block max pool, no top-k).  block_scores fp32 [batch, n_q, h, nblk]
 * receives S for every block, -inf past each row's frontier, exactly as
 * msa_index_select's optional output.  The workspace holds the status region only
 * (msa_workspace_size(params, MSA_OP_BLOCK_SCORES)).
 * Sources: "MiniMax goes sparse" section 1 step 1 (Q_idx . K_idx^T and the Block
 * Max Pool); "MiniMax M3 的 MSA ..." first layer. */
MSA_API msa_status_t msa_block_scores(const msa_params_t* params, const msa_bf16_t* q_idx,
                                      const msa_bf16_t* k_idx, float* block_scores,
                                      void* workspace, size_t workspace_bytes,
                                      msa_stream_t stream);

/* Stage 1 in one kernel for prefill: msa_index_select's ids (same order, same
 * ties, same padding) with the top-k kept in the index GEMM's epilogue, so that
 * the block scores need not be written at all (block_scores, nullable, still
 * receives them when given).  Each (query, group) row keeps its best blocks in a
 * heap in shared memory while the key tiles stream past.  Supported: n_q > 1,
 * d_idx 64 or 128, block 64 or 128, topk <= 64, else MSA_ERR_UNSUPPORTED.  The
 * workspace holds the status region only (msa_workspace_size(params,
 * MSA_OP_INDEX_TOPK)).  Sources: "MiniMax goes sparse" section 1 step 1; the
 * streaming top-k is the idea of "混合块注意力机制(MoBA)原理与实现详解" section
 * 3.1, kernel 2 (top-k lists in on-chip memory instead of the score matrix in HBM). */
MSA_API msa_status_t msa_index_topk(const msa_params_t* params, const msa_bf16_t* q_idx,
                                    const msa_bf16_t* k_idx, int32_t* block_ids,
                                    float* block_scores, void* workspace, size_t workspace_bytes,
                                    msa_stream_t stream);

/* Sequence-sharded decode.  The KV cache of every sequence is split into
 * contiguous token shards of a whole number of blocks, one per GPU; shard r holds
 * tokens [base_r, base_r + len_r) of every sequence.  The pages do not shard MSA;
 * these four calls split one decode step (n_q = 1) so that the result equals the
 * single-device result ("MiniMax goes sparse" section 1, steps 1 and 2):
 *   1. msa_shard_lengths: each sequence's token count inside this shard.
 *   2. msa_index_candidates on this shard's cache (params with the shard's
 *      lengths and capacity, force_own_block = 0): the shard's own top-k block ids
 *      (shard-local numbering) and their scores.  The lists of all shards are
 *      gathered in shard order and
 *   3. msa_select_candidates with the whole problem's params: the global top-k of
 *      each row (the global top-k blocks are each in the top-k of their shard),
 *      and the ids of the winners inside this shard in shard-local numbering.
 *   4. msa_sparse_attn on this shard with those local ids (a row with no winner
 *      here gets out = 0, lse = -inf), then the (out, lse) pairs of all shards are
 *      gathered and msa_merge_partials weights them by their log-sum-exps.
 * block_sparse_gqa_03_b200/seqshard.py runs these steps with NCCL all-gathers. */

/* shard_lens[b] = clamp(L_b - token_base, 0, token_count) (device int32 [batch]),
 * L_b from params->seq_lens (NULL: max_kv).  Workspace: the status region
 * (msa_workspace_size(params, MSA_OP_SHARD_LENGTHS)). */
MSA_API msa_status_t msa_shard_lengths(const msa_params_t* params, int64_t token_base,
                                       int64_t token_count, int32_t* shard_lens,
                                       void* workspace, size_t workspace_bytes,
                                       msa_stream_t stream);

/* msa_index_select plus the score of every kept block: block_ids int32 [batch,
 * n_q, h, topk] as msa_index_select writes them (ascending, -1 padding) and
 * kept_scores fp32 [batch, n_q, h, topk] = S[block_ids] (-inf for padding).
 * Workspace: msa_workspace_size(params, MSA_OP_INDEX_CANDIDATES) bytes. */
MSA_API msa_status_t msa_index_candidates(const msa_params_t* params, const msa_bf16_t* q_idx,
                                          const msa_bf16_t* k_idx, int32_t* block_ids,
                                          float* kept_scores, void* workspace,
                                          size_t workspace_bytes, msa_stream_t stream);

/* Top-k of each row (b, t, g) from candidate blocks, in msa_index_select's order:
 * score descending, block id ascending, and with params->force_own_block the
 * block holding position p = L_b - n_q + t first (also when no list holds it).
 *   cand_scores fp32 / cand_ids int32 [nlists, batch, n_q, h, list_len]: the
 *     lists of the shards in shard order, as an all-gather of every shard's
 *     msa_index_candidates output leaves them.  List r holds ascending ids local
 *     to shard r (global id = id + r * shard_blocks), -1 for empty entries;
 *     1 <= nlists * list_len <= 16384.
 *   block_ids (nullable) int32 [batch, n_q, h, topk]: the global winners,
 *     ascending, -1 padded (m = min(topk, listed candidates plus the forced block)).
 *   local_ids (nullable) int32 [batch, n_q, h, topk]: slot by slot, id -
 *     block_base when block_base <= id < block_base + nblk_local, else -1.
 * params: the whole problem (global seq_lens and max_kv, h, block, topk,
 * force_own_block).  Workspace: the status region
 * (msa_workspace_size(params, MSA_OP_SELECT_CANDIDATES)). */
MSA_API msa_status_t msa_select_candidates(const msa_params_t* params, int32_t nlists,
                                           int32_t list_len, int32_t shard_blocks,
                                           const float* cand_scores, const int32_t* cand_ids,
                                           int32_t block_base, int32_t nblk_local,
                                           int32_t* block_ids, int32_t* local_ids,
                                           void* workspace, size_t workspace_bytes,
                                           msa_stream_t stream);

/* Merge of nparts attention results over disjoint key sets of the same rows:
 *   part_out bf16 [nparts, batch, n_q, H, d] and part_lse fp32 [nparts, batch,
 *   n_q, H] (dense; a part with lse = -inf saw no key of the row);
 *   out = sum_r e^(lse_r - M) out_r / sum_r e^(lse_r - M), M = max_r lse_r,
 *   written with params->o_strides; lse (nullable, dense [batch, n_q, H]) =
 *   M + log sum_r e^(lse_r - M).  Rows no part saw: out = 0, lse = -inf.
 * Uses params batch, n_q, H, d and o_strides; no workspace. */
MSA_API msa_status_t msa_merge_partials(const msa_params_t* params, int32_t nparts,
                                        const msa_bf16_t* part_out, const float* part_lse,
                                        msa_bf16_t* out, float* lse, msa_stream_t stream);

/* Synchronises `stream`, returns the first error a kernel recorded in this
 * workspace since the last reset (MSA_OK if none) and, after an error, clears the
 * workspace's 4096-byte status region (the word, and the merge counters that a
 * call which stopped early may have left set). */
MSA_API msa_status_t msa_get_device_status(void* workspace, msa_stream_t stream);

/* Zeroes the workspace's 4096-byte status region, asynchronously on `stream`.
 * Call it once on every new workspace before its first use.  The region holds the
 * sticky status word (kernels only ever set it, msa_get_device_status() clears
 * it) and the decode attention's merge counters (each call leaves them at zero). */
MSA_API msa_status_t msa_workspace_init(void* workspace, size_t workspace_bytes, msa_stream_t stream);

/* Self-test of the device error path: launches one tiny kernel that waits, with
 * a bound of `wait_ns` nanoseconds, on a barrier that nothing completes, so the
 * wait runs out and records MSA_ERR_TIMEOUT in the workspace; nothing faults or
 * hangs.  Read the result with msa_get_device_status(). */
MSA_API msa_status_t msa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint64_t wait_ns,
                                       msa_stream_t stream);

/* msa_sparse_attn without a workspace, for callers that cannot allocate device
 * memory: code running where an allocation is forbidden or would stall the GPU
 * (an inference engine's enqueue path, a real-time loop, a host framework that
 * owns every allocation), which therefore cannot provide the workspace that
 * msa_sparse_attn needs for its intermediate results.  This entry point has no
 * counterpart in the pages; it is a deployment convenience.
 *   - Same arguments and results as msa_sparse_attn, minus the workspace.  The
 *     caller still passes inputs and outputs.
 *   - The intermediates live in one fixed 8 MiB array in the library's own
 *     device memory (every GPU that loads libmsa.so holds it until the process
 *     exits): the split-KV partials of decode-like shapes (batch * n_q * H *
 *     splits * (d + 1) * 4 bytes) and, for prefill with d 64/128 and block
 *     64/128, the inverted index and the per-block partial outputs of the
 *     KV-major kernel (about n_q * h * topk * (G * (2 * d + 4) + 13) bytes per
 *     sequence, plus 2 * d * 128 bytes per (group, block)), so only small
 *     prefills fit.  Prefill with block 16/32 needs none.  Whatever does not
 *     fit returns MSA_ERR_WORKSPACE before anything is launched
 *     (msa_workspace_size(params, MSA_OP_SPARSE_ATTN) minus 4096 is the need).
 *   - All calls share that array and it keeps the last call's contents (the
 *     parts that must start at zero are cleared on the stream by every call):
 *     calls whose work overlaps on the GPU (two streams, or two host threads)
 *     race and must be serialised by the caller.
 *   - The first call on a device looks up the array's device address; make that
 *     first call before any stream capture.
 *   - Device-side precondition failures (ids >= nblk, lengths outside
 *     [0, max_kv]) are skipped but not recorded, as there is no status word. */
MSA_API msa_status_t msa_sparse_attn_noalloc(const msa_params_t* params, const msa_bf16_t* q,
                                             const msa_bf16_t* k, const msa_bf16_t* v,
                                             const int32_t* block_ids, msa_bf16_t* out,
                                             float* lse, msa_stream_t stream);

/* Number of kernel launches `op` makes on the stream for these shapes (its
 * plan depends on the current device's SM count); -1 on invalid params. */
MSA_API int msa_launch_count(const msa_params_t* params, msa_op_t op);

/* A static description of a status code. */
MSA_API const char* msa_status_string(msa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
