// Launchers of the MSA kernels, called by the C-ABI layer (msa_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace msa {

// Problem description after validation; strides in elements.
struct Shape {
  int batch, n_q, max_kv, H, h, G, d, d_idx, block, topk, nblk;
  int causal, force_own;
  float scale;
  const int32_t* seq_lens;
  int64_t q_s[3], k_s[3], v_s[3], qi_s[3], ki_s[2], o_s[3];
  KvPages pages;  // table == nullptr: contiguous K/V/K_idx
};

// Stage 1a/1b: block-max-pooled index scores, fp32 [batch, n_q, h, nblk].
// Blocks past a row's frontier are written -inf only when fill_tail is set.
cudaError_t launch_index_scores(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                float* scores, bool fill_tail, DeviceStatus* st,
                                cudaStream_t stream);

// Stage 1a/1b for prefill on tcgen05 (d_idx 64 or 128, n_q > 1).
bool index_scores_tc_supported(const Shape& s);
cudaError_t launch_index_scores_tc(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                   float* scores, bool fill_tail, DeviceStatus* st,
                                   cudaStream_t stream);

// Stage 1 in one kernel for prefill (d_idx 64/128, block 64/128, topk <= 64): the
// index GEMM keeps a per-row top-k in shared memory; block scores written only
// when `scores` is given (every block, -inf past the frontier).
bool index_topk_tc_supported(const Shape& s);
cudaError_t launch_index_topk_tc(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                 int32_t* ids, float* scores, DeviceStatus* st,
                                 cudaStream_t stream);

// Stage 1c: top-k block ids, int32 [batch, n_q, h, topk], from the scores.  When
// `zero` is given, the kernel also clears zero[0, nzero) (the attention's merge
// counters, so that a fused forward needs no separate memset between the stages).
// `kept` (nullable) receives the score of each kept id, -inf for padding.
cudaError_t launch_topk(const Shape& s, const float* scores, int32_t* ids, DeviceStatus* st,
                        cudaStream_t stream, int* zero = nullptr, int nzero = 0,
                        float* kept = nullptr);

// Global top-k from the candidate lists of KV shards (sequence-sharded decode):
// cscores / cids [nlists, rows, len], list r ascending ids local to the shard
// starting at block r * shard_blocks; writes global ids and/or the ids local to
// the shard [base, base + nloc) (-1 elsewhere).  nlists * len <= 16384.
cudaError_t launch_candidates_topk(const Shape& s, int nlists, int len, int shard_blocks,
                                   const float* cscores, const int32_t* cids, int base, int nloc,
                                   int32_t* ids, int32_t* local, DeviceStatus* st,
                                   cudaStream_t stream);

// LSE merge of `nparts` partial results of the same rows: part_out bf16
// [nparts, rows * H, d] (dense), part_lse fp32 [nparts, rows * H]; out with the
// shape's output strides, lse (nullable) dense [rows * H].
cudaError_t launch_merge_partials(const Shape& s, int nparts, const uint16_t* part_out,
                                  const float* part_lse, uint16_t* out, float* lse,
                                  cudaStream_t stream);

// Token lengths of the shard [base, base + len) of each sequence:
// out[b] = clamp(L_b - base, 0, len).
cudaError_t launch_shard_lengths(const int32_t* seq_lens, int batch, int max_kv, int64_t base,
                                 int64_t len, int32_t* out, DeviceStatus* st, cudaStream_t stream);

// Decode-step cache write: the n_q new tokens of every sequence (dense
// [batch, n_q, h, d] K and V, [batch, n_q, d_idx] K_idx; any may be null) go to
// positions L_b - n_q + t of the contiguous or paged cache.
cudaError_t launch_append_kv(const Shape& s, const uint16_t* k_new, const uint16_t* v_new,
                             const uint16_t* ki_new, uint16_t* k, uint16_t* v, uint16_t* ki,
                             DeviceStatus* st, cudaStream_t stream);

// Stage 2: workspace bytes for the split-KV partials, then the attention.
size_t attn_partial_bytes(const Shape& s);
int attn_launches(const Shape& s);
// The streaming (decode) kernel's per-row merge counters inside `partials`, or
// nullptr when the shape takes another kernel; *count receives their number.
int* attn_merge_counters(const Shape& s, void* partials, int* count);
// Merge counters: `fixed_counters` (kFixedCounters words that are zero between
// calls, nullable) when the shape needs no more of them; otherwise the ones in
// `partials`, cleared by a memset unless `counters_zeroed` (the top-k kernel of
// the same forward cleared them already).  The kernel puts every counter it uses
// back to zero.
cudaError_t launch_sparse_attn(const Shape& s, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const int32_t* ids, uint16_t* out, float* lse,
                               void* partials, size_t partial_bytes, DeviceStatus* st,
                               cudaStream_t stream, bool counters_zeroed = false,
                               int* fixed_counters = nullptr);

// Stage 2 for prefill, KV-major on tcgen05 (d 64/128, block 64/128, n_q > 1):
// inverted index, tiles of gathered (query, head) rows per selected block,
// partials merged by a combine kernel; processed in query chunks.
bool kv_attn_supported(const Shape& s);
// Rows of d bf16 as a 2-D tensor map with 64 x 32 boxes (128-byte swizzle), for
// TMA stores of partial outputs.
bool make_rows_map(CUtensorMap* map, uint16_t* base, int64_t rows, int d);
size_t kv_workspace_bytes(const Shape& s);
int kv_launches(const Shape& s);
cudaError_t launch_kv_attn(const Shape& s, const CUtensorMap& tmq, const CUtensorMap& tmk,
                           const CUtensorMap& tmv,
                           const uint16_t* q, const int32_t* ids, uint16_t* out, float* lse,
                           void* ws, size_t ws_bytes, DeviceStatus* st, cudaStream_t stream);

// Test hook: one bounded wait that runs out and records kErrTimeout.
cudaError_t launch_wait_timeout_probe(DeviceStatus* st, uint64_t wait_ns, cudaStream_t stream);

int num_sms();
int max_smem_optin();

// cuTensorMapEncodeTiled from the driver (nullptr when the driver lacks it).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();

}  // namespace msa
