// C ABI of libmsa.so (declared in include/msa.h): argument validation, workspace
// carve-up and launch sequencing on the caller's stream.  No allocation, no
// host synchronisation (except msa_get_device_status), no CPU fallback.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/msa.h"
#include "kernels.h"

namespace msa {

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Largest dynamic shared memory a CTA may opt in to (227 KB on sm_100).
int max_smem_optin() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 232448;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        n <= 0)
      n = 232448;
    cached[dev] = n;
  }
  return cached[dev];
}

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

namespace {

__global__ void wait_timeout_probe_kernel(DeviceStatus* st, uint64_t wait_ns) {
  __shared__ uint64_t bar;
  const uint32_t addr = smem_u32(&bar);
  mbar_init(addr, 1);
  fence_mbar_init();
  // Nothing arrives on this barrier: the bounded wait runs out and records the error.
  mbar_wait_bounded(addr, 0, st, 0xffffu, wait_ns);
}

}  // namespace

cudaError_t launch_wait_timeout_probe(DeviceStatus* st, uint64_t wait_ns, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 1, 0, stream>>>(st, wait_ns);
  return cudaGetLastError();
}

}  // namespace msa

using msa::Shape;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool good_stride(int64_t s) { return s > 0 && (s % 8) == 0; }

// Validates the parameters that every operation shares and fills `s`.
msa_status_t make_shape(const msa_params_t* p, Shape* s) {
  if (p == nullptr) return MSA_ERR_INVALID_ARG;
  if (p->batch < 1 || p->n_q < 1 || p->max_kv < 1 || p->H < 1 || p->h < 1 || p->topk < 1 ||
      p->block < 1)
    return MSA_ERR_INVALID_ARG;
  if (p->n_q > p->max_kv || p->H % p->h != 0) return MSA_ERR_INVALID_ARG;
  if ((p->causal != 0 && p->causal != 1) || (p->force_own_block != 0 && p->force_own_block != 1))
    return MSA_ERR_INVALID_ARG;
  if (!(p->softmax_scale <= 0.f || isfinite(p->softmax_scale))) return MSA_ERR_INVALID_ARG;
  const int G = p->H / p->h;
  if (p->d != 64 && p->d != 128) return MSA_ERR_UNSUPPORTED;
  if (p->d_idx != 32 && p->d_idx != 64 && p->d_idx != 128) return MSA_ERR_UNSUPPORTED;
  if (p->block != 16 && p->block != 32 && p->block != 64 && p->block != 128)
    return MSA_ERR_UNSUPPORTED;
  if (G > 16 || p->h > 16 || p->topk > 4096) return MSA_ERR_UNSUPPORTED;
  const int64_t nblk = ((int64_t)p->max_kv + p->block - 1) / p->block;
  if (nblk > 65536) return MSA_ERR_UNSUPPORTED;
  if ((int64_t)p->batch * p->n_q * p->H > (int64_t)INT32_MAX) return MSA_ERR_UNSUPPORTED;
  s->batch = p->batch;
  s->n_q = p->n_q;
  s->max_kv = p->max_kv;
  s->H = p->H;
  s->h = p->h;
  s->G = G;
  s->d = p->d;
  s->d_idx = p->d_idx;
  s->block = p->block;
  s->topk = p->topk;
  s->nblk = (int)nblk;
  s->causal = p->causal;
  s->force_own = p->force_own_block;
  s->scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf((float)p->d);
  s->seq_lens = p->seq_lens;
  for (int i = 0; i < 3; ++i) {
    s->q_s[i] = p->q_strides[i];
    s->k_s[i] = p->k_strides[i];
    s->v_s[i] = p->v_strides[i];
    s->qi_s[i] = p->qi_strides[i];
    s->o_s[i] = p->o_strides[i];
  }
  s->ki_s[0] = p->ki_strides[0];
  s->ki_s[1] = p->ki_strides[1];
  s->pages.table = p->block_table;
  s->pages.stride = p->table_stride;
  s->pages.pages = p->num_pages;
  if (p->block_table != nullptr) {
    // one page per block; page coordinates are int32 in the tensor maps
    if ((reinterpret_cast<uintptr_t>(p->block_table) & 3u) != 0 || p->table_stride < nblk ||
        p->num_pages < 1 || p->num_pages > (int64_t)INT32_MAX - 1)
      return MSA_ERR_INVALID_ARG;
  }
  return MSA_OK;
}

msa_status_t check_strides3(const int64_t* st) {
  for (int i = 0; i < 3; ++i)
    if (!good_stride(st[i])) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

msa_status_t check_select_args(const Shape& s, const void* q_idx, const void* k_idx) {
  if (!q_idx || !k_idx || !aligned16(q_idx) || !aligned16(k_idx)) return MSA_ERR_INVALID_ARG;
  if (check_strides3(s.qi_s) != MSA_OK) return MSA_ERR_INVALID_ARG;
  if (!good_stride(s.ki_s[0]) || !good_stride(s.ki_s[1])) return MSA_ERR_INVALID_ARG;
  if (s.qi_s[2] < s.d_idx || s.ki_s[1] < s.d_idx) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

msa_status_t check_attn_args(const Shape& s, const void* q, const void* k, const void* v,
                             const void* out) {
  if (!q || !k || !v || !out) return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return MSA_ERR_INVALID_ARG;
  if (check_strides3(s.q_s) != MSA_OK || check_strides3(s.k_s) != MSA_OK ||
      check_strides3(s.v_s) != MSA_OK || check_strides3(s.o_s) != MSA_OK)
    return MSA_ERR_INVALID_ARG;
  if (s.q_s[2] < s.d || s.k_s[2] < s.d || s.v_s[2] < s.d || s.o_s[2] < s.d)
    return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

size_t scores_bytes(const Shape& s) {
  return (size_t)s.batch * s.n_q * s.h * s.nblk * sizeof(float);
}

size_t ids_bytes(const Shape& s) {
  return (size_t)s.batch * s.n_q * s.h * s.topk * sizeof(int32_t);
}

// Workspace layout: [status region (status word, decode merge counters) | scores |
// ids | attention partials], 256-aligned parts.
struct Layout {
  size_t scores_off, ids_off, part_off, part_bytes, total;
};

Layout layout(const Shape& s, msa_op_t op) {
  Layout l;
  size_t off = msa::kStatusBytes;
  l.scores_off = l.ids_off = l.part_off = 0;
  l.part_bytes = 0;
  if (op == MSA_OP_INDEX_SELECT || op == MSA_OP_INDEX_CANDIDATES || op == MSA_OP_FORWARD) {
    l.scores_off = off;
    off = align_up(off + scores_bytes(s));
  }
  if (op == MSA_OP_FORWARD) {
    l.ids_off = off;
    off = align_up(off + ids_bytes(s));
  }
  if (op == MSA_OP_SPARSE_ATTN || op == MSA_OP_FORWARD) {
    l.part_bytes = msa::attn_partial_bytes(s);
    l.part_off = off;
    off = align_up(off + l.part_bytes);
  }
  l.total = off;
  return l;
}

// Operations whose workspace holds the status word only.
bool status_only(msa_op_t op) {
  return op == MSA_OP_APPEND_KV || op == MSA_OP_BLOCK_SCORES || op == MSA_OP_SELECT_CANDIDATES ||
         op == MSA_OP_SHARD_LENGTHS || op == MSA_OP_INDEX_TOPK;
}

msa_status_t check_ws(const Shape& s, msa_op_t op, void* ws, size_t bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return MSA_ERR_WORKSPACE;
  if (bytes < (status_only(op) ? msa::kStatusBytes : layout(s, op).total))
    return MSA_ERR_WORKSPACE;
  return MSA_OK;
}

msa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

uint8_t* at(void* ws, size_t off) { return reinterpret_cast<uint8_t*>(ws) + off; }

// The decode attention's merge counters in the workspace's status region.
int* fixed_counters(void* ws) { return reinterpret_cast<int*>(at(ws, msa::kCounterOffset)); }

cudaError_t run_scores(const Shape& s, const msa_bf16_t* q_idx, const msa_bf16_t* k_idx,
                       float* scores, bool fill_tail, msa::DeviceStatus* st,
                       cudaStream_t stream) {
  return msa::index_scores_tc_supported(s)
             ? msa::launch_index_scores_tc(s, q_idx, k_idx, scores, fill_tail, st, stream)
             : msa::launch_index_scores(s, q_idx, k_idx, scores, fill_tail, st, stream);
}

msa_status_t run_select(const Shape& s, const msa_bf16_t* q_idx, const msa_bf16_t* k_idx,
                        int32_t* ids, float* user_scores, void* ws, const Layout& l,
                        cudaStream_t stream, int* zero = nullptr, int nzero = 0,
                        float* kept = nullptr) {
  msa::DeviceStatus* st = reinterpret_cast<msa::DeviceStatus*>(ws);
  float* scores = user_scores ? user_scores : reinterpret_cast<float*>(at(ws, l.scores_off));
  if (run_scores(s, q_idx, k_idx, scores, user_scores != nullptr, st, stream) != cudaSuccess)
    return MSA_ERR_CUDA;
  return cuda_status(msa::launch_topk(s, scores, ids, st, stream, zero, nzero, kept));
}

}  // namespace

extern "C" {

size_t msa_workspace_size(const msa_params_t* params, msa_op_t op) {
  Shape s;
  if (make_shape(params, &s) != MSA_OK) return 0;
  if (status_only(op)) return msa::kStatusBytes;
  if (op != MSA_OP_INDEX_SELECT && op != MSA_OP_SPARSE_ATTN && op != MSA_OP_FORWARD &&
      op != MSA_OP_INDEX_CANDIDATES)
    return 0;
  return layout(s, op).total;
}

msa_status_t msa_block_scores(const msa_params_t* params, const msa_bf16_t* q_idx,
                              const msa_bf16_t* k_idx, float* block_scores, void* workspace,
                              size_t workspace_bytes, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((rc = check_select_args(s, q_idx, k_idx)) != MSA_OK) return rc;
  if (block_scores == nullptr) return MSA_ERR_INVALID_ARG;
  if ((rc = check_ws(s, MSA_OP_BLOCK_SCORES, workspace, workspace_bytes)) != MSA_OK) return rc;
  return cuda_status(run_scores(s, q_idx, k_idx, block_scores, true,
                                reinterpret_cast<msa::DeviceStatus*>(workspace),
                                reinterpret_cast<cudaStream_t>(stream)));
}

msa_status_t msa_index_topk(const msa_params_t* params, const msa_bf16_t* q_idx,
                            const msa_bf16_t* k_idx, int32_t* block_ids, float* block_scores,
                            void* workspace, size_t workspace_bytes, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((rc = check_select_args(s, q_idx, k_idx)) != MSA_OK) return rc;
  if (block_ids == nullptr) return MSA_ERR_INVALID_ARG;
  if (!msa::index_topk_tc_supported(s)) return MSA_ERR_UNSUPPORTED;
  if ((rc = check_ws(s, MSA_OP_INDEX_TOPK, workspace, workspace_bytes)) != MSA_OK) return rc;
  return cuda_status(msa::launch_index_topk_tc(s, q_idx, k_idx, block_ids, block_scores,
                                               reinterpret_cast<msa::DeviceStatus*>(workspace),
                                               reinterpret_cast<cudaStream_t>(stream)));
}

msa_status_t msa_index_candidates(const msa_params_t* params, const msa_bf16_t* q_idx,
                                  const msa_bf16_t* k_idx, int32_t* block_ids,
                                  float* kept_scores, void* workspace, size_t workspace_bytes,
                                  msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((rc = check_select_args(s, q_idx, k_idx)) != MSA_OK) return rc;
  if (block_ids == nullptr || kept_scores == nullptr) return MSA_ERR_INVALID_ARG;
  if ((rc = check_ws(s, MSA_OP_INDEX_CANDIDATES, workspace, workspace_bytes)) != MSA_OK)
    return rc;
  return run_select(s, q_idx, k_idx, block_ids, nullptr, workspace,
                    layout(s, MSA_OP_INDEX_CANDIDATES), reinterpret_cast<cudaStream_t>(stream),
                    nullptr, 0, kept_scores);
}

msa_status_t msa_select_candidates(const msa_params_t* params, int32_t nlists, int32_t list_len,
                                   int32_t shard_blocks, const float* cand_scores,
                                   const int32_t* cand_ids, int32_t block_base,
                                   int32_t nblk_local, int32_t* block_ids, int32_t* local_ids,
                                   void* workspace, size_t workspace_bytes, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if (!cand_scores || !cand_ids || (!block_ids && !local_ids)) return MSA_ERR_INVALID_ARG;
  if (nlists < 1 || list_len < 1 || shard_blocks < 0 || block_base < 0 || nblk_local < 0)
    return MSA_ERR_INVALID_ARG;
  if ((int64_t)nlists * list_len > 16384) return MSA_ERR_UNSUPPORTED;
  if ((int64_t)(nlists - 1) * shard_blocks >= (int64_t)INT32_MAX / 2) return MSA_ERR_INVALID_ARG;
  if ((rc = check_ws(s, MSA_OP_SELECT_CANDIDATES, workspace, workspace_bytes)) != MSA_OK)
    return rc;
  return cuda_status(msa::launch_candidates_topk(
      s, nlists, list_len, shard_blocks, cand_scores, cand_ids, block_base, nblk_local, block_ids,
      local_ids, reinterpret_cast<msa::DeviceStatus*>(workspace),
      reinterpret_cast<cudaStream_t>(stream)));
}

msa_status_t msa_merge_partials(const msa_params_t* params, int32_t nparts,
                                const msa_bf16_t* part_out, const float* part_lse,
                                msa_bf16_t* out, float* lse, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if (!part_out || !part_lse || !out || !aligned16(part_out) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(part_lse) & 3u) != 0)
    return MSA_ERR_INVALID_ARG;
  if (nparts < 1 || nparts > 1024) return MSA_ERR_INVALID_ARG;
  if (check_strides3(s.o_s) != MSA_OK || s.o_s[2] < s.d) return MSA_ERR_INVALID_ARG;
  return cuda_status(msa::launch_merge_partials(s, nparts, part_out, part_lse, out, lse,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

msa_status_t msa_shard_lengths(const msa_params_t* params, int64_t token_base,
                               int64_t token_count, int32_t* shard_lens, void* workspace,
                               size_t workspace_bytes, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if (shard_lens == nullptr || token_base < 0 || token_count < 0 ||
      token_base > (int64_t)INT32_MAX || token_count > (int64_t)INT32_MAX)
    return MSA_ERR_INVALID_ARG;
  if ((rc = check_ws(s, MSA_OP_SHARD_LENGTHS, workspace, workspace_bytes)) != MSA_OK) return rc;
  return cuda_status(msa::launch_shard_lengths(
      s.seq_lens, s.batch, s.max_kv, token_base, token_count, shard_lens,
      reinterpret_cast<msa::DeviceStatus*>(workspace), reinterpret_cast<cudaStream_t>(stream)));
}

msa_status_t msa_index_select(const msa_params_t* params, const msa_bf16_t* q_idx,
                              const msa_bf16_t* k_idx, int32_t* block_ids, float* block_scores,
                              void* workspace, size_t workspace_bytes, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((rc = check_select_args(s, q_idx, k_idx)) != MSA_OK) return rc;
  if (block_ids == nullptr) return MSA_ERR_INVALID_ARG;
  if ((rc = check_ws(s, MSA_OP_INDEX_SELECT, workspace, workspace_bytes)) != MSA_OK) return rc;
  return run_select(s, q_idx, k_idx, block_ids, block_scores, workspace,
                    layout(s, MSA_OP_INDEX_SELECT), reinterpret_cast<cudaStream_t>(stream));
}

msa_status_t msa_sparse_attn(const msa_params_t* params, const msa_bf16_t* q, const msa_bf16_t* k,
                             const msa_bf16_t* v, const int32_t* block_ids, msa_bf16_t* out,
                             float* lse, void* workspace, size_t workspace_bytes,
                             msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((rc = check_attn_args(s, q, k, v, out)) != MSA_OK) return rc;
  if (block_ids == nullptr) return MSA_ERR_INVALID_ARG;
  if ((rc = check_ws(s, MSA_OP_SPARSE_ATTN, workspace, workspace_bytes)) != MSA_OK) return rc;
  const Layout l = layout(s, MSA_OP_SPARSE_ATTN);
  return cuda_status(msa::launch_sparse_attn(
      s, q, k, v, block_ids, out, lse, at(workspace, l.part_off), l.part_bytes,
      reinterpret_cast<msa::DeviceStatus*>(workspace), reinterpret_cast<cudaStream_t>(stream),
      false, fixed_counters(workspace)));
}

msa_status_t msa_forward(const msa_params_t* params, const msa_bf16_t* q, const msa_bf16_t* k,
                         const msa_bf16_t* v, const msa_bf16_t* q_idx, const msa_bf16_t* k_idx,
                         msa_bf16_t* out, int32_t* block_ids, float* block_scores, float* lse,
                         void* workspace, size_t workspace_bytes, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((rc = check_select_args(s, q_idx, k_idx)) != MSA_OK) return rc;
  if ((rc = check_attn_args(s, q, k, v, out)) != MSA_OK) return rc;
  if ((rc = check_ws(s, MSA_OP_FORWARD, workspace, workspace_bytes)) != MSA_OK) return rc;
  const Layout l = layout(s, MSA_OP_FORWARD);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int32_t* ids = block_ids ? block_ids : reinterpret_cast<int32_t*>(at(workspace, l.ids_off));
  // The attention's merge counters are the status region's (zero between calls)
  // when the shape needs no more of them; otherwise the top-k kernel clears the
  // ones in the partials, so that the two stages follow each other with no memset
  // in between.
  int ncounters = 0;
  int* counters = msa::attn_merge_counters(s, at(workspace, l.part_off), &ncounters);
  if (counters != nullptr && ncounters <= msa::kFixedCounters) counters = nullptr;
  if ((rc = run_select(s, q_idx, k_idx, ids, block_scores, workspace, l, cs, counters,
                       ncounters)) != MSA_OK)
    return rc;
  return cuda_status(msa::launch_sparse_attn(s, q, k, v, ids, out, lse, at(workspace, l.part_off),
                                             l.part_bytes,
                                             reinterpret_cast<msa::DeviceStatus*>(workspace), cs,
                                             counters != nullptr, fixed_counters(workspace)));
}

msa_status_t msa_append_kv(const msa_params_t* params, const msa_bf16_t* k_new,
                           const msa_bf16_t* v_new, const msa_bf16_t* k_idx_new, msa_bf16_t* k,
                           msa_bf16_t* v, msa_bf16_t* k_idx, void* workspace,
                           size_t workspace_bytes, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((k_new != nullptr && (!k || !aligned16(k) || !aligned16(k_new) ||
                            check_strides3(s.k_s) != MSA_OK || s.k_s[2] < s.d)) ||
      (v_new != nullptr && (!v || !aligned16(v) || !aligned16(v_new) ||
                            check_strides3(s.v_s) != MSA_OK || s.v_s[2] < s.d)) ||
      (k_idx_new != nullptr &&
       (!k_idx || !aligned16(k_idx) || !aligned16(k_idx_new) || !good_stride(s.ki_s[0]) ||
        !good_stride(s.ki_s[1]) || s.ki_s[1] < s.d_idx)))
    return MSA_ERR_INVALID_ARG;
  if ((rc = check_ws(s, MSA_OP_APPEND_KV, workspace, workspace_bytes)) != MSA_OK) return rc;
  return cuda_status(msa::launch_append_kv(s, k_new, v_new, k_idx_new, k, v, k_idx,
                                           reinterpret_cast<msa::DeviceStatus*>(workspace),
                                           reinterpret_cast<cudaStream_t>(stream)));
}

msa_status_t msa_get_device_status(void* workspace, msa_stream_t stream) {
  if (workspace == nullptr) return MSA_ERR_WORKSPACE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  msa::DeviceStatus h{0, 0};
  if (cudaMemcpyAsync(&h, workspace, sizeof h, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  if (h.code != 0) {
    // the whole status region: a call that stopped early may have left merge
    // counters set
    if (cudaMemsetAsync(workspace, 0, msa::kStatusBytes, cs) != cudaSuccess) return MSA_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return MSA_ERR_CUDA;
  }
  return static_cast<msa_status_t>(h.code);
}

msa_status_t msa_workspace_init(void* workspace, size_t workspace_bytes, msa_stream_t stream) {
  if (workspace == nullptr || workspace_bytes < msa::kStatusBytes ||
      (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return MSA_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(workspace, 0, msa::kStatusBytes,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

msa_status_t msa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint64_t wait_ns,
                                       msa_stream_t stream) {
  if (workspace == nullptr || workspace_bytes < msa::kStatusBytes ||
      (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return MSA_ERR_WORKSPACE;
  if (wait_ns == 0 || wait_ns > 1000000000ull) return MSA_ERR_INVALID_ARG;
  return cuda_status(msa::launch_wait_timeout_probe(
      reinterpret_cast<msa::DeviceStatus*>(workspace), wait_ns,
      reinterpret_cast<cudaStream_t>(stream)));
}

int msa_launch_count(const msa_params_t* params, msa_op_t op) {
  Shape s;
  if (make_shape(params, &s) != MSA_OK) return -1;
  switch (op) {
    case MSA_OP_INDEX_SELECT: return 2;
    case MSA_OP_SPARSE_ATTN: return msa::attn_launches(s);
    case MSA_OP_FORWARD: return 2 + msa::attn_launches(s);
    case MSA_OP_APPEND_KV: return 1;
    case MSA_OP_BLOCK_SCORES: return 1;
    case MSA_OP_INDEX_CANDIDATES: return 2;
    case MSA_OP_SELECT_CANDIDATES: return 1;
    case MSA_OP_SHARD_LENGTHS: return 1;
    case MSA_OP_INDEX_TOPK: return 1;
  }
  return -1;
}

const char* msa_status_string(msa_status_t status) {
  switch (status) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported size";
    case MSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_TIMEOUT: return "device wait timed out";
    case MSA_ERR_DEVICE_ASSERT: return "device-side precondition failed";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// msa_sparse_attn_noalloc: the sparse branch for callers that cannot allocate
// device memory.  Its split-KV partial results live in one fixed array in the
// library's own device memory instead of a caller-provided workspace.
namespace {

// Scratch for the split-KV partials of msa_sparse_attn_noalloc.  Every GPU that
// loads this library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and kept.  Host threads may call at the
// same time: the entries are atomics and the lookup itself runs under a lock
// (a failed lookup leaves the entry empty, so a later call tries again).
std::atomic<void*> g_noalloc_ptr[64];
std::mutex g_noalloc_lock;

msa_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MSA_ERR_CUDA;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> guard(g_noalloc_lock);
    p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return MSA_ERR_CUDA;
      g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return MSA_OK;
}

}  // namespace

extern "C" msa_status_t msa_sparse_attn_noalloc(const msa_params_t* params, const msa_bf16_t* q,
                                                const msa_bf16_t* k, const msa_bf16_t* v,
                                                const int32_t* block_ids, msa_bf16_t* out,
                                                float* lse, msa_stream_t stream) {
  Shape s;
  msa_status_t rc = make_shape(params, &s);
  if (rc != MSA_OK) return rc;
  if ((rc = check_attn_args(s, q, k, v, out)) != MSA_OK) return rc;
  if (block_ids == nullptr) return MSA_ERR_INVALID_ARG;
  const size_t need = msa::attn_partial_bytes(s);
  if (need > kNoAllocScratchBytes) return MSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch)) != MSA_OK) return rc;
  // What must start at zero inside the scratch (the decode kernel's per-row merge
  // counters, the KV-major kernel's per-block counts) is cleared on the stream by
  // every call; the partials themselves are always written before they are read.
  // No status word: device-side errors are skipped, not recorded.
  return cuda_status(msa::launch_sparse_attn(s, q, k, v, block_ids, out, lse, scratch,
                                             kNoAllocScratchBytes, nullptr,
                                             reinterpret_cast<cudaStream_t>(stream)));
}
