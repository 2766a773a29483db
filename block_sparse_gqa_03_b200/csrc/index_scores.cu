// Index branch, part 1: index scores with Block Max Pool fused into the epilogue.
//
// "MiniMax goes sparse" (atlascloud.ai), section 1, step 1: one index query per
// GQA group is scored against a single-head index key shared by all heads
// (Q_idx . K_idx^T), and Block Max Pool compresses the token scores to block
// scores.  "MiniMax M3 的 MSA ..." (ai.air7.fun), first layer, says the same.
// The causal mask is applied to token scores before pooling, so a query's own
// block pools only tokens at or before its position; token scores never leave
// the registers.
//
// Mapping.  The contraction is [tokens x d_idx] . [d_idx x columns], where a
// column is one (query, group) index vector.  It runs on the warp-level bf16
// tensor-core MMA (m16n8k16): rows are tokens, so the block max over tokens is
// a max over accumulator rows (in-thread, then across the 8 row-lanes).  The
// decode scan streams K_idx from HBM exactly once with 16-byte coalesced loads
// straight into MMA fragments: each thread loads 8 consecutive dims of a token
// row, and the same dim permutation is applied to the index-query fragments,
// which leaves the dot products unchanged.
#include "kernels.h"

namespace msa {
namespace {

struct ScanArgs {
  const uint16_t* q_idx;
  const uint16_t* k_idx;
  int64_t qi_s0, qi_s1, qi_s2, ki_s0, ki_s1;
  const int32_t* seq_lens;
  int batch, n_q, max_kv, h, block, nblk, causal, qt, ntiles;
  float* scores;
  int fill_tail;
  DeviceStatus* st;
  KvPages pg;
};

constexpr int kScanWarps = 8;

// k_idx row of the first token of block beta of sequence b, offset by this lane's
// 8 dims; nullptr for a page outside the pool (the block then reads as zeros).
__device__ __forceinline__ const uint16_t* kidx_block(const ScanArgs& a, int b, int beta, int q) {
  if (a.pg.table == nullptr)
    return a.k_idx + b * a.ki_s0 + (int64_t)beta * a.block * a.ki_s1 + 8 * q;
  const int64_t page = kv_page(a.pg, b, beta, a.st);
  return page < 0 ? nullptr : a.k_idx + page * a.ki_s0 + 8 * q;
}

// Loads the B fragments (index-query columns) of this lane: column c = nt*8 + r,
// dims [32kc + 8q, 32kc + 8q + 8).  Columns past `ncols` or t >= n_q are zero.
template <int DI, int NT>
__device__ __forceinline__ void load_columns(const ScanArgs& a, int b, int t0, int r, int q,
                                             uint4 (&bq)[NT][DI / 32]) {
  const int ncols = a.qt * a.h;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int c = nt * 8 + r;
    const int t = t0 + c / a.h, g = c % a.h;
    const bool ok = c < ncols && t < a.n_q;
    const uint16_t* src = a.q_idx + b * a.qi_s0 + (int64_t)t * a.qi_s1 + g * a.qi_s2 + 8 * q;
#pragma unroll
    for (int kc = 0; kc < DI / 32; ++kc)
      bq[nt][kc] = ok ? ld_u4(src + 32 * kc) : make_uint4(0, 0, 0, 0);
  }
}

// Block max of the visible token scores of block `beta` for this lane's
// accumulator columns (c = nt*8 + 2q + e, visible tokens j < lim[nt][e]),
// reduced over the warp: every lane returns the maxima of its own columns.
// `kbb` is the block's first k_idx row (kidx_block).
template <int DI, int NT>
__device__ __forceinline__ void block_max(const ScanArgs& a, const uint16_t* kbb, int L, int beta,
                                          int r, const uint4 (&bq)[NT][DI / 32],
                                          const int (&lim)[NT][2], float (&cm)[NT][2]) {
  constexpr int KC = DI / 32;
  const float ninf = -__int_as_float(0x7f800000);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) cm[nt][0] = cm[nt][1] = ninf;
  const int nmt = a.block / 16;
#pragma unroll 2
  for (int mt = 0; mt < nmt; ++mt) {
    const int ol = mt * 16 + r, oh = ol + 8;  // tokens in the block
    const int jl = beta * a.block + ol, jh = jl + 8;
    const bool okl = kbb != nullptr && jl < L, okh = kbb != nullptr && jh < L;
    uint4 X[KC], Y[KC];
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
      X[kc] = okl ? ld_stream_u4(kbb + (int64_t)ol * a.ki_s1 + 32 * kc) : make_uint4(0, 0, 0, 0);
      Y[kc] = okh ? ld_stream_u4(kbb + (int64_t)oh * a.ki_s1 + 32 * kc) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kc = 0; kc < KC; ++kc) {
        mma_bf16_16816(acc, X[kc].x, Y[kc].x, X[kc].y, Y[kc].y, bq[nt][kc].x, bq[nt][kc].y);
        mma_bf16_16816(acc, X[kc].z, Y[kc].z, X[kc].w, Y[kc].w, bq[nt][kc].z, bq[nt][kc].w);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        cm[nt][e] = fmaxf(cm[nt][e], jl < lim[nt][e] ? acc[e] : ninf);
        cm[nt][e] = fmaxf(cm[nt][e], jh < lim[nt][e] ? acc[2 + e] : ninf);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = cm[nt][e];
      v = warp_max_xor(v, 4);
      v = warp_max_xor(v, 8);
      v = warp_max_xor(v, 16);
      cm[nt][e] = v;
    }
}

// Decode (one query per sequence): one warp per (sequence, block) item, so the
// grid is many short CTAs and no wave leaves the GPU half idle.  The columns are
// the h groups of the sequence's query.
template <int DI, int NT>
__global__ void __launch_bounds__(kScanWarps * 32) index_scan_decode_kernel(ScanArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, q = lane & 3;
  const int64_t item = (int64_t)blockIdx.x * kScanWarps + warp;
  const int b = (int)(item / a.nblk), beta = (int)(item % a.nblk);
  if (b >= a.batch) return;
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int nb_b = (L + a.block - 1) / a.block;
  const float ninf = -__int_as_float(0x7f800000);
  if (beta >= nb_b) {
    if (a.fill_tail && lane < a.h) a.scores[((int64_t)b * a.h + lane) * a.nblk + beta] = ninf;
    return;
  }
  const uint16_t* kbb = kidx_block(a, b, beta, q);  // the page lookup overlaps the q loads
  uint4 bq[NT][DI / 32];
  load_columns<DI, NT>(a, b, 0, r, q, bq);
  int lim[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) lim[nt][0] = lim[nt][1] = L;  // p = L - 1: all j < L visible
  float cm[NT][2];
  block_max<DI, NT>(a, kbb, L, beta, r, bq, lim, cm);
  if (r == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int g = nt * 8 + 2 * q + e;
        if (g < a.h) a.scores[((int64_t)b * a.h + g) * a.nblk + beta] = cm[nt][e];
      }
  }
}

// Prefill: a CTA per (sequence, tile of queries); the columns are the tile's
// (query, group) pairs and each warp walks the blocks up to the tile's frontier.
template <int DI, int NT>
__global__ void __launch_bounds__(kScanWarps * 32) index_scan_kernel(ScanArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, q = lane & 3;
  const int tile = blockIdx.x % a.ntiles;
  const int b = blockIdx.x / a.ntiles;
  const int t0 = tile * a.qt;
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int ncols = a.qt * a.h;
  uint4 bq[NT][DI / 32];
  load_columns<DI, NT>(a, b, t0, r, q, bq);
  int lim[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = nt * 8 + 2 * q + e;
      const int t = t0 + c / a.h;
      const int p = L - a.n_q + t;
      lim[nt][e] = a.causal ? min(L, p + 1) : L;
    }
  const int t_last = min(t0 + a.qt, a.n_q) - 1;
  const int p_last = L - a.n_q + t_last;
  const int nb_b = (L + a.block - 1) / a.block;
  const int F = a.causal ? (p_last < 0 ? 0 : min(nb_b, p_last / a.block + 1)) : nb_b;
  const int nw = gridDim.y * kScanWarps;
  const int wid = blockIdx.y * kScanWarps + warp;
  const float ninf = -__int_as_float(0x7f800000);
  for (int beta = wid; beta < F; beta += nw) {
    float cm[NT][2];
    block_max<DI, NT>(a, kidx_block(a, b, beta, q), L, beta, r, bq, lim, cm);
    if (r == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = nt * 8 + 2 * q + e;
          const int t = t0 + c / a.h, g = c % a.h;
          if (c < ncols && t < a.n_q)
            a.scores[(((int64_t)b * a.n_q + t) * a.h + g) * a.nblk + beta] = cm[nt][e];
        }
    }
  }
  if (a.fill_tail && r == 0) {
    for (int beta = F + wid; beta < a.nblk; beta += nw) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = nt * 8 + 2 * q + e;
          const int t = t0 + c / a.h, g = c % a.h;
          if (c < ncols && t < a.n_q)
            a.scores[(((int64_t)b * a.n_q + t) * a.h + g) * a.nblk + beta] = ninf;
        }
    }
  }
}

template <int DI, int NT>
cudaError_t run_scan(const ScanArgs& a, int batch, cudaStream_t stream) {
  if (a.n_q == 1) {
    const int64_t items = (int64_t)batch * a.nblk;
    return launch_pdl(index_scan_decode_kernel<DI, NT>,
                      dim3((unsigned)((items + kScanWarps - 1) / kScanWarps)), dim3(kScanWarps * 32),
                      0, stream, a);
  }
  const int ctas_per_row = a.ntiles * batch;
  // Spread the block range of each query tile over enough warps to fill the
  // GPU a few times over; each warp then walks its blocks with a stride.
  const int want = num_sms() * 4;
  int split = (want + ctas_per_row - 1) / ctas_per_row;
  const int max_split = (a.nblk + kScanWarps - 1) / kScanWarps;
  split = max(1, min(split, max_split));
  dim3 grid(ctas_per_row, split);
  return launch_pdl(index_scan_kernel<DI, NT>, grid, dim3(kScanWarps * 32), 0, stream, a);
}

}  // namespace

cudaError_t launch_index_scores(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                float* scores, bool fill_tail, DeviceStatus* st,
                                cudaStream_t stream) {
  ScanArgs a;
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.qi_s0 = s.qi_s[0];
  a.qi_s1 = s.qi_s[1];
  a.qi_s2 = s.qi_s[2];
  a.ki_s0 = s.ki_s[0];
  a.ki_s1 = s.ki_s[1];
  a.pg = s.pages;
  a.seq_lens = s.seq_lens;
  a.batch = s.batch;
  a.n_q = s.n_q;
  a.max_kv = s.max_kv;
  a.h = s.h;
  a.block = s.block;
  a.nblk = s.nblk;
  a.causal = s.causal;
  a.scores = scores;
  a.fill_tail = fill_tail ? 1 : 0;
  a.st = st;
  // Columns per warp: all h groups of one query in decode; in prefill a tile of
  // queries whose columns fill four 8-wide MMA tiles.
  int nt;
  if (s.n_q == 1) {
    nt = (s.h + 7) / 8;
    a.qt = 1;
  } else {
    nt = 4;
    a.qt = max(1, 32 / s.h);
  }
  a.ntiles = (s.n_q + a.qt - 1) / a.qt;
  const int B = s.batch;
#define MSA_SCAN_CASE(DI_, NT_) \
  if (s.d_idx == DI_ && nt == NT_) return run_scan<DI_, NT_>(a, B, stream);
  MSA_SCAN_CASE(32, 1)
  MSA_SCAN_CASE(32, 2)
  MSA_SCAN_CASE(32, 4)
  MSA_SCAN_CASE(64, 1)
  MSA_SCAN_CASE(64, 2)
  MSA_SCAN_CASE(64, 4)
  MSA_SCAN_CASE(128, 1)
  MSA_SCAN_CASE(128, 2)
  MSA_SCAN_CASE(128, 4)
#undef MSA_SCAN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace msa
