// Index branch, part 2: deterministic top-k over block scores.
//
// "MiniMax goes sparse" (atlascloud.ai), section 1, step 1: a TopK decides which
// KV blocks this layer and this GQA group keep ("MiniMax M3 的 MSA ...", first
// layer).  Order: score descending, then block id ascending (the lower id wins a
// tie); with the own block forced it comes first.  min(topk, F) ids are written
// in ascending order, then -1 padding, F being the number of blocks at or before
// the causal frontier.
//
// Method: scores become order-preserving 32-bit keys (blocks past the frontier
// get key 0, a forced own block the largest key).  The k-th largest key T is
// found bit by bit from the most significant end: T is the largest value with
// count(key >= T) >= m.  Keys above T are all taken; keys equal to T are taken
// in ascending id order until m are chosen.  Rows of up to 1024 blocks use one
// warp per row with keys in registers (counts by warp reductions, ids emitted in
// order with ballots); wider rows (long-context decode) use one CTA per row.
#include "kernels.h"

namespace msa {
namespace {

struct TopkArgs {
  const float* scores;
  int32_t* ids;
  const int32_t* seq_lens;
  int rows, n_q, max_kv, h, block, nblk, topk, causal, force_own;
  DeviceStatus* st;
};

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct RowInfo {
  int F, own, m;
};

__device__ __forceinline__ RowInfo row_info(const TopkArgs& a, int row) {
  const int bt = row / a.h;
  const int t = bt % a.n_q, b = bt / a.n_q;
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int p = L - a.n_q + t;
  const int nb = (L + a.block - 1) / a.block;
  RowInfo ri;
  ri.F = a.causal ? (p < 0 ? 0 : min(nb, p / a.block + 1)) : nb;
  ri.own = (a.force_own && p >= 0) ? p / a.block : -1;
  if (ri.own >= ri.F) ri.own = -1;
  ri.m = min(a.topk, ri.F);
  return ri;
}

// Top-m of one row by one warp, element i = e*32 + lane for e < EE: keys in
// registers, the threshold found bit by bit, ids emitted in order with ballots.
template <int EE>
__device__ __forceinline__ void warp_row_topk(const float* s, int32_t* out, const RowInfo& ri,
                                              int lane) {
  uint32_t key[EE];
#pragma unroll
  for (int e = 0; e < EE; ++e) {
    const int i = e * 32 + lane;
    key[e] = i < ri.F ? order_key(s[i]) : 0u;
    if (i == ri.own) key[e] = 0xffffffffu;
  }
  const int m = ri.m;
  // The threshold lies between the smallest and the largest visible key (the
  // forced block, key 0xffffffff, always counts): it shares their common high
  // bits, and the search starts below them.
  uint32_t kmax = 0u, kmin = 0xffffffffu;
#pragma unroll
  for (int e = 0; e < EE; ++e) {
    const bool vis = key[e] != 0u && key[e] != 0xffffffffu;
    kmax = vis ? max(kmax, key[e]) : kmax;
    kmin = vis ? min(kmin, key[e]) : kmin;
  }
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  uint32_t T;
  if (m <= (ri.own >= 0 ? 1 : 0) || kmax < kmin) {
    T = 0xffffffffu;  // only the forced block is taken
  } else {
    const uint32_t diff = kmax ^ kmin;
    const int top = diff ? 31 - __clz(diff) : -1;
    T = top < 0 ? kmax : kmax & ~((2u << top) - 1u);
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      unsigned c4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < EE; ++e) c4[e & 3] += key[e] >= cand;
      const unsigned cnt = __reduce_add_sync(0xffffffffu, (c4[0] + c4[1]) + (c4[2] + c4[3]));
      if ((int)cnt >= m) T = cand;
    }
  }
  unsigned gt = 0;
#pragma unroll
  for (int e = 0; e < EE; ++e) gt += key[e] > T;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need = m - (int)gt;
  const unsigned lt = (1u << lane) - 1u;
  int base = 0, eqbase = 0;
#pragma unroll
  for (int e = 0; e < EE; ++e) {
    const bool eq = key[e] == T;
    const unsigned be = __ballot_sync(0xffffffffu, eq);
    const int eqr = eqbase + __popc(be & lt);
    eqbase += __popc(be);
    const bool sel = key[e] > T || (eq && eqr < need);
    const unsigned bs = __ballot_sync(0xffffffffu, sel);
    if (sel) out[base + __popc(bs & lt)] = e * 32 + lane;
    base += __popc(bs);
  }
}

// One warp per row of up to 32 * E blocks.  A row sees only its F blocks at or
// before the frontier, so it is handled with the smallest power-of-two number
// of 32-block groups covering F (blocks past F have key 0 and the threshold is
// at least 1, so leaving them out changes nothing); a row with m = F keeps all
// of its visible blocks and needs no threshold.
template <int E>
__global__ void __launch_bounds__(256) topk_warp_kernel(TopkArgs a) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  const RowInfo ri = row_info(a, row);
  const float* s = a.scores + (int64_t)row * a.nblk;
  int32_t* out = a.ids + (int64_t)row * a.topk;
  const int m = ri.m, ne = (ri.F + 31) >> 5;
  if (m == ri.F) {
    for (int i = lane; i < m; i += 32) out[i] = i;
  } else if (ne <= 1 || E == 1) {
    warp_row_topk<1>(s, out, ri, lane);
  } else if (ne <= 2 || E == 2) {
    warp_row_topk<(E < 2 ? E : 2)>(s, out, ri, lane);
  } else if (ne <= 4 || E == 4) {
    warp_row_topk<(E < 4 ? E : 4)>(s, out, ri, lane);
  } else if (ne <= 8 || E == 8) {
    warp_row_topk<(E < 8 ? E : 8)>(s, out, ri, lane);
  } else if (ne <= 16 || E == 16) {
    warp_row_topk<(E < 16 ? E : 16)>(s, out, ri, lane);
  } else {
    warp_row_topk<E>(s, out, ri, lane);
  }
  for (int i = m + lane; i < a.topk; i += 32) out[i] = -1;
}

// Sum over the CTA (NW warps); `buf` alternates between calls so one barrier
// per call suffices.  Each warp reads the NW partial sums with one load per lane.
template <int NW>
__device__ __forceinline__ unsigned cta_sum(unsigned v, unsigned (*red)[32], int& buf) {
  const int lane = threadIdx.x & 31;
  v = __reduce_add_sync(0xffffffffu, v);
  if (lane == 0) red[buf][threadIdx.x >> 5] = v;
  __syncthreads();
  const unsigned tot = __reduce_add_sync(0xffffffffu, lane < NW ? red[buf][lane] : 0u);
  buf ^= 1;
  return tot;
}

// Exclusive prefix over the CTA in thread order.
template <int NW>
__device__ __forceinline__ unsigned cta_exclusive_scan(unsigned v, unsigned* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  const unsigned x = lane < NW ? wsum[lane] : 0u;
  const unsigned before = __reduce_add_sync(0xffffffffu, lane < warp ? x : 0u);
  __syncthreads();
  return before + inc - v;
}

// One CTA of NT threads per row; thread i holds elements [i*E, i*E + E).
template <int NT, int E>
__global__ void __launch_bounds__(NT) topk_cta_kernel(TopkArgs a) {
  constexpr int NW = NT / 32;
  __shared__ unsigned red[2][32];
  __shared__ unsigned wsum[32];
  const int row = blockIdx.x;
  const RowInfo ri = row_info(a, row);
  const float* s = a.scores + (int64_t)row * a.nblk;
  int32_t* out = a.ids + (int64_t)row * a.topk;
  const int i0 = threadIdx.x * E;
  uint32_t key[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = i0 + e;
    key[e] = i < ri.F ? order_key(s[i]) : 0u;
    if (i == ri.own) key[e] = 0xffffffffu;
  }
  const int m = ri.m;
  int buf = 0;
  if (m > 0) {
    uint32_t T = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      unsigned cnt = 0;
#pragma unroll
      for (int e = 0; e < E; ++e) cnt += key[e] >= cand;
      if ((int)cta_sum<NW>(cnt, red, buf) >= m) T = cand;
    }
    unsigned gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      gt += key[e] > T;
      eq += key[e] == T;
    }
    const int need = m - (int)cta_sum<NW>(gt, red, buf);
    unsigned eqr = cta_exclusive_scan<NW>(eq, wsum);
    unsigned nsel = 0;
    bool sel[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const bool is_eq = key[e] == T;
      sel[e] = key[e] > T || (is_eq && (int)eqr < need);
      eqr += is_eq;
      nsel += sel[e];
    }
    unsigned pos = cta_exclusive_scan<NW>(nsel, wsum);
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (sel[e]) out[pos++] = i0 + e;
  }
  for (int i = m + threadIdx.x; i < a.topk; i += NT) out[i] = -1;
}

}  // namespace

cudaError_t launch_topk(const Shape& s, const float* scores, int32_t* ids, DeviceStatus* st,
                        cudaStream_t stream) {
  TopkArgs a;
  a.scores = scores;
  a.ids = ids;
  a.seq_lens = s.seq_lens;
  a.rows = s.batch * s.n_q * s.h;
  a.n_q = s.n_q;
  a.max_kv = s.max_kv;
  a.h = s.h;
  a.block = s.block;
  a.nblk = s.nblk;
  a.topk = s.topk;
  a.causal = s.causal;
  a.force_own = s.force_own;
  a.st = st;
  const int n = s.nblk;
  if (n <= 1024) {
    const dim3 grid((a.rows + 7) / 8);
#define MSA_TOPK_WARP(E_)                                             \
  if (n <= 32 * E_) {                                                 \
    topk_warp_kernel<E_><<<grid, 256, 0, stream>>>(a);                \
    return cudaGetLastError();                                        \
  }
    MSA_TOPK_WARP(1)
    MSA_TOPK_WARP(2)
    MSA_TOPK_WARP(4)
    MSA_TOPK_WARP(8)
    MSA_TOPK_WARP(16)
    MSA_TOPK_WARP(32)
#undef MSA_TOPK_WARP
  }
  const dim3 grid(a.rows);
#define MSA_TOPK_CTA(NT_, E_)                                      \
  if (n <= NT_ * E_) {                                             \
    topk_cta_kernel<NT_, E_><<<grid, NT_, 0, stream>>>(a);         \
    return cudaGetLastError();                                     \
  }
  MSA_TOPK_CTA(256, 8)
  MSA_TOPK_CTA(256, 16)
  MSA_TOPK_CTA(512, 16)
  MSA_TOPK_CTA(1024, 16)
  MSA_TOPK_CTA(1024, 32)
  MSA_TOPK_CTA(1024, 64)
#undef MSA_TOPK_CTA
  return cudaErrorInvalidValue;
}

}  // namespace msa
