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
// get key 0, a forced own block the largest key).  T, the m-th largest key
// (counted with multiplicity), is found from the most significant bit down: the
// visible keys share the high bits of the row's largest and smallest key, and
// each step halves the bucket of keys that can still be T by counting the keys
// at or above its midpoint (the CTA kernel first narrows a large bucket eight bits
// at a time with a shared histogram).  Once at most 32 keys remain in the bucket they are
// gathered in id order and T is the one of the right rank among them (exact
// ranks by key, ties by id), so the count steps stop long before the last bit.
// Keys above T are all taken; keys equal to T are taken in ascending id order
// until m are chosen.  Rows of up to 1024 blocks use one warp
// per row with keys in registers (ids emitted in order with ballots); wider rows
// (long-context decode) use one CTA per row.
#include "kernels.h"

namespace msa {
namespace {

struct TopkArgs {
  const float* scores;
  int32_t* ids;
  float* kept;  // when not null: the score of each kept id (-inf for padding)
  const int32_t* seq_lens;
  int rows, n_q, max_kv, h, block, nblk, topk, causal, force_own;
  DeviceStatus* st;
  int* zero;  // cleared by CTA 0 when not null (nzero words)
  int nzero;
};

// CTA 0 clears the words the caller asked for (before any early exit).
__device__ __forceinline__ void clear_words(const TopkArgs& a) {
  if (blockIdx.x == 0 && a.zero != nullptr)
    for (int i = threadIdx.x; i < a.nzero; i += blockDim.x) a.zero[i] = 0;
}

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

// Search state: T's bits above `hi` are known (`prefix`); the bucket is the keys
// sharing them (`cnt` keys, the forced block excluded), `above` keys (the forced
// block included) are larger than the whole bucket, and T is the key of rank
// `need` = m - above in the bucket.  Keys 0 (past the frontier) and 0xffffffff
// (the forced block) are never in the bucket.
struct Bucket {
  uint32_t prefix;
  int hi, cnt, above;
};

// Mask of the bits above `hi` (hi in [-1, 31]).
__device__ __forceinline__ uint32_t bits_above(int hi) {
  return hi >= 31 ? 0u : (hi < 0 ? 0xffffffffu : ~((2u << hi) - 1u));
}

__device__ __forceinline__ bool in_bucket(uint32_t key, const Bucket& r) {
  return key != 0u && key != 0xffffffffu && (key & bits_above(r.hi)) == r.prefix;
}

// Bucket of a row whose visible keys lie in [kmin, kmax] (kmin <= kmax): their
// common high bits are known, all `cnt` visible keys are in it.
__device__ __forceinline__ Bucket bucket_start(uint32_t kmax, uint32_t kmin, int cnt, int above) {
  const uint32_t diff = kmax ^ kmin;
  Bucket r;
  r.hi = diff ? 31 - __clz(diff) : -1;
  r.prefix = kmax & bits_above(r.hi);
  r.cnt = cnt;
  r.above = above;
  return r;
}

// One halving step at bit r.hi, given c = count(key >= prefix | 1 << hi) over all
// of the row's keys.
__device__ __forceinline__ void bucket_split(Bucket& r, int c, int m) {
  if (c >= m) {
    r.prefix |= 1u << r.hi;  // T is in the upper half
    r.cnt = c - r.above;
  } else {
    r.cnt -= c - r.above;  // lower half; the upper half is above T
    r.above = c;
  }
  --r.hi;
}

// Among the (at most 32) bucket keys gathered in id order in `ck` (lane i holds
// the i-th, `n` of them), the key of rank need - 1 by (key desc, id asc).
__device__ __forceinline__ uint32_t rank_pick(uint32_t ck, int n, int need, int lane) {
  int rank = 0;
  for (int j = 0; j < n; ++j) {
    const uint32_t o = __shfl_sync(0xffffffffu, ck, j);
    rank += (o > ck) || (o == ck && j < lane);
  }
  const unsigned hit = __ballot_sync(0xffffffffu, lane < n && rank == need - 1);
  return __shfl_sync(0xffffffffu, ck, __ffs(hit) - 1);
}

// Top-m of one row by one warp, element i = e*32 + lane for e < EE: keys in
// registers, counts by warp reductions, the last bucket gathered in `cbuf` (32
// words private to the warp), ids emitted in order with ballots.
template <int EE>
__device__ __forceinline__ void warp_row_topk(const float* s, int32_t* out, const RowInfo& ri,
                                              int lane, uint32_t* cbuf) {
  // The threshold lies between the smallest and the largest visible key: it
  // shares their common high bits, and the search starts below them.  (The
  // forced block's own score may widen that range; that is harmless.)  Keys
  // past the frontier are 0, which k - 1 turns into the largest value for the
  // minimum.
  uint32_t key[EE];
  uint32_t kmax = 0u, kmin1 = 0xffffffffu;
#pragma unroll
  for (int e = 0; e < EE; ++e) {
    const int i = e * 32 + lane;
    key[e] = i < ri.F ? order_key(s[i]) : 0u;
    kmax = max(kmax, key[e]);
    kmin1 = min(kmin1, key[e] - 1u);
    if (i == ri.own) key[e] = 0xffffffffu;
  }
  const int m = ri.m;
  const int forced = ri.own >= 0 ? 1 : 0;
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const uint32_t kmin = __reduce_min_sync(0xffffffffu, kmin1) + 1u;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t T;
  if (m <= forced || kmax < kmin) {
    T = 0xffffffffu;  // only the forced block is taken
  } else {
    Bucket r = bucket_start(kmax, kmin, ri.F - forced, forced);
    while (r.cnt > 32 && r.hi >= 0) {
      const uint32_t cand = r.prefix | (1u << r.hi);
      unsigned c4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < EE; ++e) c4[e & 3] += key[e] >= cand;
      bucket_split(r, (int)__reduce_add_sync(0xffffffffu, (c4[0] + c4[1]) + (c4[2] + c4[3])), m);
    }
    if (r.cnt > 32) {
      T = r.prefix;  // every bit resolved: the remaining keys all equal T
    } else {
      int base = 0;
#pragma unroll
      for (int e = 0; e < EE; ++e) {
        const bool u = in_bucket(key[e], r);
        const unsigned bu = __ballot_sync(0xffffffffu, u);
        if (u) cbuf[base + __popc(bu & lt)] = key[e];
        base += __popc(bu);
      }
      __syncwarp();
      const uint32_t ck = lane < r.cnt ? cbuf[lane] : 0u;
      __syncwarp();
      T = rank_pick(ck, r.cnt, m - r.above, lane);
    }
  }
  unsigned ge = 0;
#pragma unroll
  for (int e = 0; e < EE; ++e) ge += key[e] >= T;
  ge = __reduce_add_sync(0xffffffffu, ge);
  int base = 0;
  if ((int)ge == m) {
    // every key equal to T is taken (the usual case: T is unique)
#pragma unroll
    for (int e = 0; e < EE; ++e) {
      const bool sel = key[e] >= T;
      const unsigned bs = __ballot_sync(0xffffffffu, sel);
      if (sel) out[base + __popc(bs & lt)] = e * 32 + lane;
      base += __popc(bs);
    }
    return;
  }
  unsigned gt = 0;
#pragma unroll
  for (int e = 0; e < EE; ++e) gt += key[e] > T;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need = m - (int)gt;
  int eqbase = 0;
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
__global__ void __launch_bounds__(256, 3) topk_warp_kernel(TopkArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  clear_words(a);
  __shared__ uint32_t cbuf[8][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + w;
  if (row >= a.rows) return;
  const RowInfo ri = row_info(a, row);
  const float* s = a.scores + (int64_t)row * a.nblk;
  int32_t* out = a.ids + (int64_t)row * a.topk;
  const int m = ri.m, ne = (ri.F + 31) >> 5;
  if (m == ri.F) {
    for (int i = lane; i < m; i += 32) out[i] = i;
  } else if (ne <= 1 || E == 1) {
    warp_row_topk<1>(s, out, ri, lane, cbuf[w]);
  } else if (ne <= 2 || E == 2) {
    warp_row_topk<(E < 2 ? E : 2)>(s, out, ri, lane, cbuf[w]);
  } else if (ne <= 4 || E == 4) {
    warp_row_topk<(E < 4 ? E : 4)>(s, out, ri, lane, cbuf[w]);
  } else if (ne <= 8 || E == 8) {
    warp_row_topk<(E < 8 ? E : 8)>(s, out, ri, lane, cbuf[w]);
  } else if (ne <= 16 || E == 16) {
    warp_row_topk<(E < 16 ? E : 16)>(s, out, ri, lane, cbuf[w]);
  } else {
    warp_row_topk<E>(s, out, ri, lane, cbuf[w]);
  }
  for (int i = m + lane; i < a.topk; i += 32) out[i] = -1;
  if (a.kept != nullptr) {
    __syncwarp();
    float* kp = a.kept + (int64_t)row * a.topk;
    for (int i = lane; i < a.topk; i += 32)
      kp[i] = i < m ? s[out[i]] : -__int_as_float(0x7f800000);
  }
}

// Sums over the CTA (NW warps) of W words per thread; `buf` alternates between
// calls so one barrier per call suffices.  Each warp reads the NW partial sums
// of a word with one load per lane.
template <int NW, int W>
__device__ __forceinline__ void cta_sums(unsigned (&v)[W], unsigned (*red)[2][32], int& buf) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < W; ++k) v[k] = __reduce_add_sync(0xffffffffu, v[k]);
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < W; ++k) red[buf][k][threadIdx.x >> 5] = v[k];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < W; ++k)
    v[k] = __reduce_add_sync(0xffffffffu, lane < NW ? red[buf][k][lane] : 0u);
  buf ^= 1;
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

// One 8-bit step of the threshold search, for a bucket with at least 8 unresolved
// bits: the bucket's keys are counted by their bits [hi - 7, hi] in a shared
// histogram (hist[hb]; the other buffer is cleared for the next step) and the
// digit holding the bucket key of rank need = m - above (counted from the top) is
// found from suffix sums over the 256 bins, taken by the first 256 threads.  The
// bucket becomes that digit's keys: eight bits resolved for three barriers.
template <int NT, int E>
__device__ __forceinline__ void bucket_radix8(Bucket& r, const uint32_t (&key)[E], int m,
                                              unsigned (*hist)[256], int& hb, unsigned* wsum8,
                                              int* res) {
  static_assert(NT >= 256, "a thread per bin");
  const int sh = r.hi - 7;
  unsigned* h = hist[hb];
  if (threadIdx.x < 256) hist[hb ^ 1][threadIdx.x] = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (in_bucket(key[e], r)) atomicAdd(&h[(key[e] >> sh) & 255u], 1u);
  __syncthreads();
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  unsigned v = 0u, inc = 0u;
  if (t < 256) {
    v = h[255 - t];
    inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    if (lane == 31) wsum8[w] = inc;
  }
  __syncthreads();
  if (t < 256) {
    unsigned before = 0u;
    for (int k = 0; k < w; ++k) before += wsum8[k];
    const unsigned incl = before + inc, excl = incl - v, need = (unsigned)(m - r.above);
    if (excl < need && need <= incl) {
      res[0] = 255 - t;
      res[1] = (int)excl;
      res[2] = (int)v;
    }
  }
  __syncthreads();
  r.prefix |= (uint32_t)res[0] << sh;
  r.above += res[1];
  r.cnt = res[2];
  r.hi = sh - 1;
  hb ^= 1;
}

// One CTA of NT threads per row; thread i holds elements [i*E, i*E + E), read
// with 16-byte loads.  While the bucket holds more than 64 keys the search takes
// eight bits per step (bucket_radix8, three barriers), then one bit per step (one
// CTA sum, one barrier).  The last
// bucket (at most 32 keys) is gathered in any order: T is a key value, so the
// order among equal keys does not change it.  One more sum counts the keys above
// and equal to T; only when some keys equal to T must be left out are they
// ranked by id.
template <int NT, int E>
__global__ void __launch_bounds__(NT) topk_cta_kernel(TopkArgs a) {
  static_assert(E % 4 == 0, "four keys per vector load");
  grid_dep_wait();
  grid_dep_launch();
  clear_words(a);
  constexpr int NW = NT / 32;
  __shared__ uint32_t cbuf[32];
  __shared__ int ccount;
  __shared__ unsigned red[2][2][32];
  __shared__ unsigned wsum[32];
  __shared__ uint32_t wmax[NW], wmin[NW];
  __shared__ uint32_t Ts;
  __shared__ unsigned hist[2][256];
  __shared__ unsigned wsum8[8];
  __shared__ int rres[3];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x;
  const RowInfo ri = row_info(a, row);
  const float* s = a.scores + (int64_t)row * a.nblk;
  int32_t* out = a.ids + (int64_t)row * a.topk;
  const int i0 = threadIdx.x * E;
  const int m = ri.m, forced = ri.own >= 0 ? 1 : 0;
  if (m == ri.F) {
    for (int i = threadIdx.x; i < m; i += NT) out[i] = i;
  } else {
    if (threadIdx.x == 0) ccount = 0;  // ordered before its use by the barriers below
    uint32_t key[E];
    uint32_t kmax = 0u, kmin = 0xffffffffu;
    const bool vec = (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
#pragma unroll
    for (int v = 0; v < E / 4; ++v) {
      const int i = i0 + 4 * v;
      float f[4];
      if (vec && i + 3 < a.nblk) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(s + i));
        f[0] = x.x;
        f[1] = x.y;
        f[2] = x.z;
        f[3] = x.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) f[u] = i + u < ri.F ? s[i + u] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = 4 * v + u;
        key[e] = i + u < ri.F ? order_key(f[u]) : 0u;
        if (i + u == ri.own) key[e] = 0xffffffffu;
        const bool vis = key[e] != 0u && key[e] != 0xffffffffu;
        kmax = vis ? max(kmax, key[e]) : kmax;
        kmin = vis ? min(kmin, key[e]) : kmin;
      }
    }
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    if (lane == 0) {
      wmax[warp] = kmax;
      wmin[warp] = kmin;
    }
    if (threadIdx.x < 256) hist[0][threadIdx.x] = 0u;
    __syncthreads();
    kmax = __reduce_max_sync(0xffffffffu, lane < NW ? wmax[lane] : 0u);
    kmin = __reduce_min_sync(0xffffffffu, lane < NW ? wmin[lane] : 0xffffffffu);
    uint32_t T;
    int buf = 0;
    if (m <= forced || kmax < kmin) {
      T = 0xffffffffu;  // only the forced block is taken
    } else {
      Bucket r = bucket_start(kmax, kmin, ri.F - forced, forced);
      int hb = 0;
      while (r.cnt > 32 && r.hi >= 0) {
        if (r.cnt > 64 && r.hi >= 7) {
          bucket_radix8<NT, E>(r, key, m, hist, hb, wsum8, rres);
          continue;
        }
        const uint32_t cand = r.prefix | (1u << r.hi);
        unsigned c[1] = {0u};
#pragma unroll
        for (int e = 0; e < E; ++e) c[0] += key[e] >= cand;
        cta_sums<NW, 1>(c, red, buf);
        bucket_split(r, (int)c[0], m);
      }
      if (r.cnt > 32) {
        T = r.prefix;  // every bit resolved: the remaining keys all equal T
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e)
          if (in_bucket(key[e], r)) {
            const int at = atomicAdd(&ccount, 1);
            if (at < 32) cbuf[at] = key[e];  // r.cnt <= 32 keys are in the bucket
          }
        __syncthreads();
        if (warp == 0) {
          const uint32_t ck = lane < r.cnt ? cbuf[lane] : 0u;
          const uint32_t t = rank_pick(ck, r.cnt, m - r.above, lane);
          if (lane == 0) Ts = t;
        }
        __syncthreads();
        T = Ts;
      }
    }
    unsigned ge[2] = {0u, 0u};  // keys above T, keys equal to T
#pragma unroll
    for (int e = 0; e < E; ++e) {
      ge[0] += key[e] > T;
      ge[1] += key[e] == T;
    }
    cta_sums<NW, 2>(ge, red, buf);
    const int need = m - (int)ge[0];
    unsigned nsel = 0;
    bool sel[E];
    if ((int)ge[1] <= need) {
      // every key equal to T is taken (the usual case: T is unique)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        sel[e] = key[e] >= T;
        nsel += sel[e];
      }
    } else {
      unsigned eq = 0;
#pragma unroll
      for (int e = 0; e < E; ++e) eq += key[e] == T;
      unsigned eqr = cta_exclusive_scan<NW>(eq, wsum);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const bool is_eq = key[e] == T;
        sel[e] = key[e] > T || (is_eq && (int)eqr < need);
        eqr += is_eq;
        nsel += sel[e];
      }
    }
    unsigned pos = cta_exclusive_scan<NW>(nsel, wsum);
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (sel[e]) out[pos++] = i0 + e;
  }
  for (int i = m + threadIdx.x; i < a.topk; i += NT) out[i] = -1;
  if (a.kept != nullptr) {
    __syncthreads();
    float* kp = a.kept + (int64_t)row * a.topk;
    for (int i = threadIdx.x; i < a.topk; i += NT)
      kp[i] = i < m ? s[out[i]] : -__int_as_float(0x7f800000);
  }
}

// ------------------------------------------------ merge of candidate lists
// Global top-k of a row from the candidate lists of several KV shards (each
// shard's own top-k of its blocks, with their scores): the same order as the
// single-device top-k (score descending, block id ascending, the own block first
// when forced), because a row's global top-k blocks are each in the top-k of the
// shard that holds them.  The lists arrive as an all-gather leaves them, list
// after list ([nlists, rows, len]); list r holds ascending ids local to shard r,
// whose blocks start at r * shard_blocks, so a row's valid candidates, taken
// list by list, come in ascending global id order and position order breaks
// ties by id.  A forced own block needs no score: it is taken first even when no
// shard listed it.
struct CandArgs {
  const float* cscores;  // [nlists, rows, len]
  const int32_t* cids;   // [nlists, rows, len], -1 = empty
  int32_t* ids;          // [rows, topk] global ids (nullable)
  int32_t* local;        // [rows, topk] id - base inside [base, base + nloc), else -1 (nullable)
  const int32_t* seq_lens;
  int rows, nlists, len, shard_blocks, n_q, max_kv, h, block, topk, force_own, base, nloc;
  DeviceStatus* st;
};

template <int NT, int E>
__global__ void __launch_bounds__(NT) candidates_topk_kernel(CandArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int NW = NT / 32;
  __shared__ uint32_t cbuf[32];
  __shared__ int ccount;
  __shared__ unsigned red[2][2][32];
  __shared__ unsigned wsum[32];
  __shared__ uint32_t Ts;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x;
  const int bt = row / a.h;
  const int t = bt % a.n_q, b = bt / a.n_q;
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int p = L - a.n_q + t;
  const int own = (a.force_own && p >= 0) ? p / a.block : -1;
  const int ncand = a.nlists * a.len;
  const int i0 = threadIdx.x * E;
  if (threadIdx.x == 0) ccount = 0;
  uint32_t key[E];
  int id[E];
  unsigned cnt[2] = {0u, 0u};  // valid candidates (the own block excluded), own present
  uint32_t kmax = 0u, kmin = 0xffffffffu;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = i0 + e;
    const int li = i / a.len;  // list (shard) of candidate i
    const int64_t at = ((int64_t)li * a.rows + row) * a.len + (i - li * a.len);
    id[e] = i < ncand ? __ldg(a.cids + at) : -1;
    key[e] = id[e] >= 0 ? order_key(__ldg(a.cscores + at)) : 0u;
    if (id[e] >= 0) id[e] += li * a.shard_blocks;
    if (id[e] >= 0 && id[e] == own) key[e] = 0xffffffffu;
    const bool vis = key[e] != 0u && key[e] != 0xffffffffu;
    cnt[0] += vis;
    cnt[1] += key[e] == 0xffffffffu;
    kmax = vis ? max(kmax, key[e]) : kmax;
    kmin = vis ? min(kmin, key[e]) : kmin;
  }
  int buf = 0;
  cta_sums<NW, 2>(cnt, red, buf);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  __shared__ uint32_t wmax[NW], wmin[NW];
  if (lane == 0) {
    wmax[warp] = kmax;
    wmin[warp] = kmin;
  }
  __syncthreads();
  kmax = __reduce_max_sync(0xffffffffu, lane < NW ? wmax[lane] : 0u);
  kmin = __reduce_min_sync(0xffffffffu, lane < NW ? wmin[lane] : 0xffffffffu);
  const int forced = own >= 0 ? 1 : 0;
  const bool virt = forced && cnt[1] == 0u;  // forced own block listed by no shard
  const int m = min(a.topk, (int)cnt[0] + forced);
  uint32_t T;
  if (m <= forced || kmax < kmin) {
    T = 0xffffffffu;
  } else {
    Bucket r = bucket_start(kmax, kmin, (int)cnt[0], forced);
    while (r.cnt > 32 && r.hi >= 0) {
      const uint32_t cand = r.prefix | (1u << r.hi);
      unsigned c[1] = {0u};
#pragma unroll
      for (int e = 0; e < E; ++e) c[0] += key[e] >= cand;
      if (virt && threadIdx.x == 0) c[0] += 1u;  // the unlisted forced block, counted once
      cta_sums<NW, 1>(c, red, buf);
      bucket_split(r, (int)c[0], m);
    }
    if (r.cnt > 32) {
      T = r.prefix;
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (in_bucket(key[e], r)) {
          const int at = atomicAdd(&ccount, 1);
          if (at < 32) cbuf[at] = key[e];
        }
      __syncthreads();
      if (warp == 0) {
        const uint32_t ck = lane < r.cnt ? cbuf[lane] : 0u;
        const uint32_t tt = rank_pick(ck, r.cnt, m - r.above, lane);
        if (lane == 0) Ts = tt;
      }
      __syncthreads();
      T = Ts;
    }
  }
  unsigned ge[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < E; ++e) {
    ge[0] += key[e] > T;
    ge[1] += key[e] == T;
  }
  if (virt && threadIdx.x == 0) ge[T == 0xffffffffu ? 1 : 0] += 1u;
  cta_sums<NW, 2>(ge, red, buf);
  const int need = m - (int)ge[0];
  unsigned eq = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) eq += key[e] == T;
  // a virtual own block (key T only when T is the forced key) ranks before all
  unsigned eqr = cta_exclusive_scan<NW>(eq, wsum) + ((virt && T == 0xffffffffu) ? 1u : 0u);
  bool sel[E];
  unsigned nsel = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const bool is_eq = key[e] == T;
    sel[e] = key[e] != 0u && (key[e] > T || (is_eq && (int)eqr < need));
    eqr += is_eq;
    nsel += sel[e];
  }
  // output slots in ascending id order: position order, with a virtual own
  // block placed before the first selected id above it
  unsigned pos = cta_exclusive_scan<NW>(nsel, wsum);
  unsigned below_own = 0;
  if (virt) {
#pragma unroll
    for (int e = 0; e < E; ++e) below_own += sel[e] && id[e] < own;
    unsigned tmp[1] = {below_own};
    cta_sums<NW, 1>(tmp, red, buf);
    below_own = tmp[0];
  }
  int32_t* og = a.ids ? a.ids + (int64_t)row * a.topk : nullptr;
  int32_t* ol = a.local ? a.local + (int64_t)row * a.topk : nullptr;
  auto emit = [&](int slot, int gid) {
    if (og) og[slot] = gid;
    if (ol) ol[slot] = (gid >= a.base && gid < a.base + a.nloc) ? gid - a.base : -1;
  };
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (sel[e]) {
      const int slot = (int)pos + ((virt && id[e] > own) ? 1 : 0);
      ++pos;
      if (slot < a.topk) emit(slot, id[e]);
    }
  if (virt && threadIdx.x == 0 && (int)below_own < a.topk) emit((int)below_own, own);
  for (int i = m + threadIdx.x; i < a.topk; i += NT) emit(i, -1);
}

}  // namespace

cudaError_t launch_topk(const Shape& s, const float* scores, int32_t* ids, DeviceStatus* st,
                        cudaStream_t stream, int* zero, int nzero, float* kept) {
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
  a.zero = zero;
  a.nzero = nzero;
  a.kept = kept;
  const int n = s.nblk;
  if (n <= 1024) {
    const dim3 grid((a.rows + 7) / 8);
#define MSA_TOPK_WARP(E_)                                             \
  if (n <= 32 * E_) {                                                 \
    return launch_pdl(topk_warp_kernel<E_>, grid, dim3(256), 0, stream, a); \
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
    return launch_pdl(topk_cta_kernel<NT_, E_>, grid, dim3(NT_), 0, stream, a); \
  }
  MSA_TOPK_CTA(512, 4)
  MSA_TOPK_CTA(256, 8)
  MSA_TOPK_CTA(256, 16)
  MSA_TOPK_CTA(512, 16)
  MSA_TOPK_CTA(1024, 16)
  MSA_TOPK_CTA(1024, 32)
  MSA_TOPK_CTA(1024, 64)
#undef MSA_TOPK_CTA
  return cudaErrorInvalidValue;
}

cudaError_t launch_candidates_topk(const Shape& s, int nlists, int len, int shard_blocks,
                                   const float* cscores, const int32_t* cids, int base, int nloc,
                                   int32_t* ids, int32_t* local, DeviceStatus* st,
                                   cudaStream_t stream) {
  CandArgs a;
  a.cscores = cscores;
  a.cids = cids;
  a.ids = ids;
  a.local = local;
  a.seq_lens = s.seq_lens;
  a.rows = s.batch * s.n_q * s.h;
  a.nlists = nlists;
  a.len = len;
  a.shard_blocks = shard_blocks;
  const int ncand = nlists * len;
  a.n_q = s.n_q;
  a.max_kv = s.max_kv;
  a.h = s.h;
  a.block = s.block;
  a.topk = s.topk;
  a.force_own = s.force_own;
  a.base = base;
  a.nloc = nloc;
  a.st = st;
  const dim3 grid(a.rows);
#define MSA_CAND_CTA(NT_, E_)                                            \
  if (ncand <= NT_ * E_) {                                               \
    return launch_pdl(candidates_topk_kernel<NT_, E_>, grid, dim3(NT_), 0, stream, a); \
  }
  MSA_CAND_CTA(256, 4)
  MSA_CAND_CTA(256, 16)
  MSA_CAND_CTA(1024, 16)
#undef MSA_CAND_CTA
  return cudaErrorInvalidValue;
}

}  // namespace msa
