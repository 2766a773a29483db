// Sparse branch for prefill, KV-major on the fifth-generation tensor cores.
//
// "MiniMax goes sparse" (atlascloud.ai), section 1, step 2: softmax attention over
// the raw K/V of the selected blocks only, every head of a GQA group sharing the
// group's selection ("MiniMax M3 的 MSA ...", second layer).
//
// In prefill, neighbouring queries rarely pick the same blocks, so a query-major
// kernel must bring a whole K/V block on chip for the G heads of one query.  Here
// the loop is inverted (the "KV outer, gather Q" order): for every (sequence,
// group, block) the queries that selected it are listed (an inverted index built
// by counting, scanning and scattering), and a CTA loads the block's K and V once
// and streams tiles of up to 128 (query, head) rows through it:
//   S = Q_tile K^T      tcgen05 MMA, M = 128 rows, N = block, K = d   (TMEM)
//   P = softmax(S)      registers, one thread per row, masked to visible keys
//   O = P V             tcgen05 MMA, M = 128, N = d, K = block       (TMEM)
// Each (query, head, block) gives a normalised bf16 partial output and its
// log-sum-exp; a combine kernel merges a query's partials by log-sum-exp weights.
// Queries are processed in chunks so that the partials of one chunk fit a bounded
// workspace.
//
// CTA roles (persistent CTAs, each a contiguous share of the chunk's tiles):
//   warp 0      TMA producer of K and V (a new load only when the block changes);
//   warp 1      tensor-memory allocation and the thread issuing the S = Q K^T MMAs;
//   warps 2-5   gather the tile's Q rows with 16-byte async copies (swizzled), one
//               thread per row;
//   warps 6-17  three softmax warp groups taking tiles in turn, one thread per tile
//               row: softmax from tensor memory, the P tile into shared memory, then
//               (one elected thread) the O = P V MMA, then the output epilogue.
// Buffers: 3-4 Q/P tiles (P overwrites its Q once S is computed), 2 K/V stages
// (each released by every warp group once its products are done), and 4 tile
// buffers in tensor memory where O = P V overwrites the S it was computed from.
// Every wait is bounded.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kRows = 128;                  // MMA M: (query, head) rows per tile
constexpr int kNw = 3;                     // softmax warp groups
constexpr int kKvThreads = (6 + 4 * kNw) * 32;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpGather0 = 2, kWarpSoft0 = 6;

struct KvArgs {
  // problem
  const uint16_t* q;
  int64_t q_s0, q_s1, q_s2;
  const int32_t* ids;      // [b, n_q, h, topk]
  const int32_t* seq_lens;
  int n_q, max_kv, H, h, G, topk, nblk, causal;
  float scale_log2;
  // chunk of flattened (b, t) rows handled by this launch
  int64_t bt0;
  int nbt;
  // inverted index
  int* counts;             // [batch * h * nblk]
  int* offs;               // [batch * h * nblk + 1] entry offsets
  int* toffs;              // [batch * h * nblk + 1] tile offsets
  int* entries;            // chunk-relative slot positions, grouped by (b, g, block)
  int qpt;                 // queries per tile
  int nj;                  // batch * h * nblk
  // partials (chunk-relative position p = (bt_rel * h + g) * topk + slot)
  uint16_t* part_o;        // [p][G][d] bf16
  float* part_lse;         // [p][G]
  uint16_t* out;
  int64_t o_s0, o_s1, o_s2;
  float* lse;
  DeviceStatus* st;
  uint64_t wait_ns;
};

__device__ __forceinline__ int visible_limit(const KvArgs& a, int b, int t) {
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int p = L - a.n_q + t;
  return max(0, a.causal ? min(L, p + 1) : L);
}

// Valid slot of the chunk: a block id that exists and holds a visible token.
__device__ __forceinline__ bool slot_block(const KvArgs& a, int64_t pos, int& b, int& g,
                                           int& beta, int BLK) {
  const int64_t bt_rel = pos / ((int64_t)a.h * a.topk);
  const int rem = (int)(pos % ((int64_t)a.h * a.topk));
  g = rem / a.topk;
  const int64_t bt = a.bt0 + bt_rel;
  b = (int)(bt / a.n_q);
  const int t = (int)(bt % a.n_q);
  beta = a.ids[(bt * a.h + g) * a.topk + rem % a.topk];
  if (beta < 0) return false;
  if (beta >= a.nblk) {
    record_error(a.st, kErrDeviceAssert, (uint32_t)bt);
    return false;
  }
  return (int64_t)beta * BLK < visible_limit(a, b, t);
}

// ----------------------------------------------------------- inverted index
__global__ void kv_count_kernel(KvArgs a, int BLK) {
  const int64_t n = (int64_t)a.nbt * a.h * a.topk;
  for (int64_t pos = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; pos < n;
       pos += (int64_t)gridDim.x * blockDim.x) {
    int b, g, beta;
    if (slot_block(a, pos, b, g, beta, BLK))
      atomicAdd(&a.counts[((int64_t)b * a.h + g) * a.nblk + beta], 1);
  }
}

// Exclusive scans of the counts (entry offsets) and of the tile counts
// (ceil(count / qpt)); the counts are zeroed to serve as scatter cursors.
__global__ void __launch_bounds__(1024) kv_scan_kernel(KvArgs a) {
  __shared__ int wsum[2][32];
  __shared__ int carry[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  for (int base = 0; base < a.nj; base += 1024) {
    const int j = base + threadIdx.x;
    const int c = j < a.nj ? a.counts[j] : 0;
    const int tl = (c + a.qpt - 1) / a.qpt;
    int ic = c, it = tl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nc = __shfl_up_sync(0xffffffffu, ic, o);
      const int nt = __shfl_up_sync(0xffffffffu, it, o);
      if (lane >= o) {
        ic += nc;
        it += nt;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = ic;
      wsum[1][warp] = it;
    }
    __syncthreads();
    int bc = 0, bt = 0, tc_ = 0, tt = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < warp) {
        bc += wsum[0][w];
        bt += wsum[1][w];
      }
      tc_ += wsum[0][w];
      tt += wsum[1][w];
    }
    if (j < a.nj) {
      a.offs[j] = carry[0] + bc + ic - c;
      a.toffs[j] = carry[1] + bt + it - tl;
      a.counts[j] = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      carry[0] += tc_;
      carry[1] += tt;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    a.offs[a.nj] = carry[0];
    a.toffs[a.nj] = carry[1];
  }
}

__global__ void kv_scatter_kernel(KvArgs a, int BLK) {
  const int64_t n = (int64_t)a.nbt * a.h * a.topk;
  for (int64_t pos = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; pos < n;
       pos += (int64_t)gridDim.x * blockDim.x) {
    int b, g, beta;
    if (slot_block(a, pos, b, g, beta, BLK)) {
      const int64_t j = ((int64_t)b * a.h + g) * a.nblk + beta;
      const int k = atomicAdd(&a.counts[j], 1);
      a.entries[a.offs[j] + k] = (int)pos;
    }
  }
}

// ------------------------------------------------------------ tile walker
// Tiles are numbered through the (b, g, block) lists in order; a walker moves
// forward through them, amortising the lookup of the list a tile belongs to.
struct TileWalker {
  int j;
  __device__ __forceinline__ void seek(const KvArgs& a, int tile) {
    int lo = 0, hi = a.nj;  // toffs[lo] <= tile < toffs[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a.toffs + mid) <= tile) lo = mid; else hi = mid;
    }
    j = lo;
  }
  __device__ __forceinline__ void advance(const KvArgs& a, int tile) {
    while (__ldg(a.toffs + j + 1) <= tile) ++j;
  }
};

struct TileInfo {
  int j, b, g, beta, first, nq;  // entries [first, first + nq)
};

__device__ __forceinline__ TileInfo tile_info(const KvArgs& a, int j, int tile) {
  TileInfo ti;
  ti.j = j;
  ti.beta = j % a.nblk;
  const int bg = j / a.nblk;
  ti.g = bg % a.h;
  ti.b = bg / a.h;
  const int u = tile - __ldg(a.toffs + j);
  const int cnt = __ldg(a.offs + j + 1) - __ldg(a.offs + j);
  ti.first = __ldg(a.offs + j) + u * a.qpt;
  ti.nq = min(a.qpt, cnt - u * a.qpt);
  return ti;
}

// --------------------------------------------------------- attention tiles
// Shared-memory plan of the attention kernel for one (D, BLK).
template <int D, int BLK>
struct KvSmem {
  static constexpr uint32_t QP = kRows * (D > BLK ? D : BLK) * 2;  // a Q tile or a P tile
  static constexpr uint32_t HALF = BLK * 128u;                     // one 64-dim atom of K or V
  static constexpr uint32_t KV = 2 * (D / 64) * HALF;              // K and V of one block
  static constexpr int NQ = (4 * QP + 2 * KV + 2048 <= 227u * 1024u) ? 4 : 3;
  static constexpr uint32_t BYTES = 1024 + NQ * QP + 2 * KV + 512;
};

template <int D, int BLK>
__global__ void __launch_bounds__(kKvThreads, 1)
    kv_attn_kernel(const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, KvArgs a) {
  using SM = KvSmem<D, BLK>;
  constexpr int NH = D / 64;
  constexpr int NQ = SM::NQ;                  // Q/P tile buffers
  constexpr int NB = 4;                       // tensor-memory tile buffers
  constexpr uint32_t TB = D > BLK ? D : BLK;  // columns per buffer: S, then O in place
  constexpr uint32_t QP_BYTES = SM::QP, HALF = SM::HALF, KV_BYTES = SM::KV;
  constexpr uint32_t TMEM_COLS = NB * TB <= 256 ? 256 : 512;
  static_assert(NB * TB <= 512, "tensor memory");
  if (status_failed(a.st)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sm0a = smem_u32(smem);
  const uint32_t sqp = sm0a;                     // NQ x QP_BYTES
  const uint32_t skv = sqp + NQ * QP_BYTES;      // 2 x KV_BYTES
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NQ * QP_BYTES + 2 * KV_BYTES);
  // barrier blocks (8 bytes each)
  const uint32_t b_kvfull = smem_u32(bars);                 // [2]
  const uint32_t b_kvempty = b_kvfull + 16;                 // [2][kNw]
  const uint32_t b_qfull = b_kvempty + 16 * kNw;            // [NQ]
  const uint32_t b_qempty = b_qfull + 8 * NQ;               // [NQ]
  const uint32_t b_sfull = b_qempty + 8 * NQ;               // [NB]
  const uint32_t b_ofull = b_sfull + 8 * NB;                // [NB]
  const uint32_t b_ofree = b_ofull + 8 * NB;                // [NB]
  const uint32_t b_done = b_ofree + 8 * NB;                 // [1 + kNw]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + NQ * QP_BYTES + 2 * KV_BYTES + 480);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = __ldg(a.toffs + a.nj);
  const int per = (ntiles + gridDim.x - 1) / gridDim.x;
  const int tile0 = blockIdx.x * per;
  const int tile1 = min(ntiles, tile0 + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(b_kvfull + 8 * s, 1);
      for (int w = 0; w < kNw; ++w) mbar_init(b_kvempty + 8 * (s * kNw + w), 1);
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(b_qfull + 8 * i, 128);
      mbar_init(b_qempty + 8 * i, 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(b_sfull + 8 * i, 1);
      mbar_init(b_ofull + 8 * i, 1);
      mbar_init(b_ofree + 8 * i, 4);
    }
    for (int i = 0; i <= kNw; ++i) mbar_init(b_done + 8 * i, 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tc::tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (tile0 < tile1) {
    TileWalker w;
    w.seek(a, tile0);
    if (warp == kWarpProd) {
      // ------------------------------------------------------ K/V producer
      if (lane == 0) {
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
        int use = -1, prev_j = -1, issued = 0;
        bool ok = true;
        for (int tile = tile0; tile < tile1 && ok; ++tile) {
          w.advance(a, tile);
          if (w.j == prev_j) continue;
          prev_j = w.j;
          ++use;
          const int s = use & 1;
          if (use >= 2)
            for (int g = 0; g < kNw && ok; ++g)
              ok = mbar_wait_bounded(b_kvempty + 8 * (s * kNw + g), ((use >> 1) - 1) & 1, a.st,
                                     0x201u, a.wait_ns);
          if (!ok) break;
          const TileInfo ti = tile_info(a, w.j, tile);
          mbar_arrive_expect_tx(b_kvfull + 8 * s, KV_BYTES);
          const uint32_t kd = skv + s * KV_BYTES, vd = kd + NH * HALF;
#pragma unroll
          for (int hh = 0; hh < NH; ++hh) {
            tma_load_4d(kd + hh * HALF, &tmk, b_kvfull + 8 * s, hh * 64, ti.g, ti.beta * BLK, ti.b);
            tma_load_4d(vd + hh * HALF, &tmv, b_kvfull + 8 * s, hh * 64, ti.g, ti.beta * BLK, ti.b);
          }
          issued = use + 1;
        }
        // drain: the stages of the last two blocks are released once every
        // warp group's O = P V products that read them have completed
        for (int u = max(0, issued - 2); u < issued; ++u)
          for (int g = 0; g < kNw; ++g)
            mbar_wait_bounded(b_kvempty + 8 * ((u & 1) * kNw + g), (u >> 1) & 1, a.st, 0x202u,
                              a.wait_ns);
      }
    } else if (warp == kWarpMma) {
      // ------------------------------------------------------ S = Q K^T issue
      if (lane == 0) {
        const uint32_t id_qk = tc::idesc_bf16(kRows, BLK, false);
        int use = -1, prev_j = -1, i = 0;
        bool ok = true;
        for (int tile = tile0; tile < tile1 && ok; ++tile, ++i) {
          w.advance(a, tile);
          if (w.j != prev_j) {
            prev_j = w.j;
            ++use;
            ok = mbar_wait_bounded(b_kvfull + 8 * (use & 1), (use >> 1) & 1, a.st, 0x203u,
                                   a.wait_ns);
          }
          const int qb = i % NQ, tb = i % NB;
          if (ok) ok = mbar_wait_bounded(b_qfull + 8 * qb, (i / NQ) & 1, a.st, 0x204u, a.wait_ns);
          if (ok && i >= NB)
            ok = mbar_wait_bounded(b_ofree + 8 * tb, ((i / NB) - 1) & 1, a.st, 0x205u, a.wait_ns);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t kd = skv + (use & 1) * KV_BYTES;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t koff = (ks >> 2) * (kRows * 128u) + (ks & 3) * 32;
            const uint32_t kboff = (ks >> 2) * HALF + (ks & 3) * 32;
            tc::mma_bf16(tmem + tb * TB, tc::desc_k_sw128(sqp + qb * QP_BYTES + koff),
                         tc::desc_k_sw128(kd + kboff), id_qk, ks > 0 ? 1u : 0u);
          }
          tc::commit(b_sfull + 8 * tb);
        }
        tc::commit(b_done);
        mbar_wait_bounded(b_done, 0, a.st, 0x208u, a.wait_ns);
      }
    } else if (warp < kWarpSoft0) {
      // ----------------------------------------------------- Q gather warps
      const int row = threadIdx.x - kWarpGather0 * 32;  // 0..127: one tile row each
      int i = 0;
      bool ok = true;
      constexpr int CPR = D / 8;  // 16-byte chunks per row
      for (int tile = tile0; tile < tile1; ++tile, ++i) {
        w.advance(a, tile);
        const int qb = i % NQ;
        if (i >= NQ && ok)
          ok = mbar_wait_bounded(b_qempty + 8 * qb, ((i / NQ) - 1) & 1, a.st, 0x209u, a.wait_ns);
        const TileInfo ti = tile_info(a, w.j, tile);
        if (ok && row < ti.nq * a.G) {
          const int qi = row / a.G, hi = row - qi * a.G;
          const int pos = __ldg(a.entries + ti.first + qi);  // chunk-relative slot position
          const int bt = (int)a.bt0 + pos / (a.h * a.topk);
          const uint16_t* src = a.q + (int64_t)ti.b * a.q_s0 + (int64_t)(bt % a.n_q) * a.q_s1 +
                                (int64_t)(ti.g * a.G + hi) * a.q_s2;
          const uint32_t dst0 = sqp + qb * QP_BYTES + row * 128u;
#pragma unroll
          for (int ch = 0; ch < CPR; ++ch) {
            const uint32_t dst = dst0 + (ch >> 3) * (kRows * 128u) + (((ch & 7) ^ (row & 7)) << 4);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + ch * 8));
          }
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
        fence_proxy_async_smem();
        mbar_arrive(b_qfull + 8 * qb);
      }
    } else {
      // ------------------------- softmax, O = P V issue and epilogue (warp groups)
      const int wg = (warp - kWarpSoft0) >> 2;  // takes tiles with i % kNw == wg
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
      const bool leader = ((warp - kWarpSoft0) & 3) == 0 && lane == 0;
      const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
      const float ninf = -__int_as_float(0x7f800000);
      const float kLn2 = 0.69314718055994531f;
      const uint32_t id_pv = tc::idesc_bf16(kRows, D, true);
      bool ok = true;
      int i = 0, use = -1, prev_j = -1;
      for (int tile = tile0; tile < tile1; ++tile, ++i) {
        w.advance(a, tile);
        if (w.j != prev_j) {
          // Leaving block `use`: this group's O = P V products that read it have
          // all been issued; release its K/V stage once they complete.  The release
          // waits until the producer has loaded that block, so that a group owning
          // no tile of several short blocks never runs two phases ahead of the
          // producer on the stage's barrier.
          if (use >= 0 && leader) {
            mbar_wait_bounded(b_kvfull + 8 * (use & 1), (use >> 1) & 1, a.st, 0x20du, a.wait_ns);
            tc::commit(b_kvempty + 8 * ((use & 1) * kNw + wg));
          }
          prev_j = w.j;
          ++use;
        }
        if (i % kNw != wg) continue;
        const int qb = i % NQ, tb = i % NB;
        const TileInfo ti = tile_info(a, w.j, tile);
        const bool live = row < ti.nq * a.G;
        int pos = -1, hi = 0, lim = 0;
        if (live) {
          const int qi = row / a.G;
          hi = row - qi * a.G;
          pos = __ldg(a.entries + ti.first + qi);
          const int bt = (int)a.bt0 + pos / (a.h * a.topk);
          lim = visible_limit(a, ti.b, bt % a.n_q);
        }
        if (ok) ok = mbar_wait_warp(b_sfull + 8 * tb, (i / NB) & 1, a.st, 0x20bu, a.wait_ns);
        tc::fence_after_sync();
        // Scores from tensor memory in 32-column pieces: the row maximum first,
        // then probabilities, their sum and the bf16 P row (K-major, swizzled).
        const int vis = lim - ti.beta * BLK;  // keys [0, vis) of the block are visible
        const bool full = vis >= BLK;
        const uint32_t srow = lane_base + tb * TB;
        float mx = ninf;
#pragma unroll
        for (int c = 0; c < BLK / 32; ++c) {
          float v[32];
          tc::tmem_ld32(srow + c * 32, v);
          tc::tmem_wait_ld();
          if (!full) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = c * 32 + e < vis ? v[e] : ninf;
          }
          float m2[2] = {ninf, ninf};
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            m2[0] = fmax3(m2[0], v[e], v[e + 1]);
            m2[1] = fmax3(m2[1], v[e + 2], v[e + 3]);
          }
          mx = fmax3(mx, m2[0], m2[1]);
        }
        mx *= a.scale_log2;
        const float msafe = live && mx != ninf ? mx : 0.f;
        float l = 0.f;
        uint8_t* pbase = smem + qb * QP_BYTES;
#pragma unroll
        for (int c = 0; c < BLK / 32; ++c) {
          float v[32];
          tc::tmem_ld32(srow + c * 32, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = exp2_approx(fmaf(v[e], a.scale_log2, -msafe));
          if (!full) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = c * 32 + e < vis ? v[e] : 0.f;
          }
          float l2[2] = {0.f, 0.f};
#pragma unroll
          for (int e = 0; e < 32; ++e) l2[e & 1] += v[e];
          l += l2[0] + l2[1];
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const int ch = c * 4 + q8;  // 16-byte chunk of the P row
            const uint4 v4 = make_uint4(pack_bf16(v[8 * q8], v[8 * q8 + 1]),
                                        pack_bf16(v[8 * q8 + 2], v[8 * q8 + 3]),
                                        pack_bf16(v[8 * q8 + 4], v[8 * q8 + 5]),
                                        pack_bf16(v[8 * q8 + 6], v[8 * q8 + 7]));
            *reinterpret_cast<uint4*>(pbase + (ch >> 3) * (kRows * 128u) + swz128(row, ch & 7)) =
                v4;
          }
        }
        // V rows at or past the sequence end may hold anything; zero them so that a
        // zero probability never meets a non-finite value (idempotent per stage).
        {
          const int L = kv_length(a.seq_lens, ti.b, a.max_kv, a.st);
          const int r0 = max(0, L - ti.beta * BLK);
          if (r0 < BLK) {
            const int per_h = (BLK - r0) * 8;
            uint8_t* vb = smem + (skv - sm0a) + (use & 1) * KV_BYTES + NH * HALF;
            for (int x = row; x < per_h * NH; x += 128) {
              const int hh = x / per_h, rem = x % per_h;
              *reinterpret_cast<uint4*>(vb + hh * HALF + (r0 + rem / 8) * 128 + (rem % 8) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
        }
        // The P tile is complete once every warp of the group has written its rows.
        fence_proxy_async_smem();
        tc::fence_before_sync();
        asm volatile("bar.sync %0, 128;" ::"r"(3 + wg) : "memory");
        if (leader && ok) {
          tc::fence_after_sync();
          const uint32_t vd = skv + (use & 1) * KV_BYTES + NH * HALF;
#pragma unroll
          for (int ks = 0; ks < BLK / 16; ++ks) {
            const uint32_t poff = (ks >> 2) * (kRows * 128u) + (ks & 3) * 32;
            tc::mma_bf16(tmem + tb * TB, tc::desc_k_sw128(sqp + qb * QP_BYTES + poff),
                         tc::desc_mn_sw128(vd + ks * 16 * 128, HALF), id_pv, ks > 0 ? 1u : 0u);
          }
          tc::commit(b_ofull + 8 * tb);
          tc::commit(b_qempty + 8 * qb);  // the Q/P buffer may be refilled
        }
        // Output of this tile: O / l in bf16 and the log-sum-exp, for live rows.
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        if (ok) ok = mbar_wait_warp(b_ofull + 8 * tb, (i / NB) & 1, a.st, 0x20au, a.wait_ns);
        tc::fence_after_sync();
        const bool store = ok && live;
        uint16_t* dst = a.part_o + (store ? ((int64_t)pos * a.G + hi) * D : 0);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tc::tmem_ld32(lane_base + tb * TB + c * 32, v);
          tc::tmem_wait_ld();
          if (store) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_uint4(pack_bf16(v[8 * e] * inv_l, v[8 * e + 1] * inv_l),
                                 pack_bf16(v[8 * e + 2] * inv_l, v[8 * e + 3] * inv_l),
                                 pack_bf16(v[8 * e + 4] * inv_l, v[8 * e + 5] * inv_l),
                                 pack_bf16(v[8 * e + 6] * inv_l, v[8 * e + 7] * inv_l));
          }
        }
        if (store)
          a.part_lse[(int64_t)pos * a.G + hi] =
              (mx != ninf && l > 0.f) ? (msafe + log2f(l)) * kLn2 : ninf;
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_ofree + 8 * tb);
      }
      if (leader) {
        // release the last block, and wait for this group's products to complete
        if (use >= 0) {
          mbar_wait_bounded(b_kvfull + 8 * (use & 1), (use >> 1) & 1, a.st, 0x20du, a.wait_ns);
          tc::commit(b_kvempty + 8 * ((use & 1) * kNw + wg));
        }
        tc::commit(b_done + 8 * (1 + wg));
        mbar_wait_bounded(b_done + 8 * (1 + wg), 0, a.st, 0x20cu, a.wait_ns);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// -------------------------------------------------------------- combine
// One warp per (query, head): merge the head's partials over the group's valid
// slots by log-sum-exp weights; bf16 output and the natural-log LSE.  Lanes
// take 32 slots at a time, so the loads of many partials are in flight at once.
template <int D>
__global__ void __launch_bounds__(256) kv_combine_kernel(KvArgs a, int BLK) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int64_t n = (int64_t)a.nbt * a.H;
  if (wid >= n) return;
  const int hq = (int)(wid % a.H);
  const int bt_rel = (int)(wid / a.H);
  const int g = hq / a.G, hi = hq - g * a.G;
  const int bt = (int)a.bt0 + bt_rel;
  const int b = bt / a.n_q, t = bt % a.n_q;
  const int lim = visible_limit(a, b, t);
  const int32_t* row_ids = a.ids + ((int64_t)bt * a.h + g) * a.topk;
  const int64_t p0 = ((int64_t)bt_rel * a.h + g) * a.topk;
  const float ninf = -__int_as_float(0x7f800000);
  constexpr int PER = D / 32;  // dims per lane
  float M = ninf;
  for (int s0 = 0; s0 < a.topk; s0 += 32) {
    const int s = s0 + lane;
    float l = ninf;
    if (s < a.topk) {
      const int beta = __ldg(row_ids + s);
      if (beta >= 0 && beta < a.nblk && beta * BLK < lim) l = __ldg(a.part_lse + (p0 + s) * a.G + hi);
    }
    M = fmaxf(M, l);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (M != ninf) {
    for (int s0 = 0; s0 < a.topk; s0 += 32) {
      const int s = s0 + lane;
      float wgt = 0.f;
      if (s < a.topk) {
        const int beta = __ldg(row_ids + s);
        if (beta >= 0 && beta < a.nblk && beta * BLK < lim)
          wgt = __expf(__ldg(a.part_lse + (p0 + s) * a.G + hi) - M);
      }
      den += wgt;
      // Loads are issued for every slot of the pass (the buffer is allocated for all
      // of them); a slot without a partial contributes through a select, never a
      // multiply, so whatever its memory holds cannot leak into the sum.  Eight
      // slots per round keep several loads in flight per lane.
      const int cnt = min(32, a.topk - s0);
      for (int j0 = 0; j0 < cnt; j0 += 8) {
        uint2 u[8];
        float wj[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int jj = min(j0 + j, cnt - 1);
          wj[j] = __shfl_sync(0xffffffffu, wgt, jj);
          if (j0 + j >= cnt) wj[j] = 0.f;
          const uint16_t* src = a.part_o + ((p0 + s0 + jj) * a.G + hi) * D + lane * PER;
          if constexpr (PER == 4) {
            u[j] = __ldg(reinterpret_cast<const uint2*>(src));
          } else {
            u[j] = make_uint2(__ldg(reinterpret_cast<const uint32_t*>(src)), 0u);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const bool use = wj[j] != 0.f;
          acc[0] += use ? wj[j] * __uint_as_float(u[j].x << 16) : 0.f;
          acc[1] += use ? wj[j] * __uint_as_float(u[j].x & 0xffff0000u) : 0.f;
          if constexpr (PER == 4) {
            acc[2] += use ? wj[j] * __uint_as_float(u[j].y << 16) : 0.f;
            acc[3] += use ? wj[j] * __uint_as_float(u[j].y & 0xffff0000u) : 0.f;
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint16_t* o = a.out + (int64_t)b * a.o_s0 + (int64_t)t * a.o_s1 + (int64_t)hq * a.o_s2 + lane * PER;
  if constexpr (PER == 4) {
    *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv),
                                              pack_bf16(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(o) = pack_bf16(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && a.lse) a.lse[(int64_t)bt * a.H + hq] = M != ninf ? M + __logf(den) : ninf;
}

}  // namespace
}  // namespace msa

namespace msa {
namespace {

constexpr size_t kKvPartialBudget = size_t(6) << 30;  // partial bytes per query chunk

struct KvPlan {
  int64_t rows, chunk_rows;
  int nchunks, qpt;
  int64_t nj;
  size_t counts_off, offs_off, toffs_off, entries_off, lse_off, o_off, total;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

KvPlan plan_kv(const Shape& s) {
  KvPlan p;
  p.rows = (int64_t)s.batch * s.n_q;
  p.nj = (int64_t)s.batch * s.h * s.nblk;
  p.qpt = kRows / s.G;
  const size_t per_row = (size_t)s.h * s.topk * (4 + (size_t)s.G * 4 + (size_t)s.G * s.d * 2);
  int64_t cr = (int64_t)(kKvPartialBudget / per_row);
  cr = cr < 1 ? 1 : cr;
  const int64_t max_slots = (int64_t)1 << 30;  // chunk-relative positions are int32
  if (cr * s.h * s.topk > max_slots) cr = max_slots / ((int64_t)s.h * s.topk);
  p.chunk_rows = cr < p.rows ? cr : p.rows;
  p.nchunks = (int)((p.rows + p.chunk_rows - 1) / p.chunk_rows);
  const size_t slots = (size_t)p.chunk_rows * s.h * s.topk;
  size_t off = 0;
  p.counts_off = off;
  off = up256(off + p.nj * 4);
  p.offs_off = off;
  off = up256(off + (p.nj + 1) * 4);
  p.toffs_off = off;
  off = up256(off + (p.nj + 1) * 4);
  p.entries_off = off;
  off = up256(off + slots * 4);
  p.lse_off = off;
  off = up256(off + slots * s.G * 4);
  p.o_off = off;
  off = up256(off + slots * s.G * s.d * 2);
  p.total = off;
  return p;
}

template <int D, int BLK>
cudaError_t run_kv(const Shape& s, KvArgs& a, const KvPlan& p, const CUtensorMap& tmk,
                   const CUtensorMap& tmv, uint8_t* ws, cudaStream_t stream) {
  constexpr uint32_t smem = KvSmem<D, BLK>::BYTES;
  cudaError_t err = cudaFuncSetAttribute(kv_attn_kernel<D, BLK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int sms = num_sms();
  for (int c = 0; c < p.nchunks; ++c) {
    a.bt0 = (int64_t)c * p.chunk_rows;
    a.nbt = (int)((p.rows - a.bt0) < p.chunk_rows ? (p.rows - a.bt0) : p.chunk_rows);
    err = cudaMemsetAsync(ws + p.counts_off, 0, p.nj * 4, stream);
    if (err != cudaSuccess) return err;
    const int64_t n = (int64_t)a.nbt * s.h * s.topk;
    const int grid = (int)((n + 255) / 256 < (int64_t)sms * 8 ? (n + 255) / 256 : (int64_t)sms * 8);
    kv_count_kernel<<<grid, 256, 0, stream>>>(a, BLK);
    kv_scan_kernel<<<1, 1024, 0, stream>>>(a);
    kv_scatter_kernel<<<grid, 256, 0, stream>>>(a, BLK);
    kv_attn_kernel<D, BLK><<<sms, kKvThreads, smem, stream>>>(tmk, tmv, a);
    const int64_t warps = (int64_t)a.nbt * s.H;
    kv_combine_kernel<D><<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(a, BLK);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace

bool kv_attn_supported(const Shape& s) {
  return s.n_q > 1 && (s.d == 64 || s.d == 128) && (s.block == 64 || s.block == 128) &&
         (int64_t)s.batch * s.h * s.nblk < ((int64_t)1 << 30);
}

size_t kv_workspace_bytes(const Shape& s) { return plan_kv(s).total; }

int kv_launches(const Shape& s) { return 5 * plan_kv(s).nchunks; }

cudaError_t launch_kv_attn(const Shape& s, const CUtensorMap& tmk, const CUtensorMap& tmv,
                           const uint16_t* q, const int32_t* ids, uint16_t* out, float* lse,
                           void* ws, size_t ws_bytes, DeviceStatus* st, cudaStream_t stream) {
  const KvPlan p = plan_kv(s);
  if (ws == nullptr || ws_bytes < p.total) return cudaErrorInvalidValue;
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  KvArgs a;
  a.q = q;
  a.q_s0 = s.q_s[0];
  a.q_s1 = s.q_s[1];
  a.q_s2 = s.q_s[2];
  a.ids = ids;
  a.seq_lens = s.seq_lens;
  a.n_q = s.n_q;
  a.max_kv = s.max_kv;
  a.H = s.H;
  a.h = s.h;
  a.G = s.G;
  a.topk = s.topk;
  a.nblk = s.nblk;
  a.causal = s.causal;
  a.scale_log2 = s.scale * 1.4426950408889634f;
  a.counts = reinterpret_cast<int*>(w + p.counts_off);
  a.offs = reinterpret_cast<int*>(w + p.offs_off);
  a.toffs = reinterpret_cast<int*>(w + p.toffs_off);
  a.entries = reinterpret_cast<int*>(w + p.entries_off);
  a.qpt = p.qpt;
  a.nj = (int)p.nj;
  a.part_lse = reinterpret_cast<float*>(w + p.lse_off);
  a.part_o = reinterpret_cast<uint16_t*>(w + p.o_off);
  a.out = out;
  a.o_s0 = s.o_s[0];
  a.o_s1 = s.o_s[1];
  a.o_s2 = s.o_s[2];
  a.lse = lse;
  a.st = st;
  a.wait_ns = 4000000000ull;
  if (s.d == 128 && s.block == 128) return run_kv<128, 128>(s, a, p, tmk, tmv, w, stream);
  if (s.d == 128 && s.block == 64) return run_kv<128, 64>(s, a, p, tmk, tmv, w, stream);
  if (s.d == 64 && s.block == 128) return run_kv<64, 128>(s, a, p, tmk, tmv, w, stream);
  if (s.d == 64 && s.block == 64) return run_kv<64, 64>(s, a, p, tmk, tmv, w, stream);
  return cudaErrorInvalidValue;
}

}  // namespace msa
