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
//   P = softmax(S)      registers, one thread per row, masked to visible keys,
//                       written to tensor memory as bf16
//   O = P V             tcgen05 MMA with A = P from tensor memory, N = d, into
//                       the columns that held S (TMEM)
// Each (query, head, block) gives a normalised bf16 partial output and its
// log-sum-exp; a combine kernel merges a query's partials by log-sum-exp weights.
// Queries are processed in chunks so that the partials of one chunk fit a bounded
// workspace.
//
// CTA roles (persistent CTAs, each a contiguous share of the chunk's tiles), four
// warpgroups with registers moved from the first and last to the softmax ones:
//   warp 0        TMA producer of K and V (a new load only when the block changes;
//                 V rows past the sequence end are zeroed after the load lands),
//                 and a third of the Q gather;
//   warp 1        tensor-memory allocation and the thread issuing all MMAs: S and
//                 O = P V as two in-order streams, each issued as soon as its
//                 inputs are ready;
//   warps 0, 2-3  gather the tile's Q rows with TMA, one load per (query, 64-dim
//                 atom) bringing the query's G heads into the swizzled layout, the
//                 loads dealt round-robin to the three warps;
//   warps 4-11    two softmax warpgroups taking tiles in turn, one thread per tile
//                 row, each owning one P region in tensor memory;
//   warps 12-15   output warpgroup: O / l from tensor memory to the partials
//                 (staged per warp in shared memory, written by TMA stores).
// Buffers: 2-4 Q tiles (released when S is computed), 2 K/V stages, and in tensor
// memory 3-4 slots, each holding a tile's S and then its O, plus the two P
// regions.  Every wait is bounded.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kRows = 128;  // MMA M: (query, head) rows per tile
constexpr int kKvThreads = 512;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpGather = 2;
// Registers per thread after reallocation.  The four warpgroups' shares add up to
// what the kernel is launched with (128 per thread; the host refuses to launch a
// build that was given another count, since the softmax warpgroups would then
// wait for registers that are never released).
constexpr int kRegsLaunch = 128, kRegsLoad = 40, kRegsSoft = 184, kRegsOut = 104;
static_assert(kRegsLoad + 2 * kRegsSoft + kRegsOut == 4 * kRegsLaunch, "register split");

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
  int2* entries;           // {chunk-relative slot position, query index t} of each
                           // entry, grouped by (b, g, block)
  int* slot_row;           // [slot] partial row of a valid slot's query (head 0) in its
                           // tile; -1 for an empty or invalid slot, whose log-sum-exps
                           // are then -inf (both written by the scatter kernel)
  int qpt;                 // queries per tile
  int nj;                  // batch * h * nblk
  // partial outputs: 128 rows per tile, row = tile * 128 + query-in-tile * G +
  // head, so that a tile's output is one contiguous block; their log-sum-exps by
  // chunk-relative slot position p = (bt_rel * h + g) * topk + slot, so that a
  // query's are contiguous
  uint16_t* part_o;        // [row][d] bf16
  float* part_lse;         // [p][G]
  uint16_t* out;
  int64_t o_s0, o_s1, o_s2;
  float* lse;
  DeviceStatus* st;
  uint64_t wait_ns;
  KvPages pg;  // table == nullptr: contiguous K/V
};

__device__ __forceinline__ int visible_from_length(const KvArgs& a, int L, int t) {
  const int p = L - a.n_q + t;
  return max(0, a.causal ? min(L, p + 1) : L);
}

__device__ __forceinline__ int visible_limit(const KvArgs& a, int b, int t) {
  return visible_from_length(a, kv_length(a.seq_lens, b, a.max_kv, a.st), t);
}

// Valid slot of the chunk: a block id that exists and holds a visible token.
__device__ __forceinline__ bool slot_block(const KvArgs& a, int64_t pos, int& b, int& g, int& t,
                                           int& beta, int BLK) {
  const int64_t bt_rel = pos / ((int64_t)a.h * a.topk);
  const int rem = (int)(pos % ((int64_t)a.h * a.topk));
  g = rem / a.topk;
  const int64_t bt = a.bt0 + bt_rel;
  b = (int)(bt / a.n_q);
  t = (int)(bt % a.n_q);
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
  grid_dep_wait();
  grid_dep_launch();
  const int64_t n = (int64_t)a.nbt * a.h * a.topk;
  for (int64_t pos = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; pos < n;
       pos += (int64_t)gridDim.x * blockDim.x) {
    int b, g, t, beta;
    if (slot_block(a, pos, b, g, t, beta, BLK))
      atomicAdd(&a.counts[((int64_t)b * a.h + g) * a.nblk + beta], 1);
  }
}

// Exclusive scans of the counts (entry offsets) and of the tile counts
// (ceil(count / qpt)); the counts are zeroed to serve as scatter cursors.
__global__ void __launch_bounds__(1024) kv_scan_kernel(KvArgs a) {
  grid_dep_wait();
  grid_dep_launch();
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
  grid_dep_wait();
  grid_dep_launch();
  const int64_t n = (int64_t)a.nbt * a.h * a.topk;
  for (int64_t pos = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; pos < n;
       pos += (int64_t)gridDim.x * blockDim.x) {
    int b, g, t, beta;
    if (slot_block(a, pos, b, g, t, beta, BLK)) {
      const int64_t j = ((int64_t)b * a.h + g) * a.nblk + beta;
      const int k = atomicAdd(&a.counts[j], 1);
      a.entries[a.offs[j] + k] = make_int2((int)pos, t);
      a.slot_row[pos] = (a.toffs[j] + k / a.qpt) * kRows + (k % a.qpt) * a.G;
    } else {
      // no partial for this slot: the merge reads the marks, not the ids
      a.slot_row[pos] = -1;
      for (int hh = 0; hh < a.G; ++hh) a.part_lse[pos * a.G + hh] = -__int_as_float(0x7f800000);
    }
  }
}

// ------------------------------------------------------------ tile walker
// Tiles are numbered through the (b, g, block) lists in order.  A walker moves
// forward through them and steps the list's (b, g, block) along, so that only
// the initial seek divides.
struct Walker {
  int j, b, g, beta;  // current list
  int t0, t1;         // its tiles [t0, t1)
  int e0, cnt;        // its entries [e0, e0 + cnt)

  __device__ __forceinline__ void load_list(const KvArgs& a) {
    e0 = __ldg(a.offs + j);
    cnt = __ldg(a.offs + j + 1) - e0;
  }
  __device__ __forceinline__ void seek(const KvArgs& a, int tile) {
    int lo = 0, hi = a.nj;  // toffs[lo] <= tile < toffs[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a.toffs + mid) <= tile) lo = mid; else hi = mid;
    }
    j = lo;
    beta = j % a.nblk;
    const int bg = j / a.nblk;
    g = bg % a.h;
    b = bg / a.h;
    t0 = __ldg(a.toffs + j);
    t1 = __ldg(a.toffs + j + 1);
    load_list(a);
  }
  // Moves to the list holding `tile` (visited in increasing order); true when
  // the list changed.
  __device__ __forceinline__ bool advance(const KvArgs& a, int tile) {
    if (tile < t1) return false;
    do {
      ++j;
      if (++beta == a.nblk) {
        beta = 0;
        if (++g == a.h) {
          g = 0;
          ++b;
        }
      }
      t0 = t1;
      t1 = __ldg(a.toffs + j + 1);
    } while (tile >= t1);
    load_list(a);
    return true;
  }
  __device__ __forceinline__ int first(const KvArgs& a, int tile) const {
    return e0 + (tile - t0) * a.qpt;
  }
  __device__ __forceinline__ int count(const KvArgs& a, int tile) const {
    return min(a.qpt, cnt - (tile - t0) * a.qpt);
  }
};

// --------------------------------------------------------- attention tiles
// Shared-memory plan of the attention kernel for one (D, BLK).
template <int D, int BLK>
struct KvSmem {
  static constexpr uint32_t Q = kRows * D * 2;         // one Q tile
  static constexpr uint32_t HALF = BLK * 128u;         // one 64-dim atom of K or V
  static constexpr uint32_t KV = 2 * (D / 64) * HALF;  // K and V of one block
  // row statistics [4][128] float2, row table [128] int, barriers, TMEM address
  // (barriers from 4608, the TMEM address at 4992)
  static constexpr uint32_t MISC = 5120;
  static constexpr uint32_t STAGE = 4 * 32 * 128;  // output staging, one tile per warp
  static constexpr uint32_t LIMIT = 227u * 1024u;
  static constexpr uint32_t FIXED = 1024 + 2 * KV + MISC + STAGE;
  static constexpr int NQ = FIXED + 4 * Q <= LIMIT ? 4 : FIXED + 3 * Q <= LIMIT ? 3 : 2;
  static constexpr uint32_t BYTES = FIXED + NQ * Q;
  static_assert(BYTES <= LIMIT, "shared memory");
};

template <int D, int BLK>
__global__ void __launch_bounds__(kKvThreads, 1)
    kv_attn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                   KvArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  using SM = KvSmem<D, BLK>;
  constexpr int NH = D / 64;
  constexpr int NQ = SM::NQ;
  constexpr uint32_t QB = SM::Q, HALF = SM::HALF, KV_BYTES = SM::KV;
  // Tensor memory: NS slots of W columns, each holding a tile's S and then its
  // O (O = P V overwrites the S it was computed from), and two P regions of
  // BLK / 2 columns (bf16 pairs), one per softmax warpgroup.
  constexpr uint32_t W = BLK > D ? BLK : D;
  constexpr int NS = (512 - BLK) / W < 4 ? (512 - BLK) / W : 4;
  constexpr uint32_t PB = NS * W;
  constexpr uint32_t TMEM_COLS = PB + BLK <= 256 ? 256 : 512;
  static_assert(NS >= 3 && PB + BLK <= 512, "tensor memory");
  if (status_failed(a.st)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sq = smem_u32(smem);         // NQ Q tiles
  const uint32_t skv = sq + NQ * QB;          // 2 K/V stages
  uint8_t* misc = smem + NQ * QB + 2 * KV_BYTES;
  float2* rstat = reinterpret_cast<float2*>(misc);      // [4][128]: 1 / l, log-sum-exp
  int* rowtab = reinterpret_cast<int*>(misc + 4096);    // [128]: query | head << 16
  const uint32_t b_kvfull = smem_u32(misc + 4608);      // [2] K/V usable
  const uint32_t b_kvland = b_kvfull + 16;              // [2] K/V landed (before fix-up)
  const uint32_t b_kvempty = b_kvland + 16;             // [2]
  const uint32_t b_qfull = b_kvempty + 16;              // [NQ]
  const uint32_t b_qempty = b_qfull + 8 * NQ;           // [NQ]
  const uint32_t b_sfull = b_qempty + 8 * NQ;           // [4] S of a slot computed
  const uint32_t b_ofull = b_sfull + 32;                // [4] O of a slot computed
  const uint32_t b_sfree = b_ofull + 32;                // [4] O of a slot read out
  const uint32_t b_pfull = b_sfree + 32;                // [2] P written
  const uint32_t b_pfree = b_pfull + 16;                // [2] P consumed
  const uint32_t b_lfull = b_pfree + 16;                // [4] row statistics written
  const uint32_t b_done = b_lfull + 32;                 // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 4992);
  uint8_t* staging = misc + SM::MISC;                   // [4 warps][32 rows][128 bytes]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = __ldg(a.toffs + a.nj);
  const int per = (ntiles + gridDim.x - 1) / gridDim.x;
  const int tile0 = blockIdx.x * per;
  const int n = max(0, min(ntiles, tile0 + per) - tile0);

  if (threadIdx.x < kRows) rowtab[threadIdx.x] = (threadIdx.x / a.G) | ((threadIdx.x % a.G) << 16);
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(b_kvfull + 8 * s, 1);
      mbar_init(b_kvland + 8 * s, 1);
      mbar_init(b_kvempty + 8 * s, 1);
      mbar_init(b_pfull + 8 * s, 4);
      mbar_init(b_pfree + 8 * s, 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(b_sfull + 8 * i, 1);
      mbar_init(b_ofull + 8 * i, 1);
      mbar_init(b_sfree + 8 * i, 4);
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(b_qfull + 8 * i, 3);
      mbar_init(b_qempty + 8 * i, 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(b_lfull + 8 * i, 4);
    mbar_init(b_done, 1);
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
  // Each role sets its register limit first thing in its own branch, so that the
  // code under each limit is exactly that branch.
  const int wg = warp >> 2;
  Walker w;
  if (warp == kWarpProd || warp == kWarpGather || warp == kWarpGather + 1) {
    // ------------------------------------------ K/V producer (warp 0), Q gather
    // Warp 0 loads a block's K/V when the tile walk reaches a new block.  The Q
    // gather: one TMA load per (query, 64-dim atom) brings the query's G heads,
    // i.e. G consecutive tile rows, into the swizzled operand layout; a tile's
    // loads are dealt round-robin to warps 0, 2 and 3 (a warp issues its loads one
    // lane after another, so the more warps, the sooner a tile's Q is requested).
    // A tile's query positions are read while the previous tile is issued.
    tc::regs_dec<kRegsLoad>();
    if (n > 0) {
      const bool kv_role = warp == kWarpProd;
      const int gi = kv_role ? 0 : warp - kWarpGather + 1;  // gather share
      w.seek(a, tile0);
      if (lane == 0) {
        prefetch_tensormap(&tmq);
        if (kv_role) {
          prefetch_tensormap(&tmk);
          prefetch_tensormap(&tmv);
        }
      }
      const uint32_t rows_bytes = (uint32_t)a.G * 128u;
      // loads o = gi + 3 (lane + 32 k) of a tile: query o / NH, atom o % NH
      auto load_t = [&](int first, int nq, int (&tq)[3]) {
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const int o = gi + 3 * (lane + 32 * k);
          tq[k] = o < NH * nq ? __ldg(&a.entries[first + o / NH].y) : 0;
        }
      };
      int nq = w.count(a, tile0), qg = w.g, qbb = w.b;
      bool new_block = true;
      int tq[3];
      load_t(w.first(a, tile0), nq, tq);
      int use = -1;
      uint32_t land_par = 0;  // bit s: parity of the next wait on kv_land[s]
      bool ok = true, q_ok = true;
      for (int idx = 0; idx < n; ++idx) {
        if (kv_role && new_block && ok) {
          ++use;
          const int s = use & 1;
          if (use >= 2)
            ok = mbar_wait_warp(b_kvempty + 8 * s, ((use >> 1) - 1) & 1, a.st, 0x201u, a.wait_ns);
          if (ok) {
          // V rows [r0, BLK) lie past the sequence end and may hold anything: they
          // are zeroed once the block has landed, so that a zero probability never
          // meets a non-finite value.
          const int L = kv_length(a.seq_lens, w.b, a.max_kv, a.st);
          const int r0 = max(0, L - w.beta * BLK);
          const bool fix = r0 < BLK;
          const uint32_t bar = (fix ? b_kvland : b_kvfull) + 8 * s;
          const uint32_t kd = skv + s * KV_BYTES, vd = kd + NH * HALF;
          if (lane == 0) {
            int tok, plane;
            kv_block_coords(a.pg, w.b, w.beta, BLK, a.st, tok, plane);
            mbar_arrive_expect_tx(bar, KV_BYTES);
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
              tma_load_4d(kd + hh * HALF, &tmk, bar, hh * 64, w.g, tok, plane);
              tma_load_4d(vd + hh * HALF, &tmv, bar, hh * 64, w.g, tok, plane);
            }
          }
          if (fix) {
            ok = mbar_wait_warp(b_kvland + 8 * s, (land_par >> s) & 1u, a.st, 0x202u, a.wait_ns);
            land_par ^= 1u << s;
            if (ok) {
              const int per_h = (BLK - r0) * 8;  // 16-byte pieces per 64-dim atom
              uint8_t* vb = smem + (vd - sq);
              for (int x = lane; x < per_h * NH; x += 32) {
                const int hh = x / per_h, rem = x - hh * per_h;
                *reinterpret_cast<uint4*>(vb + hh * HALF + (r0 + rem / 8) * 128 + (rem % 8) * 16) =
                    make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(b_kvfull + 8 * s);
          }
          }
        }
        // this warp's share of the tile's Q loads
        const int qb = idx % NQ;
        if (idx >= NQ && q_ok)
          q_ok = mbar_wait_warp(b_qempty + 8 * qb, ((idx / NQ) - 1) & 1, a.st, 0x20au, a.wait_ns);
        const int total = NH * nq;
        const int mine = q_ok ? (total - gi + 2) / 3 : 0;
        const uint32_t bar = b_qfull + 8 * qb;
        if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)mine * rows_bytes);
        __syncwarp();
        if (q_ok) {
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            const int o = gi + 3 * (lane + 32 * k);
            if (o < total) {
              const int qi = o / NH, hh = o % NH;
              tma_load_4d(sq + qb * QB + hh * (kRows * 128u) + qi * rows_bytes, &tmq, bar, hh * 64,
                          qg * a.G, tq[k], qbb);
            }
          }
        }
        if (idx + 1 < n) {
          const int tile = tile0 + idx + 1;
          new_block = w.advance(a, tile);
          nq = w.count(a, tile);
          qg = w.g;
          qbb = w.b;
          load_t(w.first(a, tile), nq, tq);
        }
      }
      if (kv_role) {
        // drain: the last two stages are released once their products complete
        for (int u = max(0, use - 1); u <= use; ++u)
          mbar_wait_warp(b_kvempty + 8 * (u & 1), (u >> 1) & 1, a.st, 0x203u, a.wait_ns);
      }
    }
  } else if (warp == kWarpMma) {
    // ----------------------------------------------- MMA issue (one thread)
    tc::regs_dec<kRegsLoad>();
    if (n > 0) {
      w.seek(a, tile0);
      if (lane == 0) {
        // Two in-order streams, S = Q K^T by tile and O = P V by tile, issued as
        // their inputs become ready, O = P V first: a blocking wait on one stream
        // would hold back the other (an S waits for its slot to be read out, which
        // waits for an O).  Two bits of `hist` per tile (ring of 8; O never lags S
        // by more than NS tiles) hold its K/V stage and whether it is the last
        // tile of its block.  No progress for wait_ns records a timeout.
        const uint32_t id_qk = tc::idesc_bf16(kRows, BLK, false);
        const uint32_t id_pv = tc::idesc_bf16(kRows, D, true);
        // Shared-memory descriptors of the first Q tile, the first K stage and the
        // first V stage; an operand elsewhere is the base plus its byte offset / 16
        // (the start-address field never carries: shared addresses are < 2^18).
        const uint64_t dq0 = tc::desc_k_sw128(sq);
        const uint64_t dk0 = tc::desc_k_sw128(skv);
        const uint64_t dv0 = tc::desc_mn_sw128(skv + NH * HALF, HALF);
        int use = -1, nq = 0, np = 0;
        uint32_t hist = 0, spins = 0;
        uint64_t stall = 0;
        bool looked = false, new_block = false;  // tile nq's list, once looked up
        while (np < n) {
          bool progress = false;
          if (np < nq && mbar_test(b_pfull + 8 * (np & 1), (np >> 1) & 1)) {
            const int p = np & 1, sk = np % NS;
            const uint32_t h = hist >> (2 * (np & 7));
            const uint64_t dv = dv0 + (h & 1u) * (KV_BYTES >> 4);
            const uint32_t pa = tmem + PB + p * (BLK / 2), oa = tmem + sk * W;
            tc::fence_after_sync();
#pragma unroll
            for (int ks = 0; ks < BLK / 16; ++ks)
              tc::mma_bf16_ts(oa, pa + ks * 8, dv + ks * (16 * 128 / 16), id_pv, ks > 0 ? 1u : 0u);
            tc::commit(b_ofull + 8 * sk);
            tc::commit(b_pfree + 8 * p);
            if (h & 2u) tc::commit(b_kvempty + 8 * (h & 1u));  // K/V stage released
            ++np;
            progress = true;
          } else if (nq < n) {
            const int tile = tile0 + nq;
            if (!looked) {
              new_block = w.advance(a, tile) || nq == 0;
              looked = true;
            }
            const int u = use + (new_block ? 1 : 0), sk = nq % NS, qb = nq % NQ;
            bool ready = !new_block || mbar_test(b_kvfull + 8 * (u & 1), (u >> 1) & 1);
            ready = ready && mbar_test(b_qfull + 8 * qb, (nq / NQ) & 1);
            // the slot's previous O has been read out
            ready = ready && (nq < NS || mbar_test(b_sfree + 8 * sk, ((nq / NS) - 1) & 1));
            if (ready) {
              use = u;
              tc::fence_after_sync();
              const uint64_t dq = dq0 + qb * (QB >> 4), dk = dk0 + (use & 1) * (KV_BYTES >> 4);
              const uint32_t sa = tmem + sk * W;
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t qoff = (ks >> 2) * (kRows * 128u) + (ks & 3) * 32;
                const uint32_t koff = (ks >> 2) * HALF + (ks & 3) * 32;
                tc::mma_bf16(sa, dq + (qoff >> 4), dk + (koff >> 4), id_qk, ks > 0 ? 1u : 0u);
              }
              tc::commit(b_sfull + 8 * sk);
              tc::commit(b_qempty + 8 * qb);  // the Q tile may be refilled
              const bool last = tile + 1 >= w.t1 || nq == n - 1;
              hist = (hist & ~(3u << (2 * (nq & 7)))) |
                     (((uint32_t)(use & 1) | (last ? 2u : 0u)) << (2 * (nq & 7)));
              ++nq;
              looked = false;
              progress = true;
            }
          }
          if (progress) {
            stall = 0;
          } else if (stall == 0) {
            stall = global_timer_ns();
          } else if ((++spins & 63u) == 0 && global_timer_ns() - stall > a.wait_ns) {
            record_error(a.st, kErrTimeout, 0x204u);
            break;
          }
        }
        tc::commit(b_done);
        mbar_wait_bounded(b_done, 0, a.st, 0x209u, a.wait_ns);
      }
    }
  } else if (wg < 3) {
    // ------------------------------------------------------ softmax warpgroups
    tc::regs_inc<kRegsSoft>();
    if (n > 0) {
      w.seek(a, tile0);
      const int sw = wg - 1;  // tiles idx with idx % 2 == sw; P region sw
      const int quarter = warp & 3, row = quarter * 32 + lane;
      const uint32_t lanes = tmem + ((uint32_t)(quarter * 32) << 16);
      const uint32_t pr = lanes + PB + sw * (BLK / 2);
      const int qi = rowtab[row] & 0xffff;
      const float ninf = -__int_as_float(0x7f800000);
      const float kLn2 = 0.69314718055994531f;
      int Lb = -1, L = 0;
      bool ok = true;
      // keys [0, vis) of a tile's block are visible to this row.  With block 64 the
      // query position behind it is loaded a tile of this warpgroup ahead, so that
      // its latency is not on the path from S to P (measured 8% faster at 32K);
      // with block 128 the look-ahead measured 4% slower (more spills) and the
      // position is loaded at the top of the tile's turn.
      constexpr int LA = BLK == 64 ? 2 : 0;
      auto row_visible = [&](int tile, int& t_row, int& beta_row, int& b_row) {
        w.advance(a, tile);
        t_row = -1;
        if (qi < w.count(a, tile)) t_row = __ldg(&a.entries[w.first(a, tile) + qi].y);
        beta_row = w.beta;
        b_row = w.b;
      };
      int t_n = -1, beta_n = 0, b_n = 0;
      if (LA > 0 && sw < n) row_visible(tile0 + sw, t_n, beta_n, b_n);
      for (int idx = sw; idx < n; idx += 2) {
        if (LA == 0) row_visible(tile0 + idx, t_n, beta_n, b_n);
        const int t_row = t_n, beta_row = beta_n, b_row = b_n;
        if (LA > 0 && idx + LA < n) row_visible(tile0 + idx + LA, t_n, beta_n, b_n);
        int vis = BLK;
        if (t_row >= 0) {
          if (b_row != Lb) {
            Lb = b_row;
            L = kv_length(a.seq_lens, b_row, a.max_kv, a.st);
          }
          vis = visible_from_length(a, L, t_row) - beta_row * BLK;
        }
        const int sk = idx % NS;
        if (ok) ok = mbar_wait_warp(b_sfull + 8 * sk, (idx / NS) & 1, a.st, 0x20bu, a.wait_ns);
        tc::fence_after_sync();
        float v[BLK];
#pragma unroll
        for (int c = 0; c < BLK / 32; ++c) tc::tmem_ld32_at(lanes + sk * W + c * 32, v + c * 32);
        tc::tmem_wait_ld();
        if (vis < BLK) {
#pragma unroll
          for (int e = 0; e < BLK; ++e) v[e] = e < vis ? v[e] : ninf;
        }
        float m4[4] = {ninf, ninf, ninf, ninf};
#pragma unroll
        for (int e = 0; e < BLK; e += 8) {
          m4[0] = fmax3(m4[0], v[e], v[e + 1]);
          m4[1] = fmax3(m4[1], v[e + 2], v[e + 3]);
          m4[2] = fmax3(m4[2], v[e + 4], v[e + 5]);
          m4[3] = fmax3(m4[3], v[e + 6], v[e + 7]);
        }
        const float ms = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * a.scale_log2;
        const float msafe = ms != ninf ? ms : 0.f;
        // probabilities (masked keys hold -inf and give exactly 0), their sum and
        // the bf16 P row, written to this warpgroup's P region once the O = P V of
        // its previous tile has consumed it
        if (ok && idx >= 2)
          ok = mbar_wait_warp(b_pfree + 8 * sw, ((idx >> 1) - 1) & 1, a.st, 0x20eu, a.wait_ns);
        tc::fence_after_sync();
        float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < BLK / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            fma2(x0, x1, v[c * 32 + 2 * e], v[c * 32 + 2 * e + 1], a.scale_log2, a.scale_log2,
                 -msafe, -msafe);
            const float p0 = exp2_approx(x0), p1 = exp2_approx(x1);
            const int h2 = 2 * (e & 1);  // two packed pairs of partial sums
            add2(l4[h2], l4[h2 + 1], l4[h2], l4[h2 + 1], p0, p1);
            pk[e] = pack_bf16(p0, p1);
          }
          tc::tmem_st16(pr + c * 16, pk);
        }
        tc::tmem_wait_st();
        const float l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
        rstat[(idx & 3) * kRows + row] =
            make_float2(l > 0.f ? 1.f / l : 0.f, (ms != ninf && l > 0.f) ? (msafe + log2f(l)) * kLn2 : ninf);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(b_pfull + 8 * sw);
          mbar_arrive(b_lfull + 8 * (idx & 3));
        }
      }
    }
  } else {
    // -------------------------------------------------------- output warpgroup
    // Each warp writes its 32 rows of a 64-dim half into a 128-byte-swizzled
    // staging tile (four shared-memory wavefronts per instruction) and one TMA
    // store moves the tile to the partials; a tile's padding rows receive
    // whatever the unused tensor-memory lanes hold and are never read.
    tc::regs_dec<kRegsOut>();
    if (n > 0) {
      w.seek(a, tile0);
      const int quarter = warp & 3, row = quarter * 32 + lane;
      const int info = rowtab[row];
      const int qi = info & 0xffff, hi = info >> 16;
      const uint32_t lanes = tmem + ((uint32_t)(quarter * 32) << 16);
      const uint32_t stg = smem_u32(staging) + quarter * 4096u;
      if (lane == 0) prefetch_tensormap(&tmo);
      bool ok = true;
      // a tile's slot position (where this row's log-sum-exp goes): with block 64
      // loaded one tile ahead, so that its latency is not on the per-tile path of
      // this warpgroup, which handles every tile (see the softmax warpgroups)
      constexpr int LA = BLK == 64 ? 1 : 0;
      bool live_n = false;
      int pos_n = 0;
      auto slot_of = [&](int tile) {
        w.advance(a, tile);
        live_n = qi < w.count(a, tile);
        pos_n = live_n ? __ldg(&a.entries[w.first(a, tile) + qi].x) : 0;
      };
      if (LA > 0) slot_of(tile0);
      for (int idx = 0; idx < n; ++idx) {
        if (LA == 0) slot_of(tile0 + idx);
        const bool live = live_n;
        const int pos = pos_n;
        if (LA > 0 && idx + LA < n) slot_of(tile0 + idx + LA);
        const int tile = tile0 + idx;
        if (ok) ok = mbar_wait_warp(b_lfull + 8 * (idx & 3), (idx >> 2) & 1, a.st, 0x20cu, a.wait_ns);
        const float2 rs = rstat[(idx & 3) * kRows + row];
        const int sk = idx % NS;
        if (ok) ok = mbar_wait_warp(b_ofull + 8 * sk, (idx / NS) & 1, a.st, 0x20du, a.wait_ns);
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < D / 32; c += 2) {
          float v[64];
          tc::tmem_ld32_at(lanes + sk * W + c * 32, v);
          tc::tmem_ld32_at(lanes + sk * W + c * 32 + 32, v + 32);
          tc::tmem_wait_ld();
          if (c + 2 >= D / 32) {
            // the slot has been read out: the next S may overwrite it
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_sfree + 8 * sk);
          }
          // the previous store has finished reading the staging tile
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t u0 = pack_bf16(v[8 * e] * rs.x, v[8 * e + 1] * rs.x);
            const uint32_t u1 = pack_bf16(v[8 * e + 2] * rs.x, v[8 * e + 3] * rs.x);
            const uint32_t u2 = pack_bf16(v[8 * e + 4] * rs.x, v[8 * e + 5] * rs.x);
            const uint32_t u3 = pack_bf16(v[8 * e + 6] * rs.x, v[8 * e + 7] * rs.x);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg + swz128(lane, e)),
                         "r"(u0), "r"(u1), "r"(u2), "r"(u3)
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && ok) {
            tma_store_2d(&tmo, stg, (c / 2) * 64, tile * kRows + quarter * 32);
            bulk_commit();
          }
        }
        if (ok && live) a.part_lse[(int64_t)pos * a.G + hi] = rs.y;
      }
      if (lane == 0) bulk_wait0();
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// m[base + rl] for rl < RPI, as selects (an indexed pick would put m in local memory).
template <int RPI>
__device__ __forceinline__ float pick_row(const float* m, int base, int rl) {
  if constexpr (RPI == 2) {
    return rl ? m[base + 1] : m[base];
  } else {
    static_assert(RPI == 4, "rows per load");
    return (rl & 2) ? ((rl & 1) ? m[base + 3] : m[base + 2]) : ((rl & 1) ? m[base + 1] : m[base]);
  }
}

// One warp per (query, group) for groups of GC heads: merge the heads' partials over
// the group's valid slots by log-sum-exp weights; bf16 output and the natural-log
// LSE.  A slot's GC partial rows are consecutive rows of its tile, read as one
// contiguous piece, 16 bytes per lane.
template <int D, int GC>
__global__ void __launch_bounds__(256, 2) kv_combine_group_kernel(KvArgs a, int BLK) {
  grid_dep_wait();
  grid_dep_launch();
  // One warp per (query, group): a slot's G partial rows are consecutive rows of
  // its tile, read as one contiguous piece, 16 bytes per lane.  Lane = (row rl of
  // a load, 16-byte chunk c); a load covers RPI rows, ni loads cover the G heads.
  constexpr int LPR = D / 8;         // lanes per partial row
  constexpr int RPI = 32 / LPR;      // rows per warp-wide load
  constexpr int MI = (GC + RPI - 1) / RPI;  // loads per slot
  constexpr int U = MI >= 3 ? 3 : 4;        // slots whose loads are in flight together
  const int lane = threadIdx.x & 31;
  const int64_t wid = blockIdx.x * 8LL + (threadIdx.x >> 5);
  if (wid >= (int64_t)a.nbt * a.h) return;
  const int g = (int)(wid % a.h);
  const int bt_rel = (int)(wid / a.h);
  const int bt = (int)a.bt0 + bt_rel;
  const int b = bt / a.n_q, t = bt % a.n_q;
  constexpr int G = GC;
  const int rl = lane / LPR, c = lane % LPR;
  const int64_t p0 = ((int64_t)bt_rel * a.h + g) * a.topk;
  const float ninf = -__int_as_float(0x7f800000);
  // pass 1: per-head maximum of the slots' log-sum-exps (empty or invalid slots
  // hold -inf), slots spread over the lanes; a slot's row is kept for pass 2
  float M[GC];
#pragma unroll
  for (int h = 0; h < GC; ++h) M[h] = ninf;
  for (int s0 = 0; s0 < a.topk; s0 += 32) {
    const int s = s0 + lane;
    if (s < a.topk) {
      const float* l = a.part_lse + (p0 + s) * G;
#pragma unroll
      for (int h = 0; h < GC; ++h) M[h] = fmaxf(M[h], __ldg(l + h));
    }
  }
#pragma unroll
  for (int h = 0; h < GC; ++h)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M[h] = fmaxf(M[h], __shfl_xor_sync(0xffffffffu, M[h], o));
  // this lane's heads hi = i * RPI + rl
  float Mp[MI * RPI];
#pragma unroll
  for (int h = 0; h < MI * RPI; ++h) Mp[h] = h < GC ? M[h] : ninf;
  float Mi[MI], den[MI], acc[MI][8];
#pragma unroll
  for (int i = 0; i < MI; ++i) {
    Mi[i] = pick_row<RPI>(Mp, i * RPI, rl);
    den[i] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
  }
  // pass 2: weighted sum, slot by slot (the warp on one slot at a time, U slots'
  // loads in flight); an empty slot reads row 0 with weight 0, through a select,
  // so that whatever row 0 holds cannot leak into the sum
  for (int s0 = 0; s0 < a.topk; s0 += 32) {
    const int s = s0 + lane;
    const int prow = s < a.topk ? __ldg(a.slot_row + p0 + s) : -1;
    const bool ok = prow >= 0;
    const int cnt = min(32, a.topk - s0);
    for (int j0 = 0; j0 < cnt; j0 += U) {
      uint4 u[U][MI];
      float l[U][MI];
      bool use[U];
#pragma unroll
      for (int jj = 0; jj < U; ++jj) {
        const int j = min(j0 + jj, cnt - 1);
        use[jj] = j0 + jj < cnt && __shfl_sync(0xffffffffu, ok ? 1 : 0, j) != 0;
        const int rj = max(0, __shfl_sync(0xffffffffu, prow, j));
        const float* lp = a.part_lse + (p0 + s0 + j) * G;
#pragma unroll
        for (int i = 0; i < MI; ++i) {
          const int hi = i * RPI + rl;
          const bool live = use[jj] && hi < G;
          u[jj][i] = __ldg(reinterpret_cast<const uint4*>(
                             a.part_o + (int64_t)(live ? rj + hi : 0) * D) +
                         c);
          l[jj][i] = live ? __ldg(lp + hi) : ninf;
        }
      }
#pragma unroll
      for (int jj = 0; jj < U; ++jj)
#pragma unroll
        for (int i = 0; i < MI; ++i) {
          const bool live = l[jj][i] != ninf;
          const float w = live ? __expf(l[jj][i] - Mi[i]) : 0.f;
          den[i] += w;
          const uint32_t x[4] = {u[jj][i].x, u[jj][i].y, u[jj][i].z, u[jj][i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[i][2 * e] += live ? w * __uint_as_float(x[e] << 16) : 0.f;
            acc[i][2 * e + 1] += live ? w * __uint_as_float(x[e] & 0xffff0000u) : 0.f;
          }
        }
    }
  }
  uint16_t* ob = a.out + (int64_t)b * a.o_s0 + (int64_t)t * a.o_s1 + c * 8;
#pragma unroll
  for (int i = 0; i < MI; ++i) {
    const int hi = i * RPI + rl;
    if (hi >= G) continue;
    const int hq = g * G + hi;
    const float inv = den[i] > 0.f ? 1.f / den[i] : 0.f;
    *reinterpret_cast<uint4*>(ob + (int64_t)hq * a.o_s2) =
        make_uint4(pack_bf16(acc[i][0] * inv, acc[i][1] * inv),
                   pack_bf16(acc[i][2] * inv, acc[i][3] * inv),
                   pack_bf16(acc[i][4] * inv, acc[i][5] * inv),
                   pack_bf16(acc[i][6] * inv, acc[i][7] * inv));
    if (c == 0 && a.lse)
      a.lse[(int64_t)bt * a.H + hq] = Mi[i] != ninf && den[i] > 0.f ? Mi[i] + __logf(den[i]) : ninf;
  }
}

// -------------------------------------------------------------- combine
// One warp per (query, head): merge the head's partials over the group's valid
// slots by log-sum-exp weights; bf16 output and the natural-log LSE.  Lanes
// take 32 slots at a time, so the loads of many partials are in flight at once.
template <int D>
__global__ void __launch_bounds__(256) kv_combine_kernel(KvArgs a, int BLK) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t wid = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int64_t n = (int64_t)a.nbt * a.H;
  if (wid >= n) return;
  const int hq = (int)(wid % a.H);
  const int bt_rel = (int)(wid / a.H);
  const int g = hq / a.G, hi = hq - g * a.G;
  const int bt = (int)a.bt0 + bt_rel;
  const int b = bt / a.n_q, t = bt % a.n_q;
  const int64_t p0 = ((int64_t)bt_rel * a.h + g) * a.topk;
  const float ninf = -__int_as_float(0x7f800000);
  constexpr int PER = D / 32;  // dims per lane
  // pass 1: the slots' log-sum-exps and partial rows (empty or invalid slots hold
  // -inf and row -1, written by the scatter kernel), both loaded at once; the
  // first 64 slots stay in registers for pass 2
  constexpr int KR = 2;  // slot groups of 32 kept in registers
  float lk[KR];
  int rk[KR];
  float M = ninf;
#pragma unroll
  for (int r = 0; r < KR; ++r) {
    const int s = r * 32 + lane;
    lk[r] = ninf;
    rk[r] = -1;
    if (s < a.topk) {
      lk[r] = __ldg(a.part_lse + (p0 + s) * a.G + hi);
      rk[r] = __ldg(a.slot_row + p0 + s);
    }
  }
  for (int s0 = KR * 32; s0 < a.topk; s0 += 32) {
    const int s = s0 + lane;
    if (s < a.topk) M = fmaxf(M, __ldg(a.part_lse + (p0 + s) * a.G + hi));
  }
#pragma unroll
  for (int r = 0; r < KR; ++r) M = fmaxf(M, lk[r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (M != ninf) {
    for (int s0 = 0; s0 < a.topk; s0 += 32) {
      const int s = s0 + lane;
      const int r = s0 / 32;
      float l = ninf;
      int prow = -1;
      if (r < KR) {
        l = r == 0 ? lk[0] : lk[1];
        prow = r == 0 ? rk[0] : rk[1];
      } else if (s < a.topk) {
        l = __ldg(a.part_lse + (p0 + s) * a.G + hi);
        prow = __ldg(a.slot_row + p0 + s);
      }
      const float wgt = (prow >= 0 && l != ninf) ? __expf(l - M) : 0.f;
      prow = prow >= 0 ? prow + hi : 0;  // row 0 stands in for none
      den += wgt;
      // Loads are issued for every slot of the pass (a slot without a partial reads
      // row 0, which exists); such a slot contributes through a select, never a
      // multiply, so whatever that row holds cannot leak into the sum.  Sixteen slots
      // per round keep several loads in flight per lane.
      const int cnt = min(32, a.topk - s0);
      for (int j0 = 0; j0 < cnt; j0 += 16) {
        uint2 u[16];
        float wj[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int jj = min(j0 + j, cnt - 1);
          wj[j] = __shfl_sync(0xffffffffu, wgt, jj);
          if (j0 + j >= cnt) wj[j] = 0.f;
          const int rj = __shfl_sync(0xffffffffu, prow, jj);
          const uint16_t* src = a.part_o + (int64_t)rj * D + lane * PER;
          if constexpr (PER == 4) {
            u[j] = __ldg(reinterpret_cast<const uint2*>(src));
          } else {
            u[j] = make_uint2(__ldg(reinterpret_cast<const uint32_t*>(src)), 0u);
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
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
  int64_t nj, max_tiles;
  size_t counts_off, offs_off, toffs_off, entries_off, slot_row_off, lse_off, o_off, total;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

KvPlan plan_kv(const Shape& s) {
  KvPlan p;
  p.rows = (int64_t)s.batch * s.n_q;
  p.nj = (int64_t)s.batch * s.h * s.nblk;
  p.qpt = kRows / s.G;
  // A chunk's tiles number at most ceil(slots / qpt) + nj (one partly filled
  // tile per list); each holds 128 partial rows of d bf16.  Per slot: its entry,
  // its partial row and G log-sum-exps.
  const size_t row_bytes = (size_t)s.d * 2;
  const size_t fixed = (size_t)(p.nj + 1) * kRows * row_bytes;
  const size_t per_bt =
      (size_t)s.h * s.topk * (12 + (size_t)s.G * 4 + kRows * row_bytes / p.qpt + 1);
  int64_t cr = fixed < kKvPartialBudget ? (int64_t)((kKvPartialBudget - fixed) / per_bt) : 1;
  cr = cr < 1 ? 1 : cr;
  const int64_t max_slots = (int64_t)1 << 30;  // chunk-relative positions are int32
  if (cr * s.h * s.topk > max_slots) cr = max_slots / ((int64_t)s.h * s.topk);
  p.chunk_rows = cr < p.rows ? cr : p.rows;
  p.nchunks = (int)((p.rows + p.chunk_rows - 1) / p.chunk_rows);
  const size_t slots = (size_t)p.chunk_rows * s.h * s.topk;
  p.max_tiles = (int64_t)((slots + p.qpt - 1) / p.qpt) + p.nj;
  size_t off = 0;
  p.counts_off = off;
  off = up256(off + p.nj * 4);
  p.offs_off = off;
  off = up256(off + (p.nj + 1) * 4);
  p.toffs_off = off;
  off = up256(off + (p.nj + 1) * 4);
  p.entries_off = off;
  off = up256(off + slots * 8);
  p.slot_row_off = off;
  off = up256(off + slots * 4);
  p.lse_off = off;
  off = up256(off + slots * s.G * 4);
  p.o_off = off;
  off = up256(off + (size_t)p.max_tiles * kRows * s.d * 2);
  p.total = off;
  return p;
}

template <int D, int BLK>
cudaError_t run_kv(const Shape& s, KvArgs& a, const KvPlan& p, const CUtensorMap& tmq,
                   const CUtensorMap& tmk, const CUtensorMap& tmv, const CUtensorMap& tmo,
                   uint8_t* ws, cudaStream_t stream) {
  constexpr uint32_t smem = KvSmem<D, BLK>::BYTES;
  // The register reallocation inside the kernel is sized for a launch with
  // kRegsLaunch registers per thread; any other build would wait forever.
  cudaFuncAttributes fa;
  cudaError_t err = cudaFuncGetAttributes(&fa, kv_attn_kernel<D, BLK>);
  if (err != cudaSuccess) return err;
  if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidKernelImage;
  err = cudaFuncSetAttribute(kv_attn_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
  if (err != cudaSuccess) return err;
  const int sms = num_sms();
  for (int c = 0; c < p.nchunks; ++c) {
    a.bt0 = (int64_t)c * p.chunk_rows;
    a.nbt = (int)((p.rows - a.bt0) < p.chunk_rows ? (p.rows - a.bt0) : p.chunk_rows);
    err = cudaMemsetAsync(ws + p.counts_off, 0, p.nj * 4, stream);
    if (err != cudaSuccess) return err;
    const int64_t n = (int64_t)a.nbt * s.h * s.topk;
    const int grid = (int)((n + 255) / 256 < (int64_t)sms * 8 ? (n + 255) / 256 : (int64_t)sms * 8);
    const int64_t warps = (int64_t)a.nbt * s.H;
    if ((err = launch_pdl(kv_count_kernel, dim3(grid), dim3(256), 0, stream, a, BLK)) !=
            cudaSuccess ||
        (err = launch_pdl(kv_scan_kernel, dim3(1), dim3(1024), 0, stream, a)) != cudaSuccess ||
        (err = launch_pdl(kv_scatter_kernel, dim3(grid), dim3(256), 0, stream, a, BLK)) !=
            cudaSuccess ||
        (err = launch_pdl(kv_attn_kernel<D, BLK>, dim3(sms), dim3(kKvThreads), smem, stream, tmq,
                          tmk, tmv, tmo, a)) != cudaSuccess)
      return err;
    // The combine is launched plainly: as a programmatic dependent of kv_attn
    // (its CTAs taking the SMs that kv_attn leaves early) it measured ~6% slower.
    // Groups of 8 heads: one warp per (query, group) (measured 4% faster at G = 8,
    // no faster at G = 6, where a warp per (query, head) has more loads in flight).
    if (s.G == 8)
      kv_combine_group_kernel<D, 8><<<(unsigned)(((int64_t)a.nbt * s.h + 7) / 8), 256, 0, stream>>>(
          a, BLK);
    else
      kv_combine_kernel<D><<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(a, BLK);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace

bool kv_attn_supported(const Shape& s) {
  // partial rows are addressed with int32
  return s.n_q > 1 && (s.d == 64 || s.d == 128) && (s.block == 64 || s.block == 128) &&
         plan_kv(s).max_tiles * kRows < ((int64_t)1 << 31);
}

size_t kv_workspace_bytes(const Shape& s) { return plan_kv(s).total; }

int kv_launches(const Shape& s) { return 5 * plan_kv(s).nchunks; }

cudaError_t launch_kv_attn(const Shape& s, const CUtensorMap& tmq, const CUtensorMap& tmk,
                           const CUtensorMap& tmv,
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
  a.entries = reinterpret_cast<int2*>(w + p.entries_off);
  a.slot_row = reinterpret_cast<int*>(w + p.slot_row_off);
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
  a.pg = s.pages;
  CUtensorMap tmo;
  if (!make_rows_map(&tmo, a.part_o, p.max_tiles * kRows, s.d)) return cudaErrorInvalidValue;
  if (s.d == 128 && s.block == 128) return run_kv<128, 128>(s, a, p, tmq, tmk, tmv, tmo, w, stream);
  if (s.d == 128 && s.block == 64) return run_kv<128, 64>(s, a, p, tmq, tmk, tmv, tmo, w, stream);
  if (s.d == 64 && s.block == 128) return run_kv<64, 128>(s, a, p, tmq, tmk, tmv, tmo, w, stream);
  if (s.d == 64 && s.block == 64) return run_kv<64, 64>(s, a, p, tmq, tmk, tmv, tmo, w, stream);
  return cudaErrorInvalidValue;
}

}  // namespace msa
