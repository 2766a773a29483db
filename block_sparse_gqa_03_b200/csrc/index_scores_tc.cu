// Index branch for prefill on the fifth-generation tensor cores (tcgen05).
//
// "MiniMax goes sparse" (atlascloud.ai), section 1, step 1 and "MiniMax M3 的 MSA
// ..." (ai.air7.fun), first layer: token scores Q_idx . K_idx^T (one index query
// per GQA group, one index key shared by all heads), compressed by Block Max Pool.
// In prefill this is a dense causal GEMM per group (the pages note that the index
// branch still scans the whole length there), so it runs on tcgen05 MMAs with the
// accumulators in tensor memory; the causal mask and the block max are applied in
// the tensor-memory -> register epilogue, and only fp32 block scores reach HBM.
//
// One CTA per (sequence, pair of groups, tile of 128 queries).  Both groups share
// every 128-token key tile, which TMA streams through a ring of shared-memory
// stages; the two query tiles stay resident.  Warp roles:
//   warp 0     TMA producer (query tiles once, then the key ring);
//   warp 1     tensor-memory allocation, and one thread issuing the MMAs
//              (M = 128 queries, N = 128 keys, K = 16 per instruction);
//   warps 2-9  epilogue: one warp per (group, 32 tensor-memory lanes = 32
//              query rows); masks invisible keys, takes the block maxima,
//              stores them.  Tiles wholly below the causal frontier skip the
//              mask.
// Accumulators are double-buffered (2 x 2 groups x 128 columns = 512 columns), so
// the epilogue of one key tile overlaps the MMAs of the next.  Every mbarrier wait
// is bounded and records an error instead of hanging.
//
// Streaming top-k (the TOPK instantiation): the block scores need not reach HBM
// at all.  Each epilogue thread owns one (query, group) row and keeps the row's
// best blocks so far in a min-heap in shared memory (the root is the worst kept
// block: lowest score, then highest id), laid out [entry][row] so that the 32
// lanes of a warp touch 32 banks.  Blocks arrive in increasing id order, so a new
// block enters exactly when its score beats the root's (on equal scores the kept,
// lower id wins).  After the sweep the thread sorts its ids and writes them.  This
// follows the FlashMoBA top-k kernel's idea ("混合块注意力机制(MoBA)原理与实现详解",
// section 3.1, kernel 2: sorted top-k lists in SRAM instead of the score matrix in
// HBM); the heap costs the key ring two of its stages at d_idx 128.
#include "kernels.h"
#include "sm100.cuh"

namespace msa {
namespace {

constexpr int kQT = 128;  // queries per tile (MMA M, tensor-memory lanes)
constexpr int kKT = 128;  // keys per tile (MMA N)
constexpr int kNG = 2;    // groups per CTA
constexpr int kTcThreads = (2 + 4 * kNG) * 32;
constexpr uint32_t kTmemCols = 512;

struct TcArgs {
  int batch, n_q, max_kv, h, block, nblk, causal;
  const int32_t* seq_lens;
  int n_mtiles, n_gpairs, stages;
  float* scores;
  int fill_tail;
  DeviceStatus* st;
  uint64_t wait_ns;
  KvPages pg;  // table == nullptr: contiguous K_idx
  // streaming top-k: ids [b, n_q, h, topk]; scores (above) optional
  int32_t* ids;
  int topk, force_own;
};

constexpr int kHeapMax = 64;    // top-k the streaming variant takes
constexpr int kHeapRows = kNG * kQT;  // rows (query, group) of a CTA

// Sorts v[0..N) ascending (bitonic network, fully unrolled: v stays in registers).
template <int N>
__device__ __forceinline__ void bitonic_sort(uint32_t (&v)[N]) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const bool up = (i & k) == 0;
          const uint32_t x = v[i], y = v[l];
          v[i] = up ? min(x, y) : max(x, y);
          v[l] = up ? max(x, y) : min(x, y);
        }
      }
}

template <int DI, int BLK, bool TOPK>
__global__ void __launch_bounds__(kTcThreads, 1)
    index_score_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                          const __grid_constant__ CUtensorMap tmk, TcArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int NATOM = DI / 64;               // 128-byte K atoms per row
  constexpr uint32_t ATOM = 128u * 128u;       // one atom of a 128-row tile
  constexpr uint32_t Q_BYTES = NATOM * ATOM;   // one group's query tile
  constexpr uint32_t K_BYTES = NATOM * ATOM;   // one key tile
  if (status_failed(a.st)) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t q_base = smem_u32(smem);
  const uint32_t k_base = q_base + kNG * Q_BYTES;
  // streaming top-k heaps: scores [kHeapMax][kHeapRows] f32, ids [kHeapMax][kHeapRows] u16
  float* heap_s = reinterpret_cast<float*>(smem + kNG * Q_BYTES + a.stages * K_BYTES);
  uint16_t* heap_i = reinterpret_cast<uint16_t*>(heap_s + (TOPK ? kHeapMax * kHeapRows : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + kNG * Q_BYTES + a.stages * K_BYTES + (TOPK ? kHeapMax * kHeapRows * 6 : 0));
  const uint32_t b_qfull = smem_u32(bars);
  const uint32_t b_kfull = b_qfull + 8;
  const uint32_t b_kempty = b_kfull + 8 * a.stages;
  const uint32_t b_afull = b_kempty + 8 * a.stages;
  const uint32_t b_aempty = b_afull + 16;
  const uint32_t b_done = b_aempty + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1 + 2 * a.stages + 5);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = blockIdx.x;
  const int mt = a.n_mtiles - 1 - (x % a.n_mtiles);  // late (long) query tiles first
  x /= a.n_mtiles;
  const int gp = x % a.n_gpairs;
  const int b = x / a.n_gpairs;
  const int t0 = mt * kQT;
  const int ng_valid = min(kNG, a.h - gp * kNG);
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int t_last = min(t0 + kQT, a.n_q) - 1;
  const int p_last = L - a.n_q + t_last;
  const int lim_last = max(0, a.causal ? min(L, p_last + 1) : L);
  const int n_kt = (lim_last + kKT - 1) / kKT;  // key tiles holding a visible key

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(b_kfull + 8 * s, 1);
      mbar_init(b_kempty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_afull + 8 * i, 1);
      mbar_init(b_aempty + 8 * i, 4 * ng_valid);
    }
    mbar_init(b_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_kt > 0) {
      prefetch_tensormap(&tmq);
      prefetch_tensormap(&tmk);
      mbar_arrive_expect_tx(b_qfull, ng_valid * Q_BYTES);
      for (int ng = 0; ng < ng_valid; ++ng)
#pragma unroll
        for (int at = 0; at < NATOM; ++at)
          tma_load_4d(q_base + ng * Q_BYTES + at * ATOM, &tmq, b_qfull, at * 64, gp * kNG + ng,
                      t0, b);
      int issued = 0;
      for (int kt = 0; kt < n_kt; ++kt) {
        const int s = kt % a.stages;
        if (kt >= a.stages &&
            !mbar_wait_bounded(b_kempty + 8 * s, ((kt / a.stages) - 1) & 1, a.st, 0x101u,
                               a.wait_ns))
          break;
        mbar_arrive_expect_tx(b_kfull + 8 * s, K_BYTES);
        if (a.pg.table == nullptr) {
#pragma unroll
          for (int at = 0; at < NATOM; ++at)
            tma_load_3d(k_base + s * K_BYTES + at * ATOM, &tmk, b_kfull + 8 * s, at * 64,
                        kt * kKT, b);
        } else {
          // one box per page of BLK tokens; blocks past the sequence end are not
          // looked up and read as zeros (their keys are masked anyway)
          const int nb_b = (L + BLK - 1) / BLK;
          for (int pi = 0; pi < kKT / BLK; ++pi) {
            const int beta = kt * (kKT / BLK) + pi;
            const int64_t page = beta < nb_b ? kv_page(a.pg, b, beta, a.st) : -1;
            const int plane = page < 0 ? (int)a.pg.pages : (int)page;
#pragma unroll
            for (int at = 0; at < NATOM; ++at)
              tma_load_3d(k_base + s * K_BYTES + at * ATOM + pi * BLK * 128u, &tmk,
                          b_kfull + 8 * s, at * 64, 0, plane);
          }
        }
        ++issued;
      }
      // Drain: the last stages are released by the MMA commits, i.e. after their
      // copies landed and were read.
      for (int kt = max(0, issued - a.stages); kt < issued; ++kt)
        mbar_wait_bounded(b_kempty + 8 * (kt % a.stages), (kt / a.stages) & 1, a.st, 0x102u,
                          a.wait_ns);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0 && n_kt > 0) {
      const uint32_t idesc = tc::idesc_bf16(kQT, kKT, false);
      bool ok = mbar_wait_bounded(b_qfull, 0, a.st, 0x103u, a.wait_ns);
      for (int kt = 0; kt < n_kt && ok; ++kt) {
        const int s = kt % a.stages, buf = kt & 1;
        ok = mbar_wait_bounded(b_kfull + 8 * s, (kt / a.stages) & 1, a.st, 0x104u, a.wait_ns);
        if (ok && kt >= 2)
          ok = mbar_wait_bounded(b_aempty + 8 * buf, ((kt >> 1) - 1) & 1, a.st, 0x105u,
                                 a.wait_ns);
        if (!ok) break;
        tc::fence_after_sync();
        for (int ng = 0; ng < ng_valid; ++ng) {
          const uint32_t d_tmem = tmem + (uint32_t)(buf * kNG * kKT + ng * kKT);
#pragma unroll
          for (int ks = 0; ks < DI / 16; ++ks) {
            const uint32_t koff = (ks >> 2) * ATOM + (ks & 3) * 32;
            tc::mma_bf16(d_tmem, tc::desc_k_sw128(q_base + ng * Q_BYTES + koff),
                         tc::desc_k_sw128(k_base + s * K_BYTES + koff), idesc, ks > 0 ? 1u : 0u);
          }
        }
        tc::commit(b_kempty + 8 * s);
        tc::commit(b_afull + 8 * buf);
      }
      // Every MMA this thread issued has completed before tensor memory is freed.
      tc::commit(b_done);
      mbar_wait_bounded(b_done, 0, a.st, 0x107u, a.wait_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // tensor-memory lanes [32q, 32q + 32)
    const int ng = (warp - 2) >> 2;  // this warp's group of the pair
    const int row = quarter * 32 + lane;
    const int t = t0 + row;
    const bool row_ok = t < a.n_q;
    const int p = L - a.n_q + t;
    const int lim = row_ok ? max(0, a.causal ? min(L, p + 1) : L) : 0;
    constexpr int bpt = kKT / BLK;  // blocks per key tile
    const float ninf = -__int_as_float(0x7f800000);
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int64_t rowi = ((int64_t)b * a.n_q + t) * a.h + gp * kNG + ng;
    float* srow = a.scores ? a.scores + rowi * (int64_t)a.nblk : nullptr;
    // streaming top-k state: the heap holds `cap` entries (the forced own block is
    // kept aside), `root` caches the heap root's score
    const int hr = ng * kQT + row;  // this thread's heap column
    const int nb_row = (L + BLK - 1) / BLK;
    const int F = row_ok ? (a.causal ? (p < 0 ? 0 : min(nb_row, p / BLK + 1)) : nb_row) : 0;
    const int own = (TOPK && a.force_own && row_ok && p >= 0 && p / BLK < F) ? p / BLK : -1;
    const int cap = TOPK ? a.topk - (own >= 0 ? 1 : 0) : 0;
    float root = ninf;
    if (TOPK) {
      for (int i = 0; i < cap; ++i) {
        heap_s[i * kHeapRows + hr] = ninf;
        heap_i[i * kHeapRows + hr] = 0xffffu;
      }
    }
    for (int kt = 0; kt < n_kt && ng < ng_valid; ++kt) {
      const int buf = kt & 1;
      if (!mbar_wait_warp(b_afull + 8 * buf, (kt >> 1) & 1, a.st, 0x106u, a.wait_ns)) break;
      tc::fence_after_sync();
      const int j0 = kt * kKT;
      const int vis = lim - j0;  // columns [0, vis) of this tile are visible keys
      float v[kKT];
#pragma unroll
      for (int c = 0; c < kKT / 32; ++c)
        tc::tmem_ld32_at(lane_base + (uint32_t)(buf * kNG * kKT + ng * kKT + c * 32), v + c * 32);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_aempty + 8 * buf);
      float bm[bpt];
      if (vis >= kKT) {
#pragma unroll
        for (int k = 0; k < bpt; ++k) {
          float m0 = fmaxf(v[k * BLK], v[k * BLK + 1]), m1 = fmaxf(v[k * BLK + 2], v[k * BLK + 3]);
#pragma unroll
          for (int i = 4; i + 3 < BLK; i += 4) {
            m0 = fmax3(m0, v[k * BLK + i], v[k * BLK + i + 1]);
            m1 = fmax3(m1, v[k * BLK + i + 2], v[k * BLK + i + 3]);
          }
          bm[k] = fmaxf(m0, m1);
        }
      } else {
#pragma unroll
        for (int k = 0; k < bpt; ++k) bm[k] = ninf;
#pragma unroll
        for (int col = 0; col < kKT; ++col)
          bm[col / BLK] = fmaxf(bm[col / BLK], col < vis ? v[col] : ninf);
      }
      if (row_ok) {
        if (srow != nullptr) {
#pragma unroll
          for (int k = 0; k < bpt; ++k)
            if (j0 / BLK + k < a.nblk) srow[j0 / BLK + k] = bm[k];
        }
        if constexpr (TOPK) {
#pragma unroll
          for (int k = 0; k < bpt; ++k) {
            const int beta = j0 / BLK + k;
            const float sc = bm[k];
            if (sc > root && beta != own && cap > 0) {
              // replace the root, sift the new entry down (worse children move up)
              int pos = 0;
              for (;;) {
                int c = 2 * pos + 1;
                if (c >= cap) break;
                float cs = heap_s[c * kHeapRows + hr];
                uint32_t ci = heap_i[c * kHeapRows + hr];
                if (c + 1 < cap) {
                  const float s2 = heap_s[(c + 1) * kHeapRows + hr];
                  const uint32_t i2 = heap_i[(c + 1) * kHeapRows + hr];
                  if (s2 < cs || (s2 == cs && i2 > ci)) {
                    c = c + 1;
                    cs = s2;
                    ci = i2;
                  }
                }
                if (cs < sc || (cs == sc && ci > (uint32_t)beta)) {
                  heap_s[pos * kHeapRows + hr] = cs;
                  heap_i[pos * kHeapRows + hr] = (uint16_t)ci;
                  pos = c;
                } else {
                  break;
                }
              }
              heap_s[pos * kHeapRows + hr] = sc;
              heap_i[pos * kHeapRows + hr] = (uint16_t)beta;
              root = heap_s[hr];
            }
          }
        }
      }
    }
    if (srow != nullptr && a.fill_tail && row_ok && ng < ng_valid)
      for (int beta = n_kt * bpt; beta < a.nblk; ++beta) srow[beta] = ninf;
    if constexpr (TOPK) {
      if (row_ok && ng < ng_valid) {
        // the kept ids (empty entries are 0xffff and sort last) and the forced own
        // block, in ascending order, then -1 padding
        uint32_t v[kHeapMax];
#pragma unroll
        for (int i = 0; i < kHeapMax; ++i)
          v[i] = i < cap ? (uint32_t)heap_i[i * kHeapRows + hr]
                         : (i == cap && own >= 0 ? (uint32_t)own : 0xffffu);
        bitonic_sort<kHeapMax>(v);
        const int m = min(a.topk, F);
        int32_t* out = a.ids + rowi * a.topk;
#pragma unroll
        for (int i = 0; i < kHeapMax; ++i)
          if (i < a.topk) out[i] = i < m ? (int32_t)v[i] : -1;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DI, int BLK, bool TOPK>
cudaError_t run_tc(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx, TcArgs& a,
                   cudaStream_t stream) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorInvalidValue;
  CUtensorMap tmq, tmk;
  {
    cuuint64_t dims[4] = {(cuuint64_t)s.d_idx, (cuuint64_t)s.h, (cuuint64_t)s.n_q,
                          (cuuint64_t)s.batch};
    cuuint64_t str[3] = {(cuuint64_t)s.qi_s[2] * 2, (cuuint64_t)s.qi_s[1] * 2,
                         (cuuint64_t)s.qi_s[0] * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kQT, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    if (enc(&tmq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(q_idx), dims, str,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // contiguous [d_idx, token, batch] with 128-token boxes, or a page pool
    // [d_idx, token in page, page] with one-page boxes
    const bool paged = s.pages.table != nullptr;
    cuuint64_t dims[3] = {(cuuint64_t)s.d_idx, (cuuint64_t)(paged ? BLK : s.max_kv),
                          (cuuint64_t)(paged ? s.pages.pages : s.batch)};
    cuuint64_t str[2] = {(cuuint64_t)s.ki_s[1] * 2, (cuuint64_t)s.ki_s[0] * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)(paged ? BLK : kKT), 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tmk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(k_idx), dims, str,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  constexpr uint32_t tile = (DI / 64) * 128u * 128u;
  constexpr size_t heap = TOPK ? (size_t)kHeapMax * kHeapRows * 6 : 0;
  a.stages = DI == 128 ? 4 : 8;
  auto bytes = [&](int st) {
    return 1024 + kNG * tile + (size_t)st * tile + heap + 8 * (1 + 2 * st + 5) + 16;
  };
  while (a.stages > 2 && bytes(a.stages) > (size_t)max_smem_optin()) --a.stages;
  const size_t smem = bytes(a.stages);
  cudaError_t err = cudaFuncSetAttribute(index_score_tc_kernel<DI, BLK, TOPK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const unsigned grid = (unsigned)((int64_t)s.batch * a.n_gpairs * a.n_mtiles);
  return launch_pdl(index_score_tc_kernel<DI, BLK, TOPK>, dim3(grid), dim3(kTcThreads), smem,
                    stream, tmq, tmk, a);
}

}  // namespace

bool index_scores_tc_supported(const Shape& s) {
  return s.n_q > 1 && (s.d_idx == 64 || s.d_idx == 128);
}

cudaError_t launch_index_scores_tc(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                   float* scores, bool fill_tail, DeviceStatus* st,
                                   cudaStream_t stream) {
  TcArgs a;
  a.batch = s.batch;
  a.n_q = s.n_q;
  a.max_kv = s.max_kv;
  a.h = s.h;
  a.block = s.block;
  a.nblk = s.nblk;
  a.causal = s.causal;
  a.seq_lens = s.seq_lens;
  a.n_mtiles = (s.n_q + kQT - 1) / kQT;
  a.n_gpairs = (s.h + kNG - 1) / kNG;
  a.scores = scores;
  a.fill_tail = fill_tail ? 1 : 0;
  a.st = st;
  a.wait_ns = 4000000000ull;
  a.pg = s.pages;
  a.ids = nullptr;
  a.topk = s.topk;
  a.force_own = s.force_own;
#define MSA_TC_CASE(DI_, BLK_) \
  if (s.d_idx == DI_ && s.block == BLK_) return run_tc<DI_, BLK_, false>(s, q_idx, k_idx, a, stream);
  MSA_TC_CASE(128, 16)
  MSA_TC_CASE(128, 32)
  MSA_TC_CASE(128, 64)
  MSA_TC_CASE(128, 128)
  MSA_TC_CASE(64, 16)
  MSA_TC_CASE(64, 32)
  MSA_TC_CASE(64, 64)
  MSA_TC_CASE(64, 128)
#undef MSA_TC_CASE
  return cudaErrorInvalidValue;
}

bool index_topk_tc_supported(const Shape& s) {
  return index_scores_tc_supported(s) && (s.block == 64 || s.block == 128) &&
         s.topk <= kHeapMax && s.nblk <= 0xffff;
}

cudaError_t launch_index_topk_tc(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                 int32_t* ids, float* scores, DeviceStatus* st,
                                 cudaStream_t stream) {
  if (!index_topk_tc_supported(s)) return cudaErrorInvalidValue;
  TcArgs a;
  a.batch = s.batch;
  a.n_q = s.n_q;
  a.max_kv = s.max_kv;
  a.h = s.h;
  a.block = s.block;
  a.nblk = s.nblk;
  a.causal = s.causal;
  a.seq_lens = s.seq_lens;
  a.n_mtiles = (s.n_q + kQT - 1) / kQT;
  a.n_gpairs = (s.h + kNG - 1) / kNG;
  a.scores = scores;
  a.fill_tail = 1;
  a.st = st;
  a.wait_ns = 4000000000ull;
  a.pg = s.pages;
  a.ids = ids;
  a.topk = s.topk;
  a.force_own = s.force_own;
  if (s.d_idx == 128 && s.block == 128) return run_tc<128, 128, true>(s, q_idx, k_idx, a, stream);
  if (s.d_idx == 128 && s.block == 64) return run_tc<128, 64, true>(s, q_idx, k_idx, a, stream);
  if (s.d_idx == 64 && s.block == 128) return run_tc<64, 128, true>(s, q_idx, k_idx, a, stream);
  if (s.d_idx == 64 && s.block == 64) return run_tc<64, 64, true>(s, q_idx, k_idx, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace msa
