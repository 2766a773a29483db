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
//
// Decode with d_idx 64 or 128 takes a persistent streaming scan instead: one
// CTA per SM owns an equal, contiguous share of the (sequence, block) items; a
// producer lane brings each item's K_idx block into a ring of shared-memory
// stages with TMA (128-byte swizzle, waits bounded), and consumer warp w takes
// items w, w + 8, ...: token rows as A fragments by ldmatrix, the sequence's h
// index queries as B fragments held in registers, the block max reduced over
// the warp.  The ring keeps a steady stream of bulk copies in flight per SM.
#include "kernels.h"
#include "sm100.cuh"

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


// ------------------------------------------------ decode: streaming TMA scan
struct StreamScanArgs {
  const uint16_t* q_idx;
  int64_t qi_s0, qi_s2;
  const int32_t* seq_lens;
  int batch, max_kv, h, block, nblk, stages;
  uint32_t stage_bytes;
  float* scores;
  int fill_tail;
  DeviceStatus* st;
  uint64_t wait_ns;
  KvPages pg;
};

constexpr int kStreamScanWarps = 8;  // consumer warps; one more warp produces

__device__ __forceinline__ int seq_blocks(const StreamScanArgs& a, int b) {
  return (kv_length(a.seq_lens, b, a.max_kv, a.st) + a.block - 1) / a.block;
}

// B fragments of sequence b's index queries: column c = nt*8 + r is group c,
// k-step ks holds dims [16ks + 2q, +2) and [16ks + 8 + 2q, +2).
template <int DI, int NT>
__device__ __forceinline__ void load_query_frags(const StreamScanArgs& a, int b, int r, int q,
                                                 uint32_t (&bf)[NT][DI / 16][2]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int g = nt * 8 + r;
    const bool ok = g < a.h;
    const uint16_t* src = a.q_idx + b * a.qi_s0 + (int64_t)g * a.qi_s2 + 2 * q;
#pragma unroll
    for (int ks = 0; ks < DI / 16; ++ks) {
      bf[nt][ks][0] = ok ? *reinterpret_cast<const uint32_t*>(src + 16 * ks) : 0u;
      bf[nt][ks][1] = ok ? *reinterpret_cast<const uint32_t*>(src + 16 * ks + 8) : 0u;
    }
  }
}

template <int DI, int NT>
__global__ void __launch_bounds__((kStreamScanWarps + 1) * 32, 1)
    index_scan_stream_kernel(const __grid_constant__ CUtensorMap tmk, StreamScanArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int NW = kStreamScanWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int S = a.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * a.stage_bytes);
  int2* info = reinterpret_cast<int2*>(bars + 2 * S);  // [S] (sequence, block) of a stage
  int* n_items = reinterpret_cast<int*>(info + S);
  int4* coord = reinterpret_cast<int4*>(bars + 3 * S + 2);  // [32] next items: tok, plane, b, beta
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t box_bytes = (uint32_t)a.block * 128u;

  if (warp == NW) {
    // Producer warp: barriers, this CTA's share of the items (counted over the
    // sequences' block counts), then one lane streams them.
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(full0 + 8 * s, 1);
        mbar_init(empty0 + 8 * s, 1);
      }
      fence_mbar_init();
      prefetch_tensormap(&tmk);
    }
    const bool skip = status_failed(a.st);
    int total = 0;
    for (int b = lane; b < a.batch; b += 32) total += seq_blocks(a, b);
    total = (int)__reduce_add_sync(0xffffffffu, (unsigned)total);
    const int per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int i0 = (int)blockIdx.x * per;
    const int n = max(0, min(total, i0 + per) - i0);
    // first item: the sequence whose block range holds i0
    int b0 = 0, beta0 = 0, carry = 0;
    bool found = false;
    for (int base = 0; base < a.batch && !found; base += 32) {
      const int b = base + lane;
      const int nb = b < a.batch ? seq_blocks(a, b) : 0;
      int inc = nb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      const int excl = carry + inc - nb;
      const unsigned hit = __ballot_sync(0xffffffffu, nb > 0 && i0 >= excl && i0 < excl + nb);
      if (hit) {
        const int src = __ffs(hit) - 1;
        b0 = base + src;
        beta0 = i0 - __shfl_sync(0xffffffffu, excl, src);
        found = true;
      }
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) *n_items = skip ? -1 : n;
    __syncwarp();
    named_arrive(2, (NW + 1) * 32);
    if (skip || n == 0) return;
    int b = b0, beta = beta0, issued = 0;
    bool failed = false;
    if (a.pg.table == nullptr) {
      // contiguous K_idx: lane 0 walks the items itself (no table loads)
      if (lane != 0) return;
      int nb = seq_blocks(a, b0);
      for (int k = 0; k < n; ++k) {
        const int s = k % S;
        if (k >= S &&
            !mbar_wait_bounded(empty0 + 8 * s, ((k / S) - 1) & 1, a.st, 0x201u, a.wait_ns))
          break;
        info[s] = make_int2(b, beta);
        const uint32_t full = full0 + 8 * s, dst = sbase + (uint32_t)s * a.stage_bytes;
        mbar_arrive_expect_tx(full, a.stage_bytes);
#pragma unroll
        for (int hh = 0; hh < DI / 64; ++hh)
          tma_load_3d(dst + hh * box_bytes, &tmk, full, hh * 64, beta * a.block, b);
        issued = k + 1;
        if (++beta == nb) {
          beta = 0;
          do {
            ++b;
            nb = b < a.batch ? seq_blocks(a, b) : 1;
          } while (nb == 0);
        }
      }
    }
    // Paged K_idx, groups of 32 items: every lane resolves one item's sequence,
    // block and page (the table loads run in parallel), and lane 0 streams the
    // group from shared memory.
    for (int k0 = 0; k0 < n && !failed && a.pg.table != nullptr; k0 += 32) {
      if (k0 + lane < n) {
        int bb = b, bt = beta + lane, nbb = seq_blocks(a, bb);
        while (bt >= nbb) {  // the item exists, so bb stays below the batch
          bt -= nbb;
          nbb = seq_blocks(a, ++bb);
        }
        int tok, plane;
        kv_block_coords(a.pg, bb, bt, a.block, a.st, tok, plane);
        coord[lane] = make_int4(tok, plane, bb, bt);
      }
      __syncwarp();
      if (lane == 0) {
        for (int j = 0; j < 32 && k0 + j < n; ++j) {
          const int k = k0 + j, s = k % S;
          if (k >= S &&
              !mbar_wait_bounded(empty0 + 8 * s, ((k / S) - 1) & 1, a.st, 0x201u, a.wait_ns)) {
            failed = true;
            break;
          }
          const int4 c = coord[j];
          info[s] = make_int2(c.z, c.w);
          const uint32_t full = full0 + 8 * s, dst = sbase + (uint32_t)s * a.stage_bytes;
          mbar_arrive_expect_tx(full, a.stage_bytes);
#pragma unroll
          for (int hh = 0; hh < DI / 64; ++hh)
            tma_load_3d(dst + hh * box_bytes, &tmk, full, hh * 64, c.x, c.y);
          issued = k + 1;
        }
      }
      failed = __shfl_sync(0xffffffffu, failed, 0);
      const int4 last = coord[31];  // next group starts after this group's last item
      b = last.z;
      beta = last.w + 1;
      __syncwarp();
    }
    if (lane != 0) return;
    // before leaving, wait (bounded) for the copies still in flight
    for (int k = max(0, issued - S); k < issued; ++k)
      mbar_wait_bounded(full0 + 8 * (k % S), (k / S) & 1, a.st, 0x203u, a.wait_ns);
    return;
  }

  named_sync(2, (NW + 1) * 32);
  const int n = *n_items;
  if (n < 0) return;
  const int r = lane >> 2, q = lane & 3;
  const float ninf = -__int_as_float(0x7f800000);
  uint32_t bf[NT][DI / 16][2];
  int cur_b = -1, L = 0;
  for (int k = warp; k < n; k += NW) {
    const int s = k % S;
    if (!mbar_wait_warp(full0 + 8 * s, (k / S) & 1, a.st, 0x202u, a.wait_ns)) break;
    const int2 it = info[s];
    if (it.x != cur_b) {
      cur_b = it.x;
      L = kv_length(a.seq_lens, cur_b, a.max_kv, a.st);
      load_query_frags<DI, NT>(a, cur_b, r, q, bf);
    }
    const uint32_t base = sbase + (uint32_t)s * a.stage_bytes;
    float cm[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) cm[nt][0] = cm[nt][1] = ninf;
    for (int mt = 0; mt < a.block / 16; ++mt) {
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      const uint32_t row = (uint32_t)(mt * 16 + (lane & 15));
#pragma unroll
      for (int ks = 0; ks < DI / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(base + (uint32_t)(ks >> 2) * box_bytes +
                        swz128(row, (uint32_t)((ks & 3) * 2 + (lane >> 4))),
                    a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16_16816(acc[nt], a0, a1, a2, a3, bf[nt][ks][0], bf[nt][ks][1]);
      }
      const int jl = it.y * a.block + mt * 16 + r, jh = jl + 8;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          cm[nt][e] = fmaxf(cm[nt][e], jl < L ? acc[nt][e] : ninf);
          cm[nt][e] = fmaxf(cm[nt][e], jh < L ? acc[nt][2 + e] : ninf);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = cm[nt][e];
        v = warp_max_xor(v, 4);
        v = warp_max_xor(v, 8);
        v = warp_max_xor(v, 16);
        const int g = nt * 8 + 2 * q + e;
        if (r == 0 && g < a.h) a.scores[((int64_t)it.x * a.h + g) * a.nblk + it.y] = v;
      }
  }
  if (a.fill_tail) {
    // blocks past each sequence's end: -inf, spread over every consumer thread
    const int nthr = (int)gridDim.x * NW * 32;
    const int gt = (int)blockIdx.x * NW * 32 + (int)threadIdx.x;
    for (int b = 0; b < a.batch; ++b)
      for (int beta = seq_blocks(a, b) + gt; beta < a.nblk; beta += nthr)
        for (int g = 0; g < a.h; ++g) a.scores[((int64_t)b * a.h + g) * a.nblk + beta] = ninf;
  }
}

template <int DI, int NT>
cudaError_t run_stream_scan(const Shape& s, const uint16_t* k_idx, StreamScanArgs& a,
                            cudaStream_t stream, bool& done) {
  done = false;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaSuccess;
  // contiguous [d_idx, token, batch], or a page pool [d_idx, token in page, page];
  // one box is 64 dims x one block of tokens
  const bool paged = s.pages.table != nullptr;
  cuuint64_t dims[3] = {(cuuint64_t)DI, (cuuint64_t)(paged ? s.block : s.max_kv),
                        (cuuint64_t)(paged ? s.pages.pages : s.batch)};
  cuuint64_t str[2] = {(cuuint64_t)s.ki_s[1] * 2, (cuuint64_t)s.ki_s[0] * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)s.block, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUtensorMap tmk;
  if (enc(&tmk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(k_idx), dims, str,
          box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaSuccess;  // not expressible as a tensor map: the direct-load scan runs
  a.stage_bytes = (uint32_t)DI * 2u * (uint32_t)s.block;
  // alignment slack, the item count and the 32 resolved items after the stages'
  // barriers and (sequence, block) words
  const size_t fixed = 1024 + 16 + 32 * 16;
  const size_t cap = (size_t)max_smem_optin();
  // Consumer warp w takes items w, w + NW, ... and item k uses stage k % S.  With
  // S a multiple of NW every stage is only ever consumed by one warp, which has
  // consumed the stage's previous fill itself before it waits on the next: a
  // parity wait then never meets a phase two fills behind (a stage shared by
  // several warps would let one warp pass the parity test on a fill that
  // another warp's item has not completed).
  const size_t fit = (cap - fixed) / (a.stage_bytes + 24);
  const int nw = kStreamScanWarps;
  a.stages = (int)(fit >= 2 * (size_t)nw ? 2 * nw : (fit >= (size_t)nw ? nw : 0));
  if (a.stages == 0) return cudaSuccess;  // too few stages fit: the direct-load scan runs
  const size_t smem = fixed + (size_t)a.stages * (a.stage_bytes + 24);
  cudaError_t err = cudaFuncSetAttribute(index_scan_stream_kernel<DI, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  done = true;
  return launch_pdl(index_scan_stream_kernel<DI, NT>, dim3(num_sms()),
                    dim3((kStreamScanWarps + 1) * 32), smem, stream, tmk, a);
}

// Decode scans that the streaming kernel covers; `done` is false when the
// direct-load kernel must run instead.
cudaError_t launch_stream_scan(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                               float* scores, bool fill_tail, DeviceStatus* st,
                               cudaStream_t stream, bool& done) {
  done = false;
  if (s.n_q != 1 || s.h > 16 || (s.d_idx != 64 && s.d_idx != 128) || s.block < 16 ||
      s.block > 128 || s.block % 16 != 0 || (int64_t)s.batch * s.nblk >= (1LL << 31))
    return cudaSuccess;
  StreamScanArgs a;
  a.q_idx = q_idx;
  a.qi_s0 = s.qi_s[0];
  a.qi_s2 = s.qi_s[2];
  a.seq_lens = s.seq_lens;
  a.batch = s.batch;
  a.max_kv = s.max_kv;
  a.h = s.h;
  a.block = s.block;
  a.nblk = s.nblk;
  a.scores = scores;
  a.fill_tail = fill_tail ? 1 : 0;
  a.st = st;
  a.wait_ns = 4000000000ull;
  a.pg = s.pages;
  const bool two = s.h > 8;
  if (s.d_idx == 128)
    return two ? run_stream_scan<128, 2>(s, k_idx, a, stream, done)
               : run_stream_scan<128, 1>(s, k_idx, a, stream, done);
  return two ? run_stream_scan<64, 2>(s, k_idx, a, stream, done)
             : run_stream_scan<64, 1>(s, k_idx, a, stream, done);
}

}  // namespace

cudaError_t launch_index_scores(const Shape& s, const uint16_t* q_idx, const uint16_t* k_idx,
                                float* scores, bool fill_tail, DeviceStatus* st,
                                cudaStream_t stream) {
  bool done = false;
  const cudaError_t e = launch_stream_scan(s, q_idx, k_idx, scores, fill_tail, st, stream, done);
  if (e != cudaSuccess || done) return e;
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
