// Sparse branch: exact softmax attention over the selected KV blocks.
//
// "MiniMax goes sparse" (atlascloud.ai), section 1, step 2: with the block ids of
// step 1, the matching block subsets are taken from the raw K/V and ordinary
// softmax attention runs over them; all query heads of a GQA group share the
// group's top-k selection, so one load of a block serves the whole group
// ("MiniMax M3 的 MSA ...", second layer).
//
// A "row" is one (sequence, query, group); its G query heads are the 16 rows of
// a bf16 m16n8k16 tensor-core tile (rows >= G are zero), or, in the streaming
// kernel for G <= 8, the 8 columns of the tile with the operands swapped
// (WarpStateT).  Both kernels below share the same engine:
//  * one producer warp streams each selected block's K and V tiles into a ring of
//    shared-memory stages with TMA (4-D tensor maps over [batch, token, kv head,
//    dim], 128-byte swizzle), completion tracked by mbarriers whose waits are
//    bounded (a wait that runs out records an error; nothing hangs);
//  * consumer warps take 16-token slices of the blocks in turn: S = Q K^T and
//    O += P V on MMAs fed by ldmatrix from the swizzled tiles, with an fp32
//    online softmax in the exp2 domain; each warp keeps its own running max, sum
//    and output, and the warps' states are merged through shared memory.
//
// sparse_attn_rows_kernel: one CTA per row (prefill: many rows, each with a
// modest block list).  Writes bf16 output and the log-sum-exp directly.
//
// sparse_attn_stream_kernel: decode-style work, few rows with long block lists.
// A persistent grid of one CTA per SM splits the flattened (row, slot) list into
// equal contiguous ranges, so every SM streams the same number of blocks through
// one pipeline that never drains.  At each row boundary the consumers merge their
// states; a row covered by several CTAs gets one fp32 partial per CTA, and the
// last CTA to finish the row (a per-row counter, zero before the launch and put
// back to zero by the merging CTA) merges them by log-sum-exp weights.  The row's first CTA, which reaches the
// row at the end of its range, usually finds the others' partials already
// published and merges them into its own state without writing its own.
#include "kernels.h"

namespace msa {
namespace {

struct AttnArgs {
  const uint16_t* q;
  int64_t q_s0, q_s1, q_s2;
  const int32_t* ids;
  const int32_t* seq_lens;
  int n_q, max_kv, H, h, G, topk, block, nblk, causal;
  float scale_log2;
  int stages;
  uint32_t stage_bytes, region_bytes, merge_off;
  int list_cap;
  // stream kernel only
  int64_t total_slots;
  int per, smax;
  float* part_o;
  float* part_lse;
  int* counters;
  uint16_t* out;
  int64_t o_s0, o_s1, o_s2;
  float* lse;
  DeviceStatus* st;
  uint64_t wait_ns;
  KvPages pg;  // table == nullptr: contiguous K/V
};

constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t ld_b32(const uint16_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

__device__ __forceinline__ float neg_inf() { return -__int_as_float(0x7f800000); }

// Geometry of one row: sequence b, query t, group g, and the visible-token bound.
struct RowGeo {
  int b, t, g, bt, lim;
};

__device__ __forceinline__ RowGeo row_geo(const AttnArgs& a, int64_t rowg) {
  RowGeo r;
  r.g = (int)(rowg % a.h);
  r.bt = (int)(rowg / a.h);
  r.t = r.bt % a.n_q;
  r.b = r.bt / a.n_q;
  const int L = kv_length(a.seq_lens, r.b, a.max_kv, a.st);
  const int p = L - a.n_q + r.t;
  r.lim = a.causal ? min(L, p + 1) : L;  // visible tokens: j < lim
  return r;
}

// Running softmax state of one warp: rows r and r + 8 of the 16-row tile.
template <int D>
struct WarpState {
  uint32_t qa[D / 16][4];
  float o[D / 8][4];
  float m_a, m_b, l_a, l_b;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m_a = m_b = neg_inf();
    l_a = l_b = 0.f;
  }

  // A-operand fragments of the group's G query heads (rows >= G are zero).
  __device__ __forceinline__ void load_q(const AttnArgs& a, const RowGeo& rg, int lane) {
    const int r = lane >> 2, q4 = lane & 3;
    const bool vlo = r < a.G, vhi = r + 8 < a.G;
    const uint16_t* qb = a.q + rg.b * a.q_s0 + (int64_t)rg.t * a.q_s1 +
                         (int64_t)(rg.g * a.G) * a.q_s2 + 2 * q4;
    const uint16_t* qlo = qb + (int64_t)r * a.q_s2;
    const uint16_t* qhi = qb + (int64_t)(r + 8) * a.q_s2;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qa[kk][0] = vlo ? ld_b32(qlo + 16 * kk) : 0u;
      qa[kk][1] = vhi ? ld_b32(qhi + 16 * kk) : 0u;
      qa[kk][2] = vlo ? ld_b32(qlo + 16 * kk + 8) : 0u;
      qa[kk][3] = vhi ? ld_b32(qhi + 16 * kk + 8) : 0u;
    }
  }

  // One 16-token slice (rows `tok`.. of the stage tiles, absolute first token j0).
  __device__ __forceinline__ void attend(const AttnArgs& a, uint8_t* smem, uint32_t sbase,
                                         uint32_t kbase, uint32_t vbase, uint32_t half_bytes,
                                         int tok, int j0, int lim, int lane, bool& wrote_smem) {
    constexpr int NH = D / 64;
    const int q4 = lane & 3;
    const float ninf = neg_inf();
    if (j0 + 16 > lim) {
      // Tokens j >= lim of this slice may be uninitialised memory: zero their V rows
      // so that a zero probability never meets a non-finite value.
      const int r0 = lim - j0;
      const int per_h = (16 - r0) * 8;
      uint8_t* vrow = smem + (vbase - sbase);
      for (int x = lane; x < per_h * NH; x += 32) {
        const int hh = x / per_h, rem = x % per_h;
        const int row = tok + r0 + rem / 8;
        *reinterpret_cast<uint4*>(vrow + hh * half_bytes + row * 128 + (rem % 8) * 16) =
            make_uint4(0, 0, 0, 0);
      }
      wrote_smem = true;
      __syncwarp();
    }
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    {
      const int mi = lane >> 3, rr = lane & 7;
      const uint32_t row = tok + (mi >> 1) * 8 + rr;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t chunk = (kk & 3) * 2 + (mi & 1);
        uint32_t k0, k1, k2, k3;
        ldmatrix_x4(kbase + (kk >> 2) * half_bytes + swz128(row, chunk), k0, k1, k2, k3);
        mma_bf16_16816(sc[0], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], k0, k1);
        mma_bf16_16816(sc[1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], k2, k3);
      }
    }
    float mx_a = ninf, mx_b = ninf;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = j0 + nt * 8 + 2 * q4 + e < lim;
        sc[nt][e] = ok ? sc[nt][e] * a.scale_log2 : ninf;
        sc[nt][2 + e] = ok ? sc[nt][2 + e] * a.scale_log2 : ninf;
        mx_a = fmaxf(mx_a, sc[nt][e]);
        mx_b = fmaxf(mx_b, sc[nt][2 + e]);
      }
    mx_a = warp_max_xor(warp_max_xor(mx_a, 1), 2);
    mx_b = warp_max_xor(warp_max_xor(mx_b, 1), 2);
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float c_a = exp2f(m_a - mn_a), c_b = exp2f(m_b - mn_b);
    m_a = mn_a;
    m_b = mn_b;
    float ps_a = 0.f, ps_b = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        sc[nt][e] = exp2f(sc[nt][e] - mn_a);
        sc[nt][2 + e] = exp2f(sc[nt][2 + e] - mn_b);
        ps_a += sc[nt][e];
        ps_b += sc[nt][2 + e];
      }
    l_a = l_a * c_a + ps_a;
    l_b = l_b * c_b + ps_b;
#pragma unroll
    for (int i2 = 0; i2 < D / 8; ++i2) {
      o[i2][0] *= c_a;
      o[i2][1] *= c_a;
      o[i2][2] *= c_b;
      o[i2][3] *= c_b;
    }
    const uint32_t pa0 = pack_bf16(sc[0][0], sc[0][1]);
    const uint32_t pa1 = pack_bf16(sc[0][2], sc[0][3]);
    const uint32_t pa2 = pack_bf16(sc[1][0], sc[1][1]);
    const uint32_t pa3 = pack_bf16(sc[1][2], sc[1][3]);
    const int mi = lane >> 3, rr = lane & 7;
    const uint32_t row = tok + (mi & 1) * 8 + rr;
#pragma unroll
    for (int c2 = 0; c2 < D / 16; ++c2) {
      const uint32_t chunk = (c2 & 3) * 2 + (mi >> 1);
      uint32_t v0, v1, v2, v3;
      ldmatrix_x4_trans(vbase + (c2 >> 2) * half_bytes + swz128(row, chunk), v0, v1, v2, v3);
      mma_bf16_16816(o[2 * c2], pa0, pa1, pa2, pa3, v0, v1);
      mma_bf16_16816(o[2 * c2 + 1], pa0, pa1, pa2, pa3, v2, v3);
    }
  }

  // Stores this warp's state in the merge buffer: o [16][D], m [16], l [16].
  // Writes this warp's state for the merge: O rows [warp][gr][D] (only the gr
  // head rows in use), running max and sum [warp][16].
  __device__ __forceinline__ void stash(float* mo, float* mm, float* ml, int warp, int lane,
                                        int gr) {
    const int r = lane >> 2, q4 = lane & 3;
    float la = l_a, lb = l_b;
    la += __shfl_xor_sync(0xffffffffu, la, 1);
    la += __shfl_xor_sync(0xffffffffu, la, 2);
    lb += __shfl_xor_sync(0xffffffffu, lb, 1);
    lb += __shfl_xor_sync(0xffffffffu, lb, 2);
    float* mw = mo + warp * gr * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const int c = nt * 8 + 2 * q4;
      if (r < gr) *reinterpret_cast<float2*>(mw + r * D + c) = make_float2(o[nt][0], o[nt][1]);
      if (r + 8 < gr)
        *reinterpret_cast<float2*>(mw + (r + 8) * D + c) = make_float2(o[nt][2], o[nt][3]);
    }
    if (q4 == 0) {
      mm[warp * 16 + r] = m_a;
      mm[warp * 16 + r + 8] = m_b;
      ml[warp * 16 + r] = la;
      ml[warp * 16 + r + 8] = lb;
    }
  }
};

// The same state for groups of at most 8 heads with the MMA operands swapped:
// S^T = K Q^T puts a slice's 16 tokens on the MMA rows and the G heads on the
// n8 columns, and O^T = V^T P^T puts 16 output dims on the rows, so no MMA row
// is spent on padding (half as many MMAs and exponentials as the layout above
// at G = 8).  The K and V tiles feed the A operands through the same ldmatrix
// loads (K as stored, V transposed); P^T reaches the B layout of the second MMA
// through an in-register 8x8 transpose.  Each thread keeps heads 2 (lane % 4)
// and 2 (lane % 4) + 1: running max (shared by the 8 lanes of those heads) and
// its own part of the running sum.
template <int D>
struct WarpStateT {
  uint32_t qb[D / 16][2];  // B fragments of Q^T: dims 16kk + 2 (lane % 4) (+8), head lane / 4
  float o[D / 16][4];      // O^T tile mt: dims 16mt + lane / 4 (+8), heads 2 (lane % 4) (+1)
  float m0, m1, l0, l1;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int i = 0; i < D / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    m0 = m1 = neg_inf();
    l0 = l1 = 0.f;
  }

  __device__ __forceinline__ void load_q(const AttnArgs& a, const RowGeo& rg, int lane) {
    const int r = lane >> 2, q4 = lane & 3;
    const bool valid = r < a.G;
    const uint16_t* qh = a.q + rg.b * a.q_s0 + (int64_t)rg.t * a.q_s1 +
                         (int64_t)(rg.g * a.G + r) * a.q_s2 + 2 * q4;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qb[kk][0] = valid ? ld_b32(qh + 16 * kk) : 0u;
      qb[kk][1] = valid ? ld_b32(qh + 16 * kk + 8) : 0u;
    }
  }

  __device__ __forceinline__ void attend(const AttnArgs& a, uint8_t* smem, uint32_t sbase,
                                         uint32_t kbase, uint32_t vbase, uint32_t half_bytes,
                                         int tok, int j0, int lim, int lane, bool& wrote_smem) {
    constexpr int NH = D / 64;
    const int r = lane >> 2;
    const float ninf = neg_inf();
    if (j0 + 16 > lim) {
      // Tokens j >= lim of this slice may be uninitialised memory: zero their V rows
      // so that a zero probability never meets a non-finite value.
      const int r0 = lim - j0;
      const int per_h = (16 - r0) * 8;
      uint8_t* vrow = smem + (vbase - sbase);
      for (int x = lane; x < per_h * NH; x += 32) {
        const int hh = x / per_h, rem = x % per_h;
        const int row = tok + r0 + rem / 8;
        *reinterpret_cast<uint4*>(vrow + hh * half_bytes + row * 128 + (rem % 8) * 16) =
            make_uint4(0, 0, 0, 0);
      }
      wrote_smem = true;
      __syncwarp();
    }
    // S^T: tokens tok + r (s[0], s[1]) and tok + r + 8 (s[2], s[3]), heads 2q4, 2q4 + 1
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int mi = lane >> 3, rr = lane & 7;
      const uint32_t row = tok + (mi >> 1) * 8 + rr;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t chunk = (kk & 3) * 2 + (mi & 1);
        uint32_t k0, k1, k2, k3;  // tokens 0-7 / 8-15 x dims low / high of the k-step
        ldmatrix_x4(kbase + (kk >> 2) * half_bytes + swz128(row, chunk), k0, k1, k2, k3);
        mma_bf16_16816(s, k0, k2, k1, k3, qb[kk][0], qb[kk][1]);
      }
    }
    const bool ok_lo = j0 + r < lim, ok_hi = j0 + r + 8 < lim;
    s[0] = ok_lo ? s[0] * a.scale_log2 : ninf;
    s[1] = ok_lo ? s[1] * a.scale_log2 : ninf;
    s[2] = ok_hi ? s[2] * a.scale_log2 : ninf;
    s[3] = ok_hi ? s[3] * a.scale_log2 : ninf;
    float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
    mx0 = warp_max_xor(warp_max_xor(warp_max_xor(mx0, 4), 8), 16);
    mx1 = warp_max_xor(warp_max_xor(warp_max_xor(mx1, 4), 8), 16);
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float c0 = exp2f(m0 - mn0), c1 = exp2f(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    s[0] = exp2f(s[0] - mn0);
    s[1] = exp2f(s[1] - mn1);
    s[2] = exp2f(s[2] - mn0);
    s[3] = exp2f(s[3] - mn1);
    l0 = l0 * c0 + (s[0] + s[2]);
    l1 = l1 * c1 + (s[1] + s[3]);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      o[mt][0] *= c0;
      o[mt][1] *= c1;
      o[mt][2] *= c0;
      o[mt][3] *= c1;
    }
    // P^T as the B operand: tokens 2q4 (+1) (+8), head r
    const uint32_t pb0 = movmatrix_trans(pack_bf16(s[0], s[1]));
    const uint32_t pb1 = movmatrix_trans(pack_bf16(s[2], s[3]));
    const int mi = lane >> 3, rr = lane & 7;
    const uint32_t row = tok + (mi & 1) * 8 + rr;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const uint32_t chunk = (mt & 3) * 2 + (mi >> 1);
      uint32_t v0, v1, v2, v3;  // dims low / high x tokens 0-7 / 8-15, transposed
      ldmatrix_x4_trans(vbase + (mt >> 2) * half_bytes + swz128(row, chunk), v0, v1, v2, v3);
      mma_bf16_16816(o[mt], v0, v2, v1, v3, pb0, pb1);
    }
  }

  // Same merge-buffer layout as WarpState::stash: O rows [warp][gr][D], running
  // max and sum [warp][16].
  __device__ __forceinline__ void stash(float* mo, float* mm, float* ml, int warp, int lane,
                                        int gr) {
    const int r = lane >> 2, h0 = 2 * (lane & 3), h1 = h0 + 1;
    float s0 = l0, s1 = l1;
#pragma unroll
    for (int x = 4; x < 32; x <<= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, x);
      s1 += __shfl_xor_sync(0xffffffffu, s1, x);
    }
    float* mw = mo + warp * gr * D;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const int dd = mt * 16 + r;
      if (h0 < gr) {
        mw[h0 * D + dd] = o[mt][0];
        mw[h0 * D + dd + 8] = o[mt][2];
      }
      if (h1 < gr) {
        mw[h1 * D + dd] = o[mt][1];
        mw[h1 * D + dd + 8] = o[mt][3];
      }
    }
    if (r == 0) {
      mm[warp * 16 + h0] = m0;
      mm[warp * 16 + h1] = m1;
      ml[warp * 16 + h0] = s0;
      ml[warp * 16 + h1] = s1;
    }
  }
};

// Merge of NC warp states for tile row `row`, dims [dim, dim + 4) (dim a
// multiple of 4): normalised output and natural-log LSE (-inf and 0 when no key
// was seen).  The warps' weights are computed once for the four dims.
template <int D, int NC>
__device__ __forceinline__ void merge_warps4(const float* mo, const float* mm, const float* ml,
                                             int gr, int row, int dim, float4& val, float& lsev) {
  const float ninf = neg_inf();
  float M = ninf;
#pragma unroll
  for (int w = 0; w < NC; ++w) M = fmaxf(M, mm[w * 16 + row]);
  val = make_float4(0.f, 0.f, 0.f, 0.f);
  lsev = ninf;
  if (M == ninf) return;
  float wsum = 0.f;
  float4 acc = val;
#pragma unroll
  for (int w = 0; w < NC; ++w) {
    const float f = exp2f(mm[w * 16 + row] - M);
    wsum += f * ml[w * 16 + row];
    const float4 o = *reinterpret_cast<const float4*>(mo + (w * gr + row) * D + dim);
    acc.x += f * o.x;
    acc.y += f * o.y;
    acc.z += f * o.z;
    acc.w += f * o.w;
  }
  val = make_float4(acc.x / wsum, acc.y / wsum, acc.z / wsum, acc.w / wsum);
  lsev = (M + log2f(wsum)) * kLn2;
}

// Four consecutive bf16 outputs of head hq (one 8-byte store when aligned).
__device__ __forceinline__ void store_out4(const AttnArgs& a, const RowGeo& rg, int hq, int dim,
                                           const float4& v) {
  uint16_t* p = a.out + rg.b * a.o_s0 + (int64_t)rg.t * a.o_s1 + (int64_t)hq * a.o_s2 + dim;
  const uint32_t lo = pack_bf16(v.x, v.y), hi = pack_bf16(v.z, v.w);
  if ((reinterpret_cast<uintptr_t>(p) & 7u) == 0) {
    *reinterpret_cast<uint2*>(p) = make_uint2(lo, hi);
  } else {
    p[0] = (uint16_t)lo;
    p[1] = (uint16_t)(lo >> 16);
    p[2] = (uint16_t)hi;
    p[3] = (uint16_t)(hi >> 16);
  }
}

__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Producer: streams the K and V tiles of list entries [0, n) into the stage ring.
// Each entry is (block id in the low 16 bits, row offset in the high bits); the
// row supplies the sequence and the KV head.  Waits are bounded; before leaving,
// the producer waits for its copies still in flight.
template <int D>
__device__ __forceinline__ void produce(const AttnArgs& a, const CUtensorMap* tmk,
                                        const CUtensorMap* tmv, const int32_t* list,
                                        const int32_t* plist, const int32_t* glist, int n,
                                        uint32_t sbase, uint32_t full0, uint32_t empty0) {
  constexpr int NH = D / 64;
  const uint32_t half_bytes = (uint32_t)a.block * 128u;
  prefetch_tensormap(tmk);
  prefetch_tensormap(tmv);
  // (head, token, plane) of entry i: the head and the plane (sequence, or page of
  // a paged cache, -1 for a page outside the pool) were resolved when the list
  // was built
  auto coords = [&](int i, int& g, int& tok, int& plane) {
    const int e = list[i];
    g = glist[i];
    if (a.pg.table == nullptr) {
      tok = (e & 0xffff) * a.block;
      plane = plist[i];
    } else {
      tok = 0;
      plane = plist[i] < 0 ? (int)a.pg.pages : plist[i];
    }
  };
  int g_n = 0, tok_n = 0, plane_n = 0;
  if (n > 0) coords(0, g_n, tok_n, plane_n);
  int issued = 0;
  for (int i = 0; i < n; ++i) {
    const int g = g_n, tok = tok_n, plane = plane_n;
    if (i + 1 < n) coords(i + 1, g_n, tok_n, plane_n);
    const int s = i % a.stages;
    if (i >= a.stages &&
        !mbar_wait_bounded(empty0 + 8 * s, ((i / a.stages) - 1) & 1, a.st, 1u, a.wait_ns))
      break;
    const uint32_t full = full0 + 8 * s;
    mbar_arrive_expect_tx(full, a.stage_bytes);
    const uint32_t kdst = sbase + (uint32_t)s * a.stage_bytes;
    const uint32_t vdst = kdst + NH * half_bytes;
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      tma_load_4d(kdst + hh * half_bytes, tmk, full, hh * 64, g, tok, plane);
      tma_load_4d(vdst + hh * half_bytes, tmv, full, hh * 64, g, tok, plane);
    }
    ++issued;
  }
  for (int i = max(0, issued - a.stages); i < issued; ++i)
    mbar_wait_bounded(full0 + 8 * (i % a.stages), (i / a.stages) & 1, a.st, 2u, a.wait_ns);
}

// Compacts slots [s0, s1) of the flattened id array into the entry list: only
// blocks holding a visible token are kept.  For each kept block, glist gets its
// KV head and plist its sequence (with a paged cache: its page, looked up by the
// lanes in parallel), so that the producer's loop does no index arithmetic.  Run
// by one full warp; returns the count.
__device__ __forceinline__ int compact_ids(const AttnArgs& a, int64_t s0, int64_t s1,
                                           int64_t row0, int32_t* list, int32_t* plist,
                                           int32_t* glist, int lane) {
  constexpr int PF = 8;  // 32-slot groups whose ids are loaded together
  const unsigned lt = (1u << lane) - 1u;
  // Slot i belongs to row row0 + (i - first) / topk; the range is one CTA's
  // list (at most list_cap slots), so the offsets fit 32 bits.
  const int64_t first = row0 * a.topk;
  int ids[PF];
  auto load_ids = [&](int64_t base) {
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int64_t i = base + k * 32 + lane;
      ids[k] = i < s1 ? __ldg(a.ids + i) : -1;
    }
  };
  load_ids(s0);  // issued before the row geometry: the two loads overlap
  const int64_t span = (s1 - 1) / a.topk - row0 + 1;
  const int nrows = span < 32 ? (int)span : 32;
  // visible-token limit, head and sequence of rows row0 .. row0 + 31, one per lane
  RowGeo geo_l;
  geo_l.lim = geo_l.g = geo_l.b = 0;
  if (lane < nrows) geo_l = row_geo(a, row0 + lane);
  int n = 0;
  for (int64_t base = s0; base < s1; base += 32 * PF) {
    if (base != s0) load_ids(base);
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      if (base + k * 32 >= s1) break;
      const int64_t i = base + k * 32 + lane;
      const int beta = ids[k];
      const int rr = i < s1 ? (int)(i - first) / a.topk : 0;
      const int64_t rowg = row0 + rr;
      const int src = rr < 31 ? rr : 31;
      int lim = __shfl_sync(0xffffffffu, geo_l.lim, src);
      int g = __shfl_sync(0xffffffffu, geo_l.g, src);
      int b = __shfl_sync(0xffffffffu, geo_l.b, src);
      if (rr >= 32) {
        const RowGeo gr = row_geo(a, rowg);
        lim = gr.lim;
        g = gr.g;
        b = gr.b;
      }
      const bool bad = beta >= a.nblk;
      if (bad) record_error(a.st, kErrDeviceAssert, (uint32_t)rowg);
      const bool keep = beta >= 0 && !bad && (int64_t)beta * a.block < lim;
      const unsigned msk = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int at = n + __popc(msk & lt);
        list[at] = beta | (rr << 16);
        glist[at] = g;
        plist[at] = a.pg.table != nullptr ? (int)kv_page(a.pg, b, beta, a.st) : b;
      }
      n += __popc(msk);
    }
  }
  return n;
}

// ------------------------------------------------------- one CTA per row
template <int D>
__global__ void __launch_bounds__(5 * 32, 1)
    sparse_attn_rows_kernel(const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, AttnArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int NC = 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.region_bytes);
  int32_t* list = reinterpret_cast<int32_t*>(bars + 2 * a.stages);
  int32_t* n_list = list + a.list_cap;
  int32_t* plist = n_list + 1;       // [list_cap] sequence or page of each entry
  int32_t* glist = plist + a.list_cap;  // [list_cap] KV head of each entry
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t rowg = blockIdx.x;
  const int nsub = a.block / 16;
  const uint32_t half_bytes = (uint32_t)a.block * 128u;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, min(NC, nsub));
    }
    fence_mbar_init();
  }
  // the consumers load their queries while the list is built
  WarpState<D> ws;
  const RowGeo rg = row_geo(a, rowg);
  if (warp == NC) {
    // after an earlier timeout the kernel does nothing (status read first: its
    // latency overlaps the compaction)
    const bool skip = status_failed(a.st);
    const int n = compact_ids(a, rowg * a.topk, (rowg + 1) * a.topk, rowg, list, plist, glist, lane);
    if (lane == 0) *n_list = skip ? -1 : n;
  } else {
    ws.reset();
    ws.load_q(a, rg, lane);
  }
  __syncthreads();
  const int n = *n_list;
  if (n < 0) return;
  if (warp == NC) {
    if (lane == 0 && n > 0) produce<D>(a, &tmk, &tmv, list, plist, glist, n, sbase, full0, empty0);
    return;
  }
  for (int i = 0; i < n; ++i) {
    const int u0 = i * nsub;
    const int st0 = (warp - (u0 % NC) + NC) % NC;  // first slice of block i owned by this warp
    if (st0 >= nsub) continue;
    const int s = i % a.stages;
    if (!mbar_wait_warp(full0 + 8 * s, (i / a.stages) & 1, a.st, 3u, a.wait_ns)) break;
    const uint32_t kbase = sbase + (uint32_t)s * a.stage_bytes;
    const uint32_t vbase = kbase + (D / 64) * half_bytes;
    const int beta = list[i] & 0xffff;
    bool wrote = false;
    for (int st = st0; st < nsub; st += NC) {
      const int j0 = beta * a.block + st * 16;
      if (j0 < rg.lim) ws.attend(a, smem, sbase, kbase, vbase, half_bytes, st * 16, j0, rg.lim, lane, wrote);
    }
    if (wrote) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
  }
  // Merge the warps' states (the stages are free: every load was consumed).
  consumer_sync(NC * 32);
  float* mo = reinterpret_cast<float*>(smem);
  float* mm = mo + NC * a.G * D;
  float* ml = mm + NC * 16;
  ws.stash(mo, mm, ml, warp, lane, a.G);
  consumer_sync(NC * 32);
  for (int x = tid; x < a.G * (D / 4); x += NC * 32) {
    const int row = x / (D / 4), dim = (x % (D / 4)) * 4;
    float4 val;
    float lsev;
    merge_warps4<D, NC>(mo, mm, ml, a.G, row, dim, val, lsev);
    const int hq = rg.g * a.G + row;
    store_out4(a, rg, hq, dim, val);
    if (dim == 0 && a.lse) a.lse[(int64_t)rg.bt * a.H + hq] = lsev;
  }
}

// ----------------------------------------- persistent, balanced streaming
template <int D, int NC, class WS>
__global__ void __launch_bounds__((NC + 1) * 32, 1)
    sparse_attn_stream_kernel(const __grid_constant__ CUtensorMap tmk,
                              const __grid_constant__ CUtensorMap tmv, AttnArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* mo = reinterpret_cast<float*>(smem + a.merge_off);  // [NC][G][D]
  float* mm = mo + NC * a.G * D;                              // [NC][16]
  float* ml = mm + NC * 16;                                   // [NC][16]
  int* flag = reinterpret_cast<int*>(ml + NC * 16);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.region_bytes);
  int32_t* list = reinterpret_cast<int32_t*>(bars + 2 * a.stages);
  int32_t* n_list = list + a.list_cap;
  int32_t* plist = n_list + 1;       // [list_cap] sequence or page of each entry
  int32_t* glist = plist + a.list_cap;  // [list_cap] KV head of each entry
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nsub = a.block / 16;
  const uint32_t half_bytes = (uint32_t)a.block * 128u;
  const int64_t c = blockIdx.x;
  const int64_t s0 = c * a.per;
  const int64_t s1 = min(s0 + a.per, a.total_slots);
  if (s0 >= s1) return;
  const int64_t r0 = s0 / a.topk, r1 = (s1 - 1) / a.topk;

  if (warp == NC) {
    // The producer warp sets up the stage barriers, builds the list and starts
    // streaming at once; the arrive on barrier 2 publishes both to the consumers.
    // After an earlier timeout the kernel does nothing; the status load is issued
    // first so that its latency overlaps the compaction.
    if (lane == 0) {
      for (int s = 0; s < a.stages; ++s) {
        mbar_init(full0 + 8 * s, 1);
        mbar_init(empty0 + 8 * s, min(NC, nsub));
      }
      fence_mbar_init();
    }
    const bool skip = status_failed(a.st);
    const int n = compact_ids(a, s0, s1, r0, list, plist, glist, lane);
    if (lane == 0) *n_list = skip ? -1 : n;
    __syncwarp();
    named_arrive(2, (NC + 1) * 32);
    if (lane == 0 && !skip && n > 0)
      produce<D>(a, &tmk, &tmv, list, plist, glist, n, sbase, full0, empty0);
    return;
  }
  // the consumers load their first row's queries while the list is built
  WS ws;
  int64_t cur = r0;
  RowGeo rg = row_geo(a, cur);
  ws.reset();
  ws.load_q(a, rg, lane);
  named_sync(2, (NC + 1) * 32);
  const int n = *n_list;
  if (n < 0) return;
  bool failed = false;

  // Ends the segment of row `cur` held by this CTA: merge the warps, then write
  // the output (row entirely in this CTA) or a partial (and merge the row's
  // partials if this CTA is the last of the row to finish).
  //
  // A row's first CTA reaches it at the end of its range, while the row's other
  // CTAs start their ranges with it, so their partials are usually published
  // long before.  The first CTA reads the row's counter as it arrives: if every
  // other segment is in, it merges them straight into its own state (its own
  // partial is never written, and no atomic is taken; no other CTA can then be
  // the last, since the count never reaches nseg).  Otherwise it publishes like
  // the others.
  auto flush = [&]() {
    const int64_t c_first = (cur * a.topk) / a.per;
    const int64_t c_last = ((cur + 1) * a.topk - 1) / a.per;
    const int nseg = (int)(c_last - c_first + 1);
    const int seg = (int)(c - c_first);
    const bool first = nseg > 1 && seg == 0;
    if (first && tid == 0) {
      *flag = ld_acquire_gpu(a.counters + cur);
      __threadfence();
    }
    ws.stash(mo, mm, ml, warp, lane, a.G);
    consumer_sync(NC * 32);
    const bool fast = first && *flag == nseg - 1;
    for (int x = tid; x < a.G * (D / 4); x += NC * 32) {
      const int row = x / (D / 4), dim = (x % (D / 4)) * 4;
      const int hq = rg.g * a.G + row;
      const int64_t pr0 = ((int64_t)rg.bt * a.H + hq) * a.smax;
      // the second segment's partial, loaded before the warps' merge
      float l1 = neg_inf();
      float4 o1 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (fast) {
        l1 = __ldcg(a.part_lse + pr0 + 1);
        o1 = __ldcg(reinterpret_cast<const float4*>(a.part_o + (pr0 + 1) * D + dim));
      }
      float4 val;
      float lsev;
      merge_warps4<D, NC>(mo, mm, ml, a.G, row, dim, val, lsev);
      if (fast) {
        // the same operations in the same order as the last CTA's merge below,
        // so that the result does not depend on which of the two ran
        const float ninf = neg_inf();
        float M = fmaxf(fmaxf(ninf, lsev), l1);
        for (int sp = 2; sp < nseg; ++sp) M = fmaxf(M, __ldcg(a.part_lse + pr0 + sp));
        float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
        float lres = ninf;
        if (M != ninf) {
          float den = 0.f;
          float4 acc = res;
          auto add = [&](float l, const float4& o) {
            const float w = exp2f((l - M) * kLog2e);
            den += w;
            acc.x += w * o.x;
            acc.y += w * o.y;
            acc.z += w * o.z;
            acc.w += w * o.w;
          };
          add(lsev, val);
          add(l1, o1);
          for (int sp = 2; sp < nseg; ++sp)
            add(__ldcg(a.part_lse + pr0 + sp),
                __ldcg(reinterpret_cast<const float4*>(a.part_o + (pr0 + sp) * D + dim)));
          res = make_float4(acc.x / den, acc.y / den, acc.z / den, acc.w / den);
          lres = M + log2f(den) * kLn2;
        }
        val = res;
        lsev = lres;
      }
      if (nseg == 1 || fast) {
        store_out4(a, rg, hq, dim, val);
        if (dim == 0 && a.lse) a.lse[(int64_t)rg.bt * a.H + hq] = lsev;
      } else {
        const int64_t pr = pr0 + seg;
        *reinterpret_cast<float4*>(a.part_o + pr * D + dim) = val;
        if (dim == 0) a.part_lse[pr] = lsev;
      }
    }
    if (nseg > 1 && !fast) {
      // One thread publishes the CTA's partial (its stores ordered before the
      // fence by the barrier) and learns whether it is the row's last; its
      // second fence orders the other CTAs' partials before the loads below.
      consumer_sync(NC * 32);
      if (tid == 0) {
        __threadfence();
        const int f = atomicAdd(&a.counters[cur], 1);
        __threadfence();
        *flag = f;
      }
      consumer_sync(NC * 32);
      if (*flag == nseg - 1 && nseg <= NC) {
        // Last CTA of the row: stage the row's partials in the (now free) merge
        // buffer with independent loads, then merge them from shared memory.
        float* so = mo;              // [G][nseg][D]
        float* sl = mo + NC * a.G * D;  // [G][nseg], over the free max/sum arrays
        const int64_t pr_g = ((int64_t)rg.bt * a.H + rg.g * a.G) * a.smax;
        const int q4n = nseg * (D / 4);
#pragma unroll 4
        for (int y = tid; y < a.G * q4n; y += NC * 32) {
          const int row = y / q4n, sp = (y % q4n) / (D / 4), c4 = y % (D / 4);
          const float4 v = __ldcg(reinterpret_cast<const float4*>(
                                      a.part_o + (pr_g + (int64_t)row * a.smax + sp) * D) +
                                  c4);
          reinterpret_cast<float4*>(so)[(row * nseg + sp) * (D / 4) + c4] = v;
        }
        for (int y = tid; y < a.G * nseg; y += NC * 32)
          sl[y] = __ldcg(a.part_lse + pr_g + (int64_t)(y / nseg) * a.smax + y % nseg);
        consumer_sync(NC * 32);
        for (int x = tid; x < a.G * (D / 4); x += NC * 32) {
          const int row = x / (D / 4), dim = (x % (D / 4)) * 4;
          const int hq = rg.g * a.G + row;
          const float ninf = neg_inf();
          float M = ninf;
          for (int sp = 0; sp < nseg; ++sp) M = fmaxf(M, sl[row * nseg + sp]);
          float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
          float lsev = ninf;
          if (M != ninf) {
            float den = 0.f;
            float4 acc = val;
            for (int sp = 0; sp < nseg; ++sp) {
              const float w = exp2f((sl[row * nseg + sp] - M) * kLog2e);
              den += w;
              const float4 o = *reinterpret_cast<const float4*>(so + (row * nseg + sp) * D + dim);
              acc.x += w * o.x;
              acc.y += w * o.y;
              acc.z += w * o.z;
              acc.w += w * o.w;
            }
            val = make_float4(acc.x / den, acc.y / den, acc.z / den, acc.w / den);
            lsev = M + log2f(den) * kLn2;
          }
          store_out4(a, rg, hq, dim, val);
          if (dim == 0 && a.lse) a.lse[(int64_t)rg.bt * a.H + hq] = lsev;
        }
      } else if (*flag == nseg - 1) {
        // more segments than the merge buffer holds: merge from global memory
        for (int x = tid; x < a.G * D; x += NC * 32) {
          const int row = x / D, dim = x % D;
          const int hq = rg.g * a.G + row;
          const int64_t pr0 = ((int64_t)rg.bt * a.H + hq) * a.smax;
          const float ninf = neg_inf();
          float M = ninf;
          for (int sp = 0; sp < nseg; ++sp) M = fmaxf(M, __ldcg(a.part_lse + pr0 + sp));
          float val = 0.f, lsev = ninf;
          if (M != ninf) {
            float den = 0.f, acc = 0.f;
            for (int sp = 0; sp < nseg; ++sp) {
              const float w = exp2f((__ldcg(a.part_lse + pr0 + sp) - M) * kLog2e);
              den += w;
              acc += w * __ldcg(a.part_o + (pr0 + sp) * D + dim);
            }
            val = acc / den;
            lsev = M + log2f(den) * kLn2;
          }
          a.out[rg.b * a.o_s0 + (int64_t)rg.t * a.o_s1 + (int64_t)hq * a.o_s2 + dim] =
              __bfloat16_as_ushort(__float2bfloat16_rn(val));
          if (dim == 0 && a.lse) a.lse[(int64_t)rg.bt * a.H + hq] = lsev;
        }
      }
    }
    // the row's merge is done: its counter goes back to zero for the next call
    if (nseg > 1 && tid == 0 && *flag == nseg - 1) a.counters[cur] = 0;
    consumer_sync(NC * 32);  // the merge buffer is free again
  };

  for (int i = 0; i < n; ++i) {
    const int e = list[i];
    const int64_t row = r0 + (e >> 16);
    while (cur < row) {
      flush();
      ++cur;
      rg = row_geo(a, cur);
      ws.reset();
      ws.load_q(a, rg, lane);
    }
    const int u0 = i * nsub;
    const int st0 = (warp - (u0 % NC) + NC) % NC;
    if (st0 >= nsub || failed) continue;
    const int s = i % a.stages;
    // After a wait runs out this warp stops computing but keeps walking the list,
    // so that every consumer warp still reaches the same row-boundary barriers.
    if (!mbar_wait_warp(full0 + 8 * s, (i / a.stages) & 1, a.st, 3u, a.wait_ns)) {
      failed = true;
      continue;
    }
    const uint32_t kbase = sbase + (uint32_t)s * a.stage_bytes;
    const uint32_t vbase = kbase + (D / 64) * half_bytes;
    const int beta = e & 0xffff;
    bool wrote = false;
    for (int st = st0; st < nsub; st += NC) {
      const int j0 = beta * a.block + st * 16;
      if (j0 < rg.lim) ws.attend(a, smem, sbase, kbase, vbase, half_bytes, st * 16, j0, rg.lim, lane, wrote);
    }
    if (wrote) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
  }
  while (true) {
    flush();
    if (cur >= r1) break;
    ++cur;
    rg = row_geo(a, cur);
    ws.reset();
  }
}

// ------------------------------------------------------------ host helpers
// K or V as a 4-D tensor [batch][token][kv head][dim], or for a paged cache
// [page][token in page][kv head][dim]; one box is 64 dims x 1 head x `block`
// tokens (128 bytes per row, 128-byte swizzle).
bool make_kv_map(CUtensorMap* map, const uint16_t* base, const Shape& s, const int64_t* str) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const bool paged = s.pages.table != nullptr;
  cuuint64_t dims[4] = {(cuuint64_t)s.d, (cuuint64_t)s.h,
                        (cuuint64_t)(paged ? s.block : s.max_kv),
                        (cuuint64_t)(paged ? s.pages.pages : s.batch)};
  cuuint64_t strides[3] = {(cuuint64_t)str[2] * 2, (cuuint64_t)str[1] * 2,
                           (cuuint64_t)str[0] * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)s.block, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(base), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Q as a 4-D tensor [batch][token][head][dim]; one box is 64 dims x the G heads
// of a group x 1 token, i.e. G rows of 128 bytes (128-byte swizzle).
bool make_q_group_map(CUtensorMap* map, const uint16_t* base, const Shape& s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)s.d, (cuuint64_t)s.H, (cuuint64_t)s.n_q, (cuuint64_t)s.batch};
  cuuint64_t strides[3] = {(cuuint64_t)s.q_s[2] * 2, (cuuint64_t)s.q_s[1] * 2,
                           (cuuint64_t)s.q_s[0] * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)s.G, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(base), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

constexpr int kStreamNC = 8;       // consumer warps of the streaming kernel
constexpr int kMaxList = 4096;     // entries a streaming CTA compacts up front
constexpr uint32_t kSmemCap = 227u * 1024u;

struct AttnPlan {
  bool stream;
  int stages, ctas, per, smax, list_cap;
  int64_t total;
  uint32_t stage_bytes, region_bytes, merge_off;
  size_t smem_bytes;
};

// Stage count that keeps every block of a stage on the same warps (a warp waits
// only on the stages of blocks it processes): with fewer 16-token slices per
// block than consumer warps, a multiple of the warp cycle.
int stage_count(int want, int nsub, int nc) {
  const int cycle = nsub >= nc ? 1 : nc / nsub;
  want = max(2, min(8, want));
  return max(cycle, want - want % cycle);
}

AttnPlan plan_attn(const Shape& s) {
  AttnPlan pl;
  pl.stage_bytes = 4u * s.d * s.block;  // K and V tiles of one block, bf16
  const int nsub = s.block / 16;
  const int64_t rows_g = (int64_t)s.batch * s.n_q * s.h;
  pl.total = rows_g * s.topk;
  // merge buffer: O [warps][G][d], max and sum [warps][16], one flag word
  const uint32_t merge_bytes =
      (uint32_t)kStreamNC * s.G * s.d * 4 + (uint32_t)kStreamNC * 16 * 2 * 4 + 16;
  // Few rows with many blocks (decode): the persistent streaming kernel.
  pl.stream = rows_g < 4LL * num_sms();
  if (pl.stream) {
    pl.ctas = num_sms();
    pl.per = (int)((pl.total + pl.ctas - 1) / pl.ctas);
    if (pl.per > kMaxList) {
      pl.per = kMaxList;
      pl.ctas = (int)((pl.total + kMaxList - 1) / kMaxList);
    }
    pl.ctas = (int)((pl.total + pl.per - 1) / pl.per);
    pl.smax = (s.topk - 1) / pl.per + 2;
    pl.list_cap = pl.per;
    // as many stages as the shared memory holds: the bytes in flight per SM set
    // the streaming rate
    const size_t merge_r = (merge_bytes + 1023) & ~1023u;
    const size_t fixed = 1024 + merge_r + 4 * (3 * (size_t)pl.list_cap + 1);
    const size_t cap = (size_t)max_smem_optin();
    const int fit = cap > fixed ? (int)((cap - fixed) / (pl.stage_bytes + 16)) : 0;
    pl.stages = stage_count(fit, nsub, kStreamNC);  // fit >= 3 for every supported shape
    pl.region_bytes = pl.stages * pl.stage_bytes + merge_r;
    pl.merge_off = pl.stages * pl.stage_bytes;
  } else {
    // Two CTAs per SM when the stages allow it, else one with deeper buffering.
    int want = (int)((100u * 1024u) / pl.stage_bytes);
    if (want < 2) want = min(4, (int)((200u * 1024u) / pl.stage_bytes));
    pl.stages = stage_count(want, nsub, 4);
    pl.region_bytes = max(pl.stages * pl.stage_bytes, merge_bytes);
    pl.merge_off = 0;
    pl.ctas = (int)rows_g;
    pl.per = s.topk;
    pl.smax = 1;
    pl.list_cap = s.topk;
  }
  pl.smem_bytes = 1024 + pl.region_bytes + 16 * pl.stages + 4 * (3 * (size_t)pl.list_cap + 1);
  return pl;
}

}  // namespace

bool make_rows_map(CUtensorMap* map, uint16_t* base, int64_t rows, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_partial_bytes(const Shape& s) {
  const AttnPlan pl = plan_attn(s);
  if (!pl.stream) return kv_attn_supported(s) ? kv_workspace_bytes(s) : 0;
  const size_t n = (size_t)s.batch * s.n_q * s.H * pl.smax;
  const size_t rows_g = (size_t)s.batch * s.n_q * s.h;
  return n * (size_t)(s.d + 1) * sizeof(float) + rows_g * sizeof(int) + 512;
}

int attn_launches(const Shape& s) {
  const AttnPlan pl = plan_attn(s);
  return !pl.stream && kv_attn_supported(s) ? kv_launches(s) : 1;
}

int* attn_merge_counters(const Shape& s, void* partials, int* count) {
  const AttnPlan pl = plan_attn(s);
  *count = 0;
  if (!pl.stream || partials == nullptr) return nullptr;
  const size_t nrow_h = (size_t)s.batch * s.n_q * s.H;
  const float* part_lse = reinterpret_cast<float*>(partials) + nrow_h * pl.smax * s.d;
  *count = s.batch * s.n_q * s.h;
  return reinterpret_cast<int*>(
      (reinterpret_cast<uintptr_t>(part_lse + nrow_h * pl.smax) + 255) & ~uintptr_t(255));
}

cudaError_t launch_sparse_attn(const Shape& s, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const int32_t* ids, uint16_t* out, float* lse,
                               void* partials, size_t partial_bytes, DeviceStatus* st,
                               cudaStream_t stream, bool counters_zeroed, int* fixed_counters) {
  const AttnPlan pl = plan_attn(s);
  if (pl.smem_bytes > kSmemCap) return cudaErrorInvalidValue;
  CUtensorMap tmk, tmv;
  if (!make_kv_map(&tmk, k, s, s.k_s) || !make_kv_map(&tmv, v, s, s.v_s))
    return cudaErrorInvalidValue;
  AttnArgs a;
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
  a.block = s.block;
  a.nblk = s.nblk;
  a.causal = s.causal;
  a.scale_log2 = s.scale * kLog2e;
  a.stages = pl.stages;
  a.stage_bytes = pl.stage_bytes;
  a.region_bytes = pl.region_bytes;
  a.merge_off = pl.merge_off;
  a.list_cap = pl.list_cap;
  a.total_slots = pl.total;
  a.per = pl.per;
  a.smax = pl.smax;
  a.part_o = nullptr;
  a.part_lse = nullptr;
  a.counters = nullptr;
  a.out = out;
  a.o_s0 = s.o_s[0];
  a.o_s1 = s.o_s[1];
  a.o_s2 = s.o_s[2];
  a.lse = lse;
  a.st = st;
  a.wait_ns = 4000000000ull;  // 4 s: far above any healthy wait, even under a profiler
  a.pg = s.pages;
  cudaError_t err;
  if (!pl.stream && kv_attn_supported(s)) {
    CUtensorMap tmq;
    if (!make_q_group_map(&tmq, q, s)) return cudaErrorInvalidValue;
    return launch_kv_attn(s, tmq, tmk, tmv, q, ids, out, lse, partials, partial_bytes, st, stream);
  }
  if (!pl.stream) {
    const dim3 grid((unsigned)pl.ctas);
    if (s.d == 128) {
      err = cudaFuncSetAttribute(sparse_attn_rows_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem_bytes);
      if (err != cudaSuccess) return err;
      err = launch_pdl(sparse_attn_rows_kernel<128>, grid, dim3(5 * 32), pl.smem_bytes, stream, tmk,
                       tmv, a);
    } else {
      err = cudaFuncSetAttribute(sparse_attn_rows_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem_bytes);
      if (err != cudaSuccess) return err;
      err = launch_pdl(sparse_attn_rows_kernel<64>, grid, dim3(5 * 32), pl.smem_bytes, stream, tmk,
                       tmv, a);
    }
    return err;
  }
  const size_t nrow_h = (size_t)s.batch * s.n_q * s.H;
  if (partials == nullptr || partial_bytes < attn_partial_bytes(s)) return cudaErrorInvalidValue;
  a.part_o = reinterpret_cast<float*>(partials);
  a.part_lse = a.part_o + nrow_h * pl.smax * s.d;
  int ncounters = 0;
  a.counters = attn_merge_counters(s, partials, &ncounters);
  if (fixed_counters != nullptr && ncounters <= kFixedCounters) {
    a.counters = fixed_counters;  // zero already, and left at zero
  } else if (!counters_zeroed) {
    err = cudaMemsetAsync(a.counters, 0, (size_t)ncounters * sizeof(int), stream);
    if (err != cudaSuccess) return err;
  }
  const dim3 grid((unsigned)pl.ctas);
  constexpr int NT = (kStreamNC + 1) * 32;
  auto run = [&](auto kernel) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)pl.smem_bytes);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, dim3(NT), pl.smem_bytes, stream, tmk, tmv, a);
  };
  // groups of up to 8 heads take the swapped MMA operands
  if (s.d == 128)
    return s.G <= 8 ? run(sparse_attn_stream_kernel<128, kStreamNC, WarpStateT<128>>)
                    : run(sparse_attn_stream_kernel<128, kStreamNC, WarpState<128>>);
  return s.G <= 8 ? run(sparse_attn_stream_kernel<64, kStreamNC, WarpStateT<64>>)
                  : run(sparse_attn_stream_kernel<64, kStreamNC, WarpState<64>>);
}

}  // namespace msa
