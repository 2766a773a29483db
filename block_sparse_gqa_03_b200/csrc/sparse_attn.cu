// Sparse branch: exact softmax attention over the selected KV blocks.
//
// "MiniMax goes sparse" (atlascloud.ai), section 1, step 2: with the block ids of
// step 1, the matching block subsets are taken from the raw K/V and ordinary
// softmax attention runs over them; all query heads of a GQA group share the
// group's top-k selection, so one load of a block serves the whole group
// ("MiniMax M3 的 MSA ...", second layer).
//
// Kernel design (one CTA per (query, group, KV split)):
//  * warp 4 is the producer: one lane streams the selected blocks' K and V tiles
//    into a ring of shared-memory stages with TMA (4-D tensor maps over
//    [batch, token, kv head, dim], 128-byte swizzle), completion tracked by
//    mbarriers (bounded waits: a wait that runs out records an error and the
//    kernel returns, it never hangs);
//  * warps 0-3 consume: the group's G query heads are the 16 rows of a bf16
//    tensor-core MMA tile (rows >= G are zero), S = Q K^T and O += P V run on
//    m16n8k16 MMAs fed by ldmatrix from the swizzled tiles, with an fp32 online
//    softmax in the exp2 domain.  Each warp takes 16-token slices of the blocks in
//    turn and keeps its own running max / sum / output; the four are merged at
//    the end through shared memory;
//  * with one split the CTA writes bf16 output and the log-sum-exp; with several
//    (decode, where a row has few queries but many blocks) it writes fp32
//    partials that a combine kernel merges by log-sum-exp weights.
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
  int splits, chunk, stages;
  uint32_t stage_bytes, region_bytes;
  uint16_t* out;
  int64_t o_s0, o_s1, o_s2;
  float* lse;
  float* part_o;
  float* part_lse;
  DeviceStatus* st;
  uint64_t wait_ns;
};

constexpr int kConsumerWarps = 4;
constexpr int kAttnThreads = (kConsumerWarps + 1) * 32;

__device__ __forceinline__ uint32_t ld_b32(const uint16_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.region_bytes);
  int32_t* list = reinterpret_cast<int32_t*>(bars + 2 * a.stages);
  int32_t* n_list = list + a.chunk;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + a.stages);

  // After a timed-out wait anywhere in this launch, the remaining CTAs stop early.
  if (status_failed(a.st)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rowg = blockIdx.x;  // ((b * n_q) + t) * h + g
  const int g = rowg % a.h;
  const int bt = rowg / a.h;
  const int t = bt % a.n_q, b = bt / a.n_q;
  const int split = blockIdx.y;
  const int BLK = a.block;
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int p = L - a.n_q + t;
  const int lim = a.causal ? min(L, p + 1) : L;  // visible tokens: j < lim
  const int nsub = BLK / 16;
  const uint32_t half_bytes = (uint32_t)BLK * 128u;
  constexpr int NH = D / 64;  // 128-byte halves of a row

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, min(kConsumerWarps, nsub));
    }
    fence_mbar_init();
  }
  if (warp == kConsumerWarps) {
    // Compact this split's slots into the list of blocks that hold a visible token.
    const int s0 = split * a.chunk, s1 = min(a.topk, s0 + a.chunk);
    const int32_t* row_ids = a.ids + (int64_t)rowg * a.topk;
    const unsigned lt = (1u << lane) - 1u;
    int n = 0;
    for (int base = s0; base < s1; base += 32) {
      const int i = base + lane;
      const int beta = i < s1 ? row_ids[i] : -1;
      const bool bad = beta >= a.nblk;
      if (bad) record_error(a.st, kErrDeviceAssert, (uint32_t)rowg);
      const bool keep = beta >= 0 && !bad && (int64_t)beta * BLK < lim;
      const unsigned msk = __ballot_sync(0xffffffffu, keep);
      if (keep) list[n + __popc(msk & lt)] = beta;
      n += __popc(msk);
    }
    if (lane == 0) *n_list = n;
  }
  __syncthreads();
  const int n = *n_list;

  if (warp == kConsumerWarps) {
    if (lane == 0 && n > 0) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int s = i % a.stages;
        if (i >= a.stages &&
            !mbar_wait_bounded(empty0 + 8 * s, ((i / a.stages) - 1) & 1, a.st, 1u, a.wait_ns))
          break;
        const uint32_t full = full0 + 8 * s;
        mbar_arrive_expect_tx(full, a.stage_bytes);
        const uint32_t kdst = sbase + (uint32_t)s * a.stage_bytes;
        const uint32_t vdst = kdst + NH * half_bytes;
        const int tok = list[i] * BLK;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          tma_load_4d(kdst + hh * half_bytes, &tmk, full, hh * 64, g, tok, b);
          tma_load_4d(vdst + hh * half_bytes, &tmv, full, hh * 64, g, tok, b);
        }
        ++issued;
      }
      // Drain: make sure no copy into this CTA's shared memory is in flight at exit.
      for (int i = max(0, issued - a.stages); i < issued; ++i)
        mbar_wait_bounded(full0 + 8 * (i % a.stages), (i / a.stages) & 1, a.st, 2u, a.wait_ns);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int r = lane >> 2, q4 = lane & 3;
  const float ninf = -__int_as_float(0x7f800000);
  uint32_t qa[D / 16][4];
  {
    const bool vlo = r < a.G, vhi = r + 8 < a.G;
    const uint16_t* qb = a.q + b * a.q_s0 + (int64_t)t * a.q_s1 + (int64_t)(g * a.G) * a.q_s2 + 2 * q4;
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
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = ninf, m_b = ninf, l_a = 0.f, l_b = 0.f;

  for (int i = 0; i < n; ++i) {
    const int u0 = i * nsub;
    const int st0 = (warp - (u0 & 3) + 4) & 3;  // first slice of block i owned by this warp
    if (st0 >= nsub) continue;
    const int s = i % a.stages;
    if (!mbar_wait_bounded(full0 + 8 * s, (i / a.stages) & 1, a.st, 3u, a.wait_ns)) break;
    const uint32_t kbase = sbase + (uint32_t)s * a.stage_bytes;
    const uint32_t vbase = kbase + NH * half_bytes;
    const int beta = list[i];
    bool wrote_smem = false;
    for (int st = st0; st < nsub; st += kConsumerWarps) {
      const int j0 = beta * BLK + st * 16;
      if (j0 >= lim) continue;
      const int tok = st * 16;
      if (j0 + 16 > lim) {
        // Tokens j >= lim of this slice may be uninitialised memory: zero their V rows.
        const int r0 = lim - j0;
        const int cnt = (16 - r0) * 8 * NH;
        uint8_t* vrow = smem + (vbase - sbase);
        for (int x = lane; x < cnt; x += 32) {
          const int hh = x / ((16 - r0) * 8);
          const int rem = x % ((16 - r0) * 8);
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
      {
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
    }
    if (wrote_smem) fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
  }
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

  // ------------------------------------------- merge the four warps' states
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  float* mo = reinterpret_cast<float*>(smem);           // [4][16][D]
  float* mm = mo + kConsumerWarps * 16 * D;              // [4][16]
  float* ml = mm + kConsumerWarps * 16;                  // [4][16]
  {
    float* mw = mo + warp * 16 * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const int c = nt * 8 + 2 * q4;
      mw[r * D + c] = o[nt][0];
      mw[r * D + c + 1] = o[nt][1];
      mw[(r + 8) * D + c] = o[nt][2];
      mw[(r + 8) * D + c + 1] = o[nt][3];
    }
    if (q4 == 0) {
      mm[warp * 16 + r] = m_a;
      mm[warp * 16 + r + 8] = m_b;
      ml[warp * 16 + r] = l_a;
      ml[warp * 16 + r + 8] = l_b;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  const float kLn2 = 0.69314718055994531f;
  for (int x = tid; x < a.G * D; x += kConsumerWarps * 32) {
    const int row = x / D, dim = x % D;
    float M = ninf;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mm[w * 16 + row]);
    float val = 0.f, lsev = ninf;
    if (M != ninf) {
      float wsum = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float f = exp2f(mm[w * 16 + row] - M);
        wsum += f * ml[w * 16 + row];
        acc += f * mo[(w * 16 + row) * D + dim];
      }
      val = acc / wsum;
      lsev = (M + log2f(wsum)) * kLn2;
    }
    const int hq = g * a.G + row;
    if (a.splits == 1) {
      a.out[b * a.o_s0 + (int64_t)t * a.o_s1 + (int64_t)hq * a.o_s2 + dim] =
          __bfloat16_as_ushort(__float2bfloat16_rn(val));
      if (dim == 0 && a.lse) a.lse[(int64_t)bt * a.H + hq] = lsev;
    } else {
      const int64_t pr = ((int64_t)bt * a.H + hq) * a.splits + split;
      a.part_o[pr * D + dim] = val;
      if (dim == 0) a.part_lse[pr] = lsev;
    }
  }
}

// Log-sum-exp merge of the split partials of one (query, head) per CTA.
__global__ void __launch_bounds__(128) combine_kernel(const float* part_o, const float* part_lse,
                                                      int splits, int D, int H, int n_q,
                                                      uint16_t* out, int64_t o_s0, int64_t o_s1,
                                                      int64_t o_s2, float* lse) {
  const int64_t rh = blockIdx.x;  // bt * H + hq
  const int hq = (int)(rh % H);
  const int64_t bt = rh / H;
  const int t = (int)(bt % n_q);
  const int64_t b = bt / n_q;
  const float* pl = part_lse + rh * splits;
  const float ninf = -__int_as_float(0x7f800000);
  float M = ninf;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, pl[s]);
  for (int dim = threadIdx.x; dim < D; dim += blockDim.x) {
    float val = 0.f;
    if (M != ninf) {
      float den = 0.f, acc = 0.f;
      for (int s = 0; s < splits; ++s) {
        const float w = __expf(pl[s] - M);
        den += w;
        acc += w * part_o[(rh * splits + s) * D + dim];
      }
      val = acc / den;
    }
    out[b * o_s0 + t * o_s1 + hq * o_s2 + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
  }
  if (threadIdx.x == 0 && lse) {
    float l = ninf;
    if (M != ninf) {
      float den = 0.f;
      for (int s = 0; s < splits; ++s) den += __expf(pl[s] - M);
      l = M + __logf(den);
    }
    lse[rh] = l;
  }
}

// ------------------------------------------------------------ host helpers
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

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

// K or V as a 4-D tensor [batch][token][kv head][dim]; one box is 64 dims x 1
// head x `block` tokens (128 bytes per row, 128-byte swizzle).
bool make_kv_map(CUtensorMap* map, const uint16_t* base, const Shape& s, const int64_t* str) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)s.d, (cuuint64_t)s.h, (cuuint64_t)s.max_kv,
                        (cuuint64_t)s.batch};
  cuuint64_t strides[3] = {(cuuint64_t)str[2] * 2, (cuuint64_t)str[1] * 2,
                           (cuuint64_t)str[0] * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)s.block, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(base), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

struct AttnPlan {
  int splits, chunk, stages;
  uint32_t stage_bytes, region_bytes;
  size_t smem_bytes;
};

AttnPlan plan_attn(const Shape& s) {
  AttnPlan pl;
  pl.stage_bytes = 4u * s.d * s.block;  // K and V tiles of one block, bf16
  // Two CTAs per SM when the stages allow it, otherwise one with deeper buffering.
  int stages = (int)((100u * 1024u) / pl.stage_bytes);
  if (stages < 2) stages = min(4, (int)((200u * 1024u) / pl.stage_bytes));
  stages = max(2, min(8, stages));
  // A warp waits only on the stages of the blocks it processes, so every block
  // that lands in a given stage must be processed by the same warps: with fewer
  // than four 16-token slices per block, the stage count is a multiple of the
  // warp cycle (4 / slices).
  const int nsub = s.block / 16;
  const int cycle = nsub >= kConsumerWarps ? 1 : kConsumerWarps / nsub;
  stages = max(cycle, stages - stages % cycle);
  pl.stages = stages;
  const uint32_t merge_bytes = kConsumerWarps * 16 * (s.d + 2) * 4;
  pl.region_bytes = max(pl.stages * pl.stage_bytes, merge_bytes);
  const int64_t rows_g = (int64_t)s.batch * s.n_q * s.h;
  const int ctas_per_sm = (pl.region_bytes <= 100u * 1024u) ? 2 : 1;
  const int64_t want = (int64_t)num_sms() * ctas_per_sm * 2;
  const int64_t by_fill = (want + rows_g - 1) / rows_g;
  int splits = (int)(by_fill < (s.topk + 3) / 4 ? by_fill : (s.topk + 3) / 4);
  splits = max(splits, (s.topk + 511) / 512);
  pl.splits = max(1, splits);
  pl.chunk = (s.topk + pl.splits - 1) / pl.splits;
  pl.splits = (s.topk + pl.chunk - 1) / pl.chunk;
  pl.smem_bytes = 1024 + pl.region_bytes + 16 * pl.stages + 4 * (pl.chunk + 1);
  return pl;
}

}  // namespace

size_t attn_partial_bytes(const Shape& s) {
  const AttnPlan pl = plan_attn(s);
  if (pl.splits <= 1) return 0;
  const size_t n = (size_t)s.batch * s.n_q * s.H * pl.splits;
  return n * (size_t)(s.d + 1) * sizeof(float) + 256;
}

int attn_launches(const Shape& s) { return plan_attn(s).splits > 1 ? 2 : 1; }

cudaError_t launch_sparse_attn(const Shape& s, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const int32_t* ids, uint16_t* out, float* lse,
                               void* partials, size_t partial_bytes, DeviceStatus* st,
                               cudaStream_t stream) {
  const AttnPlan pl = plan_attn(s);
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
  a.scale_log2 = s.scale * 1.4426950408889634f;
  a.splits = pl.splits;
  a.chunk = pl.chunk;
  a.stages = pl.stages;
  a.stage_bytes = pl.stage_bytes;
  a.region_bytes = pl.region_bytes;
  a.out = out;
  a.o_s0 = s.o_s[0];
  a.o_s1 = s.o_s[1];
  a.o_s2 = s.o_s[2];
  a.lse = lse;
  a.st = st;
  a.wait_ns = 500000000ull;  // 0.5 s; a healthy wait takes microseconds
  a.part_o = nullptr;
  a.part_lse = nullptr;
  const size_t nrow_h = (size_t)s.batch * s.n_q * s.H;
  if (pl.splits > 1) {
    if (partials == nullptr || partial_bytes < attn_partial_bytes(s)) return cudaErrorInvalidValue;
    a.part_o = reinterpret_cast<float*>(partials);
    a.part_lse = a.part_o + nrow_h * pl.splits * s.d;
  }
  const dim3 grid((unsigned)((int64_t)s.batch * s.n_q * s.h), pl.splits);
  cudaError_t err;
  if (s.d == 128) {
    err = cudaFuncSetAttribute(sparse_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)pl.smem_bytes);
    if (err != cudaSuccess) return err;
    sparse_attn_kernel<128><<<grid, kAttnThreads, pl.smem_bytes, stream>>>(tmk, tmv, a);
  } else {
    err = cudaFuncSetAttribute(sparse_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)pl.smem_bytes);
    if (err != cudaSuccess) return err;
    sparse_attn_kernel<64><<<grid, kAttnThreads, pl.smem_bytes, stream>>>(tmk, tmv, a);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess || pl.splits == 1) return err;
  combine_kernel<<<(unsigned)nrow_h, 128, 0, stream>>>(a.part_o, a.part_lse, pl.splits, s.d, s.H,
                                                       s.n_q, out, s.o_s[0], s.o_s[1], s.o_s[2],
                                                       lse);
  return cudaGetLastError();
}

}  // namespace msa
