// Kernels of sequence-sharded decode: the KV cache of every sequence is split
// into contiguous token shards, one per GPU, and a decode step is
//   1. per shard: the index scan and the shard's own top-k of its blocks, with
//      the kept blocks' scores (msa_index_candidates);
//   2. the candidate lists of all shards gathered on every GPU, and the global
//      top-k taken from them (candidates_topk_kernel in topk.cu); each GPU keeps
//      the winners inside its own shard;
//   3. per shard: exact attention over its own winners, giving a partial output
//      and its log-sum-exp for every head;
//   4. the partials gathered and merged by their log-sum-exps (here).
// The result is the single-device result: the global top-k blocks of a row are
// each in the top-k of the shard that holds them, and softmax attention over a
// union of disjoint key sets is the log-sum-exp-weighted mean of the parts.
// The method is the one of "MiniMax goes sparse" (atlascloud.ai), section 1,
// steps 1 and 2; the pages do not shard it, this is a deployment layout.
#include "kernels.h"

namespace msa {
namespace {

struct MergeArgs {
  const uint16_t* part_out;  // [nparts, rows_h, D]
  const float* part_lse;     // [nparts, rows_h]
  uint16_t* out;
  int64_t o_s0, o_s1, o_s2;
  float* lse;
  int nparts, n_q, H;
  int64_t rows_h;
};

// One warp per (sequence, query, head): weights e^(lse_r - max) of the parts that
// saw a key, the weighted mean of their outputs, the merged log-sum-exp.
template <int D>
__global__ void __launch_bounds__(256) merge_partials_kernel(MergeArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x * 8LL + (threadIdx.x >> 5);
  if (r >= a.rows_h) return;
  const float ninf = -__int_as_float(0x7f800000);
  float M = ninf;
  for (int p = 0; p < a.nparts; ++p) M = fmaxf(M, __ldg(a.part_lse + p * a.rows_h + r));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (M != ninf) {
    for (int p = 0; p < a.nparts; ++p) {
      const float l = __ldg(a.part_lse + p * a.rows_h + r);
      if (l == ninf) continue;  // this part saw no key of the row
      const float w = __expf(l - M);
      den += w;
      const uint16_t* src = a.part_out + (p * a.rows_h + r) * D + lane * PER;
      if constexpr (PER == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
        acc[0] += w * __uint_as_float(u.x << 16);
        acc[1] += w * __uint_as_float(u.x & 0xffff0000u);
        acc[2] += w * __uint_as_float(u.y << 16);
        acc[3] += w * __uint_as_float(u.y & 0xffff0000u);
      } else {
        const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(src));
        acc[0] += w * __uint_as_float(u << 16);
        acc[1] += w * __uint_as_float(u & 0xffff0000u);
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const int hq = (int)(r % a.H);
  const int64_t bt = r / a.H;
  const int t = (int)(bt % a.n_q);
  const int64_t b = bt / a.n_q;
  uint16_t* o = a.out + b * a.o_s0 + (int64_t)t * a.o_s1 + (int64_t)hq * a.o_s2 + lane * PER;
  if constexpr (PER == 4) {
    *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv),
                                              pack_bf16(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(o) = pack_bf16(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && a.lse) a.lse[r] = den > 0.f ? M + __logf(den) : ninf;
}

__global__ void shard_lengths_kernel(const int32_t* seq_lens, int batch, int max_kv, int64_t base,
                                     int64_t len, int32_t* out, DeviceStatus* st) {
  grid_dep_wait();
  grid_dep_launch();
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    const int64_t L = kv_length(seq_lens, b, max_kv, st);
    out[b] = (int32_t)min(max(L - base, (int64_t)0), len);
  }
}

}  // namespace

cudaError_t launch_merge_partials(const Shape& s, int nparts, const uint16_t* part_out,
                                  const float* part_lse, uint16_t* out, float* lse,
                                  cudaStream_t stream) {
  MergeArgs a;
  a.part_out = part_out;
  a.part_lse = part_lse;
  a.out = out;
  a.o_s0 = s.o_s[0];
  a.o_s1 = s.o_s[1];
  a.o_s2 = s.o_s[2];
  a.lse = lse;
  a.nparts = nparts;
  a.n_q = s.n_q;
  a.H = s.H;
  a.rows_h = (int64_t)s.batch * s.n_q * s.H;
  const dim3 grid((unsigned)((a.rows_h + 7) / 8));
  if (s.d == 128) return launch_pdl(merge_partials_kernel<128>, grid, dim3(256), 0, stream, a);
  return launch_pdl(merge_partials_kernel<64>, grid, dim3(256), 0, stream, a);
}

cudaError_t launch_shard_lengths(const int32_t* seq_lens, int batch, int max_kv, int64_t base,
                                 int64_t len, int32_t* out, DeviceStatus* st, cudaStream_t stream) {
  const int threads = 256;
  const dim3 grid((unsigned)((batch + threads - 1) / threads));
  return launch_pdl(shard_lengths_kernel, grid, dim3(threads), 0, stream, seq_lens, batch, max_kv,
                    base, len, out, st);
}

}  // namespace msa
