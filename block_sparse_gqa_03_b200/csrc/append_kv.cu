// Decode-step cache write: the new tokens' K, V and K_idx rows go into the KV
// cache (contiguous or paged) at their positions, so that a decode step needs one
// copy of its packed inputs and no per-row copies.
//
// "MiniMax M3 的 MSA 与阶跃 Step 3.7 Flash 的 MFA" (ai.air7.fun), section
// "三条有意为之的减法", first item: MSA keeps the plain GQA KV layout that serving
// engines already use, which is what these rows are written into.
// "深度解析M3多模态模型与Token Plan" (cloud.baidu.com), list of MSA's innovations,
// first item: each physical block of the cache holds whole K/V slices, i.e. the
// paged layout's page.
#include "kernels.h"

namespace msa {
namespace {

struct AppendArgs {
  int n_new, max_kv, h, d, d_idx, block;
  const int32_t* seq_lens;
  const uint16_t *k_new, *v_new, *ki_new;  // dense [batch, n_new, h, d] / [batch, n_new, d_idx]
  uint16_t *k, *v, *ki;
  int64_t k_s[3], v_s[3], ki_s[2];
  KvPages pg;
  DeviceStatus* st;
};

// One CTA per new token: 16-byte pieces of its h K rows, h V rows and index key.
__global__ void __launch_bounds__(128) append_kv_kernel(AppendArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const int b = blockIdx.x / a.n_new, t = blockIdx.x % a.n_new;
  const int L = kv_length(a.seq_lens, b, a.max_kv, a.st);
  const int pos = L - a.n_new + t;
  if (pos < 0) {
    if (threadIdx.x == 0) record_error(a.st, kErrDeviceAssert, 0x30000u | (uint32_t)b);
    return;
  }
  int64_t plane = b, row = pos;
  if (a.pg.table != nullptr) {
    plane = kv_page(a.pg, b, pos / a.block, a.st);
    if (plane < 0) return;  // recorded by kv_page
    row = pos % a.block;
  }
  const int64_t src_tok = (int64_t)blockIdx.x;  // (b, t) in the dense inputs
  const int per_row = a.d / 8;                  // 16-byte pieces per K or V row
  for (int u = threadIdx.x; u < a.h * per_row; u += blockDim.x) {
    const int g = u / per_row, c = u % per_row;
    const int64_t src = (src_tok * a.h + g) * a.d + c * 8;
    if (a.k_new != nullptr)
      *reinterpret_cast<uint4*>(a.k + plane * a.k_s[0] + row * a.k_s[1] + g * a.k_s[2] + c * 8) =
          __ldg(reinterpret_cast<const uint4*>(a.k_new + src));
    if (a.v_new != nullptr)
      *reinterpret_cast<uint4*>(a.v + plane * a.v_s[0] + row * a.v_s[1] + g * a.v_s[2] + c * 8) =
          __ldg(reinterpret_cast<const uint4*>(a.v_new + src));
  }
  if (a.ki_new != nullptr)
    for (int c = threadIdx.x; c < a.d_idx / 8; c += blockDim.x)
      *reinterpret_cast<uint4*>(a.ki + plane * a.ki_s[0] + row * a.ki_s[1] + c * 8) =
          __ldg(reinterpret_cast<const uint4*>(a.ki_new + src_tok * a.d_idx + c * 8));
}

}  // namespace

cudaError_t launch_append_kv(const Shape& s, const uint16_t* k_new, const uint16_t* v_new,
                             const uint16_t* ki_new, uint16_t* k, uint16_t* v, uint16_t* ki,
                             DeviceStatus* st, cudaStream_t stream) {
  AppendArgs a;
  a.n_new = s.n_q;
  a.max_kv = s.max_kv;
  a.h = s.h;
  a.d = s.d;
  a.d_idx = s.d_idx;
  a.block = s.block;
  a.seq_lens = s.seq_lens;
  a.k_new = k_new;
  a.v_new = v_new;
  a.ki_new = ki_new;
  a.k = k;
  a.v = v;
  a.ki = ki;
  for (int i = 0; i < 3; ++i) {
    a.k_s[i] = s.k_s[i];
    a.v_s[i] = s.v_s[i];
  }
  a.ki_s[0] = s.ki_s[0];
  a.ki_s[1] = s.ki_s[1];
  a.pg = s.pages;
  a.st = st;
  const int64_t grid = (int64_t)s.batch * s.n_q;
  if (grid <= 0 || grid > INT32_MAX) return cudaErrorInvalidValue;
  return launch_pdl(append_kv_kernel, dim3((unsigned)grid), dim3(128), 0, stream, a);
}

}  // namespace msa
