// Device-side building blocks shared by the MSA kernels (sm_100a).
//
// Inline PTX wrappers written from the PTX ISA: mbarrier with bounded waits,
// TMA tile loads (no multicast), ldmatrix, the bf16 m16n8k16 warp MMA, and the
// sticky device status word that the host reads back.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msa {

// Status codes mirrored from the public header.
enum : uint32_t { kOk = 0, kErrTimeout = 5, kErrDeviceAssert = 6 };

// First bytes of every workspace: the sticky status word.
struct DeviceStatus {
  uint32_t code;    // first error recorded (0 = none)
  uint32_t detail;  // kernel-specific detail of that error
};

// Reserved at the start of the workspace: the status word, and from byte
// kCounterOffset the decode attention's per-row merge counters.  The counters are
// zero between calls: msa_workspace_init clears the region, every row's merging
// CTA puts its counter back to zero, and msa_get_device_status clears the region
// again after an error (a call that stopped early may leave counters set).
constexpr size_t kStatusBytes = 4096;
constexpr size_t kCounterOffset = 256;
constexpr int kFixedCounters = (int)((kStatusBytes - kCounterOffset) / sizeof(int));

__device__ __forceinline__ void record_error(DeviceStatus* st, uint32_t code, uint32_t detail) {
  if (st == nullptr) return;
  if (atomicCAS(&st->code, 0u, code) == 0u) atomicExch(&st->detail, detail);
}

// KV length of sequence b: seq_lens[b] clamped to [0, max_kv]; a value outside
// that range is recorded as a broken precondition.
__device__ __forceinline__ int kv_length(const int32_t* seq_lens, int b, int max_kv,
                                         DeviceStatus* st) {
  if (seq_lens == nullptr) return max_kv;
  const int L = seq_lens[b];
  if (L < 0 || L > max_kv) {
    record_error(st, kErrDeviceAssert, 0x10000u | (uint32_t)b);
    return L < 0 ? 0 : max_kv;
  }
  return L;
}

// Paged K, V and K_idx: table[b * stride + beta] is the pool page holding tokens
// [beta * block, (beta + 1) * block) of sequence b.  table == nullptr: the tensors
// are contiguous per sequence.
struct KvPages {
  const int32_t* table;
  int64_t stride, pages;
};

// The page of block beta of sequence b, or -1 (recorded as a broken precondition)
// when the table names a page outside the pool.
__device__ __forceinline__ int64_t kv_page(const KvPages& pg, int b, int beta, DeviceStatus* st) {
  const int64_t page = __ldg(pg.table + (int64_t)b * pg.stride + beta);
  if (page < 0 || page >= pg.pages) {
    record_error(st, kErrDeviceAssert, 0x20000u | (uint32_t)b);
    return -1;
  }
  return page;
}

// TMA coordinates (token, plane) of the first token of block beta of sequence b:
// [beta * block, b] in contiguous tensors, [0, page] in a page pool.  A bad page
// gives the plane just past the pool, which a TMA load reads as zeros.
__device__ __forceinline__ void kv_block_coords(const KvPages& pg, int b, int beta, int block,
                                                DeviceStatus* st, int& tok, int& plane) {
  if (pg.table == nullptr) {
    tok = beta * block;
    plane = b;
    return;
  }
  const int64_t page = kv_page(pg, b, beta, st);
  tok = 0;
  plane = page < 0 ? (int)pg.pages : (int)page;
}

// True once any kernel sharing this status word has recorded an error; kernels
// check it on entry so that a failure is not repeated by every later CTA.
__device__ __forceinline__ bool status_failed(const DeviceStatus* st) {
  return st != nullptr && *reinterpret_cast<const volatile uint32_t*>(&st->code) == kErrTimeout;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Programmatic dependent launch.  Every kernel of the library starts with
// grid_dep_wait(), which returns once the grid launched before it on the stream
// has completed and its writes are visible (immediately when the kernel was not
// launched as a dependent), and then allows its own dependent to be scheduled:
// the next kernel's CTAs take free SM slots and wait there, so its launch overlaps
// this kernel's tail.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches `kernel` on `stream` as a programmatic dependent of the previous
// kernel on the stream (see grid_dep_wait).
template <typename... K, typename... A>
inline cudaError_t launch_pdl(void (*kernel)(K...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, A... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Load with acquire semantics at GPU scope (pairs with a writer's fence + atomic).
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Named barrier `id` over `nthreads` threads: arrive without waiting, or wait.
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed, for at most
// `limit_ns` nanoseconds.  On expiry it records kErrTimeout and returns false;
// it never traps and never spins without bound.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  DeviceStatus* st, uint32_t detail,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0u && global_timer_ns() - t0 > limit_ns) {
      record_error(st, kErrTimeout, detail);
      return false;
    }
  }
}

// Bounded wait taken by a whole warp: the result is the same on every lane (all
// lanes succeed or all report failure), so that warp-collective instructions that
// follow (ldmatrix, mma.sync, tcgen05.ld) never run on a diverged warp.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, DeviceStatus* st,
                                               uint32_t detail, uint64_t limit_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, st, detail, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// -------------------------------------------------------------- TMA loads
// 4-D tiled tensor load into shared memory, completion counted in bytes on an
// mbarrier.  No cluster multicast.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------ warp-level tensor ops
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A * B for one 16x8x16 tile, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 matrix held in the m8n8 fragment layout (thread t
// holds row t / 4, columns 2 (t % 4) and 2 (t % 4) + 1) into the same layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Two floats to a packed bf16 pair (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_u4(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a tile stored
// with the 128-byte TMA swizzle (rows of 128 bytes, tile base 1024-aligned).
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed two-wide fp32 arithmetic of sm_100 (one instruction for two lanes of
// work, round to nearest even as the scalar forms): d = a * b + c, d = a + b and
// d = a * b element-wise on (lo, hi) pairs.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// 2^x with the hardware approximation (subnormal results flush to zero).
__device__ __forceinline__ float exp2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// 2^x for x <= 0 on the FMA and integer pipes, leaving the special-function unit
// free: x = n + f with n = round(x) and f in [-1/2, 1/2]; 2^f from a cubic fitted
// to it on that interval by iterated weighted least squares on the relative
// error (largest relative error 7.5e-5 evaluated in float), and 2^n added to the
// exponent field.  Adding 1.5 * 2^23 rounds x to an integer held in the low
// mantissa bits, which the shift by 23 moves into the exponent field.  Inputs
// below -125 (-inf included) give exactly 0; they are clamped first so that the
// exponent arithmetic stays in range.
__device__ __forceinline__ float exp2_poly(float x) {
  const float xc = fmaxf(x, -125.f);
  const float t = __fadd_rn(xc, 12582912.f);
  const float f = __fsub_rn(xc, __fsub_rn(t, 12582912.f));
  const float p = fmaf(fmaf(fmaf(0.0551716685f, f, 0.2426111400f), f, 0.6932609677f), f,
                       0.9999280572f);
  const float r = __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
  return x > -125.f ? r : 0.f;
}

// Two floats to bf16x2 (lo in the low half) on the integer pipe: half a bf16 unit
// in the last place is added to the magnitude and the high halves are kept, i.e.
// rounding to nearest with ties away from zero.  Finite inputs only.
__device__ __forceinline__ uint32_t pack_bf16_int(float lo, float hi) {
  return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
}

__device__ __forceinline__ float warp_max_xor(float v, int mask) {
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, mask));
}

}  // namespace msa
