// Shared device helpers for the Sparse GQA kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sgqa {

// Device status word, one per device (a __device__ variable lives in each
// device's copy of the module).  Kernels never trap: a bounded wait that runs
// out or a failed device-side check records a code here and the kernel
// returns.  sgqa_check() reads and clears it.
enum DeviceStatus : int { kDevOk = 0, kDevTimeout = 1, kDevBounds = 2 };
__device__ int g_status;

// Every spin-wait gives up after this many nanoseconds of %globaltimer.  The
// pipeline waits (a consumer waiting for data, a producer for a free slot)
// read the limit from g_wait_limit_ns (constant memory: a cached read), which
// sgqa_set_wait_limit_ns() may lower between launches; the drains that let in-flight copies and MMAs land before a kernel
// exits always use the full kWaitLimitNs.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__constant__ uint64_t g_wait_limit_ns = kWaitLimitNs;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report(int code) { atomicCAS(&g_status, 0, code); }

// Monotone map float -> uint32 for "larger score = larger key" comparisons.
// -0.0 is first turned into +0.0 so the two compare equal; every non-NaN
// value maps above 0x007FFFFF, so 0 works as "accept everything".
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(b);
}

// Head-wise output gate: the sigmoid of a head's BF16 gate logit, 1 without
// a gate (expf of a large positive argument gives inf, hence exactly 0).
__device__ __forceinline__ float gate_factor(const __nv_bfloat16* gate, int64_t head_row) {
  return gate == nullptr ? 1.f : 1.f / (1.f + expf(-__bfloat162float(gate[head_row])));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- E4M3 <-> BF16 ------------------------------------------------------
// Storage rounding FP32 -> BF16 (RNE) -> E4M3 (RNE, saturating), two at a time.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  __nv_bfloat162_raw raw = h;
  return static_cast<uint16_t>(__nv_cvt_bfloat16raw2_to_fp8x2(raw, __NV_SATFINITE, __NV_E4M3));
}

// Exact widening of two E4M3 codes to two BF16 values (packed, low = first).
// E4M3 -> half is exact (cvt.rn.f16x2.e4m3x2); half -> float -> bf16 is exact
// for every E4M3 value (3 mantissa bits, exponents 2^-9 .. 2^8).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t v) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v), __NV_E4M3);
  __half2 hh = h;
  float2 f = __half22float2(hh);
  __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t*>(&b);
}

// ---- warp-level MMA (m16n8k16, bf16 in, fp32 accumulate) ----------------
// (Plain asm: registers only, so the compiler may interleave independent MMAs.)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
// Arrive on an mbarrier once every cp.async this thread issued so far has
// completed (the pending count is raised now and lowered at completion).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// 2^x with the hardware approximation (relative error ~2^-22, subnormal
// results flushed to zero; 2^-inf = 0): for softmax weights that are rounded
// to BF16 afterwards.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Two FP32 values as one 64-bit operand of the packed f32x2 instructions (lo in bits 0-31).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

}  // namespace sgqa
