// Block-wise token merging (page "Step-5-Preview: Sparse Reads Are Not a
// Compressed KV Cache", section "Eight tokens become one search key,
// coordinate by coordinate").
//
// One thread owns 8 consecutive proxy coordinates of one block: it reads the
// block's B rows of proxy keys and compression logits as 16-byte vectors
// (bf16; two 16-byte vectors for fp32), forms the per-coordinate softmax with
// the block maximum subtracted, accumulates in FP32 and writes 8 FP32 merged
// values (optional) and 8 E4M3 codes (FP32 -> BF16 -> E4M3).  Eight adjacent
// threads cover one 64-wide row, so every row read is one 128-byte segment.
// HBM-bound: per block it moves B*Di*(2+2) bytes in and Di*(1[+4]) out.
#pragma once
#include "common.cuh"

namespace sgqa {

constexpr int kMergeThreads = 256;

template <int B, bool F32IN>
__device__ __forceinline__ void load8(const void* base, int64_t elem_off, float (&v)[8]) {
  if constexpr (F32IN) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_off);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem_off));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
}

// Di is fixed at 64 (8 threads x 8 coordinates).
template <int B, bool F32IN>
__global__ void __launch_bounds__(kMergeThreads)
merge_blocks_kernel(const void* __restrict__ kp, const void* __restrict__ logits,
                    int64_t cache_cap, int64_t blk_begin, int64_t nblk, int64_t num_seqs,
                    float* __restrict__ merged, uint8_t* __restrict__ store) {
  constexpr int Di = 64;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * kMergeThreads + threadIdx.x;
  if (gid >= num_seqs * nblk * 8) return;
  const int part = static_cast<int>(gid & 7);
  const int64_t rb = gid >> 3;
  const int64_t seq = rb / nblk;
  const int64_t r = blk_begin + rb % nblk;
  const int64_t row0 = seq * cache_cap + r * B;

  float c[B][8], k[B][8];
#pragma unroll
  for (int j = 0; j < B; ++j) {
    load8<B, F32IN>(logits, (row0 + j) * Di + part * 8, c[j]);
    load8<B, F32IN>(kp, (row0 + j) * Di + part * 8, k[j]);
  }
  float out[8];
#pragma unroll
  for (int d = 0; d < 8; ++d) {
    float m = c[0][d];
#pragma unroll
    for (int j = 1; j < B; ++j) m = fmaxf(m, c[j][d]);
    // The sums start from the first term (not from +0), so a block whose
    // terms are all -0 keeps the sign of zero, as a plain sum does.
    float den = expf(c[0][d] - m);
    float num = den * k[0][d];
#pragma unroll
    for (int j = 1; j < B; ++j) {
      const float e = expf(c[j][d] - m);
      den += e;
      num = fmaf(e, k[j][d], num);
    }
    out[d] = num / den;
  }
  const int64_t orow = (seq * (cache_cap / B) + r) * Di + part * 8;
  if (merged != nullptr) {
    float4* o = reinterpret_cast<float4*>(merged + orow);
    o[0] = make_float4(out[0], out[1], out[2], out[3]);
    o[1] = make_float4(out[4], out[5], out[6], out[7]);
  }
  uint2 codes;
  codes.x = static_cast<uint32_t>(f32x2_to_e4m3x2(out[0], out[1])) |
            (static_cast<uint32_t>(f32x2_to_e4m3x2(out[2], out[3])) << 16);
  codes.y = static_cast<uint32_t>(f32x2_to_e4m3x2(out[4], out[5])) |
            (static_cast<uint32_t>(f32x2_to_e4m3x2(out[6], out[7])) << 16);
  *reinterpret_cast<uint2*>(store + orow) = codes;
}

}  // namespace sgqa
