// Indexer score and top-k selection, materialised-row form.
//
// Page "Step-5-Preview: Sparse Reads Are Not a Compressed KV Cache", section
// "Selection is a weighted ReLU score, not attention softmax":
//   I[t,g,r] = sum_i w[t,g,i] * max(0, q[t,g,i] . widen(store[r])), r < floor(t/B),
// then the k largest, equal scores to the smaller block id.
//
// Three kernels:
//  * widen_store_kernel   E4M3 store -> BF16 keys (exact), once per call;
//  * index_score_kernel   warp-level BF16 MMA (m16n8k16, FP32 accumulate) of
//                         candidate keys against a tile of (query, head) rows,
//                         then the weighted-ReLU head sum in FP32 registers;
//                         writes one FP32 score row per (query, group);
//  * topk_rows_kernel     exact radix select (11/11/10-bit digits over the
//                         order-preserving key of the FP32 score) per row, then
//                         an index-order compaction that takes every score
//                         above the k-th and the lowest-id ties at it, which
//                         leaves the ids already ascending.
// This form suits decode (one query per sequence, a few MB of scores) and is
// the general fallback; long prefill uses the fused streaming kernel.
#pragma once
#include "common.cuh"

namespace sgqa {

// keys[s, r, :] = widen(store[s, r, :]) for r < n_rows; 8 codes per thread.
__global__ void widen_store_kernel(const uint8_t* __restrict__ store, int64_t store_rows_per_seq,
                                   int64_t n_rows, int64_t out_rows_per_seq, int64_t num_seqs,
                                   __nv_bfloat16* __restrict__ keys) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= num_seqs * n_rows * 8) return;
  const int part = static_cast<int>(gid & 7);
  const int64_t rr = gid >> 3;
  const int64_t s = rr / n_rows, r = rr % n_rows;
  const uint2 c = __ldg(reinterpret_cast<const uint2*>(store + (s * store_rows_per_seq + r) * 64 + part * 8));
  uint4 o;
  o.x = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.x & 0xFFFF));
  o.y = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.x >> 16));
  o.z = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.y & 0xFFFF));
  o.w = e4m3x2_to_bf16x2(static_cast<uint16_t>(c.y >> 16));
  *reinterpret_cast<uint4*>(keys + (s * out_rows_per_seq + r) * 64 + part * 8) = o;
}

constexpr int kScoreWarps = 4;
constexpr int kScoreCandPerCta = 1024;

// Grid: x = query tiles of 64/H queries, y = candidate chunks of 1024,
// z = seq * G + g.  Each warp takes 16-candidate strips; the 64 columns of the
// B operand are (query, head) pairs of the tile.
template <int H>
__global__ void __launch_bounds__(kScoreWarps * 32)
index_score_kernel(const __nv_bfloat16* __restrict__ idx_q, const float* __restrict__ idx_w,
                   const __nv_bfloat16* __restrict__ keys, float* __restrict__ scores,
                   int64_t nq, int G, int64_t q_pos0, int B, int64_t rpad) {
  constexpr int QPC = 64 / H;  // queries per CTA tile
  constexpr int Di = 64;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t seq = blockIdx.z / G;
  const int g = blockIdx.z % G;
  const int64_t qt0 = static_cast<int64_t>(blockIdx.x) * QPC;
  const int64_t q_last = min(nq, qt0 + QPC) - 1;
  const int64_t ncand_max = (q_pos0 + q_last) / B;
  const int64_t c0 = static_cast<int64_t>(blockIdx.y) * kScoreCandPerCta;
  const int64_t c1 = min(ncand_max, c0 + kScoreCandPerCta);
  if (c0 >= c1) return;

  // B fragments: column n = 8j + lane/4 -> (query n / H, head n % H).
  uint32_t bf[8][4][2];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int n = 8 * j + (lane >> 2);
    const int64_t qi = qt0 + n / H;
    const bool ok = qi < nq;
    const __nv_bfloat16* row = idx_q + (((seq * nq + (ok ? qi : 0)) * G + g) * H + (n % H)) * Di;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int k0 = 16 * s + 2 * (lane & 3);
      bf[j][s][0] = ok ? *reinterpret_cast<const uint32_t*>(row + k0) : 0u;
      bf[j][s][1] = ok ? *reinterpret_cast<const uint32_t*>(row + k0 + 8) : 0u;
    }
  }
  // Head weights for the two accumulator columns this thread holds per n-tile.
  float wv[8][2];
  bool qok[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int col = 8 * j + 2 * (lane & 3);
    const int64_t qi = qt0 + col / H;
    qok[j] = qi < nq;
    const float* wr = idx_w + ((seq * nq + (qok[j] ? qi : 0)) * G + g) * H + (col % H);
    wv[j][0] = qok[j] ? wr[0] : 0.f;
    wv[j][1] = qok[j] ? wr[1] : 0.f;
  }
  const __nv_bfloat16* kbase = keys + seq * rpad * Di;
  for (int64_t r0 = c0 + 16 * warp; r0 < c1; r0 += 16 * kScoreWarps) {
    uint32_t af[4][4];
    const __nv_bfloat16* ra = kbase + (r0 + (lane >> 2)) * Di + 2 * (lane & 3);
    const __nv_bfloat16* rb = ra + 8 * Di;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      af[s][0] = *reinterpret_cast<const uint32_t*>(ra + 16 * s);
      af[s][1] = *reinterpret_cast<const uint32_t*>(rb + 16 * s);
      af[s][2] = *reinterpret_cast<const uint32_t*>(ra + 16 * s + 8);
      af[s][3] = *reinterpret_cast<const uint32_t*>(rb + 16 * s + 8);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_bf16_16816(acc, af[s], bf[j][s][0], bf[j][s][1]);
      float pa = wv[j][0] * fmaxf(acc[0], 0.f) + wv[j][1] * fmaxf(acc[1], 0.f);
      float pb = wv[j][0] * fmaxf(acc[2], 0.f) + wv[j][1] * fmaxf(acc[3], 0.f);
#pragma unroll
      for (int m = 1; m < H / 2; m <<= 1) {
        pa += __shfl_xor_sync(0xffffffffu, pa, m);
        pb += __shfl_xor_sync(0xffffffffu, pb, m);
      }
      const int col = 8 * j + 2 * (lane & 3);
      if (((lane & 3) % (H / 2)) == 0 && qok[j]) {
        const int64_t qi = qt0 + col / H;
        float* srow = scores + ((seq * nq + qi) * G + g) * rpad;
        srow[r0 + (lane >> 2)] = pa;
        srow[r0 + (lane >> 2) + 8] = pb;
      }
    }
  }
}

constexpr int kSelThreads = 512;

// Block-wide exclusive scan of one int per thread; returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int& total, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kSelThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSelThreads / 32) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  total = warp_sums[kSelThreads / 32 - 1];
  __syncthreads();
  return before;
}

// One CTA per (seq, query, group) row of scores.
__global__ void __launch_bounds__(kSelThreads)
topk_rows_kernel(const float* __restrict__ scores, int64_t rpad, int64_t nq, int G,
                 int64_t q_pos0, int B, int k, int32_t* __restrict__ sel,
                 int32_t* __restrict__ sel_count, const int32_t* __restrict__ only_if) {
  __shared__ uint32_t hist[2048];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_prefix, s_rem;
  const int64_t row = blockIdx.x;  // (seq * nq + i) * G + g
  if (only_if != nullptr && only_if[row] == 0) return;  // row already selected
  const int64_t i = (row / G) % nq;
  const int64_t t = q_pos0 + i;
  const int64_t n = t / B;
  const float* srow = scores + row * rpad;
  int32_t* out = sel + row * k;
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int j = tid; j < k; j += kSelThreads) out[j] = j < n ? j : -1;
    if (tid == 0) sel_count[row] = static_cast<int32_t>(n);
    return;
  }
  uint32_t prefix = 0, mask = 0, rem = static_cast<uint32_t>(k);
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int p = 0; p < 3; ++p) {
    const int shift = shifts[p];
    const uint32_t nb = 1u << widths[p];
    for (uint32_t b = tid; b < 2048; b += kSelThreads) hist[b] = 0;
    __syncthreads();
    for (int64_t j = tid; j < n; j += kSelThreads) {
      const uint32_t key = score_key(srow[j]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    // Find the bin, counted from the top, that holds the rem-th largest key.
    const int per = 2048 / kSelThreads;  // 4 bins per thread, descending
    uint32_t local[4];
    int lsum = 0;
#pragma unroll
    for (int q = 0; q < per; ++q) {
      const int b = 2047 - (tid * per + q);
      local[q] = (static_cast<uint32_t>(b) < nb) ? hist[b] : 0u;
      lsum += static_cast<int>(local[q]);
    }
    int total;
    int before = block_exclusive_scan(lsum, total, warp_sums);
    if (static_cast<uint32_t>(before) < rem && rem <= static_cast<uint32_t>(before + lsum)) {
      uint32_t acc = before;
#pragma unroll
      for (int q = 0; q < per; ++q) {
        if (acc < rem && rem <= acc + local[q]) {
          const uint32_t b = 2047 - (tid * per + q);
          s_prefix = prefix | (b << shift);
          s_rem = rem - acc;
        }
        acc += local[q];
      }
    }
    __syncthreads();
    prefix = s_prefix;
    rem = s_rem;
    mask |= (nb - 1) << shift;
    __syncthreads();
  }
  // prefix is the k-th largest key; take every larger key and the first rem
  // equal keys in id order.
  const uint32_t theta = prefix;
  int written = 0, eq_seen = 0;
  for (int64_t base = 0; base < n; base += kSelThreads) {
    const int64_t j = base + tid;
    const uint32_t key = j < n ? score_key(srow[j]) : 0u;
    const int eq = (j < n && key == theta) ? 1 : 0;
    int eq_total;
    const int eq_before = block_exclusive_scan(eq, eq_total, warp_sums);
    const int keep = (j < n) && (key > theta || (eq && static_cast<uint32_t>(eq_seen + eq_before) < rem));
    int keep_total;
    const int pos = block_exclusive_scan(keep, keep_total, warp_sums);
    if (keep && written + pos < k) out[written + pos] = static_cast<int32_t>(j);
    written += keep_total;
    eq_seen += eq_total;
  }
  if (tid == 0) sel_count[row] = k;
}

}  // namespace sgqa
