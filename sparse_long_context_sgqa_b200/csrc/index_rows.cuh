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
#include <cooperative_groups.h>

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
// E4M3 = true: keys are the E4M3 store itself ([S, store_rows, 64] bytes),
// widened to BF16 in registers (decode reads the store once, no BF16 copy).
template <int H, bool E4M3>
__global__ void __launch_bounds__(kScoreWarps * 32)
index_score_kernel(const __nv_bfloat16* __restrict__ idx_q, const float* __restrict__ idx_w,
                   const void* __restrict__ keys_any, float* __restrict__ scores,
                   int64_t nq, int G, int64_t q_pos0, int B, int64_t rpad, int64_t key_rows) {
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
  for (int64_t r0 = c0 + 16 * warp; r0 < c1; r0 += 16 * kScoreWarps) {
    uint32_t af[4][4];
    if constexpr (E4M3) {
      // rows past the store's end read as zero (their scores are never selected)
      const uint8_t* kb = static_cast<const uint8_t*>(keys_any) + seq * key_rows * Di;
      const int64_t ra_row = r0 + (lane >> 2), rb_row = ra_row + 8;
      const uint8_t* ra = kb + ra_row * Di + 2 * (lane & 3);
      const uint8_t* rb = kb + rb_row * Di + 2 * (lane & 3);
      const bool oka = ra_row < key_rows, okb = rb_row < key_rows;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        af[s][0] = oka ? e4m3x2_to_bf16x2(*reinterpret_cast<const uint16_t*>(ra + 16 * s)) : 0u;
        af[s][1] = okb ? e4m3x2_to_bf16x2(*reinterpret_cast<const uint16_t*>(rb + 16 * s)) : 0u;
        af[s][2] = oka ? e4m3x2_to_bf16x2(*reinterpret_cast<const uint16_t*>(ra + 16 * s + 8)) : 0u;
        af[s][3] = okb ? e4m3x2_to_bf16x2(*reinterpret_cast<const uint16_t*>(rb + 16 * s + 8)) : 0u;
      }
    } else {
      const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(keys_any) + seq * rpad * Di;
      const __nv_bfloat16* ra = kbase + (r0 + (lane >> 2)) * Di + 2 * (lane & 3);
      const __nv_bfloat16* rb = ra + 8 * Di;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        af[s][0] = *reinterpret_cast<const uint32_t*>(ra + 16 * s);
        af[s][1] = *reinterpret_cast<const uint32_t*>(rb + 16 * s);
        af[s][2] = *reinterpret_cast<const uint32_t*>(ra + 16 * s + 8);
        af[s][3] = *reinterpret_cast<const uint32_t*>(rb + 16 * s + 8);
      }
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

// Warp-level exact selection over buf[0, n) (n > k): the k-th largest key
// theta and, among entries whose key equals theta, the largest id to keep
// (id_cut), so that {key > theta} + {key == theta, id <= id_cut} is exactly k
// entries -- every key above the k-th and the smallest ids among its ties.
// Radix select on the 32-bit order-preserving keys, 8 bits per pass from the
// top; ties by a second radix select on the (distinct) ids.  The passes start
// at the highest byte in which the entries differ: the bits above it are
// common to all of them, so the passes over those would pick them with the
// count unchanged.
__device__ __forceinline__ void common_high_bits(uint32_t and_all, uint32_t or_all, uint32_t& prefix,
                                                 uint32_t& mask, int& shift) {
  const uint32_t diff = and_all ^ or_all;
  shift = diff ? (31 - __clz(static_cast<int>(diff))) / 8 * 8 : -8;
  mask = shift >= 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
  prefix = and_all & mask;
}
__device__ __noinline__ void warp_select(const uint2* buf, int n, int k, uint32_t* hist, uint32_t& theta,
                                         uint32_t& id_cut) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, mask = 0, rem = static_cast<uint32_t>(k);
  int shift0;
  {
    uint32_t a = 0xFFFFFFFFu, o = 0u;
    for (int i = lane; i < n; i += 32) {
      a &= buf[i].x;
      o |= buf[i].x;
    }
    a = __reduce_and_sync(0xffffffffu, a);
    o = __reduce_or_sync(0xffffffffu, o);
    common_high_bits(a, o, prefix, mask, shift0);
  }
  for (int shift = shift0; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint32_t key = buf[i].x;
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    uint32_t loc[8], sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) { loc[q] = hist[255 - (lane * 8 + q)]; sum += loc[q]; }
    uint32_t inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { uint32_t y = __shfl_up_sync(0xffffffffu, inc, o); if (lane >= o) inc += y; }
    const uint32_t before = inc - sum;
    const bool mine = before < rem && rem <= inc;
    uint32_t pick = 0, newrem = 0;
    if (mine) {
      uint32_t acc = before;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (acc < rem && rem <= acc + loc[q]) { pick = 255 - (lane * 8 + q); newrem = rem - acc; }
        acc += loc[q];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    pick = __shfl_sync(0xffffffffu, pick, src);
    rem = __shfl_sync(0xffffffffu, newrem, src);
    prefix |= pick << shift;
    mask |= 255u << shift;
    __syncwarp();
  }
  theta = prefix;
  int ties = 0;
  for (int i = lane; i < n; i += 32) ties += buf[i].x == theta;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ties += __shfl_xor_sync(0xffffffffu, ties, o);
  id_cut = 0xFFFFFFFFu;
  if (static_cast<uint32_t>(ties) > rem) {
    uint32_t ipre = 0, imask = 0, irem = rem;
    int ishift0;
    {
      uint32_t a = 0xFFFFFFFFu, o = 0u;
      for (int i = lane; i < n; i += 32) {
        const uint2 e = buf[i];
        if (e.x == theta) {
          a &= e.y;
          o |= e.y;
        }
      }
      a = __reduce_and_sync(0xffffffffu, a);
      o = __reduce_or_sync(0xffffffffu, o);
      common_high_bits(a, o, ipre, imask, ishift0);
    }
    for (int shift = ishift0; shift >= 0; shift -= 8) {
      for (int b = lane; b < 256; b += 32) hist[b] = 0;
      __syncwarp();
      for (int i = lane; i < n; i += 32) {
        const uint2 e = buf[i];
        if (e.x == theta && (e.y & imask) == ipre) atomicAdd(&hist[(e.y >> shift) & 255u], 1u);
      }
      __syncwarp();
      uint32_t loc[8], sum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { loc[q] = hist[lane * 8 + q]; sum += loc[q]; }
      uint32_t inc = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) { uint32_t y = __shfl_up_sync(0xffffffffu, inc, o); if (lane >= o) inc += y; }
      const uint32_t before = inc - sum;
      const bool mine = before < irem && irem <= inc;
      uint32_t pick = 0, newrem = 0;
      if (mine) {
        uint32_t acc = before;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (acc < irem && irem <= acc + loc[q]) { pick = lane * 8 + q; newrem = irem - acc; }
          acc += loc[q];
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      pick = __shfl_sync(0xffffffffu, pick, src);
      irem = __shfl_sync(0xffffffffu, newrem, src);
      ipre |= pick << shift;
      imask |= 255u << shift;
      __syncwarp();
    }
    id_cut = ipre;
  }
  __syncwarp();
}

__device__ __forceinline__ bool kept(uint2 e, uint32_t theta, uint32_t id_cut) {
  return e.x > theta || (e.x == theta && e.y <= id_cut);
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

// One CTA per (seq, query, group) row of scores.  STAGE = true copies the row
// into shared memory first (rows of up to kSelStageMax scores), so the radix
// passes read SRAM instead of HBM.
constexpr int kSelStageMax = 40960;

// The selection of one row by the whole CTA (every thread calls it with the
// same row); srow holds the row's scores.
template <bool STAGE>
__device__ __forceinline__ void topk_row_radix_at(int64_t row, const float* __restrict__ srow, int64_t nq, int G,
                                                  int64_t q_pos0, int B, int k, int32_t* __restrict__ sel,
                                                  int32_t* __restrict__ sel_count) {
  extern __shared__ float staged_row[];
  __shared__ uint32_t hist[2048];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_prefix, s_rem;
  const int64_t i = (row / G) % nq;
  const int64_t t = q_pos0 + i;
  const int64_t n = t / B;
  int32_t* out = sel + row * k;
  const int tid = threadIdx.x;
  if (STAGE && n > k) {
    const float4* src4 = reinterpret_cast<const float4*>(srow);
    float4* dst4 = reinterpret_cast<float4*>(staged_row);
    for (int64_t j = tid; j < (n + 3) / 4; j += kSelThreads) dst4[j] = src4[j];
    __syncthreads();
    srow = staged_row;
  }
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

template <bool STAGE>
__device__ __forceinline__ void topk_row_radix(int64_t row, const float* __restrict__ scores, int64_t rpad,
                                               int64_t nq, int G, int64_t q_pos0, int B, int k,
                                               int32_t* __restrict__ sel, int32_t* __restrict__ sel_count) {
  topk_row_radix_at<STAGE>(row, scores + row * rpad, nq, G, q_pos0, B, k, sel, sel_count);
}

// one CTA per row; only_if (optional) restricts the work to flagged rows
template <bool STAGE>
__global__ void __launch_bounds__(kSelThreads)
topk_rows_kernel(const float* __restrict__ scores, int64_t rpad, int64_t nq, int G,
                 int64_t q_pos0, int B, int k, int32_t* __restrict__ sel,
                 int32_t* __restrict__ sel_count, const int32_t* __restrict__ only_if) {
  const int64_t row = blockIdx.x;  // (seq * nq + i) * G + g
  if (only_if != nullptr && only_if[row] == 0) return;  // row already selected
  topk_row_radix<STAGE>(row, scores, rpad, nq, G, q_pos0, B, k, sel, sel_count);
}

// The rows another select kernel listed as unsettled (list[0 .. *count)),
// a fixed grid striding over them: a launch with an empty list costs one
// wave of CTAs that exit at once.
__global__ void __launch_bounds__(kSelThreads)
topk_rows_list_kernel(const float* __restrict__ scores, int64_t rpad, int64_t nq, int G, int64_t q_pos0, int B,
                      int k, int32_t* __restrict__ sel, int32_t* __restrict__ sel_count,
                      const int32_t* __restrict__ list, const int32_t* __restrict__ count) {
  const int n = *count;
  for (int x = blockIdx.x; x < n; x += gridDim.x) {
    topk_row_radix<false>(list[x], scores, rpad, nq, G, q_pos0, B, k, sel, sel_count);
    __syncthreads();  // the next row reuses the shared arrays
  }
}

}  // namespace sgqa

namespace sgqa {

// Two E4M3 codes widened to FP16 (exact: every E4M3 value is an FP16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float(static_cast<uint32_t>(127 + e) << 23); }

// Decode scores: a warp scores strips of 16 candidates for the query's four
// groups at once (B operand = 4 groups x 8 heads = 32 columns, resident in
// registers), straight from the E4M3 store.
//
// The MMA runs in FP16: the E4M3 codes convert to FP16 exactly with one
// instruction per pair.  Each head's query row is scaled by a power of two
// 2^s_h that brings its largest magnitude into [2^14, 2^15) and rounded to
// FP16, which is exact (a BF16 value has 8 significant bits, FP16 11) for
// every element down to 2^-28 of the head's largest; the head's weight
// carries 2^-s_h, so sum_h w_h * ReLU(dot_h) is unchanged (the scale is a
// power of two and positive).
//
// The MMA's k index is permuted (the same permutation on both operands leaves
// every dot product unchanged) so that each lane's A fragments for all four
// k-steps come from one contiguous 16-byte piece of a key row: logical
// k = 16 s + 8 h + 2 j + e is dimension 16 j + 4 s + 2 h + e (lane j =
// lane % 4).  A warp's strip of 16 candidates is then two fully used
// 512-byte runs of the store.

// B fragments of one (sequence and query) sq for all four groups (column n =
// head lane / 4 of group g): the scaled FP16 values of dimensions
// 16 j .. 16 j + 15 of that head (j = lane % 4), k-step s taking pairs 2 s,
// 2 s + 1; wv: the weights of the lane's accumulator columns (heads 2 j and
// 2 j + 1), which carry the heads' 2^-s.
__device__ __forceinline__ void dec_query_frags(const __nv_bfloat16* __restrict__ idx_q,
                                                const float* __restrict__ idx_w, int64_t sq, int lane,
                                                uint32_t (&bf)[4][8], float (&wv)[4][2]) {
  constexpr int G = 4, H = 8, Di = 64;
  const int j = lane & 3, rl = lane >> 2;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4* qrow = reinterpret_cast<const uint4*>(idx_q + ((sq * G + g) * H + rl) * Di + 16 * j);
    const uint4 q0 = __ldg(qrow), q1 = __ldg(qrow + 1);
    const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    float mx = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m)
      mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(qw[m] << 16)), fabsf(__uint_as_float(qw[m] & 0xFFFF0000u))));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // s_h = 141 - biased exponent of the head's largest magnitude (clamped)
    const int eb = static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu);
    const int sh = min(max(141 - eb, -110), 110);
    const float up = exp2i(sh), down = exp2i(-sh);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const __half2 h2 = __floats2half2_rn(__uint_as_float(qw[m] << 16) * up, __uint_as_float(qw[m] & 0xFFFF0000u) * up);
      bf[g][m] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    const float d0 = __shfl_sync(0xffffffffu, down, 8 * j), d1 = __shfl_sync(0xffffffffu, down, 8 * j + 4);
    const float2 w2 = __ldg(reinterpret_cast<const float2*>(idx_w + (sq * G + g) * H + 2 * j));
    wv[g][0] = w2.x * d0;
    wv[g][1] = w2.y * d1;
  }
}

// Scores of one strip of 16 candidates: ka / kb are the lane's 16-byte pieces
// (piece j) of key rows rl and rl + 8 of the strip.  Every lane of a quad
// computes all four groups' sums (bit-identical across the quad); lane j
// returns group j's, for rows rl (sa) and rl + 8 (sb).
__device__ __forceinline__ void dec_strip_scores(uint4 ka, uint4 kb, const uint32_t (&bf)[4][8],
                                                 const float (&wv)[4][2], int j, float& sa_out, float& sb_out) {
  // A fragments: pair m of the lane's 16 codes = dimensions 16 j + 2 m, + 1
  uint32_t pa[8], pb[8];
  const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w};
  const uint32_t wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    pa[2 * m] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa[m] & 0xFFFFu));
    pa[2 * m + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa[m] >> 16));
    pb[2 * m] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb[m] & 0xFFFFu));
    pb[2 * m + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb[m] >> 16));
  }
  sa_out = 0.f;
  sb_out = 0.f;
  // k-steps outside, groups inside: four independent accumulations in flight
  float acc[4][4];
#pragma unroll
  for (int g = 0; g < 4; ++g) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const uint32_t af[4] = {pa[2 * ks], pb[2 * ks], pa[2 * ks + 1], pb[2 * ks + 1]};
#pragma unroll
    for (int g = 0; g < 4; ++g) mma_f16_16816(acc[g], af, bf[g][2 * ks], bf[g][2 * ks + 1]);
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float sa = wv[g][0] * fmaxf(acc[g][0], 0.f) + wv[g][1] * fmaxf(acc[g][1], 0.f);
    float sb = wv[g][0] * fmaxf(acc[g][2], 0.f) + wv[g][1] * fmaxf(acc[g][3], 0.f);
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sb += __shfl_xor_sync(0xffffffffu, sb, 1);
    sb += __shfl_xor_sync(0xffffffffu, sb, 2);
    if (j == g) {
      sa_out = sa;
      sb_out = sb;
    }
  }
}

// One (sequence and query) per blockIdx.y; blockIdx.x takes a contiguous
// range of `per_cta` candidates, which its warps walk strip by strip (warp w:
// strips w, w + 8, ...).  Each warp streams its strips' key rows through a
// private ring of cp.async copies, kDecScoreRing strips in flight; every lane
// copies exactly the two 16-byte pieces it later reads, so the ring needs no
// warp barrier.  Writes FP32 score rows (lane j: group j) and, per row, the
// largest score of every strip of 16 candidates (smax [rows, rpad / 16]),
// from which topk_rows_bound_kernel bounds the row's k-th largest score.
constexpr int kDecScoreThreads = 256;
constexpr int kDecScoreRing = 8;
constexpr size_t kDecScoreSmem = static_cast<size_t>(kDecScoreThreads / 32) * kDecScoreRing * 1024;

__global__ void __launch_bounds__(kDecScoreThreads, 2)
index_score_decode_kernel(const __nv_bfloat16* __restrict__ idx_q, const float* __restrict__ idx_w,
                          const uint8_t* __restrict__ store, float* __restrict__ scores, int64_t nq,
                          int64_t q_pos0, int B, int64_t rpad, int64_t key_rows, int64_t per_cta,
                          float* __restrict__ smax, int32_t* __restrict__ list_count) {
  constexpr int Di = 64, W = kDecScoreThreads / 32;
  extern __shared__ __align__(16) uint8_t ring[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j = lane & 3, rl = lane >> 2;
  // the select kernel that follows lists the rows it leaves to the radix kernel
  if (list_count != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *list_count = 0;
  const int64_t sq = blockIdx.y;  // seq * nq + i
  const int64_t i = sq % nq, seq = sq / nq;
  const int64_t ncand = (q_pos0 + i) / B;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * per_cta;
  const int64_t c1 = min(ncand, c0 + per_cta);
  if (c0 >= c1) return;
  const int nstrips = static_cast<int>((c1 - c0 + 15) / 16);
  const int mine = nstrips > warp ? (nstrips - warp + W - 1) / W : 0;  // strips of this warp
  const uint8_t* kseq = store + seq * key_rows * Di;
  const uint32_t wring = smem_u32(ring + static_cast<size_t>(warp) * kDecScoreRing * 1024);
  // strip s of this warp into slot s % ring: rows 8 h + rl, the lane's piece j, at h * 512 + 16 lane
  auto issue = [&](int s) {
    if (s < mine) {
      const int64_t row0 = c0 + 16 * (warp + static_cast<int64_t>(W) * s);
      const uint32_t dst = wring + (s % kDecScoreRing) * 1024 + 16 * lane;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t r = row0 + 8 * h + rl;
        const bool ok = r < key_rows;
        cp_async16_zfill(dst + 512 * h, kseq + (ok ? r * Di + 16 * j : 0), ok);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < kDecScoreRing - 1; ++s) issue(s);
  uint32_t bf[4][8];
  float wv[4][2];
  dec_query_frags(idx_q, idx_w, sq, lane, bf, wv);
  float* srow = scores + (sq * 4 + j) * rpad;
  for (int s = 0; s < mine; ++s) {
    cp_async_wait<kDecScoreRing - 2>();
    const uint32_t src = wring + (s % kDecScoreRing) * 1024 + 16 * lane;
    uint4 ka, kb;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(ka.x), "=r"(ka.y), "=r"(ka.z), "=r"(ka.w) : "r"(src));
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(kb.x), "=r"(kb.y), "=r"(kb.z), "=r"(kb.w)
                 : "r"(src + 512));
    issue(s + kDecScoreRing - 1);  // into the slot this lane emptied in the previous strip
    float sa, sb;
    dec_strip_scores(ka, kb, bf, wv, j, sa, sb);
    const int64_t r0 = c0 + 16 * (warp + static_cast<int64_t>(W) * s), ra = r0 + rl, rb = ra + 8;
    if (ra < rpad) srow[ra] = sa;
    if (rb < rpad) srow[rb] = sb;
    // the strip's largest score of group j over its real candidates (the first always is one)
    float m = fmaxf(ra < ncand ? sa : -INFINITY, rb < ncand ? sb : -INFINITY);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    if (rl == 0) smax[(sq * 4 + j) * (rpad / 16) + r0 / 16] = m;
  }
  cp_async_wait<0>();
}

// Exact top-k of rows of at most 32768 scores: 1024 threads hold 32 keys each
// in registers.  Fast path: one linear histogram of 2048 bins between the
// row's smallest and largest score finds the bin holding the k-th largest;
// every score of a better bin is kept, and the boundary bin's entries (a few
// dozen on typical rows) are ranked exactly -- score, then smaller id -- by
// one warp.  The bin function rounds monotonically, so a better score never
// lands in a worse bin.  A boundary bin larger than its buffer (massive near
// or exact ties) falls back to four 8-bit radix passes over the keys, with a
// private histogram per warp, and ties taken in id order.  The kept ids are
// marked in a bitmap and read out in id order (ascending).
constexpr int kRegSelThreads = 1024;
constexpr int kRegSelPer = 32;
constexpr int kRegSelBins = 2048;
constexpr int kRegSelBnd = 1024;  // boundary entries the fast path ranks

// The kept bits (thread t owns word t) read out in id order by the whole CTA.
__device__ __forceinline__ void topk_reg_readout(const uint32_t* keep_bits, int* sums, int tid, int lane, int warp,
                                                 int k, int32_t* __restrict__ out, int32_t* __restrict__ sel_count,
                                                 int64_t row) {
  const uint32_t kb = keep_bits[tid];
  const uint32_t cnt = __popc(kb);
  uint32_t x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) { uint32_t y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
  __syncthreads();
  if (lane == 31) sums[warp] = static_cast<int>(x);
  __syncthreads();
  uint32_t pos = x - cnt;
  for (int w = 0; w < warp; ++w) pos += sums[w];
  uint32_t b = kb;
  while (b) {
    const int t = __ffs(b) - 1;
    b &= b - 1;
    if (pos < static_cast<uint32_t>(k)) out[pos] = tid * 32 + t;
    ++pos;
  }
  if (tid == kRegSelThreads - 1) {
    sel_count[row] = k;
    if (pos != static_cast<uint32_t>(k)) report(kDevBounds);
  }
}

__global__ void __launch_bounds__(kRegSelThreads)
topk_rows_reg_kernel(const float* __restrict__ scores, int64_t rpad, int64_t nq, int G, int64_t q_pos0, int B,
                     int k, int32_t* __restrict__ sel, int32_t* __restrict__ sel_count) {
  __shared__ uint32_t wh[32][256];
  __shared__ uint32_t keep_bits[1024];
  __shared__ uint32_t tie_bits[1024];
  __shared__ int sums[32];
  __shared__ uint32_t s_pick, s_rem;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = blockIdx.x;
  const int64_t i = (row / G) % nq;
  const int n = static_cast<int>((q_pos0 + i) / B);
  const float* srow = scores + row * rpad;
  int32_t* out = sel + row * k;
  if (n <= k) {
    for (int j = tid; j < k; j += kRegSelThreads) out[j] = j < n ? j : -1;
    if (tid == 0) sel_count[row] = n;
    return;
  }
  uint32_t key[kRegSelPer];
#pragma unroll
  for (int u = 0; u < kRegSelPer; ++u) {
    const int j = tid + u * kRegSelThreads;
    key[u] = j < n ? score_key(srow[j]) : 0u;  // 0 sorts below every real key
  }
  keep_bits[tid] = 0;
  tie_bits[tid] = 0;
  // ---- fast path: linear histogram between the row's extreme scores
  __shared__ float fmx[32], fmn[32];
  __shared__ uint32_t s_cnt, s_nb;
  uint32_t* hall = &wh[0][0];  // 4 copies x 2048 bins, then reused for the boundary list
  {
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int u = 0; u < kRegSelPer; ++u) {
      if (tid + u * kRegSelThreads < n) {
        const float v = key_score(key[u]);
        mx = fmaxf(mx, v);
        mn = fminf(mn, v);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
      fmx[warp] = mx;
      fmn[warp] = mn;
    }
    for (int b = tid; b < 4 * kRegSelBins; b += kRegSelThreads) hall[b] = 0u;
    if (tid == 0) s_nb = 0;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < 32; ++w) {
      mx = fmaxf(mx, fmx[w]);
      mn = fminf(mn, fmn[w]);
    }
    const float width = mx - mn;
    const float scale = width > 0.f ? (kRegSelBins - 0.5f) / width : 0.f;
    // bins best first; both steps round monotonically
    auto bin_of = [&](uint32_t kk) -> int {
      return min(static_cast<int>(__fmul_rn(__fsub_rn(mx, key_score(kk)), scale)), kRegSelBins - 1);
    };
    uint32_t* myh = hall + (warp & 3) * kRegSelBins;
#pragma unroll
    for (int u = 0; u < kRegSelPer; ++u)
      if (tid + u * kRegSelThreads < n) atomicAdd(&myh[bin_of(key[u])], 1u);
    __syncthreads();
    // thread t owns bins 2t, 2t + 1: the bin in which the running count reaches k
    const uint32_t c0 = hall[2 * tid] + hall[kRegSelBins + 2 * tid] + hall[2 * kRegSelBins + 2 * tid] +
                        hall[3 * kRegSelBins + 2 * tid];
    const uint32_t c1 = hall[2 * tid + 1] + hall[kRegSelBins + 2 * tid + 1] + hall[2 * kRegSelBins + 2 * tid + 1] +
                        hall[3 * kRegSelBins + 2 * tid + 1];
    uint32_t x = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { uint32_t y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
    if (lane == 31) sums[warp] = static_cast<int>(x);
    __syncthreads();
    uint32_t before = x - c0 - c1;
    for (int w = 0; w < warp; ++w) before += sums[w];
    const uint32_t kk = static_cast<uint32_t>(k);
    if (before < kk && kk <= before + c0) {
      s_pick = 2 * tid; s_rem = kk - before; s_cnt = c0;
    } else if (before + c0 < kk && kk <= before + c0 + c1) {
      s_pick = 2 * tid + 1; s_rem = kk - before - c0; s_cnt = c1;
    }
    __syncthreads();
    if (s_cnt <= kRegSelBnd) {
      const int bstar = static_cast<int>(s_pick);
      const uint32_t rem = s_rem;
      uint2* bnd = reinterpret_cast<uint2*>(hall);  // [kRegSelBnd], the histogram is consumed
      uint32_t* scratch = hall + 2 * kRegSelBnd;     // warp_select's 256 counters
#pragma unroll
      for (int u = 0; u < kRegSelPer; ++u) {
        const int j = tid + u * kRegSelThreads;
        if (j < n) {
          const int b = bin_of(key[u]);
          if (b < bstar) atomicOr(&keep_bits[j >> 5], 1u << (j & 31));
          else if (b == bstar) bnd[atomicAdd(&s_nb, 1u)] = make_uint2(key[u], static_cast<uint32_t>(j));
        }
      }
      __syncthreads();
      if (warp == 0) {
        const uint32_t nb = s_nb;
        uint32_t theta = 0, id_cut = 0xFFFFFFFFu;
        if (nb > rem) warp_select(bnd, static_cast<int>(nb), static_cast<int>(rem), scratch, theta, id_cut);
        for (uint32_t c = lane; c < nb; c += 32) {
          const uint2 e = bnd[c];
          if (nb <= rem || kept(e, theta, id_cut)) atomicOr(&keep_bits[e.y >> 5], 1u << (e.y & 31));
        }
      }
      __syncthreads();
      topk_reg_readout(keep_bits, sums, tid, lane, warp, k, out, sel_count, row);
      return;
    }
    __syncthreads();
  }
  // ---- fallback: radix passes (every thread takes this branch together)
  uint32_t prefix = 0, mask = 0, rem = static_cast<uint32_t>(k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) wh[warp][b] = 0;
    __syncwarp();
#pragma unroll
    for (int u = 0; u < kRegSelPer; ++u) {
      const bool in = (key[u] & mask) == prefix && (tid + u * kRegSelThreads) < n;
      if (in) atomicAdd(&wh[warp][(key[u] >> shift) & 255u], 1u);
    }
    __syncthreads();
    // bins from the top: thread b < 256 sums bin 255-b over the warps
    uint32_t c = 0;
    if (tid < 256) {
      const int b = 255 - tid;
#pragma unroll 8
      for (int w = 0; w < 32; ++w) c += wh[w][b];
    }
    // inclusive scan over the 256 descending bins (8 warps)
    uint32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { uint32_t y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
    if (tid < 256 && lane == 31) sums[warp] = static_cast<int>(x);
    __syncthreads();
    if (tid < 256) {
      uint32_t before = x - c;
      for (int w = 0; w < warp; ++w) before += sums[w];
      if (before < rem && rem <= before + c) { s_pick = 255 - tid; s_rem = rem - before; }
    }
    __syncthreads();
    prefix |= s_pick << shift;
    mask |= 255u << shift;
    rem = s_rem;
    __syncthreads();
  }
  const uint32_t theta = prefix;  // the k-th largest key; rem of its ties are kept
#pragma unroll
  for (int u = 0; u < kRegSelPer; ++u) {
    const int j = tid + u * kRegSelThreads;
    if (j < n && key[u] > theta) atomicOr(&keep_bits[j >> 5], 1u << (j & 31));
    if (j < n && key[u] == theta) atomicOr(&tie_bits[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  // ties in id order: thread w owns word w; keep the first rem tie bits overall
  {
    const uint32_t tb = tie_bits[tid];
    uint32_t cnt = __popc(tb), x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { uint32_t y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
    if (lane == 31) sums[warp] = static_cast<int>(x);
    __syncthreads();
    uint32_t before = x - cnt;
    for (int w = 0; w < warp; ++w) before += sums[w];
    uint32_t take = tb;
    if (before >= rem) take = 0;
    else if (before + cnt > rem) {
      uint32_t need = rem - before, t2 = 0, b = tb;
      while (need--) { t2 |= b & (~b + 1u); b &= b - 1u; }
      take = t2;
    }
    keep_bits[tid] |= take;
    __syncthreads();
  }
  topk_reg_readout(keep_bits, sums, tid, lane, warp, k, out, sel_count, row);
}

// ---------------------------------------------------------------------------
// Exact top-k of decode rows (at most 32768 candidates) from a lower bound on
// the k-th largest score.  Each strip of 16 candidates has one largest score
// (the score kernel writes them); if k strip maxima are >= L, then at least k
// candidates are >= L, so L <= the row's k-th largest score and every member
// of the top k -- ties at the k-th included -- scores >= L.  The kernel takes
// as L the smallest strip maximum among the best bins of a linear 2048-bin
// histogram of the strip maxima that hold k of them (at least k maxima are
// >= L, and L sits close above the k-th largest maximum, a little below the
// row's k-th largest score), collects the candidates >= L (a few more than k
// on typical rows) in one pass over the row, each warp into its own part of
// the list, and ranks them exactly (score, then smaller id): a linear
// histogram of their scores finds the bin of the k-th largest, and one warp
// ranks that bin's few entries (by counting when there are at most 64).  A row with fewer strips than k has no such bound and keeps every
// candidate for the exact rank (the launch sends rows of fewer than 16 k + 128
// candidates to topk_rows_reg_kernel).  Ids are marked in a bitmap and read out ascending.  A row with more
// than kBndSelWarpCap such candidates in one warp's share, or a boundary bin of
// more than 1024 (massive ties), is listed for topk_rows_list_kernel, which
// ranks the full row.
// ---------------------------------------------------------------------------
constexpr int kBndSelThreads = 1024;
constexpr int kBndSelPer = 32;      // scores of the row each thread holds
constexpr int kBndSelCap = 4096;    // candidates >= L the exact rank takes
constexpr int kBndSelWarpCap = kBndSelCap / (kBndSelThreads / 32);  // of them, per warp
constexpr int kBndSelBins = 2048;

__global__ void __launch_bounds__(kBndSelThreads)
topk_rows_bound_kernel(const float* __restrict__ scores, int64_t rpad, const float* __restrict__ smax, int64_t nq,
                       int G, int64_t q_pos0, int B, int k, int32_t* __restrict__ sel,
                       int32_t* __restrict__ sel_count, int32_t* __restrict__ list, int32_t* __restrict__ list_count) {
  __shared__ uint32_t hist[kBndSelBins];
  __shared__ uint2 surv[kBndSelCap];
  __shared__ uint32_t keep_bits[kBndSelThreads];
  __shared__ int sums[32];
  __shared__ float fmx[32], fmn[32];
  __shared__ uint32_t s_nsurv, s_lkey, s_bstar, s_rem, s_cnt, s_nb, s_kmin, s_kmax, s_over;
  __shared__ uint32_t wcount[kBndSelThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = blockIdx.x;
  const int64_t i = (row / G) % nq;
  const int n = static_cast<int>((q_pos0 + i) / B);
  int32_t* out = sel + row * k;
  if (n <= k) {
    for (int j = tid; j < k; j += kBndSelThreads) out[j] = j < n ? j : -1;
    if (tid == 0) sel_count[row] = n;
    return;
  }
  const float* srow = scores + row * rpad;
  // the row's strip maxima, two per thread
  const int ns = (n + 15) / 16;
  const float* mrow = smax + row * (rpad / 16);
  const float m0 = tid < ns ? mrow[tid] : -INFINITY;
  const float m1 = tid + kBndSelThreads < ns ? mrow[tid + kBndSelThreads] : -INFINITY;
  {
    float mx = fmaxf(m0, m1);
    float mn = fminf(tid < ns ? m0 : INFINITY, tid + kBndSelThreads < ns ? m1 : INFINITY);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
      fmx[warp] = mx;
      fmn[warp] = mn;
    }
  }
  for (int b = tid; b < kBndSelBins; b += kBndSelThreads) hist[b] = 0u;
  keep_bits[tid] = 0u;
  if (tid == 0) {
    s_nsurv = 0;
    s_lkey = ns >= k ? 0xFFFFFFFFu : 0u;  // fewer strips than k: no bound, every candidate is kept
    s_bstar = 0;
    s_kmin = 0xFFFFFFFFu;
    s_kmax = 0u;
    s_over = 0;
  }
  __syncthreads();
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int w = 0; w < 32; ++w) {
    mx = fmaxf(mx, fmx[w]);
    mn = fminf(mn, fmn[w]);
  }
  const float width = mx - mn;
  const float scale = width > 0.f ? (kBndSelBins - 0.5f) / width : 0.f;
  // bins best first; both steps round monotonically
  auto bin_of = [&](float x) -> int { return min(static_cast<int>(__fmul_rn(__fsub_rn(mx, x), scale)), kBndSelBins - 1); };
  if (ns >= k) {  // (uniform over the CTA)
  if (tid < ns) atomicAdd(&hist[bin_of(m0)], 1u);
  if (tid + kBndSelThreads < ns) atomicAdd(&hist[bin_of(m1)], 1u);
  __syncthreads();
  {  // thread t owns bins 2 t, 2 t + 1: the bin in which the running count of maxima reaches k
    const uint32_t c0 = hist[2 * tid], c1 = hist[2 * tid + 1];
    uint32_t x = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sums[warp] = static_cast<int>(x);
    __syncthreads();
    uint32_t before = x - c0 - c1;
    for (int w = 0; w < warp; ++w) before += sums[w];
    const uint32_t kk = static_cast<uint32_t>(k);
    if (before < kk && kk <= before + c0) s_bstar = 2 * tid;
    else if (before + c0 < kk && kk <= before + c0 + c1) s_bstar = 2 * tid + 1;
  }
  __syncthreads();
  {  // L: the smallest maximum of the bins up to the boundary bin
    const int bstar = static_cast<int>(s_bstar);
    uint32_t lk = 0xFFFFFFFFu;
    if (tid < ns && bin_of(m0) <= bstar) lk = score_key(m0);
    if (tid + kBndSelThreads < ns && bin_of(m1) <= bstar) lk = min(lk, score_key(m1));
    lk = __reduce_min_sync(0xffffffffu, lk);
    if (lane == 0 && lk != 0xFFFFFFFFu) atomicMin(&s_lkey, lk);
  }
  }
  __syncthreads();
  const uint32_t lkey = s_lkey;
  {  // the candidates >= L, one pass (thread t reads scores 4 t .. 4 t + 3 of
     // every 4096): each warp appends to its own region of the list (no
     // shared counter), a region that fills up sends the row to the radix kernel
    constexpr int kChunks = kBndSelPer / 4;
    uint2* mine = surv + warp * kBndSelWarpCap;
    uint32_t cnt = 0, kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
      const int j0 = 4 * tid + 4 * kBndSelThreads * u;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 < n) v = *reinterpret_cast<const float4*>(srow + j0);
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t kk = score_key(vv[e]);
        const bool in = j0 + e < n && kk >= lkey;
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        const uint32_t pos = cnt + __popc(bal & ((1u << lane) - 1u));
        if (in) {
          if (pos < static_cast<uint32_t>(kBndSelWarpCap)) mine[pos] = make_uint2(kk, static_cast<uint32_t>(j0 + e));
          kmin = min(kmin, kk);
          kmax = max(kmax, kk);
        }
        cnt += __popc(bal);
      }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      wcount[warp] = cnt;
      if (cnt) {
        atomicAdd(&s_nsurv, cnt);
        atomicMin(&s_kmin, kmin);
        atomicMax(&s_kmax, kmax);
      }
      if (cnt > static_cast<uint32_t>(kBndSelWarpCap)) s_over = 1;
    }
  }
  for (int b = tid; b < kBndSelBins; b += kBndSelThreads) hist[b] = 0u;
  __syncthreads();
  if (s_over) {  // every thread leaves here together
    if (tid == 0) list[atomicAdd(list_count, 1)] = static_cast<int32_t>(row);
    return;
  }
  // slot x of the list is entry x % cap of warp x / cap's region
  auto live = [&](int x) { return static_cast<uint32_t>(x % kBndSelWarpCap) < wcount[x / kBndSelWarpCap]; };
  // the exact rank among them: a linear histogram of their scores finds the
  // bin holding the k-th largest; better bins are kept, that bin's entries
  // (typically a few) are ranked by one warp
  const float hi = key_score(s_kmax), lo = key_score(s_kmin);
  const float scale2 = hi > lo ? (kBndSelBins - 0.5f) / (hi - lo) : 0.f;
  auto bin2 = [&](uint32_t kk) -> int {
    return min(static_cast<int>(__fmul_rn(__fsub_rn(hi, key_score(kk)), scale2)), kBndSelBins - 1);
  };
  for (int x = tid; x < kBndSelCap; x += kBndSelThreads)
    if (live(x)) atomicAdd(&hist[bin2(surv[x].x)], 1u);
  __syncthreads();
  {  // thread t owns bins 2 t, 2 t + 1
    const uint32_t c0 = hist[2 * tid], c1 = hist[2 * tid + 1];
    uint32_t x = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sums[warp] = static_cast<int>(x);
    __syncthreads();
    uint32_t before = x - c0 - c1;
    for (int w = 0; w < warp; ++w) before += sums[w];
    const uint32_t kk = static_cast<uint32_t>(k);
    if (before < kk && kk <= before + c0) {
      s_bstar = 2 * tid;
      s_rem = kk - before;
      s_cnt = c0;
    } else if (before + c0 < kk && kk <= before + c0 + c1) {
      s_bstar = 2 * tid + 1;
      s_rem = kk - before - c0;
      s_cnt = c1;
    }
    if (tid == 0) s_nb = 0;
  }
  __syncthreads();
  const int bstar = static_cast<int>(s_bstar);
  const uint32_t rem = s_rem, cstar = s_cnt;
  if (cstar > static_cast<uint32_t>(kBndSelBins / 2)) {  // a huge group of near-equal scores: the radix kernel
    if (tid == 0) list[atomicAdd(list_count, 1)] = static_cast<int32_t>(row);
    return;
  }
  uint2* bnd = reinterpret_cast<uint2*>(hist);  // [kBndSelBins / 2]; the histogram is consumed
  for (int x = tid; x < kBndSelCap; x += kBndSelThreads) {
    if (!live(x)) continue;
    const uint2 e = surv[x];
    const int b = bin2(e.x);
    if (b < bstar) atomicOr(&keep_bits[e.y >> 5], 1u << (e.y & 31));
    else if (b == bstar) bnd[atomicAdd(&s_nb, 1u)] = e;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t nb = s_nb;
    if (nb <= rem) {
      for (uint32_t e = lane; e < nb; e += 32) atomicOr(&keep_bits[bnd[e].y >> 5], 1u << (bnd[e].y & 31));
    } else if (nb <= 64) {
      // rank by counting: an entry is kept if fewer than rem entries beat it (score, then smaller id)
      const uint2 e0 = lane < static_cast<int>(nb) ? bnd[lane] : make_uint2(0u, 0xFFFFFFFFu);
      const uint2 e1 = lane + 32 < static_cast<int>(nb) ? bnd[lane + 32] : make_uint2(0u, 0xFFFFFFFFu);
      uint32_t r0 = 0, r1 = 0;
      for (int q = 0; q < 32; ++q) {
        const uint2 f0 = make_uint2(__shfl_sync(0xffffffffu, e0.x, q), __shfl_sync(0xffffffffu, e0.y, q));
        const uint2 f1 = make_uint2(__shfl_sync(0xffffffffu, e1.x, q), __shfl_sync(0xffffffffu, e1.y, q));
        auto beats = [](uint2 f, uint2 e) { return f.x > e.x || (f.x == e.x && f.y < e.y); };
        const bool v0 = q < static_cast<int>(nb), v1 = q + 32 < static_cast<int>(nb);
        r0 += (v0 && beats(f0, e0)) + (v1 && beats(f1, e0));
        r1 += (v0 && beats(f0, e1)) + (v1 && beats(f1, e1));
      }
      if (lane < static_cast<int>(nb) && r0 < rem) atomicOr(&keep_bits[e0.y >> 5], 1u << (e0.y & 31));
      if (lane + 32 < static_cast<int>(nb) && r1 < rem) atomicOr(&keep_bits[e1.y >> 5], 1u << (e1.y & 31));
    } else {
      uint32_t theta = 0, id_cut = 0xFFFFFFFFu;
      // warp_select's 256 counters live in the consumed candidate list
      warp_select(bnd, static_cast<int>(nb), static_cast<int>(rem), reinterpret_cast<uint32_t*>(surv), theta, id_cut);
      for (uint32_t e = lane; e < nb; e += 32)
        if (kept(bnd[e], theta, id_cut)) atomicOr(&keep_bits[bnd[e].y >> 5], 1u << (bnd[e].y & 31));
    }
  }
  __syncthreads();
  topk_reg_readout(keep_bits, sums, tid, lane, warp, k, out, sel_count, row);
}

}  // namespace sgqa
