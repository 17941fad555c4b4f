// Sparse attention over the selected original K/V (page "Step-5-Preview:
// Sparse Reads Are Not a Compressed KV Cache", sections "Main attention still
// reads original K/V" and "Selection is a weighted ReLU score ...").
//
// Warp-level formulation: one warp owns the Hg = 16 heads of one (query,
// group) -- exactly the M = 16 rows of an m16n8k16 MMA -- and walks the
// query's attended tokens 16 at a time: S = Q K^T (12 k-steps over D = 192),
// mask, online softmax in FP32 (base-2 exponent), P (bf16) x V into 24 FP32
// accumulator tiles.  K/V rows are staged in shared memory with cp.async
// (rows padded to 400 B so ldmatrix is conflict-free).
//
// It serves attn_decode_kernel (few queries, blocks under 8 tokens) --
// split-K over the query's tokens, 4 warps per CTA, partial (m, l, O)
// combined by attn_combine_kernel.  This file also holds the union planners
// (attn_plan_kernel, attn_plan_sort_kernel) of the prefill kernel in
// attn_tc.cuh: adjacent queries' selections overlap (the second page), so the
// 8 queries of a query block share one pass over the union of their blocks.
#pragma once
#include "common.cuh"

namespace sgqa {

constexpr int kD = 192;          // head_dim
constexpr int kHg = 16;          // heads per group
constexpr int kRowPad = 200;     // bf16 per staged row (400 B)
constexpr int kStepTok = 16;     // tokens per step
constexpr int kStageElems = kStepTok * kRowPad;  // one K or V stage

// ---------------------------------------------------------------------------
// Union planner: for each (seq, query block of 8, group) the sorted union of
// the 8 queries' selected blocks, each with an 8-bit mask of the queries that
// selected it.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 512;

// The candidate ids of a unit are < floor(t_last / B); a bitmap over that range
// (one bit per block, in shared memory) turns the union into set-bit order:
// set bits, prefix-popcount the words (the prefix kept for every word, or --
// pshift = 3, wide ranges -- for every eighth word, so that a 1M-token range
// at B = 1 fits: 128 KB of bitmap, 16 KB of prefix), then every (query, id)
// finds its union position from the prefix and the counts of the words since,
// and ORs its query bit into that entry's mask, in shared memory; the masks
// go out with 8-byte stores.
__global__ void __launch_bounds__(kPlanThreads)
attn_plan_kernel(const int32_t* __restrict__ sel, const int32_t* __restrict__ sel_count,
                 int64_t nq, int G, int k, int nwords, int pshift, int64_t q_pos0, int B,
                 int32_t* __restrict__ plan_ids, uint8_t* __restrict__ plan_mask, int32_t* __restrict__ plan_count) {
  // [nwords] bitmap, [ngroups] prefix of every (1 << pshift)-th word, then the union's masks (8k bytes)
  extern __shared__ __align__(16) uint32_t sm_words[];
  const int ngroups = ((nwords - 1) >> pshift) + 1;
  uint32_t* bm = sm_words;
  uint32_t* pre = sm_words + nwords;
  uint32_t* msk = sm_words + nwords + ngroups + ((nwords + ngroups) & 1);  // 8-byte aligned
  __shared__ int warp_sums[kPlanThreads / 32];
  __shared__ int s_total;
  const int64_t nqb = (nq + 7) / 8;
  const int64_t unit = blockIdx.x;  // (seq * nqb + qb) * G + g
  const int g = static_cast<int>(unit % G);
  const int64_t qb = (unit / G) % nqb;
  const int64_t seq = unit / (G * nqb);
  const int tid = threadIdx.x;
  for (int w = tid; w < nwords; w += kPlanThreads) bm[w] = 0;
  for (int w = tid; w < 2 * k; w += kPlanThreads) msk[w] = 0;  // 8k bytes
  __syncthreads();
  const int nq_here = static_cast<int>(nq - qb * 8 < 8 ? nq - qb * 8 : 8);
  const int64_t row0 = (seq * nq + qb * 8) * G + g;
  // a query at position t may only have selected blocks below floor(t / B):
  // other ids break the call's contract, are reported and left out
  const int64_t lim0 = q_pos0 + qb * 8;
  for (int q = 0; q < nq_here; ++q) {
    const int64_t row = row0 + static_cast<int64_t>(q) * G;
    const int cnt = min(max(sel_count[row], 0), k);
    const int64_t lim = (lim0 + q) / B;
    for (int j = tid; j < cnt; j += kPlanThreads) {
      const int id = sel[row * k + j];
      if (id >= 0 && id < lim) atomicOr(&bm[id >> 5], 1u << (id & 31));
      else report(kDevBounds);
    }
  }
  __syncthreads();
  // exclusive prefix of popcounts, words split into contiguous per-thread runs
  const int per = (nwords + kPlanThreads - 1) / kPlanThreads;
  const int w0 = tid * per, w1 = min(nwords, w0 + per);
  int local = 0;
  for (int w = w0; w < w1; ++w) local += __popc(bm[w]);
  const int lane = tid & 31, warp = tid >> 5;
  int x = local;
  for (int o = 1; o < 32; o <<= 1) { int y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kPlanThreads / 32 ? warp_sums[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) { int y = __shfl_up_sync(0xffffffffu, w, o); if (lane >= o) w += y; }
    if (lane < kPlanThreads / 32) warp_sums[lane] = w;
    if (lane == kPlanThreads / 32 - 1) s_total = w;
  }
  __syncthreads();
  int run = (warp > 0 ? warp_sums[warp - 1] : 0) + x - local;
  const int64_t obase = unit * (8 * static_cast<int64_t>(k));
  for (int w = w0; w < w1; ++w) {
    if ((w & ((1 << pshift) - 1)) == 0) pre[w >> pshift] = run;
    uint32_t bits = bm[w];
    int pos = run;
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      plan_ids[obase + pos] = w * 32 + b;
      ++pos;
    }
    run = pos;
  }
  __syncthreads();
  for (int q = 0; q < nq_here; ++q) {
    const int64_t row = row0 + static_cast<int64_t>(q) * G;
    const int cnt = min(max(sel_count[row], 0), k);
    const int64_t lim = (lim0 + q) / B;
    for (int j = tid; j < cnt; j += kPlanThreads) {
      const int id = sel[row * k + j];
      if (id < 0 || id >= lim) continue;
      const int w = id >> 5;
      int pos = pre[w >> pshift] + __popc(bm[w] & ((1u << (id & 31)) - 1u));
      for (int v = (w >> pshift) << pshift; v < w; ++v) pos += __popc(bm[v]);
      atomicOr(&msk[pos >> 2], (1u << q) << (8 * (pos & 3)));
    }
  }
  __syncthreads();
  // the masks of entries [0, s_total), 8 bytes per store (a unit's 8k bytes
  // start 8-byte aligned; bytes past s_total are zeros)
  uint2* gm = reinterpret_cast<uint2*>(plan_mask + obase);
  const uint2* sm2 = reinterpret_cast<const uint2*>(msk);
  for (int x = tid; x < (s_total + 7) / 8; x += kPlanThreads) gm[x] = sm2[x];
  if (tid == 0) plan_count[unit] = s_total;
}

constexpr int kPlanSortThreads = 1024;

// Same plan by a bitonic sort of the 8 lists' (id, query) keys; used when the
// id range is too wide for a shared-memory bitmap (B = 1 at very long contexts).
__global__ void __launch_bounds__(kPlanSortThreads)
attn_plan_sort_kernel(const int32_t* __restrict__ sel, const int32_t* __restrict__ sel_count,
                 int64_t nq, int G, int k, int pow2, int64_t q_pos0, int B, int32_t* __restrict__ plan_ids,
                 uint8_t* __restrict__ plan_mask, int32_t* __restrict__ plan_count) {
  extern __shared__ uint32_t sk[];  // pow2 keys
  __shared__ int warp_sums[32];
  const int64_t nqb = (nq + 7) / 8;
  const int64_t unit = blockIdx.x;  // (seq * nqb + qb) * G + g
  const int g = static_cast<int>(unit % G);
  const int64_t qb = (unit / G) % nqb;
  const int64_t seq = unit / (G * nqb);
  const int tid = threadIdx.x;
  for (int j = tid; j < pow2; j += kPlanSortThreads) sk[j] = 0xFFFFFFFFu;
  __syncthreads();
  for (int q = 0; q < 8; ++q) {
    const int64_t i = qb * 8 + q;
    if (i >= nq) break;
    const int64_t row = (seq * nq + i) * G + g;
    const int cnt = min(max(sel_count[row], 0), k);
    const int64_t lim = (q_pos0 + i) / B;
    for (int j = tid; j < cnt; j += kPlanSortThreads) {
      const int id = sel[row * k + j];
      if (id >= 0 && id < lim) {
        sk[q * k + j] = (static_cast<uint32_t>(id) << 3) | q;
      } else {
        report(kDevBounds);  // outside the query's candidates: left out
      }
    }
  }
  __syncthreads();
  for (int size = 2; size <= pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int c = tid; c < pow2 / 2; c += kPlanSortThreads) {
        const int lo = 2 * stride * (c / stride) + (c % stride);
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint32_t a = sk[lo], b = sk[hi];
        if ((a > b) == asc) { sk[lo] = b; sk[hi] = a; }
      }
      __syncthreads();
    }
  }
  // Dedup: a run of equal ids becomes one entry whose mask ORs the run.
  const int per = pow2 / kPlanSortThreads > 0 ? pow2 / kPlanSortThreads : 1;
  const int beg = tid * per;
  int heads = 0;
  for (int j = beg; j < beg + per && j < pow2; ++j) {
    const uint32_t key = sk[j];
    if (key != 0xFFFFFFFFu && (j == 0 || (sk[j - 1] >> 3) != (key >> 3))) ++heads;
  }
  // block exclusive scan of heads
  const int lane = tid & 31, warp = tid >> 5;
  int x = heads;
  for (int o = 1; o < 32; o <<= 1) { int y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    for (int o = 1; o < 32; o <<= 1) { int y = __shfl_up_sync(0xffffffffu, w, o); if (lane >= o) w += y; }
    warp_sums[lane] = w;
  }
  __syncthreads();
  int pos = (warp > 0 ? warp_sums[warp - 1] : 0) + x - heads;
  const int64_t obase = unit * (8 * static_cast<int64_t>(k));
  for (int j = beg; j < beg + per && j < pow2; ++j) {
    const uint32_t key = sk[j];
    if (key == 0xFFFFFFFFu || (j > 0 && (sk[j - 1] >> 3) == (key >> 3))) continue;
    uint32_t m = 0;
    for (int r = j; r < pow2 && (sk[r] >> 3) == (key >> 3) && sk[r] != 0xFFFFFFFFu; ++r) m |= 1u << (sk[r] & 7);
    plan_ids[obase + pos] = static_cast<int32_t>(key >> 3);
    plan_mask[obase + pos] = static_cast<uint8_t>(m);
    ++pos;
  }
  if (tid == kPlanSortThreads - 1) plan_count[unit] = pos;
}

// ---------------------------------------------------------------------------
// Per-warp attention state and one 16-token step.
// ---------------------------------------------------------------------------
struct WarpAttn {
  uint32_t qf[12][4];  // Q as the A operand, 12 k-steps of 16
  float o[24][4];      // O accumulators, 24 n-tiles of 8 dims
  float m[2], l[2];    // running max (log2 domain) and partial sum, rows lane/4 and lane/4+8
};

__device__ __forceinline__ void warp_load_q(WarpAttn& st, const __nv_bfloat16* q16, int lane) {
  // q16: the 16 head rows of this (query, group), each kD wide.
  const __nv_bfloat16* ra = q16 + (lane >> 2) * kD + 2 * (lane & 3);
  const __nv_bfloat16* rb = ra + 8 * kD;
#pragma unroll
  for (int s = 0; s < 12; ++s) {
    st.qf[s][0] = *reinterpret_cast<const uint32_t*>(ra + 16 * s);
    st.qf[s][1] = *reinterpret_cast<const uint32_t*>(rb + 16 * s);
    st.qf[s][2] = *reinterpret_cast<const uint32_t*>(ra + 16 * s + 8);
    st.qf[s][3] = *reinterpret_cast<const uint32_t*>(rb + 16 * s + 8);
  }
#pragma unroll
  for (int j = 0; j < 24; ++j) st.o[j][0] = st.o[j][1] = st.o[j][2] = st.o[j][3] = 0.f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.f;
}

// One 16-token step.  kaddr / vaddr: this lane's ldmatrix row addresses (K:
// token 8 (mat >> 1) + mrow of the step, dims + 8 (mat & 1); V: token
// 8 (mat & 1) + mrow, dims + 8 (mat >> 1)), so a step's 16 tokens may be any
// staged rows.  tokmask bit p: token p of the step is attended by this warp's
// query.
__device__ __forceinline__ void warp_attend_at(WarpAttn& st, uint32_t kaddr, uint32_t vaddr,
                                               uint32_t tokmask, float scale_log2, int lane) {
  float s[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
  // QK^T: matrices (tok 0-7|8-15) x (dims 16s | 16s+8)
#pragma unroll
  for (int kstep = 0; kstep < 12; ++kstep) {
    uint32_t b[4];
    ldmatrix_x4(b, kaddr + kstep * 32);
    mma_bf16_16816(s[0], st.qf[kstep], b[0], b[1]);
    mma_bf16_16816(s[1], st.qf[kstep], b[2], b[3]);
  }
  // mask + scale; columns: token 8nt + 2(lane&3) + {0,1}
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = 8 * nt + 2 * (lane & 3) + (e & 1);
      const bool ok = (tokmask >> tok) & 1u;
      s[nt][e] = ok ? s[nt][e] * scale_log2 : -INFINITY;
      mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
    }
  }
  float alpha[2], muse[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    const float mnew = fmaxf(st.m[r], mx[r]);
    muse[r] = mnew == -INFINITY ? 0.f : mnew;
    alpha[r] = exp2f(st.m[r] - muse[r]);
    st.m[r] = mnew;
  }
  float p[2][4];
  float psum[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[nt][e] = exp2f(s[nt][e] - muse[e >> 1]);
      psum[e >> 1] += p[nt][e];
    }
  }
  st.l[0] = st.l[0] * alpha[0] + psum[0];
  st.l[1] = st.l[1] * alpha[1] + psum[1];
#pragma unroll
  for (int j = 0; j < 24; ++j) {
    st.o[j][0] *= alpha[0]; st.o[j][1] *= alpha[0];
    st.o[j][2] *= alpha[1]; st.o[j][3] *= alpha[1];
  }
  uint32_t pa[4];
  pa[0] = pack_bf16x2(p[0][0], p[0][1]);
  pa[1] = pack_bf16x2(p[0][2], p[0][3]);
  pa[2] = pack_bf16x2(p[1][0], p[1][1]);
  pa[3] = pack_bf16x2(p[1][2], p[1][3]);
  // PV: trans matrices (tok 0-7 | 8-15) x (dims 16jj | 16jj+8)
#pragma unroll
  for (int jj = 0; jj < 12; ++jj) {
    uint32_t b[4];
    ldmatrix_x4_trans(b, vaddr + jj * 32);
    mma_bf16_16816(st.o[2 * jj], pa, b[0], b[1]);
    mma_bf16_16816(st.o[2 * jj + 1], pa, b[2], b[3]);
  }
}

// The step over 16 consecutive staged tokens at ks / vs.
__device__ __forceinline__ void warp_attend_step(WarpAttn& st, uint32_t ks, uint32_t vs,
                                                 uint32_t tokmask, float scale_log2, int lane) {
  const int mrow = lane & 7, mat = lane >> 3;
  warp_attend_at(st, ks + ((8 * (mat >> 1) + mrow) * kRowPad + 8 * (mat & 1)) * 2,
                 vs + ((8 * (mat & 1) + mrow) * kRowPad + 8 * (mat >> 1)) * 2, tokmask, scale_log2, lane);
}

// Final normalisation and bf16 store of one warp's 16 x 192 output.
// g16: the 16 heads' gate logits (nullptr: no gate).
__device__ __forceinline__ void warp_store_out(WarpAttn& st, __nv_bfloat16* o16, const __nv_bfloat16* g16, int lane) {
  float l0 = st.l[0], l1 = st.l[1];
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = gate_factor(g16, lane >> 2) / l0, i1 = gate_factor(g16, (lane >> 2) + 8) / l1;
  __nv_bfloat16* ra = o16 + (lane >> 2) * kD + 2 * (lane & 3);
  __nv_bfloat16* rb = ra + 8 * kD;
#pragma unroll
  for (int j = 0; j < 24; ++j) {
    *reinterpret_cast<uint32_t*>(ra + 8 * j) = pack_bf16x2(st.o[j][0] * i0, st.o[j][1] * i0);
    *reinterpret_cast<uint32_t*>(rb + 8 * j) = pack_bf16x2(st.o[j][2] * i1, st.o[j][3] * i1);
  }
}

// Stage the K and V rows of ntok tokens (tok[p] < 0: zero row).  The calling
// threads [0, nthreads) share the 2 x ntok x 24 sixteen-byte chunks.
__device__ __forceinline__ void stage_tokens(uint32_t ks, uint32_t vs, const __nv_bfloat16* kc,
                                             const __nv_bfloat16* vc, const int64_t* tokbase,
                                             int tid, int nthreads, int ntok = kStepTok) {
  for (int c = tid; c < 2 * ntok * 24; c += nthreads) {
    const int which = c / (ntok * 24);
    const int cc = c % (ntok * 24);
    const int p = cc / 24, part = cc % 24;
    const int64_t base = tokbase[p];
    const bool ok = base >= 0;
    const __nv_bfloat16* src = (which ? vc : kc) + (ok ? base : 0) + part * 8;
    const uint32_t dst = (which ? vs : ks) + (p * kRowPad + part * 8) * 2;
    cp_async16_zfill(dst, src, ok);
  }
}

// ---------------------------------------------------------------------------
// Decode: split-K over one query's tokens.
// ---------------------------------------------------------------------------
constexpr int kDecWarps = 4;
constexpr int kDecStages = 3;  // per warp

template <int B>
__global__ void __launch_bounds__(kDecWarps * 32)
attn_decode_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                   const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ sel,
                   const int32_t* __restrict__ sel_count, float* __restrict__ part_o,
                   float* __restrict__ part_ml, int64_t nq, int G, int k, int64_t q_pos0,
                   int64_t cache_cap, int nsplit, float scale_log2) {
  extern __shared__ __align__(16) __nv_bfloat16 smem[];
  __shared__ int64_t s_tok[kDecWarps][kDecStages][kStepTok];
  constexpr int E = kStepTok / B;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x % nsplit;
  const int64_t row = blockIdx.x / nsplit;  // (seq * nq + i) * G + g
  const int g = static_cast<int>(row % G);
  const int64_t i = (row / G) % nq;
  const int64_t seq = row / (G * nq);
  const int64_t t = q_pos0 + i;
  const int cnt = min(max(sel_count[row], 0), k);
  const int32_t* ids = sel + row * k;
  const int n_union_steps = (cnt + E - 1) / E;
  const int n_steps = n_union_steps + 1;
  const int per = (n_steps + nsplit - 1) / nsplit;
  const int s_begin = split * per;
  const int s_end = min(n_steps, s_begin + per);
  const int64_t c0 = B * (t / B);
  const int64_t row_stride = static_cast<int64_t>(G) * kD;
  const __nv_bfloat16* kseq = kc + seq * cache_cap * row_stride + g * kD;
  const __nv_bfloat16* vseq = vc + seq * cache_cap * row_stride + g * kD;

  WarpAttn st;
  warp_load_q(st, q + ((seq * nq + i) * G + g) * kHg * kD, lane);
  __nv_bfloat16* wsm = smem + warp * (2 * kDecStages * kStageElems);

  auto token_of = [&](int step, int p) -> int64_t {
    if (step < n_union_steps) {
      const int e = step * E + p / B;
      if (e >= cnt) return -1;
      const int64_t tk = static_cast<int64_t>(ids[e]) * B + (p % B);
      return (tk >= 0 && tk <= t) ? tk : -1;
    }
    const int64_t s = c0 + p;
    return s <= t ? s : -1;
  };
  auto issue = [&](int step, int slot) {
    if (lane < kStepTok) {
      const int64_t tk = token_of(step, lane);
      s_tok[warp][slot][lane] = tk >= 0 ? tk * row_stride : -1;
    }
    __syncwarp();
    stage_tokens(smem_u32(wsm + (2 * slot) * kStageElems), smem_u32(wsm + (2 * slot + 1) * kStageElems),
                 kseq, vseq, s_tok[warp][slot], lane, 32);
  };
  // this warp's steps: s_begin + warp, + kDecWarps, ...
  int nmine = 0;
  for (int s = s_begin + warp; s < s_end; s += kDecWarps) ++nmine;
  for (int j = 0; j < kDecStages - 1; ++j) {
    if (j < nmine) issue(s_begin + warp + j * kDecWarps, j % kDecStages);
    cp_async_commit();
  }
  for (int j = 0; j < nmine; ++j) {
    cp_async_wait<kDecStages - 2>();
    __syncwarp();
    const int step = s_begin + warp + j * kDecWarps;
    uint32_t tm = 0;
    if (lane < kStepTok) tm = token_of(step, lane) >= 0 ? 1u : 0u;
    tm = __ballot_sync(0xffffffffu, tm) & 0xFFFFu;
    const int slot = j % kDecStages;
    if (tm) warp_attend_step(st, smem_u32(wsm + (2 * slot) * kStageElems),
                             smem_u32(wsm + (2 * slot + 1) * kStageElems), tm, scale_log2, lane);
    __syncwarp();
    const int jn = j + kDecStages - 1;
    if (jn < nmine) issue(s_begin + warp + jn * kDecWarps, jn % kDecStages);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();
  // combine the 4 warps in shared memory (reuse the staging area)
  float* cm = reinterpret_cast<float*>(smem);          // [4][16] max
  float* cl = cm + kDecWarps * kHg;                    // [4][16] sum
  float* co = cl + kDecWarps * kHg;                    // [4][16][192]
  float l0 = st.l[0], l1 = st.l[1];
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const int h0 = lane >> 2, h1 = h0 + 8;
  if ((lane & 3) == 0) {
    cm[warp * kHg + h0] = st.m[0]; cm[warp * kHg + h1] = st.m[1];
    cl[warp * kHg + h0] = l0;      cl[warp * kHg + h1] = l1;
  }
#pragma unroll
  for (int j = 0; j < 24; ++j) {
    const int d = 8 * j + 2 * (lane & 3);
    co[(warp * kHg + h0) * kD + d] = st.o[j][0];
    co[(warp * kHg + h0) * kD + d + 1] = st.o[j][1];
    co[(warp * kHg + h1) * kD + d] = st.o[j][2];
    co[(warp * kHg + h1) * kD + d + 1] = st.o[j][3];
  }
  __syncthreads();
  float* po = part_o + (row * nsplit + split) * kHg * kD;
  float* pml = part_ml + (row * nsplit + split) * kHg * 2;
  for (int idx = tid; idx < kHg * kD; idx += kDecWarps * 32) {
    const int h = idx / kD;
    float mm = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) mm = fmaxf(mm, cm[w * kHg + h]);
    const float mu = mm == -INFINITY ? 0.f : mm;
    float acc = 0.f, ls = 0.f;
    for (int w = 0; w < kDecWarps; ++w) {
      const float a = exp2f(cm[w * kHg + h] - mu);
      acc += a * co[(w * kHg + h) * kD + (idx % kD)];
      ls += a * cl[w * kHg + h];
    }
    po[idx] = acc;
    if (idx % kD == 0) { pml[2 * h] = mm; pml[2 * h + 1] = ls; }
  }
}

// Combine nsplit partials of each (row, head) into the bf16 output.
__global__ void attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                    __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ gate,
                                    int64_t rows, int nsplit) {
  const int64_t rh = blockIdx.x;  // row * 16 + h
  const int64_t row = rh / kHg;
  const int h = static_cast<int>(rh % kHg);
  float mm = -INFINITY;
  for (int s = 0; s < nsplit; ++s) mm = fmaxf(mm, part_ml[((row * nsplit + s) * kHg + h) * 2]);
  const float mu = mm == -INFINITY ? 0.f : mm;
  float ls = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float* ml = part_ml + ((row * nsplit + s) * kHg + h) * 2;
    ls += exp2f(ml[0] - mu) * ml[1];
  }
  const float inv = gate_factor(gate, rh) / ls;  // normalisation and output gate
  for (int d = threadIdx.x; d < kD; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float a = exp2f(part_ml[((row * nsplit + s) * kHg + h) * 2] - mu);
      acc += a * part_o[((row * nsplit + s) * kHg + h) * kD + d];
    }
    out[(row * kHg + h) * kD + d] = __float2bfloat16_rn(acc * inv);
  }
}

}  // namespace sgqa
