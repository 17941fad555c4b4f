// Indexer scores on the 5th-generation tensor cores and the top-k kernels of
// the prefill path (page "Step-5-Preview: Sparse Reads Are Not a Compressed KV
// Cache", section "Selection is a weighted ReLU score, not attention softmax").
//
// The page's standalone code materialises a [G*N, R] FP32 score matrix (its
// section "A configured million-token window is not a validated million-token
// launch": 512 GiB at 1M tokens).  Here scores exist per 8192-query chunk only,
// and for long rows not at all: one CTA owns a tile of Q queries of one group
// (Q * H = 256 (query, head) columns) and sweeps that tile's causal candidate
// blocks 128 at a time,
//   D[128 cand x 256 cols] = keys[128 x 64] . q[256 x 64]^T   (4 tcgen05.mma
//   M128 N256 K16, keys = the E4M3 store widened to BF16, both TMA-fed),
// double-buffered in TMEM, with the ReLU-weighted head sum in the epilogue
// (index_score_tc_kernel).  The select kernels below take its output.
#pragma once
#include "common.cuh"
#include "index_rows.cuh"
#include "tc.cuh"

namespace sgqa {

constexpr int kScoreTcThreads = 576;  // score kernel: producer, MMA, 16 epilogue warps
constexpr int kIdxStages = 4;
constexpr int kIdxCand = 128;    // candidates per tile (MMA M)
constexpr int kIdxCols = 256;    // (query, head) columns per CTA (MMA N)

struct __align__(1024) IndexTcSmem {
  uint8_t b[kIdxCols * 128];               // queries: 256 rows x 64 bf16 (SW128)
  uint8_t a[kIdxStages][kIdxCand * 128];   // candidate keys: 128 rows x 64 bf16 (SW128)
  float w[kIdxCols];                       // head weights, column order
  uint32_t thr[kIdxCols];                  // per-query threshold key (first Q used)
  int ncand[kIdxCols];                     // per-query candidate count floor(t / B)
  uint64_t b_full, a_full[kIdxStages], a_empty[kIdxStages], acc_full[2], acc_empty[2], drain;
  uint32_t tmem;
  int abort;
};


// Indexer scores I[t, g, r] on the tensor cores (one CTA = 256 (query, head)
// columns of one group, all candidates in tiles of 128), with one of three
// epilogues:
//   kScoreRows    every score as FP32 rows [row, rpad] (one 128-byte store per
//                 warp and query); a top-k kernel then selects from the rows;
//   kScoreSample  only every o.samp-th candidate tile, compacted into rows
//                 [row, ld] (for the per-row threshold estimate);
//   kScoreFilter  every score, but only those at or above the row's threshold
//                 are kept, as (order-preserving key, block id) pairs in the
//                 row's staging list; the row's count (which may exceed the
//                 list's capacity) is written at the end.  A CTA owns its rows,
//                 so the counters live in shared memory.
constexpr int kScoreRows = 0, kScoreSample = 1, kScoreFilter = 2;
constexpr int kSampleStride = 16;   // the smallest sample stride (in candidate tiles)
constexpr int kSampleTilesMax = 64; // sampled tiles per row: at most 8192 samples
struct ScoreOut {
  float* scores;            // kScoreRows: [rows, ld] = [rows, rpad]; kScoreSample: [rows, ld]
  int64_t ld;
  int samp;                 // kScoreSample: every samp-th candidate tile is scored
  const float* thr;         // kScoreFilter: per-row threshold
  uint2* staging;           // kScoreFilter: [rows, 4, cap] (key, id), one list per TMEM lane quadrant
  int32_t* staged;          // kScoreFilter: [rows, 4] scores at or above the threshold per list
  int cap;                  // entries per list
};

template <int H, int MODE>
__global__ void __launch_bounds__(kScoreTcThreads, 1)
index_score_tc_kernel(const __grid_constant__ CUtensorMap keymap, const __grid_constant__ CUtensorMap qmap,
                      const float* __restrict__ idx_w, ScoreOut o, int64_t nq, int G,
                      int64_t q_pos0, int B, int64_t rpad) {
  constexpr int Q = kIdxCols / H;
  extern __shared__ uint8_t smem_raw[];
  IndexTcSmem& sm = *reinterpret_cast<IndexTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                    ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles_q = (nq + Q - 1) / Q;
  const int64_t per_group = static_cast<int64_t>(gridDim.x) / G;
  const int g = static_cast<int>(blockIdx.x / per_group);
  const int64_t rest = blockIdx.x % per_group;
  const int64_t seq = rest / ntiles_q;
  const int64_t qt = ntiles_q - 1 - rest % ntiles_q;
  const int64_t q0 = qt * Q;
  const int nq_here = static_cast<int>(nq - q0 < Q ? nq - q0 : Q);
  const int64_t ncand_max = (q_pos0 + q0 + nq_here - 1) / B;
  const int n_tiles = static_cast<int>((ncand_max + kIdxCand - 1) / kIdxCand);
  // tiles this launch computes (the sample takes every kSampleStride-th) and the tile behind loop index c
  const int samp = o.samp;
  const int n_loop = MODE == kScoreSample ? (n_tiles + samp - 1) / samp : n_tiles;
  auto tile_of = [samp](int c) { return MODE == kScoreSample ? c * samp : c; };
  volatile int* abort = &sm.abort;
  auto bar = [](uint64_t& b) { return smem_u32(&b); };
  if (threadIdx.x == 0) {
    sm.abort = 0;
    tc::mbar_init(bar(sm.b_full), 1);
    for (int s = 0; s < kIdxStages; ++s) {
      tc::mbar_init(bar(sm.a_full[s]), 1);
      tc::mbar_init(bar(sm.a_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(sm.acc_full[b]), 1);
      tc::mbar_init(bar(sm.acc_empty[b]), 512);
    }
    tc::mbar_init(bar(sm.drain), 1);
    tc::mbar_fence_init();
  }
  for (int c = threadIdx.x; c < kIdxCols; c += kScoreTcThreads) {
    const int qs = c / H;
    sm.w[c] = qs < nq_here ? idx_w[((seq * nq + q0 + qs) * G + g) * H + (c % H)] : 0.f;
  }
  if (MODE == kScoreFilter) {
    for (int qs = threadIdx.x; qs < Q; qs += kScoreTcThreads) {
      const bool real = qs < nq_here;
      sm.thr[qs] = __float_as_uint(real ? o.thr[(seq * nq + q0 + qs) * G + g] : INFINITY);
      sm.ncand[qs] = real ? static_cast<int>((q_pos0 + q0 + qs) / B) : 0;
    }
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(&sm.tmem), 512);
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = sm.tmem;
  int issued = 0;  // producer: key tiles whose copies were issued
  if (n_tiles > 0) {
    if (warp == 0) {
      // producer: queries once, then the candidate tiles through the ring (converged warp, one elected issuer)
      if (tc::elect_one()) {
        tc::prefetch_tmap(&keymap);
        tc::prefetch_tmap(&qmap);
        tc::mbar_expect_tx(bar(sm.b_full), kIdxCols * 128);
        tc::tma_load_4d(smem_u32(&sm.b[0]), &qmap, 0, 0, g, static_cast<int32_t>(seq * nq + q0), bar(sm.b_full));
      }
      __syncwarp();
      for (int c = 0; c < n_loop; ++c) {
        const int s = c % kIdxStages;
        if (c >= kIdxStages && !tc::warp_wait(bar(sm.a_empty[s]), ((c / kIdxStages) - 1) & 1, abort)) break;
        if (tc::elect_one()) {
          tc::mbar_expect_tx(bar(sm.a_full[s]), kIdxCand * 128);
          tc::tma_load_2d(smem_u32(&sm.a[s][0]), &keymap, 0,
                          static_cast<int32_t>(seq * rpad + static_cast<int64_t>(tile_of(c)) * kIdxCand),
                          bar(sm.a_full[s]));
        }
        __syncwarp();
        issued = c + 1;
      }
    } else if (warp == 1) {
      // MMA issuer (converged warp, one elected issuer per tile)
      const uint32_t idesc = tc::idesc_bf16(kIdxCand, kIdxCols, false);
      const uint64_t da0 = tc::sdesc_sw128(smem_u32(&sm.a[0][0]), 16, 1024);
      const uint64_t db0 = tc::sdesc_sw128(smem_u32(&sm.b[0]), 16, 1024);
      constexpr uint32_t kStageUnits = kIdxCand * 128 / 16;  // one key stage in 16-byte units
      bool ok = tc::warp_wait(bar(sm.b_full), 0, abort);
      for (int c = 0; ok && c < n_loop; ++c) {
        const int s = c % kIdxStages, ab = c & 1;
        if (!tc::warp_wait(bar(sm.a_full[s]), (c / kIdxStages) & 1, abort)) { ok = false; break; }
        if (c >= 2 && !tc::warp_wait(bar(sm.acc_empty[ab]), ((c >> 1) - 1) & 1, abort)) { ok = false; break; }
        tc::fence_after();
        if (tc::elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // +32 B per 16 dims in both operands
            tc::mma_f16(tmem + ab * kIdxCols, da0 + s * kStageUnits + 2 * kk, db0 + 2 * kk, idesc, kk > 0 ? 1u : 0u);
          tc::mma_commit(bar(sm.a_empty[s]));
          tc::mma_commit(bar(sm.acc_full[ab]));
        }
        __syncwarp();
      }
    } else {
      // epilogue: sixteen warps, four per TMEM lane quadrant (= 32 candidates),
      // each taking 64 of the 256 (query, head) columns, read 32 at a time
      constexpr int QW = 32 / H;  // query slots per 32 columns
      const int quad = warp & 3;
      const int part = (warp - 2) >> 2;
      const int m = quad * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
      const int64_t row0 = (seq * nq + q0) * G + g;  // row of query slot 0; slot qs is row0 + qs * G
      // the CTA's smallest candidate count: tiles below it need no per-row bound check
      const int64_t ncand_min = (q_pos0 + q0) / B;
      int kept[2 * QW];  // filter: this warp's kept entries per query slot (the same in every lane)
#pragma unroll
      for (int x = 0; x < 2 * QW; ++x) kept[x] = 0;
      // FP32 outputs: slot x = (h2, qq) of this warp writes row row0 + qs * G,
      // element c * kIdxCand + m (the sample's tile c, or candidate tile c):
      // 32-bit offsets from one base (at most 32 * G rows of o.ld apart) and a
      // bit per slot for the queries the call has
      // (filter: soff[x] is instead the offset of slot x's (row, quadrant)
      // list from the CTA's first one, in entries: at most 32 * G * 4 * cap)
      int32_t soff[2 * QW];
      uint32_t vmask = 0;
#pragma unroll
      for (int x = 0; x < 2 * QW; ++x) {
        const int qs = (64 * part + 32 * (x / QW)) / H + x % QW;
        soff[x] = MODE == kScoreFilter ? static_cast<int32_t>(qs * G * 4 * o.cap)
                                       : static_cast<int32_t>(static_cast<int64_t>(qs) * G * o.ld);
        vmask |= static_cast<uint32_t>(qs < nq_here) << x;
      }
      float* const sbase = MODE == kScoreFilter ? nullptr : o.scores + row0 * o.ld + m;
      uint2* const lbase = MODE == kScoreFilter ? o.staging + (row0 * 4 + quad) * o.cap : nullptr;
      const uint32_t lt_mask = (1u << lane) - 1u;
      for (int c = 0; c < n_loop; ++c) {
        const int ab = c & 1;
        if (!tc::mbar_wait(bar(sm.acc_full[ab]), (c >> 1) & 1, abort)) break;
        tc::fence_after();
        const int64_t r = static_cast<int64_t>(tile_of(c)) * kIdxCand + m;  // candidate block id
        const bool tail = static_cast<int64_t>(tile_of(c) + 1) * kIdxCand > ncand_min;
        float* const tb = MODE == kScoreFilter ? nullptr : sbase + static_cast<int64_t>(c) * kIdxCand;
        // the warp's 64 columns in four chunks of 16 (SPC query slots each),
        // the next chunk's TMEM load in flight while this one is reduced
        constexpr int SPC = 16 / H;
        const uint32_t tcol = tmem + ab * kIdxCols + 64 * part + lane_off;
        uint32_t dbuf[2][16];
        tc::tmem_ld16(tcol, dbuf[0]);
        tc::tmem_ld_wait16(dbuf[0]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j < 3) {
            tc::tmem_ld16(tcol + 16 * (j + 1), dbuf[(j + 1) & 1]);
          } else {
            // every column of this accumulator has been read
            tc::fence_before();
            tc::mbar_arrive(bar(sm.acc_empty[ab]));
          }
          const uint32_t(&d)[16] = dbuf[j & 1];
#pragma unroll
          for (int u = 0; u < SPC; ++u) {
            const int x = j * SPC + u;  // slot index among the warp's 2 * QW
            const int qs = (64 * part) / H + x;
            const float4 w0 = *reinterpret_cast<const float4*>(&sm.w[qs * H]);
            float wv[H];
            wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
            if constexpr (H == 8) {
              const float4 w1 = *reinterpret_cast<const float4*>(&sm.w[qs * H + 4]);
              wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
            }
            // sum_i w_i * max(0, s_i): even and odd heads accumulate in the two
            // halves of a packed FP32 pair (fma.rn.f32x2), added at the end
            uint64_t acc2 = 0;
#pragma unroll
            for (int i = 0; i < H; i += 2) {
              const uint64_t x2 = pack_f32x2(fmaxf(__uint_as_float(d[u * H + i]), 0.f),
                                             fmaxf(__uint_as_float(d[u * H + i + 1]), 0.f));
              const uint64_t w2 = pack_f32x2(wv[i], wv[i + 1]);
              asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc2) : "l"(x2), "l"(w2));
            }
            const float acc = __uint_as_float(static_cast<uint32_t>(acc2)) +
                              __uint_as_float(static_cast<uint32_t>(acc2 >> 32));
            if (MODE != kScoreFilter) {
              if ((vmask >> x) & 1u) tb[soff[x]] = acc;
            } else {
              // keep the score if it reaches the row's threshold (rows past the
              // call's queries have threshold +inf); each (row, quadrant) has its
              // own list, filled in ballot order: no shared counters
              bool pass = acc >= __uint_as_float(sm.thr[qs]);
              if (tail) pass = pass && r < sm.ncand[qs];
              const uint32_t bal = __ballot_sync(0xffffffffu, pass);
              if (bal) {  // (long rows: most strips of 32 candidates have none)
                const int pos = kept[x] + __popc(bal & lt_mask);
                if (pass && pos < o.cap) lbase[soff[x] + pos] = make_uint2(score_key(acc), static_cast<uint32_t>(r));
                kept[x] += __popc(bal);
              }
            }
          }
          if (j < 3) tc::tmem_ld_wait16(dbuf[(j + 1) & 1]);
        }
      }
      if (MODE == kScoreFilter && lane == 0) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
          for (int qq = 0; qq < QW; ++qq) {
            const int qs = (64 * part + 32 * h2) / H + qq;
            if (qs < nq_here) o.staged[(row0 + static_cast<int64_t>(qs) * G) * 4 + quad] = kept[h2 * QW + qq];
          }
      }
    }
  } else if (MODE == kScoreFilter && warp >= 2 && warp < 6) {
    for (int qs = lane; qs < nq_here; qs += 32) o.staged[((seq * nq + q0 + qs) * G + g) * 4 + (warp & 3)] = 0;
  }
  // Every role has left its loop, so the abort flag is final.  After a
  // failed wait, the producer lets its copies still in flight land and the
  // MMA warp waits for its own MMAs (full time bound) before shared memory and
  // TMEM are released.
  __syncthreads();
  if (sm.abort && n_tiles > 0) {
    if (warp == 0) {
      tc::mbar_drain(bar(sm.b_full), 0);
      for (int c = issued > kIdxStages ? issued - kIdxStages : 0; c < issued; ++c)
        tc::mbar_drain(bar(sm.a_full[c % kIdxStages]), (c / kIdxStages) & 1);
    } else if (warp == 1) {
      if (tc::elect_one()) tc::mma_commit(bar(sm.drain));
      __syncwarp();
      tc::mbar_drain(bar(sm.drain), 0);
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Exact top-k of materialised score rows in two passes over the row.  Pass 1
// counts the top 11 bits of every order-preserving key into a private
// histogram per warp (two 16-bit counters per word: warps never contend);
// their sum locates the bin holding the k-th score.  Pass 2 marks every
// entry of a higher bin in a bitmap and gathers the boundary bin's (key, id)
// pairs, of which one warp radix-selects the remainder (ties to the smaller
// id).  The bitmap is read out in id order, so the output is ascending.  One
// CTA per row; a row whose boundary bin overflows the gather buffer is flagged
// in `overflow` for topk_rows_kernel.
constexpr int kRows2Threads = 512;
constexpr int kRows2Warps = kRows2Threads / 32;
constexpr int kRows2Bins = 2048;
constexpr int kRows2Cand = 4096;

__global__ void __launch_bounds__(kRows2Threads, 2)
topk_rows2_kernel(const float* __restrict__ scores, int64_t rpad, int64_t nq, int G, int64_t q_pos0, int B,
                  int k, int nwords, int32_t* __restrict__ sel, int32_t* __restrict__ sel_count,
                  int32_t* __restrict__ overflow, int32_t* __restrict__ list, int32_t* __restrict__ list_count) {
  extern __shared__ uint32_t sm2[];
  uint32_t* wh = sm2;                                                     // [16][1024] packed u16 pairs
  uint2* cand = reinterpret_cast<uint2*>(sm2 + kRows2Warps * kRows2Bins / 2);  // [kRows2Cand]
  uint32_t* bits = sm2 + kRows2Warps * kRows2Bins / 2 + 2 * kRows2Cand;       // [nwords]
  __shared__ int warp_sums[kRows2Warps];
  __shared__ uint32_t s_bin, s_rem, s_nc;
  const int64_t row = blockIdx.x;
  const int64_t i = (row / G) % nq;
  const int64_t n = (q_pos0 + i) / B;
  const float* srow = scores + row * rpad;
  int32_t* out = sel + row * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int j = tid; j < k; j += kRows2Threads) out[j] = j < n ? j : -1;
    if (tid == 0) { sel_count[row] = static_cast<int32_t>(n); overflow[row] = 0; }
    return;
  }
  uint32_t* myh = wh + warp * (kRows2Bins / 2);
  for (int b = lane; b < kRows2Bins / 2; b += 32) myh[b] = 0;
  const int nw = static_cast<int>((n + 31) / 32);
  for (int w = tid; w < nw; w += kRows2Threads) bits[w] = 0;
  if (tid == 0) s_nc = 0;
  __syncwarp();
  for (int64_t j = tid; j < n; j += kRows2Threads) {
    const uint32_t bin = score_key(srow[j]) >> 21;
    atomicAdd(&myh[bin >> 1], 1u << (16 * (bin & 1)));
  }
  __syncthreads();
  // 4 bins per thread, from the top
  {
    uint32_t loc[4], sum = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int b = kRows2Bins - 1 - (tid * 4 + q);
      uint32_t c = 0;
#pragma unroll 4
      for (int w = 0; w < kRows2Warps; ++w) c += (wh[w * (kRows2Bins / 2) + (b >> 1)] >> (16 * (b & 1))) & 0xFFFFu;
      loc[q] = c;
      sum += c;
    }
    uint32_t x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { uint32_t y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
    if (lane == 31) warp_sums[warp] = static_cast<int>(x);
    __syncthreads();
    if (warp == 0) {
      int w = lane < kRows2Warps ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) { int y = __shfl_up_sync(0xffffffffu, w, o); if (lane >= o) w += y; }
      if (lane < kRows2Warps) warp_sums[lane] = w;
    }
    __syncthreads();
    const uint32_t before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - sum;
    const uint32_t kk = static_cast<uint32_t>(k);
    if (before < kk && kk <= before + sum) {
      uint32_t acc = before;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (acc < kk && kk <= acc + loc[q]) { s_bin = kRows2Bins - 1 - (tid * 4 + q); s_rem = kk - acc; }
        acc += loc[q];
      }
    }
    __syncthreads();
  }
  const uint32_t bstar = s_bin, rem = s_rem;
  // pass 2: higher bins into the bitmap, the boundary bin gathered (one atomic per warp)
  for (int64_t j0 = 0; j0 < n; j0 += kRows2Threads) {
    const int64_t j = j0 + tid;
    uint32_t key = 0, bin = 0;
    if (j < n) {
      key = score_key(srow[j]);
      bin = key >> 21;
      if (bin > bstar) atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
    const bool g2 = j < n && bin == bstar;
    const uint32_t bal = __ballot_sync(0xffffffffu, g2);
    if (bal) {
      uint32_t base = 0;
      if (lane == __ffs(bal) - 1) base = atomicAdd(&s_nc, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, __ffs(bal) - 1);
      const uint32_t pos = base + __popc(bal & ((1u << lane) - 1u));
      if (g2 && pos < kRows2Cand) cand[pos] = make_uint2(key, static_cast<uint32_t>(j));
    }
  }
  __syncthreads();
  const uint32_t nc = s_nc;
  if (nc > kRows2Cand) {  // boundary bin too large for the gather buffer
    if (tid == 0) {
      overflow[row] = 1;
      list[atomicAdd(list_count, 1)] = static_cast<int32_t>(row);
    }
    return;
  }
  if (warp == 0) {
    uint32_t theta = 0, id_cut = 0xFFFFFFFFu;
    if (nc > rem) warp_select(cand, static_cast<int>(nc), static_cast<int>(rem), wh, theta, id_cut);
    for (uint32_t c = lane; c < nc; c += 32) {
      const uint2 e = cand[c];
      if (nc <= rem || kept(e, theta, id_cut)) atomicOr(&bits[e.y >> 5], 1u << (e.y & 31));
    }
  }
  __syncthreads();
  // read the bitmap out in id order
  const int per = (nw + kRows2Threads - 1) / kRows2Threads;
  const int w0 = tid * per, w1 = min(nw, w0 + per);
  int local = 0;
  for (int w = w0; w < w1; ++w) local += __popc(bits[w]);
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) { int y = __shfl_up_sync(0xffffffffu, x, o); if (lane >= o) x += y; }
  __syncthreads();
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kRows2Warps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) { int y = __shfl_up_sync(0xffffffffu, w, o); if (lane >= o) w += y; }
    if (lane < kRows2Warps) warp_sums[lane] = w;
  }
  __syncthreads();
  int pos = (warp > 0 ? warp_sums[warp - 1] : 0) + x - local;
  for (int w = w0; w < w1; ++w) {
    uint32_t b = bits[w];
    while (b) {
      const int t = __ffs(b) - 1;
      b &= b - 1;
      if (pos < k) out[pos] = w * 32 + t;
      ++pos;
    }
  }
  if (tid == kRows2Threads - 1) {
    sel_count[row] = k;
    overflow[row] = 0;
    if (pos != k) report(kDevBounds);
  }
}

// ---------------------------------------------------------------------------
// Top-k for rows of 2048 .. kHistMaxCand candidates (every prefill row up to a
// 131072-token context).  One 128-thread CTA per row, about 22 KB of shared
// memory, so many rows are in flight per SM; the row streams through
// registers.
//
// Survivor filter (rows of more than 4k candidates): a sample of an eighth of
// the row (every eighth float4) gives a threshold T expected to pass about 2k
// candidates; one pass over the row appends the survivors (score >= T) as
// (score, id) to a shared list, one atomic per warp and batch.  If at least k
// survive, the k largest of the row are all among them; otherwise (or if too
// many survive) the exact step below runs over the whole row instead.
//
// Exact step (over the survivors, or the whole row): a 256-bin histogram of
// the scores, linear between their minimum and maximum, finds the bin b*
// holding the k-th largest.  Every step of the bin function rounds
// monotonically, so the bin never decreases as the score falls: each entry of
// a lower bin beats each entry of b*, and only b* needs the exact (score, then
// smaller id) order.  When b* holds more entries than the boundary buffer, a
// second 256-bin level splits b* the same way.  Selected ids are set in a
// bitmap read out in ascending id order.  A row whose boundary still
// overflows (massive exact ties) is flagged and listed for the radix kernel.
// ---------------------------------------------------------------------------
constexpr int kHistThreads = 128;
constexpr int kHistWarps = kHistThreads / 32;
constexpr int kHistBins = 256;         // 16-bit counters, two per word
constexpr int kHistBnd = 256;          // boundary entries resolved in the kernel
constexpr int kHistSurv = 2048;        // survivors of the sampled threshold
constexpr int kHistMaxCand = 16384;
constexpr int kHistSampPer = kHistMaxCand / 32 / kHistThreads;  // sample float4s per thread
constexpr int kHistBatch = 8;          // float4s per thread in flight in the survivor pass
constexpr uint32_t kHistRankMax = 64;  // boundary sets up to this size are ranked by all threads at once
static_assert(kHistBins == 2 * kHistThreads, "one histogram word (two bins) per thread in the bin scan");
static_assert(kHistMaxCand < 65536, "per-warp bin counts fit 16 bits");

struct HistSmem {
  uint32_t wh[kHistWarps][kHistBins / 2];  // per-warp histograms (also warp_select scratch)
  uint2 bnd[kHistBnd];                     // (key, id) of the boundary bin
  uint2 surv[kHistSurv];                   // survivors as (score bits, id)
  uint32_t bits[kHistMaxCand / 32];        // selection bitmap
  float rmax[kHistWarps], rmin[kHistWarps];
  uint32_t wsum[kHistWarps];
  uint32_t bstar, rem, cstar, nc, nsurv;
};

// A float in [2^23, 2^24) is an integer (ulp 1); adding 1.5 * 2^23 to a value
// in [0, 2^22) rounds it to the nearest integer, readable as the bit pattern
// minus that of 1.5 * 2^23.
constexpr float kRoundBase = 12582912.0f;
constexpr int kRoundBits = 0x4B400000;

__device__ __forceinline__ void hist_add(uint32_t* h, int b) { atomicAdd(&h[b >> 1], 1u << ((b & 1) * 16)); }

// Bins are ordered best first.  Finds the bin of sm.wh in which the running
// count reaches `need` (1 <= need <= total), its count, and the rank of `need`
// inside it (sm.bstar, sm.cstar, sm.rem).  Called by every thread of the CTA.
__device__ __forceinline__ void hist_boundary(HistSmem& sm, uint32_t need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t c0 = 0, c1 = 0;
#pragma unroll
  for (int w = 0; w < kHistWarps; ++w) {
    const uint32_t pr = sm.wh[w][tid];
    c0 += pr & 0xFFFFu;
    c1 += pr >> 16;
  }
  const uint32_t c = c0 + c1;
  uint32_t inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) sm.wsum[warp] = inc;
  __syncthreads();
  uint32_t before = inc - c;
  for (int w = 0; w < warp; ++w) before += sm.wsum[w];
  if (before < need && need <= before + c0) {
    sm.bstar = 2 * tid;
    sm.rem = need - before;
    sm.cstar = c0;
  } else if (before + c0 < need && need <= before + c) {
    sm.bstar = 2 * tid + 1;
    sm.rem = need - before - c0;
    sm.cstar = c1;
  }
  __syncthreads();
}

// Maximum and minimum over the CTA (every thread gets both; NaN inputs are
// ignored).
__device__ __forceinline__ void block_minmax(HistSmem& sm, float& mx, float& mn) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if (lane == 0) {
    sm.rmax[warp] = mx;
    sm.rmin[warp] = mn;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kHistWarps; ++w) {
    mx = fmaxf(mx, sm.rmax[w]);
    mn = fminf(mn, sm.rmin[w]);
  }
}

__device__ __forceinline__ void zero_hist(HistSmem& sm) {
  for (int b = threadIdx.x; b < kHistWarps * kHistBins / 2; b += kHistThreads) (&sm.wh[0][0])[b] = 0u;
}

__global__ void __launch_bounds__(kHistThreads)
topk_rows_hist_kernel(const float* __restrict__ scores, int64_t rpad, int64_t nq, int G, int64_t q_pos0, int B,
                      int k, int32_t* __restrict__ sel, int32_t* __restrict__ sel_count,
                      int32_t* __restrict__ overflow, int32_t* __restrict__ list, int32_t* __restrict__ list_count) {
  __shared__ HistSmem sm;
  const int64_t row = blockIdx.x;  // (seq * nq + i) * G + g
  const int64_t i = (row / G) % nq;
  const int n = static_cast<int>((q_pos0 + i) / B);
  const float* srow = scores + row * rpad;  // 16-byte aligned (rpad is a multiple of 128)
  const float4* r4 = reinterpret_cast<const float4*>(srow);
  int32_t* out = sel + row * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int j = tid; j < k; j += kHistThreads) out[j] = j < n ? j : -1;
    if (tid == 0) {
      sel_count[row] = n;
      overflow[row] = 0;
    }
    return;
  }
  if (tid == 0) {
    sm.nc = 0;
    sm.nsurv = 0;
    // the whole row (rounded up to float4s; the padded row has room) into L2
    // while the sample is read and binned
    tc::prefetch_l2(srow, static_cast<uint32_t>((n + 3) / 4) * 16u);
  }
  zero_hist(sm);
  for (int w = tid; w < kHistMaxCand / 32; w += kHistThreads) sm.bits[w] = 0u;
  __syncthreads();

  const int nwords = (n + 31) / 32;
  uint32_t* myh = sm.wh[warp];
  bool use_surv = false;
  float smax_surv = -INFINITY, smin_surv = INFINITY;
  if (n > 4 * k && 2 * k <= kHistSurv / 2) {
    // ---- sampled threshold: the float4s 8 j (candidates 32 j .. 32 j + 3),
    // held in registers; samples past the row are NaN (ignored by min/max)
    const int s4 = n / 32, s = 4 * s4;
    float4 sv[kHistSampPer];
#pragma unroll
    for (int q = 0; q < kHistSampPer; ++q) {
      const int j = tid + kHistThreads * q;
      sv[q] = j < s4 ? __ldg(r4 + 8 * j) : make_float4(NAN, NAN, NAN, NAN);
    }
    float smx = -INFINITY, smn = INFINITY;
#pragma unroll
    for (int q = 0; q < kHistSampPer; ++q) {
      smx = fmaxf(smx, fmaxf(fmaxf(sv[q].x, sv[q].y), fmaxf(sv[q].z, sv[q].w)));
      smn = fminf(smn, fminf(fminf(sv[q].x, sv[q].y), fminf(sv[q].z, sv[q].w)));
    }
    block_minmax(sm, smx, smn);
    const float sw = smx - smn;
    const float sscale = sw > 0.f ? 255.5f / sw : 0.f;
    // t = (max - x) * scale: bin b holds t in [b - 0.5, b + 0.5], sub-bin u of
    // b holds t in b + [u - 128.5, u - 127.5] / 256 (the exact step's bins)
    auto sbin1 = [&](float x) -> int {
      const float y = __fmaf_rn(__fsub_rn(smx, x), sscale, kRoundBase);
      return min(__float_as_int(y) - kRoundBits, kHistBins - 1);
    };
#pragma unroll
    for (int q = 0; q < kHistSampPer; ++q) {
      if (tid + kHistThreads * q < s4) {
        hist_add(myh, sbin1(sv[q].x));
        hist_add(myh, sbin1(sv[q].y));
        hist_add(myh, sbin1(sv[q].z));
        hist_add(myh, sbin1(sv[q].w));
      }
    }
    __syncthreads();
    // the sample rank that corresponds to about 2k candidates of the row
    const uint32_t r = static_cast<uint32_t>(min(static_cast<int>((2 * static_cast<int64_t>(k) * s + n - 1) / n), s));
    hist_boundary(sm, r);
    const int sb = static_cast<int>(sm.bstar);
    // threshold half a bin below the boundary bin's lower edge, or, when that
    // bin holds many samples, a sub-bin below its boundary sub-bin's
    float t_thr = static_cast<float>(sb) + 1.0f;
    if (sm.cstar > 16u) {
      const float sscale2 = sscale * 256.f;
      const float sbase2 = kRoundBase + 128.f - 256.f * static_cast<float>(sb);
      const uint32_t srem = sm.rem;
      zero_hist(sm);
      __syncthreads();
      auto sadd2 = [&](float x) {
        if (sbin1(x) == sb) {
          const float y = __fmaf_rn(__fsub_rn(smx, x), sscale2, sbase2);
          hist_add(myh, max(min(__float_as_int(y) - kRoundBits, kHistBins - 1), 0));
        }
      };
#pragma unroll
      for (int q = 0; q < kHistSampPer; ++q) {
        if (tid + kHistThreads * q < s4) {
          sadd2(sv[q].x);
          sadd2(sv[q].y);
          sadd2(sv[q].z);
          sadd2(sv[q].w);
        }
      }
      __syncthreads();
      hist_boundary(sm, srem);
      t_thr = static_cast<float>(sb) + (static_cast<float>(sm.bstar) - 126.5f) / 256.f;
    }
    const float thr = sscale > 0.f ? smx - t_thr / sscale : smx;
    // ---- survivors, batch by batch: each lane's passes as a bit mask, one
    // atomic per warp for the batch's positions
    const int nfull = n / 4;
    float smax = -INFINITY;  // largest survivor
    for (int base = 0; base < nfull; base += kHistThreads * kHistBatch) {
      float4 v[kHistBatch];
#pragma unroll
      for (int u = 0; u < kHistBatch; ++u) {
        const int j = base + kHistThreads * u + tid;
        v[u] = j < nfull ? __ldg(r4 + j) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
      uint32_t mask = 0;
#pragma unroll
      for (int u = 0; u < kHistBatch; ++u) {
        mask |= static_cast<uint32_t>(v[u].x >= thr) << (4 * u);
        mask |= static_cast<uint32_t>(v[u].y >= thr) << (4 * u + 1);
        mask |= static_cast<uint32_t>(v[u].z >= thr) << (4 * u + 2);
        mask |= static_cast<uint32_t>(v[u].w >= thr) << (4 * u + 3);
      }
      const uint32_t cnt = __popc(mask);
      uint32_t inc = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      uint32_t pos = 0;
      if (lane == 31 && inc) pos = atomicAdd(&sm.nsurv, inc);
      pos = __shfl_sync(0xffffffffu, pos, 31) + inc - cnt;
      // the lane's survivors, re-read from L1 (their lines were just loaded)
      while (mask) {
        const int b = __ffs(mask) - 1;
        mask &= mask - 1;
        const int id = 4 * (base + kHistThreads * (b >> 2) + tid) + (b & 3);
        const float x = __ldg(srow + id);
        if (pos < static_cast<uint32_t>(kHistSurv)) sm.surv[pos] = make_uint2(__float_as_uint(x), static_cast<uint32_t>(id));
        smax = fmaxf(smax, x);
        ++pos;
      }
    }
    for (int id = 4 * nfull + tid; id < n; id += kHistThreads) {
      const float x = srow[id];
      if (x >= thr) {
        const uint32_t p = atomicAdd(&sm.nsurv, 1u);
        if (p < static_cast<uint32_t>(kHistSurv)) sm.surv[p] = make_uint2(__float_as_uint(x), static_cast<uint32_t>(id));
        smax = fmaxf(smax, x);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    if (lane == 0) sm.rmax[warp] = smax;
    __syncthreads();
    const uint32_t total = sm.nsurv;
    use_surv = total >= static_cast<uint32_t>(k) && total <= static_cast<uint32_t>(kHistSurv);
    if (use_surv) {
      // every survivor lies in [thr, largest survivor]
      smin_surv = thr;
      for (int w = 0; w < kHistWarps; ++w) smax_surv = fmaxf(smax_surv, sm.rmax[w]);
    }
    zero_hist(sm);
    __syncthreads();
  }

  // ---- exact step over entries e < m: survivor e, or candidate e of the row
  const int m = use_surv ? static_cast<int>(sm.nsurv) : n;
  auto val = [&](int e) -> float { return use_surv ? __uint_as_float(sm.surv[e].x) : srow[e]; };
  auto idx = [&](int e) -> int { return use_surv ? static_cast<int>(sm.surv[e].y) : e; };
  float mx = smax_surv, mn = smin_surv;
  if (!use_surv) {
    for (int e = tid; e < m; e += kHistThreads) {
      const float x = val(e);
      mx = fmaxf(mx, x);
      mn = fminf(mn, x);
    }
    block_minmax(sm, mx, mn);
  }
  // level-1 bin: round((max - s) * 255.5 / (max - min)), 0 for the maximum,
  // at most 255; explicit roundings so every pass computes the same bin
  const float width = mx - mn;
  const float scale = width > 0.f ? 255.5f / width : 0.f;
  auto bin1 = [&](float x) -> int {
    const float y = __fmaf_rn(__fsub_rn(mx, x), scale, kRoundBase);
    return min(__float_as_int(y) - kRoundBits, kHistBins - 1);
  };
  for (int e = tid; e < m; e += kHistThreads) hist_add(myh, bin1(val(e)));
  __syncthreads();
  hist_boundary(sm, static_cast<uint32_t>(k));
  const int bstar = static_cast<int>(sm.bstar);
  uint32_t need = sm.rem;
  // level 2 (boundary bin too full): 256 sub-bins of b*, the same construction
  // with 256 times the scale; entries of b* land in [0, 256]
  const bool lvl2 = sm.cstar > static_cast<uint32_t>(kHistBnd);
  const float scale2 = scale * 256.f;
  const float base2 = kRoundBase + 128.f - 256.f * static_cast<float>(bstar);
  auto bin2 = [&](float x) -> int {
    const float y = __fmaf_rn(__fsub_rn(mx, x), scale2, base2);
    return max(min(__float_as_int(y) - kRoundBits, kHistBins - 1), 0);
  };
  int sstar = 0;
  if (lvl2) {
    zero_hist(sm);
    __syncthreads();
    for (int e = tid; e < m; e += kHistThreads) {
      const float x = val(e);
      if (bin1(x) == bstar) hist_add(myh, bin2(x));
    }
    __syncthreads();
    hist_boundary(sm, need);
    sstar = static_cast<int>(sm.bstar);
    need = sm.rem;
  }
  // entries ranked above the boundary go straight into the selection bitmap,
  // the boundary's are gathered as (key, id)
  const int msteps = (m + kHistThreads - 1) / kHistThreads;
  for (int it = 0; it < msteps; ++it) {
    const int e = it * kHistThreads + tid;
    const bool valid = e < m;
    const float x = valid ? val(e) : 0.f;
    const int id = valid ? idx(e) : 0;
    const int b = valid ? bin1(x) : kHistBins;
    bool above = b < bstar, eq = b == bstar;
    if (lvl2 && eq) {
      const int b2 = bin2(x);
      above = b2 < sstar;
      eq = b2 == sstar;
    }
    if (above) atomicOr(&sm.bits[id >> 5], 1u << (id & 31));
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    if (eb) {
      uint32_t base = 0;
      if (lane == 0) base = atomicAdd(&sm.nc, static_cast<uint32_t>(__popc(eb)));
      base = __shfl_sync(0xffffffffu, base, 0);
      const uint32_t p = base + __popc(eb & ((1u << lane) - 1u));
      if (eq && p < static_cast<uint32_t>(kHistBnd)) sm.bnd[p] = make_uint2(score_key(x), static_cast<uint32_t>(id));
    }
  }
  __syncthreads();
  const uint32_t nc = sm.nc;
  if (nc > static_cast<uint32_t>(kHistBnd)) {
    if (tid == 0) {
      overflow[row] = 1;
      list[atomicAdd(list_count, 1)] = static_cast<int32_t>(row);
    }
    return;
  }
  // the `need` best of the nc boundary entries (need <= nc)
  if (nc == need) {
    for (uint32_t c = tid; c < nc; c += kHistThreads) {
      const uint32_t id = sm.bnd[c].y;
      atomicOr(&sm.bits[id >> 5], 1u << (id & 31));
    }
  } else if (nc <= kHistRankMax) {
    if (static_cast<uint32_t>(tid) < nc) {
      const uint2 q = sm.bnd[tid];
      uint32_t r = 0;  // entries ranked ahead: larger key, or equal key and smaller id
      for (uint32_t j = 0; j < nc; ++j) {
        const uint2 f = sm.bnd[j];
        r += (f.x > q.x) | ((f.x == q.x) & (f.y < q.y));
      }
      if (r < need) atomicOr(&sm.bits[q.y >> 5], 1u << (q.y & 31));
    }
  } else if (warp == 0) {
    uint32_t theta = 0, id_cut = 0xFFFFFFFFu;
    warp_select(sm.bnd, static_cast<int>(nc), static_cast<int>(need), &sm.wh[0][0], theta, id_cut);
    for (uint32_t c = lane; c < nc; c += 32) {
      const uint2 q = sm.bnd[c];
      if (kept(q, theta, id_cut)) atomicOr(&sm.bits[q.y >> 5], 1u << (q.y & 31));
    }
  }
  __syncthreads();
  // ascending readout: thread t owns words [t * wpt, t * wpt + wpt)
  const int wpt = (nwords + kHistThreads - 1) / kHistThreads;
  const int w0 = tid * wpt;
  uint32_t cnt = 0;
  for (int w = 0; w < wpt; ++w)
    if (w0 + w < nwords) cnt += __popc(sm.bits[w0 + w]);
  uint32_t inc = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) sm.wsum[warp] = inc;
  __syncthreads();
  uint32_t pos = inc - cnt;
  for (int w = 0; w < warp; ++w) pos += sm.wsum[w];
  for (int w = 0; w < wpt; ++w) {
    if (w0 + w >= nwords) break;
    uint32_t wb = sm.bits[w0 + w];
    while (wb) {
      const int bit = __ffs(wb) - 1;
      wb &= wb - 1;
      if (pos < static_cast<uint32_t>(k)) out[pos] = 32 * (w0 + w) + bit;
      ++pos;
    }
  }
  if (tid == 0) {
    sel_count[row] = k;
    overflow[row] = 0;
  }
}


// ---------------------------------------------------------------------------
// Filtered selection for long rows (no FP32 score rows in HBM).  A sample of
// the scores (every samp-th candidate tile) gives each row a threshold below
// its rank-th largest sampled score, so about rank * samp candidates are
// expected to reach it; the full score pass then keeps only the (key, id)
// pairs at or above the threshold.  The selection stays exact: every
// candidate at or above the threshold is in the list, so if at least k are,
// the k largest are among them.  A row with fewer than k or more than its
// lists hold is flagged and redone from recomputed scores by the radix
// kernel.  Sizes (host side): k <= 512 keeps about 2k candidates in four
// lists of 1024; larger k about 3k in four lists of 2k.
// ---------------------------------------------------------------------------
constexpr int kThrRank = 64;                 // rank at the smallest sample stride, k <= 512
constexpr int kFilterCap = 4096;             // kept entries per row for k <= 512: four lists of kFilterCap / 4
constexpr int kFilterSubCap = kFilterCap / 4;
constexpr int kThrThreads = 256;
constexpr int kThrPer = 32;  // samples per thread (kSampleTilesMax tiles of 128)

__global__ void __launch_bounds__(kThrThreads)
index_threshold_kernel(const float* __restrict__ sample, int64_t ld, int64_t nq, int G, int64_t q_pos0, int B,
                       int samp, int thr_rank, float* __restrict__ thr) {
  __shared__ uint32_t wh[kThrThreads / 32][256];
  __shared__ float rmax[kThrThreads / 32], rmin[kThrThreads / 32];
  __shared__ uint32_t wsum[kThrThreads / 32];
  __shared__ int s_bstar, s_before, s_sub;
  const int64_t row = blockIdx.x;
  const int64_t i = (row / G) % nq;
  const int64_t n = (q_pos0 + i) / B;
  const float* srow = sample + row * ld;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // sample entry j = c * 128 + m is candidate (c * samp) * 128 + m
  auto cand_of = [samp](int j) -> int64_t { return static_cast<int64_t>(j / kIdxCand) * samp * kIdxCand + j % kIdxCand; };
  const int nsamp_tiles = static_cast<int>(((n + kIdxCand - 1) / kIdxCand + samp - 1) / samp);
  const int nj_all = nsamp_tiles * kIdxCand;
  // rows with more samples than the registers hold (contexts beyond 1M) use every step-th one
  const int step = (nj_all + kThrThreads * kThrPer - 1) / (kThrThreads * kThrPer);
  const int nj = (nj_all + step - 1) / step;
  float v[kThrPer];
  int nvalid = 0;
#pragma unroll
  for (int e = 0; e < kThrPer; ++e) {
    const int j = (tid + kThrThreads * e) * step;
    const bool ok = tid + kThrThreads * e < nj && cand_of(j) < n;
    v[e] = ok ? srow[j] : -INFINITY;
    nvalid += ok;
  }
  for (int b = tid; b < (kThrThreads / 32) * 256; b += kThrThreads) (&wh[0][0])[b] = 0u;
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int e = 0; e < kThrPer; ++e) {
    mx = fmaxf(mx, v[e]);
    if (v[e] != -INFINITY) mn = fminf(mn, v[e]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    nvalid += __shfl_xor_sync(0xffffffffu, nvalid, o);
  }
  if (lane == 0) {
    rmax[warp] = mx;
    rmin[warp] = mn;
    wsum[warp] = static_cast<uint32_t>(nvalid);
  }
  __syncthreads();
  int total = 0;
#pragma unroll
  for (int w = 0; w < kThrThreads / 32; ++w) {
    mx = fmaxf(mx, rmax[w]);
    mn = fminf(mn, rmin[w]);
    total += static_cast<int>(wsum[w]);
  }
  // the threshold sits below the (thr_rank / step)-th largest of the samples read
  const int rank = max(thr_rank / step, 1);
  if (total <= rank) {  // too few samples to estimate: keep everything
    if (tid == 0) thr[row] = -INFINITY;
    return;
  }
  const float width = mx - mn;
  const float scale = width > 0.f ? 255.5f / width : 0.f;
  auto bin_of = [&](float x) -> int { return min(static_cast<int>((mx - x) * scale), 255); };
#pragma unroll
  for (int e = 0; e < kThrPer; ++e)
    if (v[e] != -INFINITY) atomicAdd(&wh[warp][bin_of(v[e])], 1u);
  __syncthreads();
  {
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < kThrThreads / 32; ++w) c += wh[w][tid];  // tid < 256: one bin per thread
    uint32_t inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    __syncthreads();
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    uint32_t before = inc - c;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (before < static_cast<uint32_t>(rank) && static_cast<uint32_t>(rank) <= before + c) {
      s_bstar = tid;
      s_before = static_cast<int>(before);
    }
  }
  __syncthreads();
  // Second level: the boundary bin's samples in 256 sub-bins, so that the
  // threshold sits close below the rank-th largest sample even where one bin
  // of the first level holds many samples (the kept count, about
  // rank * samp, would otherwise grow by that bin's samples times samp).
  const int bstar = s_bstar;
  for (int b = tid; b < (kThrThreads / 32) * 256; b += kThrThreads) (&wh[0][0])[b] = 0u;
  __syncthreads();
  const float scale2 = scale * 256.f;
  auto sub_of = [&](float x) -> int {
    return min(max(static_cast<int>((mx - x) * scale2) - 256 * bstar, 0), 255);
  };
#pragma unroll
  for (int e = 0; e < kThrPer; ++e)
    if (v[e] != -INFINITY && bin_of(v[e]) == bstar) atomicAdd(&wh[warp][sub_of(v[e])], 1u);
  __syncthreads();
  {
    const uint32_t rank2 = static_cast<uint32_t>(rank - s_before);
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < kThrThreads / 32; ++w) c += wh[w][tid];
    uint32_t inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    __syncthreads();
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    uint32_t before = inc - c;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    // the last sub-bin takes the samples the clamp moved there (rounding)
    if ((before < rank2 && rank2 <= before + c) || (tid == 255 && before + c < rank2)) s_sub = tid;
  }
  __syncthreads();
  if (tid == 0) {
    // every sample of bin b*, sub-bin s* (and above) lies above about
    // mx - (256 b* + s* + 1) / scale2; a small margin covers the rounding
    float t = scale > 0.f ? mx - static_cast<float>(256 * bstar + s_sub + 1) / scale2 : mx;
    t -= fabsf(t) * 1e-6f + 1e-30f;
    thr[row] = t;
  }
}

// Exact top-k of a row's staged (key, id) list; ascending ids.  Rows with too
// few or too many kept entries are flagged for the fallback.
constexpr int kStagedThreads = 256;
constexpr int kStagedPer = kFilterCap / kStagedThreads;  // 16

__global__ void __launch_bounds__(kStagedThreads)
topk_staged_kernel(const uint2* __restrict__ staging, const int32_t* __restrict__ staged, int64_t nq, int G,
                   int64_t q_pos0, int B, int k, int cap, int nwords_max, int32_t* __restrict__ sel,
                   int32_t* __restrict__ sel_count, int32_t* __restrict__ flags, int32_t* __restrict__ list,
                   int32_t* __restrict__ list_count) {
  extern __shared__ uint32_t dyn[];
  uint2* cand = reinterpret_cast<uint2*>(dyn);                 // [kFilterCap]
  uint32_t* bits = dyn + 2 * kFilterCap;                       // [nwords_max]
  __shared__ uint32_t wh[kStagedThreads / 32][256];
  __shared__ float rmax[kStagedThreads / 32], rmin[kStagedThreads / 32];
  __shared__ uint32_t wsum[kStagedThreads / 32];
  __shared__ uint32_t s_bstar, s_rem, s_nc;
  const int64_t row = blockIdx.x;
  const int64_t i = (row / G) % nq;
  const int n = static_cast<int>((q_pos0 + i) / B);
  int32_t* out = sel + row * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int j = tid; j < k; j += kStagedThreads) out[j] = j < n ? j : -1;
    if (tid == 0) {
      sel_count[row] = n;
      flags[row] = 0;
    }
    return;
  }
  // the row's four lists (one per candidate quadrant of the score kernel)
  const int4 c4 = *reinterpret_cast<const int4*>(staged + row * 4);
  const int cnt = c4.x + c4.y + c4.z + c4.w;
  if (cnt < k || c4.x > cap || c4.y > cap || c4.z > cap || c4.w > cap) {
    if (tid == 0) {
      flags[row] = 1;
      list[atomicAdd(list_count, 1)] = static_cast<int32_t>(row);
    }
    return;
  }
  const int p1 = c4.x, p2 = p1 + c4.y, p3 = p2 + c4.z;
  const uint2* lists = staging + row * 4 * static_cast<int64_t>(cap);
  auto entry = [&](int j) -> uint2 {
    const int q = (j >= p1) + (j >= p2) + (j >= p3);
    const int off = j - (q == 0 ? 0 : q == 1 ? p1 : q == 2 ? p2 : p3);
    return lists[q * static_cast<int64_t>(cap) + off];
  };
  const int nw = (n + 31) / 32;
  for (int w = tid; w < nw; w += kStagedThreads) bits[w] = 0u;
  for (int b = tid; b < (kStagedThreads / 32) * 256; b += kStagedThreads) (&wh[0][0])[b] = 0u;
  if (tid == 0) s_nc = 0;
  uint2 e[kStagedPer];
  float v[kStagedPer];
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int x = 0; x < kStagedPer; ++x) {
    const int j = tid + kStagedThreads * x;
    e[x] = j < cnt ? entry(j) : make_uint2(0u, 0xFFFFFFFFu);
    v[x] = j < cnt ? key_score(e[x].x) : -INFINITY;
    mx = fmaxf(mx, v[x]);
    if (j < cnt) mn = fminf(mn, v[x]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if (lane == 0) {
    rmax[warp] = mx;
    rmin[warp] = mn;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kStagedThreads / 32; ++w) {
    mx = fmaxf(mx, rmax[w]);
    mn = fminf(mn, rmin[w]);
  }
  const float width = mx - mn;
  const float scale = width > 0.f ? 255.5f / width : 0.f;
  auto bin_of = [&](float x) -> int { return min(static_cast<int>((mx - x) * scale), 255); };
#pragma unroll
  for (int x = 0; x < kStagedPer; ++x)
    if (tid + kStagedThreads * x < cnt) atomicAdd(&wh[warp][bin_of(v[x])], 1u);
  __syncthreads();
  {
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < kStagedThreads / 32; ++w) c += wh[w][tid];
    uint32_t inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    uint32_t before = inc - c;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    const uint32_t kk = static_cast<uint32_t>(k);
    if (before < kk && kk <= before + c) {
      s_bstar = static_cast<uint32_t>(tid);
      s_rem = kk - before;
    }
  }
  __syncthreads();
  const int bstar = static_cast<int>(s_bstar);
  const uint32_t rem = s_rem;
  // higher bins into the bitmap, the boundary bin gathered
#pragma unroll
  for (int x = 0; x < kStagedPer; ++x) {
    if (tid + kStagedThreads * x >= cnt) continue;
    const int b = bin_of(v[x]);
    if (b < bstar) {
      atomicOr(&bits[e[x].y >> 5], 1u << (e[x].y & 31));
    } else if (b == bstar) {
      const uint32_t pos = atomicAdd(&s_nc, 1u);
      cand[pos] = e[x];
    }
  }
  __syncthreads();
  const uint32_t nc = s_nc;
  if (warp == 0) {
    uint32_t theta = 0, id_cut = 0xFFFFFFFFu;
    if (nc > rem) warp_select(cand, static_cast<int>(nc), static_cast<int>(rem), wh[0], theta, id_cut);
    for (uint32_t c = lane; c < nc; c += 32) {
      const uint2 x = cand[c];
      if (nc <= rem || kept(x, theta, id_cut)) atomicOr(&bits[x.y >> 5], 1u << (x.y & 31));
    }
  }
  __syncthreads();
  // ascending readout: thread t owns words [t * per, t * per + per)
  const int per = (nw + kStagedThreads - 1) / kStagedThreads;
  uint32_t cntw = 0;
  for (int w = tid * per; w < min(nw, tid * per + per); ++w) cntw += __popc(bits[w]);
  uint32_t inc = cntw;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t pos = inc - cntw;
  for (int w = 0; w < warp; ++w) pos += wsum[w];
  for (int w = tid * per; w < min(nw, tid * per + per); ++w) {
    uint32_t wb = bits[w];
    while (wb) {
      const int bit = __ffs(wb) - 1;
      wb &= wb - 1;
      if (pos < static_cast<uint32_t>(k)) out[pos] = 32 * w + bit;
      ++pos;
    }
  }
  if (tid == 0) {
    sel_count[row] = k;
    flags[row] = 0;
  }
}

// Exact top-k of a row's staged (key, id) lists for k > 512 (up to 2048),
// from up to four lists of 4096 entries: 1024 threads hold 16 entries each.
// A linear 2048-bin histogram between the kept scores' minimum and maximum
// finds the bin holding the k-th largest; entries of higher bins are taken,
// the boundary bin's entries are ranked exactly (score, then smaller id) by
// one warp (by counting when there are at most 64); a boundary bin too full
// for its buffer is split once more into 2048 sub-bins, and a sub-bin still
// too full (exact ties) is resolved by key and id threshold searches.  Each list holds its ids
// ascending (the score kernel appends candidate tiles in order), so the taken
// entries of a list stay ascending: the output is the merge of four sorted
// runs -- each taken entry's place is its rank in its own run plus, in each
// other run, the number of taken ids below its own (a binary search).  Rows
// with fewer than k kept entries or an overflowing list are flagged and
// listed for the fallback.
constexpr int kStagedBigThreads = 1024;
constexpr int kStagedBigPer = 16;
constexpr int kStagedBigBnd = 4096;  // boundary entries resolved in the kernel
constexpr int kStagedBigBins = 2048;
constexpr int kStagedBigWarps = kStagedBigThreads / 32;
constexpr int kStagedBigEntries = kStagedBigThreads * kStagedBigPer;
struct StagedBigSmem {
  uint2 bnd[kStagedBigBnd];                   // boundary entries (key, id)
  uint32_t bj[kStagedBigBnd];                 // their entry indices
  uint32_t hist[kStagedBigBins];              // (then warp_select's counters)
  uint32_t tbits[kStagedBigEntries / 32];     // taken entries, bit j = entry j
  uint32_t wpre[kStagedBigEntries / 32];      // taken entries before each word
  uint32_t T[2048];                           // taken ids, the four runs one after the other
  float rmax[kStagedBigWarps], rmin[kStagedBigWarps];
  uint32_t wsum[kStagedBigWarps];
  uint32_t wk[4][kStagedBigWarps];            // per-warp key / id ranges
  uint2 cut;                                  // (key, id) thresholds of a tied sub-bin
  uint32_t bstar, rem, cstar, nb, runs[5];
};

// Bin of a score: bins ordered best first, 2048 across [mn, mx]; the product
// rounds monotonically, so a higher score never falls in a later bin.
__device__ __forceinline__ int staged_bin(float mx, float scale, float x) {
  return min(static_cast<int>(__fmul_rn(__fsub_rn(mx, x), scale)), kStagedBigBins - 1);
}
// Sub-bin of a score of bin bstar: the fractional part of the same scaled
// distance (scaling by 2048 is exact), so the order stays monotone across levels.
__device__ __forceinline__ int staged_sub(float mx, float scale2, int bstar, float x) {
  return min(max(static_cast<int>(__fmul_rn(__fsub_rn(mx, x), scale2)) - kStagedBigBins * bstar, 0),
             kStagedBigBins - 1);
}

// The rem best entries (score, then smaller id) of sub-bin sstar of bin bstar,
// when there are more of them than the boundary buffer holds: the largest key
// K with at least rem entries at or above it, then the smallest id X with
// enough entries of key K at or below it.  Entries above K, and those of key K
// with id <= X, are the ones taken (ids are distinct, so exactly rem).
// Returns (K, X).  Called by every thread of the block.
__device__ __forceinline__ uint2 staged_tie_cut(StagedBigSmem& sm, const uint2* __restrict__ lists, int cap, int p1,
                                               int p2, int p3, int cnt, float mx, float scale, float scale2,
                                               int bstar, int sstar, uint32_t rem) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // entry x of this thread, if it lies in the boundary sub-bin (else key 0);
  // read again from the lists (L2) on every pass, which keeps registers free
  auto load = [&](int x) -> uint2 {
    const int j = tid + kStagedBigThreads * x;
    if (j >= cnt) return make_uint2(0u, 0u);
    const int q = (j >= p1) + (j >= p2) + (j >= p3);
    const uint2 en = lists[q * static_cast<int64_t>(cap) + (j - (q == 0 ? 0 : q == 1 ? p1 : q == 2 ? p2 : p3))];
    const float v = key_score(en.x);
    const bool in = staged_bin(mx, scale, v) == bstar && staged_sub(mx, scale2, bstar, v) == sstar;
    return in ? en : make_uint2(0u, 0u);
  };
  uint32_t k0 = 0xFFFFFFFFu, k1 = 0u, i0 = 0xFFFFFFFFu, i1 = 0u;
#pragma unroll 4
  for (int x = 0; x < kStagedBigPer; ++x) {
    const uint2 en = load(x);
    if (en.x != 0u) {  // every real key is above 0
      k0 = min(k0, en.x);
      k1 = max(k1, en.x);
      i0 = min(i0, en.y);
      i1 = max(i1, en.y);
    }
  }
  k0 = __reduce_min_sync(0xffffffffu, k0);
  k1 = __reduce_max_sync(0xffffffffu, k1);
  i0 = __reduce_min_sync(0xffffffffu, i0);
  i1 = __reduce_max_sync(0xffffffffu, i1);
  __syncthreads();  // every thread has read the previous scan's totals
  if (lane == 0) {
    sm.wk[0][warp] = k0;
    sm.wk[1][warp] = k1;
    sm.wk[2][warp] = i0;
    sm.wk[3][warp] = i1;
  }
  __syncthreads();
  for (int w = 0; w < kStagedBigWarps; ++w) {
    k0 = min(k0, sm.wk[0][w]);
    k1 = max(k1, sm.wk[1][w]);
    i0 = min(i0, sm.wk[2][w]);
    i1 = max(i1, sm.wk[3][w]);
  }
  // number of boundary entries with key >= kmin and (key > kmax or id <= xmax), over the block
  auto block_count = [&](uint32_t kmin, uint32_t kmax, uint32_t xmax) -> uint32_t {
    uint32_t c = 0;
#pragma unroll 4
    for (int x = 0; x < kStagedBigPer; ++x) {
      const uint2 en = load(x);
      c += en.x != 0u && en.x >= kmin && (en.x > kmax || en.y <= xmax);
    }
    c = __reduce_add_sync(0xffffffffu, c);
    __syncthreads();  // every thread has read the previous counts
    if (lane == 0) sm.wsum[warp] = c;
    __syncthreads();
    uint32_t t = 0;
    for (int w = 0; w < kStagedBigWarps; ++w) t += sm.wsum[w];
    return t;
  };
  uint32_t lo = k0, hi = k1;  // every boundary entry has key >= k0, and there are >= rem of them
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo + 1) / 2;
    if (block_count(mid, 0u, 0xFFFFFFFFu) >= rem) lo = mid;  // key >= mid
    else hi = mid - 1;
  }
  const uint32_t kcut = lo;
  lo = i0;
  hi = i1;  // key > K, or key == K and id <= i1: all entries at or above K, >= rem
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo) / 2;
    if (block_count(kcut, kcut, mid) >= rem) hi = mid;
    else lo = mid + 1;
  }
  return make_uint2(kcut, lo);
}

__global__ void __launch_bounds__(kStagedBigThreads)
topk_staged_sort_kernel(const uint2* __restrict__ staging, const int32_t* __restrict__ staged, int64_t nq, int G,
                        int64_t q_pos0, int B, int k, int cap, int32_t* __restrict__ sel,
                        int32_t* __restrict__ sel_count, int32_t* __restrict__ flags, int32_t* __restrict__ list,
                        int32_t* __restrict__ list_count) {
  extern __shared__ __align__(16) uint8_t dyn_raw[];
  StagedBigSmem& sm = *reinterpret_cast<StagedBigSmem*>(dyn_raw);
  const int64_t row = blockIdx.x;
  const int64_t i = (row / G) % nq;
  const int64_t n = (q_pos0 + i) / B;
  int32_t* out = sel + row * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int j = tid; j < k; j += kStagedBigThreads) out[j] = j < n ? j : -1;
    if (tid == 0) {
      sel_count[row] = static_cast<int32_t>(n);
      flags[row] = 0;
    }
    return;
  }
  const int4 c4 = *reinterpret_cast<const int4*>(staged + row * 4);
  const int cnt = c4.x + c4.y + c4.z + c4.w;
  auto flag_row = [&]() {
    if (tid == 0) {
      flags[row] = 1;
      list[atomicAdd(list_count, 1)] = static_cast<int32_t>(row);
    }
  };
  if (cnt < k || c4.x > cap || c4.y > cap || c4.z > cap || c4.w > cap || cnt > kStagedBigEntries) {
    flag_row();
    return;
  }
  const int p1 = c4.x, p2 = p1 + c4.y, p3 = p2 + c4.z;
  const uint2* lists = staging + row * 4 * static_cast<int64_t>(cap);
  auto run_of = [&](int j) { return (j >= p1) + (j >= p2) + (j >= p3); };
  auto entry = [&](int j) -> uint2 {
    const int q = run_of(j);
    const int off = j - (q == 0 ? 0 : q == 1 ? p1 : q == 2 ? p2 : p3);
    return lists[q * static_cast<int64_t>(cap) + off];
  };
  for (int b = tid; b < kStagedBigBins; b += kStagedBigThreads) sm.hist[b] = 0u;
  for (int w = tid; w < kStagedBigEntries / 32; w += kStagedBigThreads) sm.tbits[w] = 0u;
  if (tid == 0) sm.nb = 0;
  uint2 e[kStagedBigPer];  // (key, id); the score is key_score(key)
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int x = 0; x < kStagedBigPer; ++x) {
    const int j = tid + kStagedBigThreads * x;
    e[x] = j < cnt ? entry(j) : make_uint2(0u, 0xFFFFFFFFu);
    if (j < cnt) {
      const float v = key_score(e[x].x);
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
    sm.rmax[warp] = mx;
    sm.rmin[warp] = mn;
  }
  __syncthreads();
  for (int w = 0; w < kStagedBigWarps; ++w) {
    mx = fmaxf(mx, sm.rmax[w]);
    mn = fminf(mn, sm.rmin[w]);
  }
  const float width = mx - mn;
  const float scale = width > 0.f ? (kStagedBigBins - 0.5f) / width : 0.f;
  auto bin_of = [&](float x) -> int { return staged_bin(mx, scale, x); };
#pragma unroll
  for (int x = 0; x < kStagedBigPer; ++x)
    if (tid + kStagedBigThreads * x < cnt) atomicAdd(&sm.hist[bin_of(key_score(e[x].x))], 1u);
  __syncthreads();
  {  // thread t owns bins 2 t, 2 t + 1: the bin in which the running count reaches k
    const uint32_t c0 = sm.hist[2 * tid], c1 = sm.hist[2 * tid + 1];
    uint32_t x = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sm.wsum[warp] = x;
    __syncthreads();
    uint32_t before = x - c0 - c1;
    for (int w = 0; w < warp; ++w) before += sm.wsum[w];
    const uint32_t kk = static_cast<uint32_t>(k);
    if (before < kk && kk <= before + c0) {
      sm.bstar = 2 * tid;
      sm.rem = kk - before;
      sm.cstar = c0;
    } else if (before + c0 < kk && kk <= before + c0 + c1) {
      sm.bstar = 2 * tid + 1;
      sm.rem = kk - before - c0;
      sm.cstar = c1;
    }
  }
  __syncthreads();
  const int bstar = static_cast<int>(sm.bstar);
  uint32_t rem = sm.rem;
  // A boundary bin too full for its buffer (a few outlying scores stretch the
  // bins) is split once more: its entries in 2048 sub-bins of its own width.
  const float scale2 = scale * static_cast<float>(kStagedBigBins);
  auto sub_of = [&](float x) -> int { return staged_sub(mx, scale2, bstar, x); };
  const bool split = sm.cstar > kStagedBigBnd;  // (uniform)
  int sstar = -1;
  if (split) {
    __syncthreads();  // the first level's scan has read the histogram
    for (int b = tid; b < kStagedBigBins; b += kStagedBigThreads) sm.hist[b] = 0u;
    __syncthreads();
#pragma unroll
    for (int x = 0; x < kStagedBigPer; ++x) {
      const int j = tid + kStagedBigThreads * x;
      if (j < cnt) {
        const float v = key_score(e[x].x);
        if (bin_of(v) == bstar) atomicAdd(&sm.hist[sub_of(v)], 1u);
      }
    }
    __syncthreads();
    {
      const uint32_t c0 = sm.hist[2 * tid], c1 = sm.hist[2 * tid + 1];
      uint32_t x = c0 + c1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) sm.wsum[warp] = x;
      __syncthreads();
      uint32_t before = x - c0 - c1;
      for (int w = 0; w < warp; ++w) before += sm.wsum[w];
      if (before < rem && rem <= before + c0) {
        sm.bstar = 2 * tid;  // (reused: the sub-bin)
        sm.rem = rem - before;
        sm.cstar = c0;
      } else if (before + c0 < rem && rem <= before + c0 + c1) {
        sm.bstar = 2 * tid + 1;
        sm.rem = rem - before - c0;
        sm.cstar = c1;
      }
    }
    __syncthreads();
    sstar = static_cast<int>(sm.bstar);
    rem = sm.rem;
  }
  // A sub-bin still too full for the buffer holds (nearly) equal scores, e.g.
  // many exact zeros: its rem best entries are found by threshold searches
  // (on entries it reads again from the lists, so that the registers holding
  // this thread's own stay untouched).
  const bool wide = split && sm.cstar > kStagedBigBnd;  // (uniform)
  if (wide) {
    const uint2 cut = staged_tie_cut(sm, lists, cap, p1, p2, p3, cnt, mx, scale, scale2, bstar, sstar, rem);
    if (tid == 0) sm.cut = cut;
    __syncthreads();
  }
#pragma unroll
  for (int x = 0; x < kStagedBigPer; ++x) {
    const int j = tid + kStagedBigThreads * x;
    if (j >= cnt) continue;
    const float v = key_score(e[x].x);
    int b = bin_of(v);
    if (split && b == bstar) {  // order within the boundary bin by sub-bin
      const int sb = sub_of(v);
      b = sb < sstar ? bstar - 1 : (sb == sstar ? bstar : bstar + 1);
      if (wide && b == bstar) {  // resolved by the thresholds
        const uint2 cut = sm.cut;
        b = (e[x].x > cut.x || (e[x].x == cut.x && e[x].y <= cut.y)) ? bstar - 1 : bstar + 1;
      }
    }
    if (b < bstar) {
      atomicOr(&sm.tbits[j >> 5], 1u << (j & 31));
    } else if (b == bstar) {
      const uint32_t pos = atomicAdd(&sm.nb, 1u);
      sm.bnd[pos] = e[x];
      sm.bj[pos] = static_cast<uint32_t>(j);
    }
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t nb = sm.nb;
    auto take = [&](uint32_t c) { atomicOr(&sm.tbits[sm.bj[c] >> 5], 1u << (sm.bj[c] & 31)); };
    if (nb <= rem) {
      for (uint32_t c = lane; c < nb; c += 32) take(c);
    } else if (nb <= 64) {
      // rank by counting: an entry is taken if fewer than rem entries beat it (score, then smaller id)
      const uint2 e0 = lane < static_cast<int>(nb) ? sm.bnd[lane] : make_uint2(0u, 0xFFFFFFFFu);
      const uint2 e1 = lane + 32 < static_cast<int>(nb) ? sm.bnd[lane + 32] : make_uint2(0u, 0xFFFFFFFFu);
      uint32_t r0 = 0, r1 = 0;
      for (int q = 0; q < 32; ++q) {
        const uint2 f0 = make_uint2(__shfl_sync(0xffffffffu, e0.x, q), __shfl_sync(0xffffffffu, e0.y, q));
        const uint2 f1 = make_uint2(__shfl_sync(0xffffffffu, e1.x, q), __shfl_sync(0xffffffffu, e1.y, q));
        auto beats = [](uint2 f, uint2 g) { return f.x > g.x || (f.x == g.x && f.y < g.y); };
        const bool v0 = q < static_cast<int>(nb), v1 = q + 32 < static_cast<int>(nb);
        r0 += (v0 && beats(f0, e0)) + (v1 && beats(f1, e0));
        r1 += (v0 && beats(f0, e1)) + (v1 && beats(f1, e1));
      }
      if (lane < static_cast<int>(nb) && r0 < rem) take(lane);
      if (lane + 32 < static_cast<int>(nb) && r1 < rem) take(lane + 32);
    } else {
      uint32_t theta = 0, id_cut = 0xFFFFFFFFu;
      warp_select(sm.bnd, static_cast<int>(nb), static_cast<int>(rem), sm.hist, theta, id_cut);
      for (uint32_t c = lane; c < nb; c += 32)
        if (kept(sm.bnd[c], theta, id_cut)) take(c);
    }
  }
  __syncthreads();
  // taken entries before each bitmap word (exclusive scan over 512 words)
  if (tid < kStagedBigEntries / 32) {
    const uint32_t c = __popc(sm.tbits[tid]);
    uint32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sm.wsum[warp] = x;
    sm.wpre[tid] = x - c;  // within the warp; the earlier warps' totals are added below
  }
  __syncthreads();
  if (tid < kStagedBigEntries / 32) {
    uint32_t add = 0;
    for (int w = 0; w < warp; ++w) add += sm.wsum[w];
    sm.wpre[tid] += add;
  }
  __syncthreads();
  auto rank_all = [&](int j) -> uint32_t {  // taken entries before entry j
    return sm.wpre[j >> 5] + __popc(sm.tbits[j >> 5] & ((1u << (j & 31)) - 1u));
  };
  if (tid == 0) {  // (a run that starts at cnt is empty: every taken entry lies before it)
    sm.runs[0] = 0;
    sm.runs[1] = p1 < cnt ? rank_all(p1) : static_cast<uint32_t>(k);
    sm.runs[2] = p2 < cnt ? rank_all(p2) : static_cast<uint32_t>(k);
    sm.runs[3] = p3 < cnt ? rank_all(p3) : static_cast<uint32_t>(k);
    sm.runs[4] = static_cast<uint32_t>(k);
  }
#pragma unroll
  for (int x = 0; x < kStagedBigPer; ++x) {
    const int j = tid + kStagedBigThreads * x;
    if (j < cnt && ((sm.tbits[j >> 5] >> (j & 31)) & 1u)) sm.T[rank_all(j)] = e[x].y;
  }
  __syncthreads();
  // merge of the four ascending runs: place = own rank + taken ids below it in the other runs
#pragma unroll
  for (int x = 0; x < kStagedBigPer; ++x) {
    const int j = tid + kStagedBigThreads * x;
    if (j >= cnt || !((sm.tbits[j >> 5] >> (j & 31)) & 1u)) continue;
    const int q = run_of(j);
    const uint32_t id = e[x].y;
    uint32_t pos = rank_all(j) - sm.runs[q];
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2) {
      if (q2 == q) continue;
      uint32_t lo = sm.runs[q2], hi = sm.runs[q2 + 1];  // first taken id >= id in [lo, hi)
      const uint32_t base = lo;
      while (lo < hi) {
        const uint32_t mid = (lo + hi) >> 1;
        if (sm.T[mid] < id) lo = mid + 1;
        else hi = mid;
      }
      pos += lo - base;
    }
    if (pos < static_cast<uint32_t>(k)) out[pos] = static_cast<int32_t>(id);
  }
  if (tid == 0) {
    sel_count[row] = k;
    flags[row] = 0;
  }
}

// One flagged row's scores, recomputed by the whole CTA into srow.
__device__ __forceinline__ void index_score_fallback_row(int64_t row, const __nv_bfloat16* __restrict__ idx_q,
                                                         const float* __restrict__ idx_w,
                                                         const __nv_bfloat16* __restrict__ keys,
                                                         float* __restrict__ srow, int64_t nq, int G, int H,
                                                         int64_t q_pos0, int B, int64_t rpad, float (*qf)[64],
                                                         float* wf) {
  const int64_t i = (row / G) % nq;
  const int64_t seq = row / (static_cast<int64_t>(G) * nq);
  const int64_t n = (q_pos0 + i) / B;
  for (int x = threadIdx.x; x < H * 64; x += blockDim.x) qf[x / 64][x % 64] = __bfloat162float(idx_q[row * H * 64 + x]);
  if (threadIdx.x < H) wf[threadIdx.x] = idx_w[row * H + threadIdx.x];
  __syncthreads();
  const __nv_bfloat16* kb = keys + seq * rpad * 64;
  for (int64_t r = threadIdx.x; r < n; r += blockDim.x) {
    float kv[64];
    const uint4* src = reinterpret_cast<const uint4*>(kb + r * 64);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 u = src[c];
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        kv[8 * c + 2 * x] = __uint_as_float(w4[x] << 16);
        kv[8 * c + 2 * x + 1] = __uint_as_float(w4[x] & 0xFFFF0000u);
      }
    }
    float acc = 0.f;
    for (int h = 0; h < H; ++h) {
      float d = 0.f;
#pragma unroll
      for (int x = 0; x < 64; ++x) d = fmaf(qf[h][x], kv[x], d);
      acc = fmaf(wf[h], fmaxf(d, 0.f), acc);
    }
    srow[r] = acc;
  }
}

// Listed rows only (the rows the filtered path could not settle): each CTA
// recomputes a row's scores on the CUDA cores (FP32 dot products of the row's
// indexer queries with the widened keys) into its own slot of rpad floats,
// then radix-selects the row from it; a fixed grid strides over the list, so
// the scratch is grid x rpad floats whatever the number of rows.
__global__ void __launch_bounds__(kSelThreads)
index_fallback_select_kernel(const __nv_bfloat16* __restrict__ idx_q, const float* __restrict__ idx_w,
                             const __nv_bfloat16* __restrict__ keys, const int32_t* __restrict__ list,
                             const int32_t* __restrict__ list_count, float* __restrict__ slots, int64_t nq, int G,
                             int H, int64_t q_pos0, int B, int64_t rpad, int k, int32_t* __restrict__ sel,
                             int32_t* __restrict__ sel_count) {
  __shared__ float qf[8][64];
  __shared__ float wf[8];
  float* slot = slots + static_cast<int64_t>(blockIdx.x) * rpad;
  const int nlist = *list_count;
  for (int x = blockIdx.x; x < nlist; x += gridDim.x) {
    __syncthreads();  // the previous row's scores, qf and wf are no longer read
    const int64_t row = list[x];
    index_score_fallback_row(row, idx_q, idx_w, keys, slot, nq, G, H, q_pos0, B, rpad, qf, wf);
    __syncthreads();  // the slot holds the row's scores
    topk_row_radix_at<false>(row, slot, nq, G, q_pos0, B, k, sel, sel_count);
  }
}


}  // namespace sgqa
