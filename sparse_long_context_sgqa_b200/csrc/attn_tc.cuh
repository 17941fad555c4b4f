// Sparse attention for prefill on the 5th-generation tensor cores (tcgen05,
// TMEM accumulators, TMA-fed shared memory).  Page "Step-5-Preview: Sparse
// Reads Are Not a Compressed KV Cache", sections "Main attention still reads
// original K/V" and "What gets cheaper ..."; the second page's "group
// overlapping computations" of adjacent queries.
//
// One CTA takes one unit = (sequence, block of 8 adjacent queries, KV group).
// The MMA M dimension is the 8 queries x 16 heads = 128 rows, all sharing the
// group's K/V; the unit walks the sorted union of the 8 queries' selected
// blocks (built by attn_plan_kernel) 64 tokens at a time (8 blocks of 8, or
// 64 / BS blocks of BS < 8 tokens), then one tile holding the current-block
// tokens.  Blocks of 8 tokens arrive by TMA, one box per block; smaller
// blocks by cp.async row gathers into the same swizzled layout, their masks
// applied per token.
//
// Tensor memory (512 columns, one row per TMEM lane):
//   [0, 192)    O accumulator, FP32
//   [192, 320)  two S buffers of 64 FP32 columns
//   [320, 384)  two P buffers of 32 columns, two BF16 per column
//   [384, 480)  Q, two BF16 per column, written once per unit by the softmax warps
// An S buffer is free again as soon as the softmax has loaded it, a P buffer
// once O += P V has read it.
// Per 64-token tile j (buffers j % 2):
//   S = Q K^T   12 tcgen05.mma (M128 N64 K16), A = Q from TMEM, B = K (SMEM, K-major)
//   softmax     per-row block mask (the row's query must have selected the
//               block) and causal mask on the current block, running max in
//               log2 units with lazy rescaling of O (only when the max grows
//               by more than 2^8), P rounded to BF16 into its P buffer
//   O += P V    4 tcgen05.mma (M128 N192 K16), A = P from TMEM, B = V (SMEM, MN-major)
// The QK^T warp runs up to two tiles ahead of the PV warp (as far as the S
// buffers the softmax releases allow), so the softmax always finds the next
// scores computed; it waits on an O update only for the (rare) rescale.
// Warp roles: warp 0 streams K and warp 10 streams V by TMA (one 5-D box per
// 8-token block gathers all 192 dims: 3 KB), warp 1 allocates TMEM and issues
// the QK^T MMAs, warp 11 issues the PV MMAs, warps 2-9 run the softmax and
// the epilogue.  The producer and MMA
// warps run converged and hand each TMA or MMA batch to one elected lane:
// issuing from a lone divergent lane costs the tensor pipe several hundred
// cycles per tile in synchronisation stalls.  Every mbarrier wait is bounded
// (tc::mbar_wait / tc::warp_wait).
#pragma once
#include <cooperative_groups.h>

#include "attn_mma.cuh"
#include "tc.cuh"

namespace sgqa {

constexpr int kTcStages = 4;      // K ring depth (K freed after QK^T)
constexpr int kTcVStages = 4;     // V ring depth (V freed after PV)
constexpr int kTcThreads = 384;   // K producer, QK issuer, 8 softmax warps, V producer, PV issuer
constexpr int kTcTileTok = 64;    // tokens per KV tile = 8 blocks of 8

struct __align__(1024) AttnTcSmem {
  uint8_t k[kTcStages][8][3][1024];        // K tile: [block][chunk][8 rows x 128 B] (SW128)
  uint8_t v[kTcVStages][8][3][1024];       // V tile, same layout (MN-major operand)
  uint64_t q_full;                         // Q written to TMEM (256 softmax threads)
  uint64_t k_full[kTcStages], k_empty[kTcStages];
  uint64_t v_full[kTcVStages], v_empty[kTcVStages];
  uint64_t s_full[2];                      // S(j) in S buffer j % 2
  uint64_t s_free[2];                      // S(j) loaded by the softmax (the 128 threads of tile j's warps)
  uint64_t p_full[2];                      // P(j) in P buffer j % 2 (the 128 threads of tile j's warps)
  uint64_t pv_done[2];                     // O += P(j) V(j) complete: P buffer j % 2 free, O current
  uint64_t o_final, drain, drain_pv;
  float mchain[128];                       // running reference max after the latest tile, per row
  float lsum[2][128];                      // partial row sums of the two warps of a quadrant
  float gfac[128];                         // output gate factor per row (1 without a gate)
  uint32_t tmem;
  int abort;
};

// SKIP_PAIRS: skip the exponentials of block pairs that no row of a warp
// attends (pays when selections cover a small part of the context); otherwise
// all 64 exponentials of a tile run as one branch-free block.
// PAGED: the K/V live in a pool of 16-token pages [pages, G, 16, D] reached
// through page_table [S, max_pages] (the tensor maps cover the pool); a
// block's copy starts at (row 0 or 8 of its page, page).  Otherwise the maps
// cover the contiguous caches [S, cap, G, D] and a copy starts at (token row,
// sequence).
template <bool SKIP_PAIRS, bool PAGED, int BS>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __nv_bfloat16* __restrict__ q, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const int32_t* __restrict__ plan_ids,
               const uint8_t* __restrict__ plan_mask, const int32_t* __restrict__ plan_count,
               __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ gate, int64_t nq, int G,
               int k, int64_t q_pos0, float scale_log2, const int32_t* __restrict__ page_table, int64_t max_pages,
               int64_t num_pages, const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc,
               int64_t cache_cap, int64_t cache_len) {
  static_assert(BS == 1 || BS == 2 || BS == 4 || BS == 8, "block size");
  static_assert(BS == 8 || (!PAGED && !SKIP_PAIRS), "paged pools and pair skipping are for 8-token blocks");
  constexpr int E = kTcTileTok / BS;  // union entries (blocks) per 64-token tile
  extern __shared__ uint8_t smem_raw[];
  AttnTcSmem& sm = *reinterpret_cast<AttnTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                  ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Group-major order: CTAs resident together read one group's K/V (L2 reuse).
  const int64_t nqb = (nq + 7) / 8;
  const int64_t per_group = static_cast<int64_t>(gridDim.x) / G;
  const int g = static_cast<int>(blockIdx.x / per_group);
  const int64_t sq = blockIdx.x % per_group;       // seq * nqb + qb
  const int64_t qb = sq % nqb;
  const int64_t seq = sq / nqb;
  const int64_t unit = sq * G + g;                  // index of the plan arrays
  const int U = plan_count[unit];
  const int32_t* uid = plan_ids + unit * (8 * static_cast<int64_t>(k));
  const uint8_t* umask = plan_mask + unit * (8 * static_cast<int64_t>(k));
  const int n_union_tiles = (U + E - 1) / E;
  const int n_tiles = n_union_tiles + 1;
  const int64_t t_first = q_pos0 + qb * 8;
  const int64_t t_last = q_pos0 + min(nq, qb * 8 + 8) - 1;
  const int64_t c0 = 8 * (t_first / 8);  // first token of the current segment
  volatile int* abort = &sm.abort;

  auto bar = [](uint64_t& b) { return smem_u32(&b); };
  if (threadIdx.x == 0) {
    sm.abort = 0;
    tc::mbar_init(bar(sm.q_full), 256);
    // a full K/V stage: one TMA transaction count (8-token blocks) or the
    // 32 lanes of the copying warp (smaller blocks)
    for (int s = 0; s < kTcStages; ++s) {
      tc::mbar_init(bar(sm.k_full[s]), BS == 8 ? 1 : 32);
      tc::mbar_init(bar(sm.k_empty[s]), 1);
    }
    for (int s = 0; s < kTcVStages; ++s) {
      tc::mbar_init(bar(sm.v_full[s]), BS == 8 ? 1 : 32);
      tc::mbar_init(bar(sm.v_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(sm.s_full[b]), 1);
      tc::mbar_init(bar(sm.s_free[b]), 128);
      tc::mbar_init(bar(sm.p_full[b]), 128);
      tc::mbar_init(bar(sm.pv_done[b]), 1);
    }
    tc::mbar_init(bar(sm.o_final), 1);
    tc::mbar_init(bar(sm.drain), 1);
    tc::mbar_init(bar(sm.drain_pv), 1);
    tc::mbar_fence_init();
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(&sm.tmem), 512);
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = sm.tmem;
  const uint32_t tO = tmem;           // columns [0, 192)
  const uint32_t tS0 = tmem + 192;    // S buffers at [192, 256), [256, 320)
  const uint32_t tP0 = tmem + 320;    // P buffers at [320, 352), [352, 384)
  const uint32_t tQ = tmem + 384;     // Q at [384, 480)
  int issued = 0;                     // producers: tiles whose copies this warp issued

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------ producers
    // warp 0 streams K, warp 10 streams V: the rings drain at different points
    // (K after QK^T, V after PV), so each gets its own issuer.
    const bool is_k = warp == 0;
    const int nst = is_k ? kTcStages : kTcVStages;
    if constexpr (BS < 8) {
      // Blocks of fewer than 8 tokens: the 32 lanes gather the tile's 64
      // token rows with cp.async into the layout the TMA boxes produce
      // (8-row slots, 128-byte swizzle).  Piece L = 32 it + lane of the
      // tile's 64 x 24 sixteen-byte pieces is piece L % 24 of token L / 24,
      // so consecutive lanes read consecutive bytes of a row.  Row offsets
      // are 32-bit counts of 16-byte pieces (a sequence's K of one group up
      // to 2^31 pieces: 178 M tokens at 4 groups).
      const uint4* src0 = reinterpret_cast<const uint4*>((is_k ? kc : vc) + (seq * cache_cap * G + g) * static_cast<int64_t>(kD));
      const uint32_t rstride16 = static_cast<uint32_t>(G) * (kD / 8);  // 16-byte pieces between token rows
      // this lane's row offsets (16-byte units) of tile positions lane and
      // lane + 32, -1: a zero row; the union ids are fetched a tile before
      // they are needed (id_of), the offsets formed from them (row_of)
      auto id_of = [&](int j, int p) -> int32_t {
        const int idx = j * E + p / BS;
        return (j < n_union_tiles && idx < U) ? __ldg(uid + idx) : -1;
      };
      auto row_of = [&](int j, int p, int32_t id) -> int32_t {
        int64_t tk = -1;
        if (j < n_union_tiles) {
          if (id >= 0) tk = static_cast<int64_t>(id) * BS + p % BS;
          if (tk >= cache_len) tk = -1;
        } else if (p < 16 && c0 + p < cache_len) {
          tk = c0 + p;
        }
        return tk < 0 ? -1 : static_cast<int32_t>(tk * rstride16);
      };
      // Iteration it = 3 a + r copies piece c_r of token 4 a + p_r, where
      // 32 r + lane = 24 p_r + c_r; its destination is the same for every a
      // of one parity, plus (a >> 1) slots.
      uint32_t dstc[3][2];
      int pr[3], cr[3];
#pragma unroll
      for (int r = 0; r < 3; ++r) {
        pr[r] = (32 * r + lane) / 24;
        cr[r] = (32 * r + lane) % 24;
#pragma unroll
        for (int par = 0; par < 2; ++par) {
          const int row = 4 * par + pr[r];  // row within the 8-row slot
          dstc[r][par] = (cr[r] >> 3) * 1024 + row * 128 + (((cr[r] & 7) ^ row) << 4);
        }
      }
      int32_t ra = row_of(0, lane, id_of(0, lane)), rb = row_of(0, lane + 32, id_of(0, lane + 32));
      int32_t na = id_of(1, lane), nb = id_of(1, lane + 32);  // the next tile's ids
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % nst;
        uint64_t* empty = is_k ? &sm.k_empty[s] : &sm.v_empty[s];
        uint64_t* full = is_k ? &sm.k_full[s] : &sm.v_full[s];
        if (j >= nst && !tc::warp_wait(bar(*empty), ((j / nst) - 1) & 1, abort)) break;
        const uint32_t dst0 = is_k ? smem_u32(&sm.k[s][0][0][0]) : smem_u32(&sm.v[s][0][0][0]);
#pragma unroll
        for (int a = 0; a < 16; ++a) {
#pragma unroll
          for (int r = 0; r < 3; ++r) {
            const int32_t off = __shfl_sync(0xffffffffu, a < 8 ? ra : rb, (4 * a + pr[r]) & 31);
            cp_async16_zfill(dst0 + (a >> 1) * 3072 + dstc[r][a & 1], src0 + (off >= 0 ? off + cr[r] : 0), off >= 0);
          }
        }
        // the stage is full once every lane has arrived and its copies have
        // landed (the asynchronous arrive fires when they complete)
        cp_async_mbar_arrive(bar(*full));
        tc::mbar_arrive(bar(*full));
        issued = j + 1;
        ra = row_of(j + 1, lane, na);
        rb = row_of(j + 1, lane + 32, nb);
        na = id_of(j + 2, lane);
        nb = id_of(j + 2, lane + 32);
      }
      cp_async_commit();
      cp_async_wait<0>();  // nothing may land after the CTA's shared memory is released
    } else {
      if (tc::elect_one()) tc::prefetch_tmap(is_k ? &kmap : &vmap);
      __syncwarp();
      // Copy rows of the union's blocks, one per lane in batches of four tiles
      // (32 blocks), loaded a whole batch ahead: the id fetch (an L2 round trip,
      // plus the page-table read of a paged pool) never sits between two tiles'
      // copies.  Lane 8 t + e holds block e of tile 4 b + t.  A row is a token
      // row, or page * 16 + row within the page; negative: a zero-filled box.
      auto page_row = [&](int64_t tok) -> int32_t {  // paged pool: the row of token tok
        const int32_t pg = page_table[seq * max_pages + (tok >> 4)];
        if (pg < 0 || pg >= num_pages) {
          report(kDevBounds);
          return -64;
        }
        return pg * 16 + static_cast<int32_t>(tok & 15);
      };
      // contiguous caches: the raw ids (a row is id * 8); a paged pool: the rows
      auto load_batch = [&](int bt) -> int32_t {
        const int idx = 32 * bt + lane;
        const int32_t id = idx < U ? uid[idx] : -1;
        if (!PAGED) return id;
        return id < 0 ? -64 : page_row(static_cast<int64_t>(id) * 8);
      };
      int32_t ids_cur = load_batch(0), ids_next = n_union_tiles > 4 ? load_batch(1) : -1;
      // the current-block tile: the current block and, when the unit spans two blocks, the next
      int32_t cur_rows = -64;
      if (PAGED && lane < 2 && (lane == 0 || c0 + 8 <= t_last)) cur_rows = page_row(c0 + 8 * lane);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % nst;
        if (j > 0 && (j & 3) == 0) {
          ids_cur = ids_next;
          if (4 * (j / 4 + 1) < n_union_tiles) ids_next = load_batch(j / 4 + 1);
        }
        // this tile's eight copy rows (-64: a zero-filled box)
        int32_t rows[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int32_t id = __shfl_sync(0xffffffffu, ids_cur, 8 * (j & 3) + e);
          if (PAGED) {
            const int32_t r_cur = __shfl_sync(0xffffffffu, cur_rows, e & 1);
            rows[e] = j < n_union_tiles ? id : (e < 2 ? r_cur : -64);
          } else if (j < n_union_tiles) {
            rows[e] = id >= 0 ? id * 8 : -64;
          } else {  // the current block and, when the unit spans two blocks, the next
            rows[e] = (e == 0 || (e == 1 && c0 + 8 <= t_last)) ? static_cast<int32_t>(c0 + 8 * e) : -64;
          }
        }
        uint64_t* empty = is_k ? &sm.k_empty[s] : &sm.v_empty[s];
        uint64_t* full = is_k ? &sm.k_full[s] : &sm.v_full[s];
        if (j >= nst && !tc::warp_wait(bar(*empty), ((j / nst) - 1) & 1, abort)) break;
        if (tc::elect_one()) {
          tc::mbar_expect_tx(bar(*full), 8 * 3 * 1024);
          const CUtensorMap* map = is_k ? &kmap : &vmap;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t dst = is_k ? smem_u32(&sm.k[s][e][0][0]) : smem_u32(&sm.v[s][e][0][0]);
            const int32_t c1 = PAGED ? (rows[e] & 15) : rows[e];
            const int32_t c4 = PAGED ? (rows[e] >> 4) : static_cast<int32_t>(seq);
            tc::tma_load_5d(dst, map, 0, c1, 0, g, c4, bar(*full));
          }
        }
        __syncwarp();
        issued = j + 1;
      }
    }
  } else if (warp == 1 || warp == 11) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues S(j) = Q K(j)^T, warp 11 issues O += P(j) V(j).  They
    // touch disjoint TMEM (S buffers / O and P buffers) and each commit tracks
    // its own warp's MMAs, so neither waits on the other: the scores run up
    // to two tiles ahead (bounded by the S buffers the softmax releases) while
    // PV follows the softmax.
    const bool is_qk = warp == 1;
    const uint32_t id_qk = tc::idesc_bf16(128, 64, false);
    const uint32_t id_pv = tc::idesc_bf16(128, 192, true);
    // Base descriptors once per unit; each MMA adds a constant offset (in
    // 16-byte units, the descriptor's address field).  Stages are contiguous:
    // stage x starts x * 24 KB (1536 units) after stage 0.
    const uint64_t dk0 = tc::sdesc_sw128(smem_u32(&sm.k[0][0][0][0]), 16, 3072);
    const uint64_t dv0 = tc::sdesc_sw128(smem_u32(&sm.v[0][0][0][0]), 1024, 3072);
    bool ok = true;
    if (is_qk) {
      ok = tc::warp_wait(bar(sm.q_full), 0, abort);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kTcStages, b = j % 2;
        ok = tc::warp_wait(bar(sm.k_full[s]), (j / kTcStages) & 1, abort);
        // S buffer b is free once the softmax of tile j-2 has loaded it
        if (ok && j >= 2) ok = tc::warp_wait(bar(sm.s_free[b]), ((j / 2) - 1) & 1, abort);
        if (!ok) break;
        tc::fence_after();
        if (tc::elect_one()) {
          const uint64_t b0 = dk0 + 1536 * s;
#pragma unroll
          for (int kk = 0; kk < 12; ++kk)  // Q: 8 columns per 16 dims; K: +1 KB per 64 dims, +32 B per 16
            tc::mma_f16_tmem_a(tS0 + 64 * b, tQ + 8 * kk, b0 + (kk >> 2) * 64 + (kk & 3) * 2, id_qk,
                               kk > 0 ? 1u : 0u);
          tc::mma_commit(bar(sm.k_empty[s]));
          tc::mma_commit(bar(sm.s_full[b]));
        }
        __syncwarp();
      }
    } else {
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kTcVStages, b = j % 2;
        ok = tc::warp_wait(bar(sm.v_full[s]), (j / kTcVStages) & 1, abort) &&
             tc::warp_wait(bar(sm.p_full[b]), (j / 2) & 1, abort);
        if (!ok) break;
        tc::fence_after();
        if (tc::elect_one()) {
          const uint64_t b0 = dv0 + 1536 * s;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // P: 8 columns per 16 tokens; V: +2 blocks (6144 B) per 16 tokens
            tc::mma_f16_tmem_a(tO, tP0 + 32 * b + 8 * kk, b0 + 384 * kk, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(bar(sm.v_empty[s]));
          tc::mma_commit(bar(sm.pv_done[b]));
        }
        __syncwarp();
      }
      if (ok) {
        if (tc::elect_one()) tc::mma_commit(bar(sm.o_final));
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Eight warps, two per TMEM lane quadrant (both own the same 32 rows).  The
    // two take alternate tiles, so one warp's exponentials overlap the other's
    // TMEM load and row max on the same SM sub-partition.  The running
    // reference max is handed from tile to tile through shared memory: the
    // warp of tile j publishes it (bar.arrive) right after its row max, the
    // warp of tile j+1 picks it up (bar.sync) before computing P.  Each warp
    // keeps its own partial row sum; the two are combined in the epilogue.  A
    // failed wait clears `ok` but keeps every barrier step in place.
    const int sw = warp - 2;                 // 0..7
    const int quad = warp & 3;
    const int half = sw >> 2;                // this warp takes tiles j with j % 2 == half
    const int pair_bar = 1 + quad;           // both warps of this quadrant
    const int pub_mine = 5 + 2 * quad + half;         // this warp -> the other
    const int pub_other = 5 + 2 * quad + (half ^ 1);  // the other warp -> this one
    const int m = quad * 32 + lane;          // TMEM lane = row = (query slot, head)
    const int qs = m >> 4;
    const int64_t qi = qb * 8 + qs;
    const bool qvalid = qi < nq;
    const int64_t t = q_pos0 + (qvalid ? qi : qb * 8);
    const int64_t cur_lo = BS * (t / BS);
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int64_t orow_idx = ((seq * nq + (qvalid ? qi : 0)) * G + g) * kHg + (m & 15);
    if (half == 0) sm.gfac[m] = gate_factor(gate, orow_idx);  // read by both warps at the end
    // Q row m, dims [96 half, 96 half + 96), into TMEM columns tQ + 48 half ...
    {
      const uint4* src = reinterpret_cast<const uint4*>(q + orow_idx * kD + 96 * half);
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        uint32_t r[16];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const uint4 w = qvalid ? src[4 * c + x] : make_uint4(0u, 0u, 0u, 0u);
          r[4 * x + 0] = w.x;
          r[4 * x + 1] = w.y;
          r[4 * x + 2] = w.z;
          r[4 * x + 3] = w.w;
        }
        tc::tmem_st16(tQ + lane_off + 48 * half + 16 * c, r);
      }
      tc::tmem_st_wait();
      tc::fence_before();
      tc::mbar_arrive(bar(sm.q_full));
    }
    float m_l = -INFINITY, l = 0.f;          // this warp's partial row sum, relative to 2^m_l
    bool ok = true;
    // mask bytes of this warp's next tile, loaded one own tile (two tiles) ahead
    uint2 mb_next = make_uint2(0u, 0u);
    // blocks under 8 tokens: the mask bytes of tile positions lane and lane + 32
    auto tok_bytes = [&](int jj) -> uint2 {
      const int i0 = jj * E + lane / BS, i1 = jj * E + (lane + 32) / BS;
      return make_uint2(jj < n_union_tiles && i0 < U ? umask[i0] : 0u, jj < n_union_tiles && i1 < U ? umask[i1] : 0u);
    };
    if (BS == 8) {
      if (half < n_union_tiles) mb_next = *reinterpret_cast<const uint2*>(umask + 8 * half);
    } else {
      mb_next = tok_bytes(half);
    }
    for (int j = half; j < n_tiles; j += 2) {
      const int b = j % 2;
      const uint32_t tS = tS0 + 64 * b + lane_off;
      const uint32_t tP = tP0 + 32 * b + lane_off;
      const uint2 mb = mb_next;
      if (BS == 8) {
        if (j + 2 < n_union_tiles) mb_next = *reinterpret_cast<const uint2*>(umask + 8 * (j + 2));
      } else {
        mb_next = tok_bytes(j + 2);
      }
      // blocks (8 tokens each) of this tile the row attends: the row's query
      // selected the block, or (current tile) causal positions of its own block;
      // blocks under 8 tokens: a token mask (bit p: tile position p)
      uint32_t bmask = 0, tlo = 0, thi = 0;
      if (BS < 8 && j < n_union_tiles) {
        const int qa = 2 * quad, qb2 = 2 * quad + 1;
        const uint32_t la = __ballot_sync(0xffffffffu, (mb.x >> qa) & 1u), ha = __ballot_sync(0xffffffffu, (mb.y >> qa) & 1u);
        const uint32_t lb = __ballot_sync(0xffffffffu, (mb.x >> qb2) & 1u), hb = __ballot_sync(0xffffffffu, (mb.y >> qb2) & 1u);
        tlo = (lane >> 4) ? lb : la;
        thi = (lane >> 4) ? hb : ha;
        bmask = 0xFFu;
      } else if (j < n_union_tiles) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t byte = ((e < 4 ? mb.x : mb.y) >> (8 * (e & 3))) & 0xFFu;
          if (8 * j + e < U && ((byte >> qs) & 1u)) bmask |= 1u << e;
        }
      } else {
        bmask = 3u;
      }
      ok = ok && tc::mbar_wait(bar(sm.s_full[b]), (j / 2) & 1, abort);
      tc::fence_after();
      uint32_t sr[64];
      tc::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tc::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tc::tmem_ld_wait();
      tc::fence_before();
      tc::mbar_arrive(bar(sm.s_free[b]));
      // row max over the attended scores (the scale is positive: it commutes
      // with max).  Union tiles mask whole blocks: a block the row does not
      // attend gets the exponent offset -inf below instead of masked scores.
      float bm[8];
      if (BS < 8 && j < n_union_tiles) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          bm[e] = -INFINITY;
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const bool keep = (((e < 4 ? tlo : thi) >> (8 * (e & 3) + x)) & 1u) != 0u;
            const float v = keep ? __uint_as_float(sr[8 * e + x]) : -INFINITY;
            sr[8 * e + x] = __float_as_uint(v);
            bm[e] = fmaxf(bm[e], v);
          }
        }
      } else if (j < n_union_tiles) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float* x = reinterpret_cast<const float*>(&sr[8 * e]);
          const float mb = fmaxf(fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])), fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7])));
          bm[e] = ((bmask >> e) & 1u) ? mb : -INFINITY;
        }
      } else {
        // current tile: tokens c0 .. c0 + 15, of which the row attends cur_lo .. t
        const int lo = static_cast<int>(cur_lo - c0), hi = static_cast<int>(t - c0);  // 0 <= lo <= hi <= 15
        const uint32_t tm = ((2u << hi) - 1u) & ~((1u << lo) - 1u);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          bm[e] = -INFINITY;
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const bool keep = e < 2 && ((tm >> (8 * e + x)) & 1u);
            const float v = keep ? __uint_as_float(sr[8 * e + x]) : -INFINITY;
            sr[8 * e + x] = __float_as_uint(v);
            bm[e] = fmaxf(bm[e], v);
          }
        }
      }
      const float mraw = fmaxf(fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3])),
                               fmaxf(fmaxf(bm[4], bm[5]), fmaxf(bm[6], bm[7])));
      // reference after tile j-1 (published by the other warp)
      float m_prev = -INFINITY;
      if (j > 0) {
        asm volatile("bar.sync %0, 64;" ::"r"(pub_other) : "memory");
        m_prev = sm.mchain[m];
      }
      const float m_new = fmaxf(m_prev, mraw * scale_log2);
      const bool need = (m_prev != -INFINITY) && (m_new > m_prev + 8.0f);
      const float m_use = (m_prev == -INFINITY || need) ? m_new : m_prev;
      sm.mchain[m] = m_use;
      if (j + 1 < n_tiles) asm volatile("bar.arrive %0, 64;" ::"r"(pub_mine) : "memory");
      if (__any_sync(0xffffffffu, need)) {
        // O must hold P(j-1) V(j-1) before it is rescaled
        ok = ok && tc::mbar_wait(bar(sm.pv_done[(j - 1) % 2]), ((j - 1) / 2) & 1, abort);
        tc::fence_after();
        const float alpha = need ? exp2f(m_prev - m_use) : 1.f;
#pragma unroll 1
        for (int h = 0; h < 6; ++h) {
          uint32_t o[32];
          tc::tmem_ld32(tO + lane_off + 32 * h, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
          tc::tmem_st32(tO + lane_off + 32 * h, o);
        }
      }
      if (m_l != m_use) {
        l = m_l == -INFINITY ? 0.f : l * exp2f(m_l - m_use);
        m_l = m_use;
      }
      // P = 2^(s * scale - m_use) in BF16, packed two tokens per column.  A
      // block the row does not attend has offset -inf (P = 0).  Exponentials
      // run in pairs of blocks (16 per branch-free chunk, so their latencies
      // overlap); with SKIP_PAIRS a pair no row of this warp attends is skipped.
      const float neg_m = m_use == -INFINITY ? 0.f : -m_use;
      const uint32_t wmask = SKIP_PAIRS ? __reduce_or_sync(0xffffffffu, bmask) : 0xFFu;
      float ls[8];
      uint32_t pk[32];
#pragma unroll
      for (int e2 = 0; e2 < 8; e2 += 2) {
        if (!SKIP_PAIRS || ((wmask >> e2) & 3u)) {
#pragma unroll
          for (int e = e2; e < e2 + 2; ++e) {
            const float off = ((bmask >> e) & 1u) ? neg_m : -INFINITY;
            float pe[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) pe[x] = fast_exp2(fmaf(__uint_as_float(sr[8 * e + x]), scale_log2, off));
            ls[e] = ((pe[0] + pe[1]) + (pe[2] + pe[3])) + ((pe[4] + pe[5]) + (pe[6] + pe[7]));
#pragma unroll
            for (int x = 0; x < 4; ++x) pk[4 * e + x] = pack_bf16x2(pe[2 * x], pe[2 * x + 1]);
          }
        } else {
#pragma unroll
          for (int e = e2; e < e2 + 2; ++e) {
            ls[e] = 0.f;
#pragma unroll
            for (int x = 0; x < 4; ++x) pk[4 * e + x] = 0u;
          }
        }
      }
      const float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      // P buffer b is free once O += P(j-2) V(j-2) has read it
      if (j >= 2) ok = ok && tc::mbar_wait(bar(sm.pv_done[b]), ((j / 2) - 1) & 1, abort);
      tc::fence_after();
      tc::tmem_st32(tP, pk);
      l += lsum;
      tc::tmem_st_wait();
      tc::fence_before();
      tc::mbar_arrive(bar(sm.p_full[b]));
    }
    ok = ok && tc::mbar_wait(bar(sm.o_final), 0, abort);
    // both loops done: the final reference is in mchain; combine the two partial sums
    asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
    const float m_fin = sm.mchain[m];
    const float l_adj = (m_l == -INFINITY) ? 0.f : (m_l == m_fin ? l : l * exp2f(m_l - m_fin));
    sm.lsum[half][m] = l_adj;
    asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
    const float ltot = l_adj + sm.lsum[half ^ 1][m];
    if (ok) {
      tc::fence_after();
      const float inv = sm.gfac[m] / ltot;  // softmax normalisation and output gate
      __nv_bfloat16* orow = out + orow_idx * kD;
#pragma unroll 1
      for (int h = 3 * half; h < 3 * half + 3; ++h) {
        uint32_t o[32];
        tc::tmem_ld32(tO + lane_off + 32 * h, o);
        tc::tmem_ld_wait();
        if (qvalid) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv, __uint_as_float(o[8 * v4 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv, __uint_as_float(o[8 * v4 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv, __uint_as_float(o[8 * v4 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv, __uint_as_float(o[8 * v4 + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + 32 * h + 8 * v4) = w;
          }
        }
      }
    }
  }
  // Every role has left its loop, so the abort flag is final.  After a
  // failed wait, copies and MMAs already issued may still be in flight: the
  // producers wait for their last ring's worth of copies and each MMA warp for
  // its own MMAs (full time bound) before shared memory and TMEM are released.
  __syncthreads();
  if (sm.abort) {
    if ((warp == 0 || warp == 10) && BS == 8) {  // (smaller blocks: the copies landed before the loop's end)
      const bool is_k = warp == 0;
      const int nst = is_k ? kTcStages : kTcVStages;
      for (int j = issued > nst ? issued - nst : 0; j < issued; ++j)
        tc::mbar_drain(bar(is_k ? sm.k_full[j % nst] : sm.v_full[j % nst]), (j / nst) & 1);
    } else if (warp == 1 || warp == 11) {
      uint64_t& d = warp == 1 ? sm.drain : sm.drain_pv;
      if (tc::elect_one()) tc::mma_commit(bar(d));
      __syncwarp();
      tc::mbar_drain(bar(d), 0);
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace sgqa

namespace sgqa {

// ---------------------------------------------------------------------------
// Decode attention (few queries, long context): HBM-bound gather of the
// selected 8-token blocks.  One CTA takes a contiguous range of one (query,
// group)'s blocks (split-K); four lanes of a producer warp stream the blocks'
// K and V (one 5-D TMA box each, 3 KB, 128-byte swizzled) into a 16-slot ring,
// and four compute warps consume two blocks (16 tokens) per step with the
// warp-level MMA formulation (16 heads = the m16 rows).  The splits of a row
// form one thread-block cluster: each keeps its (max, sum, unnormalised O) in
// shared memory and, after a cluster barrier, finalises a slice of the row's
// output by reading every split's partial through distributed shared memory
// (no global partials, fences or tickets).
// ---------------------------------------------------------------------------
constexpr int kDecSlots = 16;
constexpr int kDecThreads = 160;  // warp 0 producer, warps 1-4 compute
constexpr int kDecIssuers = 4;    // producer lanes issuing TMA loads side by side
static_assert(kDecSlots % kDecIssuers == 0 && kDecIssuers <= 32, "issuer groups tile the ring");

constexpr int kDecQPad = kD + 8;  // Q rows of 400 B: ldmatrix rows fall in distinct banks

struct __align__(1024) DecSmem {
  uint8_t kv[kDecSlots][2][3 * 1024];   // [slot][K|V][chunk][8 rows x 128 B]
  __nv_bfloat16 q[kHg][kDecQPad];       // the row's 16 heads (A operand, read by ldmatrix)
  int32_t rows[2049];                   // first token row of each of this CTA's blocks
  uint64_t full[kDecSlots], empty[kDecSlots];
  int abort;
  int last;
};

// byte offset of (token row r in 0..7, 16-byte piece j in 0..23) in a swizzled block tile
__device__ __forceinline__ uint32_t blk_off(uint32_t r, uint32_t j) {
  return (j >> 3) * 1024u + r * 128u + (((j & 7u) ^ r) << 4);
}

constexpr int kDecMaxSplit = 8;  // splits of a row = one (portable) cluster
constexpr int kPageTokens = 16;  // tokens per page of a paged K/V cache

__global__ void __launch_bounds__(kDecThreads, 2)
attn_decode_tma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                       const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ sel,
                       const int32_t* __restrict__ sel_count, __nv_bfloat16* __restrict__ out,
                       const __nv_bfloat16* __restrict__ gate, int64_t nq, int G, int k, int64_t q_pos0, int nsplit,
                       float scale_log2, const int32_t* __restrict__ page_table, int64_t max_pages,
                       int64_t num_pages) {
  extern __shared__ uint8_t smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % nsplit;
  const int64_t row = blockIdx.x / nsplit;  // (seq * nq + i) * G + g
  const int g = static_cast<int>(row % G);
  const int64_t i = (row / G) % nq;
  const int64_t seq = row / (G * nq);
  const int64_t t = q_pos0 + i;
  const int cnt = min(max(sel_count[row], 0), k);
  const int32_t* ids = sel + row * k;
  // A block's copy coordinates: contiguous caches (token row, sequence); a
  // paged pool [pages, G, 16, D] (row within its page, page), packed in the
  // staged row value as page * 16 + row (negative: a zero block)
  const bool paged = page_table != nullptr;
  const int nblk = cnt + 1;  // selected blocks, then the current block
  const int per = (nblk + nsplit - 1) / nsplit;
  const int b0 = min(nblk, split * per), b1 = min(nblk, b0 + per);
  const int nb = b1 - b0;
  const int64_t cur0 = 8 * (t / 8);
  volatile int* abort = &sm.abort;
  auto bar = [](uint64_t& b) { return smem_u32(&b); };
  if (threadIdx.x == 0) {
    sm.abort = 0;
    for (int s = 0; s < kDecSlots; ++s) {
      tc::mbar_init(bar(sm.full[s]), 1);
      tc::mbar_init(bar(sm.empty[s]), 1);
    }
    tc::mbar_fence_init();
  }
  // stage the block rows (one coalesced read instead of a dependent load per TMA issue);
  // a selected id outside [0, floor(t/8)) breaks the call's contract: it is
  // reported, read as zeros and masked out (row -64)
  const int64_t nhist = t / 8;
  for (int b = threadIdx.x; b < nb; b += kDecThreads) {
    const int e = b0 + b;
    int32_t r = static_cast<int32_t>(cur0);  // first token of the block
    if (e < cnt) {
      const int32_t id = ids[e];
      if (id < 0 || id >= nhist) {
        report(kDevBounds);
        sm.rows[b] = -64;
        continue;
      }
      r = id * 8;
    }
    if (page_table != nullptr) {
      // paged cache: the block's 8 tokens lie in one 16-token page of the pool
      const int32_t pg = page_table[seq * max_pages + (r >> 4)];
      if (pg < 0 || pg >= num_pages) {
        report(kDevBounds);
        r = -64;  // outside the pool: the copy reads zeros
      } else {
        r = pg * kPageTokens + (r & (kPageTokens - 1));
      }
    }
    sm.rows[b] = r;
  }
  // Q into shared memory (its fragments are re-read per k-step: held in
  // registers they pushed the O accumulators into local memory)
  {
    const uint4* q16 = reinterpret_cast<const uint4*>(q + ((seq * nq + i) * G + g) * kHg * kD);
    for (int x = threadIdx.x; x < kHg * kD / 8; x += kDecThreads)
      *reinterpret_cast<uint4*>(&sm.q[x / (kD / 8)][(x % (kD / 8)) * 8]) = q16[x];
  }
  int mine_end = 0;  // producer lanes: one past the last block this lane issued
  // per-warp attention state (compute warps)
  WarpAttn st;
#pragma unroll
  for (int j = 0; j < 24; ++j) st.o[j][0] = st.o[j][1] = st.o[j][2] = st.o[j][3] = 0.f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.f;
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tmap(&kmap);
      tc::prefetch_tmap(&vmap);
    }
    __syncwarp();
    // blocks in pairs: step s uses slots 2s, 2s+1 (mod kDecSlots); an odd tail
    // gets a zero block.  kDecIssuers lanes issue consecutive blocks side by
    // side (one thread's TMA issue rate does not keep an SM's share of HBM busy).
    const int nblocks = 2 * ((nb + 1) / 2);
    for (int bg = 0; bg < nblocks; bg += kDecIssuers) {
      const int b = bg + lane;
      bool ok = true;
      if (lane < kDecIssuers && b < nblocks) {
        const int slot = b % kDecSlots;
        if (b >= kDecSlots) ok = tc::mbar_wait(bar(sm.empty[slot]), ((b / kDecSlots) - 1) & 1, abort);
        if (ok) {
          const int32_t r = b < nb ? sm.rows[b] : -64;  // -64: zero-filled tail block
          tc::mbar_expect_tx(bar(sm.full[slot]), 2 * 3 * 1024);
          const int32_t c1 = paged ? (r & 15) : r, c4 = paged ? (r >> 4) : static_cast<int32_t>(seq);
          tc::tma_load_5d(smem_u32(&sm.kv[slot][0][0]), &kmap, 0, c1, 0, g, c4, bar(sm.full[slot]));
          tc::tma_load_5d(smem_u32(&sm.kv[slot][1][0]), &vmap, 0, c1, 0, g, c4, bar(sm.full[slot]));
          mine_end = b + 1;
        }
      }
      if (!__all_sync(0xffffffffu, ok)) break;
    }
  } else {
    const int cw = warp - 1;  // compute warp 0..3
    const int nsteps = (nb + 1) / 2;
    const int mrow = lane & 7, mat = lane >> 3;
    // ldmatrix row of this lane in the Q tile: matrices (heads 0-7 | 8-15) x (dims +0 | +8)
    const uint32_t qrow = smem_u32(&sm.q[8 * (mat & 1) + mrow][8 * (mat >> 1)]);
    for (int s = cw; s < nsteps; s += 4) {
      const int ba = 2 * s, bb = 2 * s + 1;
      const int sa = ba % kDecSlots, sb2 = bb % kDecSlots;
      if (!tc::mbar_wait(bar(sm.full[sa]), (ba / kDecSlots) & 1, abort)) break;
      if (!tc::mbar_wait(bar(sm.full[sb2]), (bb / kDecSlots) & 1, abort)) break;
      // token mask: 8 tokens per block; the current block only up to t; zero blocks none
      uint32_t tm = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int b = 2 * s + h;
        if (b < nb && sm.rows[b] >= 0) {  // -64: a zero block (bad id or page), attended by no one
          const int e = b0 + b;
          uint32_t m8 = 0xFFu;
          if (e >= cnt) m8 = (t - cur0 >= 7) ? 0xFFu : ((1u << (t - cur0 + 1)) - 1u);
          tm |= m8 << (8 * h);
        }
      }
      const uint32_t ka = smem_u32(&sm.kv[sa][0][0]), kb = smem_u32(&sm.kv[sb2][0][0]);
      const uint32_t va = smem_u32(&sm.kv[sa][1][0]), vb = smem_u32(&sm.kv[sb2][1][0]);
      // S = Q K^T: matrices (tok 0-7 = block a | 8-15 = block b) x (dims 16ks | 16ks+8)
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
      const uint32_t kblk = (mat >> 1) ? kb : ka;
#pragma unroll
      for (int ks = 0; ks < 12; ++ks) {
        uint32_t bf[4];
        ldmatrix_x4(bf, kblk + blk_off(mrow, 2 * ks + (mat & 1)));
        uint32_t qa[4];
        ldmatrix_x4(qa, qrow + 2u * (16 * ks));
        mma_bf16_16816(sc[0], qa, bf[0], bf[1]);
        mma_bf16_16816(sc[1], qa, bf[2], bf[3]);
      }
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = 8 * nt + 2 * (lane & 3) + (e & 1);
          sc[nt][e] = ((tm >> tok) & 1u) ? sc[nt][e] * scale_log2 : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], sc[nt][e]);
        }
      }
      // lazy rescale: the reference max moves only when the new max exceeds it
      // by more than 2^8 (P stays <= 256, exact in the final normalisation)
      float alpha[2], muse[2];
      bool need = false;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        alpha[r] = 1.f;
        if (st.m[r] == -INFINITY) {
          st.m[r] = mx[r];
        } else if (mx[r] > st.m[r] + 8.f) {
          alpha[r] = exp2f(st.m[r] - mx[r]);
          st.m[r] = mx[r];
          need = true;
        }
        muse[r] = st.m[r] == -INFINITY ? 0.f : st.m[r];
      }
      float p[2][4], psum[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          p[nt][e] = exp2f(sc[nt][e] - muse[e >> 1]);
          psum[e >> 1] += p[nt][e];
        }
      st.l[0] = st.l[0] * alpha[0] + psum[0];
      st.l[1] = st.l[1] * alpha[1] + psum[1];
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int j = 0; j < 24; ++j) {
          st.o[j][0] *= alpha[0]; st.o[j][1] *= alpha[0];
          st.o[j][2] *= alpha[1]; st.o[j][3] *= alpha[1];
        }
      }
      uint32_t pa[4];
      pa[0] = pack_bf16x2(p[0][0], p[0][1]);
      pa[1] = pack_bf16x2(p[0][2], p[0][3]);
      pa[2] = pack_bf16x2(p[1][0], p[1][1]);
      pa[3] = pack_bf16x2(p[1][2], p[1][3]);
      // PV: trans matrices (tok 0-7 = a | 8-15 = b) x (dims 16jj | 16jj+8)
      const uint32_t vblk = (mat & 1) ? vb : va;
#pragma unroll
      for (int jj = 0; jj < 12; ++jj) {
        uint32_t bf[4];
        ldmatrix_x4_trans(bf, vblk + blk_off(mrow, 2 * jj + (mat >> 1)));
        mma_bf16_16816(st.o[2 * jj], pa, bf[0], bf[1]);
        mma_bf16_16816(st.o[2 * jj + 1], pa, bf[2], bf[3]);
      }
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(bar(sm.empty[sa]));
        tc::mbar_arrive(bar(sm.empty[sb2]));
      }
    }
  }
  __syncthreads();
  // Every role has left its loop, so the abort flag is final.  After a failed
  // wait, this lane's loads still in flight (at most one ring's worth) land
  // (full time bound) before the ring's memory is reused below.
  if (sm.abort && warp == 0 && lane < kDecIssuers) {
    for (int b = lane; b < mine_end; b += kDecIssuers)
      if (b >= mine_end - kDecSlots) tc::mbar_drain(bar(sm.full[b % kDecSlots]), (b / kDecSlots) & 1);
  }
  __syncthreads();
  // combine the four compute warps into this split's partial (shared memory
  // of the ring reused): per-head factors once, then four FMAs per output
  constexpr int kCoStride = kD + 4;                       // padded rows: no bank conflicts
  float* cm = reinterpret_cast<float*>(&sm.kv[0][0][0]);  // [4][16]
  float* cl = cm + 4 * kHg;                               // [4][16]
  float* co = cl + 4 * kHg;                               // [4][16][196]
  float* fw = co + 4 * kHg * kCoStride;                   // [4][16] warp factors
  float* pm = reinterpret_cast<float*>(&sm.kv[0][0][0] + 65536);  // this split: max [16]
  float* pl = pm + kHg;                                           //             sum [16]
  float* pacc = pl + kHg;                                         //             O [16][192]
  float* gf = pacc + kHg * kD;                                    // row factors [kDecMaxSplit][16]
  float* ginv = gf + kDecMaxSplit * kHg;                          // [16]
  if (warp >= 1) {
    const int cw = warp - 1;
    float l0 = st.l[0], l1 = st.l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const int h0 = lane >> 2, h1 = h0 + 8;
    if ((lane & 3) == 0) {
      cm[cw * kHg + h0] = st.m[0]; cm[cw * kHg + h1] = st.m[1];
      cl[cw * kHg + h0] = l0;      cl[cw * kHg + h1] = l1;
    }
#pragma unroll
    for (int j = 0; j < 24; ++j) {
      const int d = 8 * j + 2 * (lane & 3);
      *reinterpret_cast<float2*>(&co[(cw * kHg + h0) * kCoStride + d]) = make_float2(st.o[j][0], st.o[j][1]);
      *reinterpret_cast<float2*>(&co[(cw * kHg + h1) * kCoStride + d]) = make_float2(st.o[j][2], st.o[j][3]);
    }
  }
  __syncthreads();
  if (threadIdx.x < kHg) {
    const int h = threadIdx.x;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mm = fmaxf(mm, cm[w * kHg + h]);
    const float mu = mm == -INFINITY ? 0.f : mm;
    float ls = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float a = exp2f(cm[w * kHg + h] - mu);
      fw[w * kHg + h] = a;
      ls += a * cl[w * kHg + h];
    }
    pm[h] = mm;
    pl[h] = ls;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < kHg * kD; idx += kDecThreads) {
    const int h = idx / kD, d = idx % kD;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) acc = fmaf(fw[w * kHg + h], co[(w * kHg + h) * kCoStride + d], acc);
    pacc[idx] = acc;
  }
  // every split's partial is in its shared memory: combine across the cluster
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  if (threadIdx.x < kHg) {
    const int h = threadIdx.x;
    float mm = -INFINITY;
    for (int r = 0; r < nsplit; ++r) mm = fmaxf(mm, cluster.map_shared_rank(pm, r)[h]);
    const float mu = mm == -INFINITY ? 0.f : mm;
    float ls = 0.f;
    for (int r = 0; r < nsplit; ++r) {
      const float a = exp2f(cluster.map_shared_rank(pm, r)[h] - mu);
      gf[r * kHg + h] = a;
      ls += a * cluster.map_shared_rank(pl, r)[h];
    }
    ginv[h] = gate_factor(gate, row * kHg + h) / ls;  // normalisation and output gate
  }
  __syncthreads();
  {
    // this split finalises outputs [split * per, split * per + per) of the row's 16 x 192
    const int per = (kHg * kD + nsplit - 1) / nsplit;
    const int i0 = split * per, i1 = min(kHg * kD, i0 + per);
    for (int idx = i0 + threadIdx.x; idx < i1; idx += kDecThreads) {
      const int h = idx / kD;
      float acc = 0.f;
      for (int r = 0; r < nsplit; ++r) acc = fmaf(gf[r * kHg + h], cluster.map_shared_rank(pacc, r)[idx], acc);
      out[row * kHg * kD + idx] = __float2bfloat16_rn(acc * ginv[h]);
    }
  }
  cluster.sync();  // no split leaves while others still read its shared memory
}

}  // namespace sgqa
