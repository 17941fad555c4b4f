// Sparse attention for prefill on the 5th-generation tensor cores (tcgen05,
// TMEM accumulators, TMA-fed shared memory).  Page "Step-5-Preview: Sparse
// Reads Are Not a Compressed KV Cache", sections "Main attention still reads
// original K/V" and "What gets cheaper ..."; the second page's "group
// overlapping computations" of adjacent queries.
//
// One CTA takes one unit = (sequence, block of 8 adjacent queries, KV group).
// The MMA M dimension is the 8 queries x 16 heads = 128 rows, all sharing the
// group's K/V; the unit walks the sorted union of the 8 queries' selected
// 8-token blocks (built by attn_plan_kernel) 64 tokens (8 blocks) at a time,
// then one tile holding the current-block tokens.  Per 64-token tile:
//   S = Q K^T     12 tcgen05.mma (M128 N64 K16) into TMEM, Q and K from SMEM
//   softmax       4 warps, one TMEM lane (= one (query, head) row) per thread:
//                 per-row block mask (the row's query must have selected the
//                 block) and causal mask on the current block, running max
//                 in log2 units with lazy rescaling of O (only when the max
//                 grows by more than 2^8), P rounded to BF16 into SMEM
//   O += P V      4 tcgen05.mma (M128 N192 K16), V as an MN-major operand.
// Warp roles: warp 0 issues TMA (one 5-D box per 8-token block gathers all
// 192 dims of K or V: 3 KB), warp 1 allocates TMEM and issues the MMAs from
// one thread, warps 2-5 run the softmax and the epilogue.  Every mbarrier
// wait is bounded (tc::mbar_wait).
#pragma once
#include "attn_mma.cuh"
#include "tc.cuh"

namespace sgqa {

constexpr int kTcStages = 3;      // K ring and V ring depth (K freed after QK^T, V after PV)
constexpr int kTcThreads = 192;
constexpr int kTcTileTok = 64;    // tokens per KV tile = 8 blocks of 8

struct __align__(1024) AttnTcSmem {
  uint8_t q[3][128 * 128];                 // Q: 3 column chunks x 128 rows x 128 B (SW128)
  uint8_t k[kTcStages][8][3][1024];        // K tile: [block][chunk][8 rows x 128 B]
  uint8_t v[kTcStages][8][3][1024];        // V tile, same layout (MN-major operand)
  uint8_t p[2][128 * 128];                 // P: 128 rows x 64 tokens bf16 (SW128)
  uint64_t q_full;
  uint64_t k_full[kTcStages], k_empty[kTcStages], v_full[kTcStages], v_empty[kTcStages];
  uint64_t s_full[3], s_free[3], p_full[2], p_empty[2];
  uint64_t o_done, o_final, drain;
  uint32_t tmem;
  int abort;
};

__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const int32_t* __restrict__ plan_ids,
               const uint8_t* __restrict__ plan_mask, const int32_t* __restrict__ plan_count,
               __nv_bfloat16* __restrict__ out, int64_t nq, int G, int k, int64_t q_pos0,
               float scale_log2) {
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
  const int n_union_tiles = (U + 7) / 8;
  const int n_tiles = n_union_tiles + 1;
  const int64_t t_first = q_pos0 + qb * 8;
  const int64_t t_last = q_pos0 + min(nq, qb * 8 + 8) - 1;
  const int64_t c0 = 8 * (t_first / 8);  // first token of the current segment
  volatile int* abort = &sm.abort;

  auto bar = [](uint64_t& b) { return smem_u32(&b); };
  if (threadIdx.x == 0) {
    sm.abort = 0;
    tc::mbar_init(bar(sm.q_full), 1);
    for (int s = 0; s < kTcStages; ++s) {
      tc::mbar_init(bar(sm.k_full[s]), 1);
      tc::mbar_init(bar(sm.k_empty[s]), 1);
      tc::mbar_init(bar(sm.v_full[s]), 1);
      tc::mbar_init(bar(sm.v_empty[s]), 1);
    }
    for (int b = 0; b < 3; ++b) {
      tc::mbar_init(bar(sm.s_full[b]), 1);
      tc::mbar_init(bar(sm.s_free[b]), 128);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(sm.p_full[b]), 128);
      tc::mbar_init(bar(sm.p_empty[b]), 1);
    }
    tc::mbar_init(bar(sm.o_done), 1);
    tc::mbar_init(bar(sm.o_final), 1);
    tc::mbar_init(bar(sm.drain), 1);
    tc::mbar_fence_init();
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(&sm.tmem), 512);
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = sm.tmem;
  const uint32_t tO = tmem;           // columns [0, 192)
  const uint32_t tS0 = tmem + 256;    // S buffers at [256, 320), [320, 384), [384, 448)

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_tmap(&qmap);
      tc::prefetch_tmap(&kmap);
      tc::prefetch_tmap(&vmap);
      tc::mbar_expect_tx(bar(sm.q_full), 3 * 128 * 128);
      const int32_t qrow0 = static_cast<int32_t>(((seq * nq + qb * 8) * G + g) * 16);
      const int32_t qstride = G * 16;
      for (int c = 0; c < 3; ++c)
        for (int i = 0; i < 8; ++i)
          tc::tma_load_2d(smem_u32(&sm.q[c][i * 16 * 128]), &qmap, 64 * c, qrow0 + i * qstride, bar(sm.q_full));
      int issued = 0;
      // block ids of the next union tile, fetched one tile ahead
      auto tile_rows = [&](int j, int32_t (&rows)[8]) {
        if (j < n_union_tiles) {
          const int4 a = *reinterpret_cast<const int4*>(uid + 8 * j);
          const int4 b = *reinterpret_cast<const int4*>(uid + 8 * j + 4);
          const int32_t ids[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) rows[e] = (8 * j + e < U) ? ids[e] * 8 : -64;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            rows[e] = (e == 0 || (e == 1 && c0 + 8 <= t_last)) ? static_cast<int32_t>(c0 + 8 * e) : -64;
        }
      };
      int32_t rows[8];
      tile_rows(0, rows);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kTcStages;
        const uint32_t ph = ((j / kTcStages) - 1) & 1;
        int32_t next[8];
        if (j + 1 < n_tiles) tile_rows(j + 1, next);
        if (j >= kTcStages && !tc::mbar_wait(bar(sm.k_empty[s]), ph, abort)) break;
        tc::mbar_expect_tx(bar(sm.k_full[s]), 8 * 3 * 1024);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          tc::tma_load_5d(smem_u32(&sm.k[s][e][0][0]), &kmap, 0, rows[e], 0, g, static_cast<int32_t>(seq),
                          bar(sm.k_full[s]));
        if (j >= kTcStages && !tc::mbar_wait(bar(sm.v_empty[s]), ph, abort)) { issued = -(j + 1); break; }
        tc::mbar_expect_tx(bar(sm.v_full[s]), 8 * 3 * 1024);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          tc::tma_load_5d(smem_u32(&sm.v[s][e][0][0]), &vmap, 0, rows[e], 0, g, static_cast<int32_t>(seq),
                          bar(sm.v_full[s]));
        issued = j + 1;
#pragma unroll
        for (int e = 0; e < 8; ++e) rows[e] = next[e];
      }
      if (*abort) {
        // Let the copies already issued land before the CTA's shared memory goes away.
        const bool k_only = issued < 0;
        const int n_iss = k_only ? -issued : issued;
        const uint64_t t0 = globaltimer_ns();
        while (!tc::mbar_try(bar(sm.q_full), 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
        for (int j = n_iss > kTcStages ? n_iss - kTcStages : 0; j < n_iss; ++j) {
          const uint64_t t1 = globaltimer_ns();
          while (!tc::mbar_try(bar(sm.k_full[j % kTcStages]), (j / kTcStages) & 1) &&
                 globaltimer_ns() - t1 < kWaitLimitNs) {
          }
          if (k_only && j == n_iss - 1) break;
          while (!tc::mbar_try(bar(sm.v_full[j % kTcStages]), (j / kTcStages) & 1) &&
                 globaltimer_ns() - t1 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = tc::idesc_bf16(128, 64, false);
      const uint32_t id_pv = tc::idesc_bf16(128, 192, true);
      auto pv = [&](int i) -> bool {
        const int pb = i & 1, s = i % kTcStages;
        if (!tc::mbar_wait(bar(sm.v_full[s]), (i / kTcStages) & 1, abort)) return false;
        if (!tc::mbar_wait(bar(sm.p_full[pb]), (i >> 1) & 1, abort)) return false;
        tc::fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = tc::sdesc_sw128(smem_u32(&sm.p[pb][0]) + kk * 32, 16, 1024);
          const uint64_t b = tc::sdesc_sw128(smem_u32(&sm.v[s][2 * kk][0][0]), 1024, 3072);
          tc::mma_f16(tO, a, b, id_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar(sm.v_empty[s]));
        tc::mma_commit(bar(sm.p_empty[pb]));
        tc::mma_commit(bar(sm.o_done));
        return true;
      };
      bool ok = tc::mbar_wait(bar(sm.q_full), 0, abort);
      // QK^T runs two tiles ahead of PV, so the tensor pipe has work queued
      // while the softmax of the older tile is still running.
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kTcStages, sb = j % 3;
        if (!tc::mbar_wait(bar(sm.k_full[s]), (j / kTcStages) & 1, abort)) { ok = false; break; }
        if (j >= 3 && !tc::mbar_wait(bar(sm.s_free[sb]), ((j / 3) - 1) & 1, abort)) { ok = false; break; }
        tc::fence_after();
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const uint64_t a = tc::sdesc_sw128(smem_u32(&sm.q[kk >> 2][0]) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = tc::sdesc_sw128(smem_u32(&sm.k[s][0][kk >> 2][0]) + (kk & 3) * 32, 16, 3072);
          tc::mma_f16(tS0 + 64 * sb, a, b, id_qk, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar(sm.k_empty[s]));
        tc::mma_commit(bar(sm.s_full[sb]));
        if (j >= 2 && !pv(j - 2)) { ok = false; break; }
      }
      for (int i = n_tiles >= 2 ? n_tiles - 2 : 0; ok && i < n_tiles; ++i) ok = pv(i);
      if (ok) {
        tc::mma_commit(bar(sm.o_final));
      } else {
        // Let the MMAs already issued finish before TMEM is released.
        tc::mma_commit(bar(sm.drain));
        const uint64_t t0 = globaltimer_ns();
        while (!tc::mbar_try(bar(sm.drain), 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const int m = quad * 32 + lane;          // TMEM lane = row = (query slot, head)
    const int qs = m >> 4;
    const int64_t qi = qb * 8 + qs;
    const bool qvalid = qi < nq;
    const int64_t t = q_pos0 + (qvalid ? qi : qb * 8);
    const int64_t cur_lo = 8 * (t / 8);
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    uint2 mb_next = n_union_tiles > 0 ? *reinterpret_cast<const uint2*>(umask) : make_uint2(0, 0);
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j % 3, pb = j & 1;
      const uint2 mb = mb_next;
      if (j + 1 < n_union_tiles) mb_next = *reinterpret_cast<const uint2*>(umask + 8 * (j + 1));
      // which of the 64 tokens this row attends
      uint64_t tok_mask = 0;
      if (j < n_union_tiles) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t byte = ((e < 4 ? mb.x : mb.y) >> (8 * (e & 3))) & 0xFFu;
          if (8 * j + e < U && ((byte >> qs) & 1u)) tok_mask |= 0xFFull << (8 * e);
        }
      } else {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int64_t tok = c0 + jj;
          if (tok >= cur_lo && tok <= t) tok_mask |= 1ull << jj;
        }
      }
      if (!tc::mbar_wait(bar(sm.s_full[sb]), (j / 3) & 1, abort)) { ok = false; break; }
      tc::fence_after();
      uint32_t sr[64];
      tc::tmem_ld32(tS0 + 64 * sb + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tc::tmem_ld32(tS0 + 64 * sb + 32 + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tc::tmem_ld_wait();
      tc::fence_before();
      tc::mbar_arrive(bar(sm.s_free[sb]));
      // masked scores (raw), their max; the scale is positive so it commutes with max
      float mraw = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < 64; ++jj) {
        const float x = ((tok_mask >> jj) & 1ull) ? __uint_as_float(sr[jj]) : -INFINITY;
        sr[jj] = __float_as_uint(x);
        mraw = fmaxf(mraw, x);
      }
      const float mt = mraw * scale_log2;
      const float m_new = fmaxf(m_used, mt);
      const bool need = (m_used != -INFINITY) && (m_new > m_used + 8.0f);
      if (m_used == -INFINITY) m_used = m_new;
      // P buffer pb is free once PV(j-2) has completed
      if (j >= 2 && !tc::mbar_wait(bar(sm.p_empty[pb]), ((j >> 1) - 1) & 1, abort)) { ok = false; break; }
      if (__any_sync(0xffffffffu, need)) {
        if (j >= 1 && !tc::mbar_wait(bar(sm.o_done), (j - 1) & 1, abort)) { ok = false; break; }
        tc::fence_after();
        const float alpha = need ? exp2f(m_used - m_new) : 1.f;
#pragma unroll 1
        for (int h = 0; h < 6; ++h) {
          uint32_t o[32];
          tc::tmem_ld32(tO + lane_off + 32 * h, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
          tc::tmem_st32(tO + lane_off + 32 * h, o);
        }
        tc::tmem_st_wait();
        if (need) {
          l *= alpha;
          m_used = m_new;
        }
      }
      // P = 2^(s * scale - m_used) in BF16 (masked -> exp2(-inf) = 0)
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      uint8_t* prow = &sm.p[pb][0];
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float pv8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          pv8[x] = exp2f(fmaf(__uint_as_float(sr[8 * c + x]), scale_log2, neg_m));
          lsum += pv8[x];
        }
        uint4 w;
        w.x = pack_bf16x2(pv8[0], pv8[1]);
        w.y = pack_bf16x2(pv8[2], pv8[3]);
        w.z = pack_bf16x2(pv8[4], pv8[5]);
        w.w = pack_bf16x2(pv8[6], pv8[7]);
        *reinterpret_cast<uint4*>(prow + tc::sw128_offset(static_cast<uint32_t>(m), static_cast<uint32_t>(c))) = w;
      }
      l += lsum;
      tc::fence_proxy_async_smem();
      tc::fence_before();
      tc::mbar_arrive(bar(sm.p_full[pb]));
    }
    if (ok && tc::mbar_wait(bar(sm.o_final), 0, abort)) {
      tc::fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = out + (((seq * nq + (qvalid ? qi : 0)) * G + g) * kHg + (m & 15)) * kD;
#pragma unroll 1
      for (int h = 0; h < 6; ++h) {
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
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace sgqa
