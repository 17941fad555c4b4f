// C ABI of the Sparse GQA hot path: argument validation, workspace carve-up
// and kernel launches.  All kernels live in the headers included below; this
// is the library's single translation unit (so the device status word is one
// symbol per device).
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cudaTypedefs.h>
#include <string>

#include "../../include/sgqa.h"
#include "attn_mma.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "index_rows.cuh"
#include "index_tc.cuh"
#include "merge.cuh"

namespace {

thread_local std::string g_err;

sgqa_status fail(sgqa_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
sgqa_status fail(sgqa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

sgqa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SGQA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Kernels launched by this library (all threads), read by sgqa_launch_count().
std::atomic<uint64_t> g_launches{0};

#define SGQA_LAUNCH_CHECK(what)                           \
  do {                                                    \
    cudaError_t e_ = cudaGetLastError();                  \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);    \
    g_launches.fetch_add(1, std::memory_order_relaxed);   \
  } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sgqa_status check_params(const sgqa_params* p) {
  if (p == nullptr) return fail(SGQA_ERR_INVALID_ARGUMENT, "params is NULL");
  if (p->num_kv_groups < 1 || p->heads_per_group < 1 || p->head_dim < 1 || p->idx_heads < 1 ||
      p->idx_dim < 1 || p->block_size < 1 || p->topk < 1)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "all sizes in sgqa_params must be >= 1");
  if (p->heads_per_group != 16 || p->head_dim != 192 || p->idx_dim != 64)
    return fail(SGQA_ERR_UNSUPPORTED, "this build supports heads_per_group=16, head_dim=192, idx_dim=64");
  if (p->idx_heads != 4 && p->idx_heads != 8)
    return fail(SGQA_ERR_UNSUPPORTED, "idx_heads must be 4 or 8");
  const int B = p->block_size;
  if (B != 1 && B != 2 && B != 4 && B != 8) return fail(SGQA_ERR_UNSUPPORTED, "block_size must be 1, 2, 4 or 8");
  if (p->topk > 2048) return fail(SGQA_ERR_UNSUPPORTED, "topk must be <= 2048");
  if (p->merge_in_f32 != 0 && p->merge_in_f32 != 1)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "merge_in_f32 must be 0 or 1");
  return SGQA_OK;
}

float softmax_scale(const sgqa_params* p) {
  return p->scale > 0.f ? p->scale : 1.0f / sqrtf(static_cast<float>(p->head_dim));
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Streaming multiprocessors of a B200 (grid sizing).
constexpr int64_t kSmCount = 148;

// Queries per sequence below which attention runs split-K per query.
constexpr int64_t kDecodeMaxNq = 32;

// Split-K factor for decode attention: one wave of two CTAs per SM.  On the
// 16 x 262144 decode workload this beat both two waves of shorter CTAs (their
// fixed costs -- staging, first loads, cross-warp combine -- add up) and one
// CTA per SM (four compute warps cannot keep an SM's share of HBM busy).
int decode_splits(int64_t rows) {
  int64_t s = (2 * 148) / std::max<int64_t>(rows, 1);
  return static_cast<int>(std::min<int64_t>(std::max<int64_t>(s, 1), 32));
}


int plan_pow2(int k) {
  int p = 1;
  while (p < 8 * k) p <<= 1;
  return std::max(p, 2);
}

// Index path for many queries: tcgen05 score rows and a top-k kernel over
// them.  Rows longer than the histogram top-k takes (16384 candidates) use the
// filtered path; shorter rows are cheaper to materialise and select (measured
// at 128K and 1M contexts).
constexpr int64_t kFilterMinCand = 16385;

// Sizes of the filtered path for rows of up to rneed candidates and top-k k:
// every samp-th tile of 128 candidates is sampled (at most kSampleTilesMax
// tiles per row); the threshold sits below the rank-th largest sample, so
// about rank * samp candidates -- 2k for k <= 512, 3k above -- are expected to
// pass; each row keeps four lists of subcap (key, id) pairs.
struct FilterSizes {
  int samp, rank, subcap;
  int64_t nsamp;
};
FilterSizes filter_sizes(int64_t rneed, int k) {
  FilterSizes f;
  const int64_t ntiles = (rneed + sgqa::kIdxCand - 1) / sgqa::kIdxCand;
  f.samp = static_cast<int>(std::max<int64_t>(sgqa::kSampleStride,
                                              (ntiles + sgqa::kSampleTilesMax - 1) / sgqa::kSampleTilesMax));
  f.nsamp = (ntiles + f.samp - 1) / f.samp * sgqa::kIdxCand;
  const int64_t target = k <= 512 ? 2 * static_cast<int64_t>(k) : 3 * static_cast<int64_t>(k);
  f.rank = static_cast<int>(std::max<int64_t>(16, (target + f.samp - 1) / f.samp));
  f.subcap = k <= 512 ? sgqa::kFilterSubCap : 2 * k;
  return f;
}

// CTAs of the fallback kernel (each owns one row-sized scratch slot).
constexpr int64_t kFallbackGrid = 2 * 148;

// Index workspace: widened keys, then one region used by the call's path --
// the FP32 score rows [rows, rpad] (rows of fewer than kFilterMinCand
// candidates, and decode), or in turn the sampled scores, the filtered
// (key, id) lists and the fallback's per-CTA score slots (the stages that use
// them run in that order); decode adds each row's strip maxima
// [rows, rpad / 16] after its score rows -- then four per-row arrays.
struct IndexWs {
  int64_t rpad;
  bool filtered;
  FilterSizes f;
  int64_t fb_grid;
  size_t keys_off, region_off, flags_off, staged_off, thr_off, list_off, bytes;
};
IndexWs index_ws(const sgqa_params* p, int64_t S, int64_t nq, int64_t max_ctx) {
  IndexWs w;
  const int64_t rneed = std::max<int64_t>((max_ctx - 1) / p->block_size, 1);
  w.rpad = round_up(rneed, 128);
  w.keys_off = 0;
  const size_t keys = align256(static_cast<size_t>(S * w.rpad * 64) * 2);
  const size_t rows = static_cast<size_t>(S * nq * p->num_kv_groups);
  w.filtered = nq > kDecodeMaxNq && rneed >= kFilterMinCand;
  w.f = filter_sizes(rneed, p->topk);
  w.fb_grid = std::min<int64_t>(static_cast<int64_t>(rows), kFallbackGrid);
  size_t region;
  if (w.filtered) {
    region = std::max({rows * static_cast<size_t>(w.f.nsamp) * 4, rows * 4 * static_cast<size_t>(w.f.subcap) * 8,
                       static_cast<size_t>(w.fb_grid) * static_cast<size_t>(w.rpad) * 4});
  } else {
    region = rows * static_cast<size_t>(w.rpad) * 4;
    // decode: the largest score of every 16-candidate strip, after the rows
    if (nq <= kDecodeMaxNq) region = align256(region) + rows * static_cast<size_t>(w.rpad / 16) * 4;
  }
  w.region_off = keys;
  w.flags_off = keys + align256(region);
  w.staged_off = w.flags_off + align256(rows * 4);
  w.thr_off = w.staged_off + align256(rows * 4 * 4);  // staged: [rows, 4] counts
  w.list_off = w.thr_off + align256(rows * 4);       // unsettled rows [rows], then their count
  w.bytes = w.list_off + align256(rows * 4) + 256;
  return w;
}

// Workspace for every call with q_pos0 + nq <= max_ctx: the largest call of
// each path (score rows, filtered).
size_t index_ws_bytes_upto(const sgqa_params* p, int64_t S, int64_t nq, int64_t max_ctx) {
  const int64_t rows_max_ctx = (kFilterMinCand - 1) * p->block_size + 1;  // longest context on the score-rows path
  return std::max(index_ws(p, S, nq, max_ctx).bytes,
                  index_ws(p, S, nq, std::min(max_ctx, rows_max_ctx)).bytes);
}

struct AttnWs {
  int nsplit;
  size_t ids_off, mask_off, cnt_off, po_off, pml_off, tick_off, bytes;
};
AttnWs attn_ws(const sgqa_params* p, int64_t S, int64_t nq) {
  AttnWs w{};
  const int64_t G = p->num_kv_groups;
  if (nq <= kDecodeMaxNq) {
    const int64_t rows = S * nq * G;
    w.nsplit = decode_splits(rows);
    w.po_off = 0;
    size_t po = align256(static_cast<size_t>(rows * w.nsplit) * 16 * 192 * 4);
    w.pml_off = po;
    size_t pml = align256(static_cast<size_t>(rows * w.nsplit) * 16 * 2 * 4);
    w.tick_off = po + pml;
    size_t tick = align256(static_cast<size_t>(rows) * 4);
    w.bytes = po + pml + tick;
  } else {
    const int64_t units = S * ((nq + 7) / 8) * G;
    const int64_t cap = 8 * static_cast<int64_t>(p->topk);
    w.ids_off = 0;
    size_t ids = align256(static_cast<size_t>(units * cap) * 4);
    w.mask_off = ids;
    size_t mask = align256(static_cast<size_t>(units * cap) + 64);
    w.cnt_off = ids + mask;
    size_t cnt = align256(static_cast<size_t>(units) * 4);
    w.bytes = ids + mask + cnt;
  }
  return w;
}

template <typename T>
T* ws_at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

sgqa_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return SGQA_OK;
  if (ws == nullptr) return fail(SGQA_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (!aligned(ws, 256)) return fail(SGQA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (have < need) return fail(SGQA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", have, need);
  return SGQA_OK;
}

template <int B>
void launch_merge(bool f32, const void* kp, const void* c, int64_t cap, int64_t b0, int64_t nblk,
                  int64_t S, float* merged, uint8_t* store, cudaStream_t st) {
  const int64_t threads = S * nblk * 8;
  const unsigned grid = static_cast<unsigned>((threads + sgqa::kMergeThreads - 1) / sgqa::kMergeThreads);
  if (f32)
    sgqa::merge_blocks_kernel<B, true><<<grid, sgqa::kMergeThreads, 0, st>>>(kp, c, cap, b0, nblk, S, merged, store);
  else
    sgqa::merge_blocks_kernel<B, false><<<grid, sgqa::kMergeThreads, 0, st>>>(kp, c, cap, b0, nblk, S, merged, store);
}

sgqa_status do_merge(const sgqa_params* p, int64_t S, int64_t cap, const void* kp, const void* c,
                     int64_t b0, int64_t b1, float* merged, uint8_t* store, cudaStream_t st) {
  const int64_t nblk = b1 - b0;
  if (nblk <= 0) return SGQA_OK;
  const bool f32 = p->merge_in_f32 != 0;
  switch (p->block_size) {
    case 1: launch_merge<1>(f32, kp, c, cap, b0, nblk, S, merged, store, st); break;
    case 2: launch_merge<2>(f32, kp, c, cap, b0, nblk, S, merged, store, st); break;
    case 4: launch_merge<4>(f32, kp, c, cap, b0, nblk, S, merged, store, st); break;
    default: launch_merge<8>(f32, kp, c, cap, b0, nblk, S, merged, store, st); break;
  }
  SGQA_LAUNCH_CHECK("merge_blocks_kernel");
  return SGQA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims/strides innermost first, strides in bytes for dims >= 1.
sgqa_status encode_bf16(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                        const cuuint64_t* strides, const cuuint32_t* box, const char* what) {
  auto enc = tmap_encoder();
  if (enc == nullptr) return fail(SGQA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SGQA_ERR_CUDA, "tensor map for %s: CUresult %d", what, (int)r);
  return SGQA_OK;
}

// Where the K/V of an attention call live: the contiguous caches
// [S, cap, G, D], or a pool of 16-token pages [pages, G, 16, D] with a page
// table [S, max_pages].
struct KvSource {
  const void* k;
  const void* v;
  int64_t cap, clen;                    // contiguous
  const int32_t* page_table = nullptr;  // paged
  int64_t max_pages = 0, num_pages = 0;
  bool paged() const { return page_table != nullptr; }
};

// Tensor maps over K and V with 8-token boxes of all 192 dims (three 128-byte
// column chunks, SW128): contiguous caches as (64 elements, token row, chunk,
// group, sequence); a page pool as (64 elements, row in page, chunk, group,
// page), where one group's 8-token block is a contiguous 3 KB run.
sgqa_status kv_maps(const KvSource& kv, int G, int64_t S, CUtensorMap* km, CUtensorMap* vm) {
  cuuint32_t box[5] = {64, 8, 3, 1, 1};
  sgqa_status s;
  if (kv.paged()) {
    cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(sgqa::kPageTokens), 3, static_cast<cuuint64_t>(G),
                          static_cast<cuuint64_t>(kv.num_pages)};
    cuuint64_t strides[4] = {384, 128, static_cast<cuuint64_t>(sgqa::kPageTokens) * 384,
                             static_cast<cuuint64_t>(G) * sgqa::kPageTokens * 384};
    if ((s = encode_bf16(km, kv.k, 5, dims, strides, box, "k_pool")) != SGQA_OK) return s;
    return encode_bf16(vm, kv.v, 5, dims, strides, box, "v_pool");
  }
  cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(kv.clen), 3, static_cast<cuuint64_t>(G), static_cast<cuuint64_t>(S)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(G) * 384, 128, 384, static_cast<cuuint64_t>(kv.cap) * G * 384};
  if ((s = encode_bf16(km, kv.k, 5, dims, strides, box, "k_cache")) != SGQA_OK) return s;
  return encode_bf16(vm, kv.v, 5, dims, strides, box, "v_cache");
}

template <int BS>
sgqa_status launch_attn_tc(const sgqa_params* p, int64_t S, int64_t q0, int64_t nq, const void* q,
                           const KvSource& kv, const int32_t* ids, const uint8_t* msk, const int32_t* cnt, void* out,
                           const void* gate, int64_t units, cudaStream_t st) {
  const int G = p->num_kv_groups;
  const float scale_log2 = softmax_scale(p) * 1.4426950408889634f;
  CUtensorMap km, vm;
  sgqa_status s;
  if ((s = kv_maps(kv, G, S, &km, &vm)) != SGQA_OK) return s;
  static_assert(sizeof(sgqa::AttnTcSmem) + 1024 <= 232448, "attention tile exceeds shared memory");
  const size_t smem = sizeof(sgqa::AttnTcSmem) + 1024;
  // Selections covering under a quarter of the candidates leave many block
  // pairs unattended by both queries of a warp: skip their exponentials.
  // (Blocks under 8 tokens: pools are not paged here, and no pairs are skipped.)
  const bool skip_pairs = (q0 + nq - 1) / p->block_size > 4 * static_cast<int64_t>(p->topk);
  auto kern = BS < 8 ? sgqa::attn_tc_kernel<false, false, BS>
              : kv.paged()
                  ? (skip_pairs ? sgqa::attn_tc_kernel<BS == 8, BS == 8, BS> : sgqa::attn_tc_kernel<false, BS == 8, BS>)
                  : (skip_pairs ? sgqa::attn_tc_kernel<BS == 8, false, BS> : sgqa::attn_tc_kernel<false, false, BS>);
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kern<<<static_cast<unsigned>(units), sgqa::kTcThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(q), km, vm, ids, msk, cnt, static_cast<__nv_bfloat16*>(out),
      static_cast<const __nv_bfloat16*>(gate), nq, G, p->topk, q0, scale_log2, kv.page_table, kv.max_pages,
      kv.num_pages, static_cast<const __nv_bfloat16*>(kv.k), static_cast<const __nv_bfloat16*>(kv.v), kv.cap, kv.clen);
  SGQA_LAUNCH_CHECK("attn_tc_kernel");
  return SGQA_OK;
}

sgqa_status do_index(const sgqa_params* p, int64_t S, int64_t q0, int64_t nq, const void* idx_q,
                     const float* idx_w, int64_t cap, const uint8_t* store, int32_t* sel,
                     int32_t* sel_count, void* ws, cudaStream_t st) {
  const int B = p->block_size, G = p->num_kv_groups, H = p->idx_heads;
  const IndexWs w = index_ws(p, S, nq, q0 + nq);
  const int64_t rneed = (q0 + nq - 1) / B;
  __nv_bfloat16* keys = ws_at<__nv_bfloat16>(ws, w.keys_off);
  if (rneed > 0 && nq > kDecodeMaxNq) {
    const int64_t threads = S * rneed * 8;
    sgqa::widen_store_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(
        store, cap / B, rneed, w.rpad, S, keys);
    SGQA_LAUNCH_CHECK("widen_store_kernel");
  }
  const __nv_bfloat16* iq = static_cast<const __nv_bfloat16*>(idx_q);
  float* scores = ws_at<float>(ws, w.region_off);
  int32_t* flags = ws_at<int32_t>(ws, w.flags_off);
  // rows a select kernel could not settle, for the radix kernel (count after the list)
  int32_t* list = ws_at<int32_t>(ws, w.list_off);
  int32_t* list_count = list + align256(static_cast<size_t>(S * nq * G) * 4) / 4;
  if (rneed > 0 && nq > kDecodeMaxNq) {
    // tcgen05 scores: 256 (query, head) columns per CTA, 128 candidates per MMA
    const int Q = sgqa::kIdxCols / H;
    sgqa_status s;
    CUtensorMap km, qm;
    {
      cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(S * w.rpad)};
      cuuint64_t strides[1] = {128};
      cuuint32_t box[2] = {64, static_cast<cuuint32_t>(sgqa::kIdxCand)};
      if ((s = encode_bf16(&km, keys, 2, dims, strides, box, "indexer keys")) != SGQA_OK) return s;
    }
    {
      cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(G),
                            static_cast<cuuint64_t>(S * nq)};
      cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(H) * 128, static_cast<cuuint64_t>(G) * H * 128};
      cuuint32_t box[4] = {64, static_cast<cuuint32_t>(H), 1, static_cast<cuuint32_t>(Q)};
      if ((s = encode_bf16(&qm, iq, 4, dims, strides, box, "idx_q")) != SGQA_OK) return s;
    }
    const int64_t grid = static_cast<int64_t>(G) * S * ((nq + Q - 1) / Q);
    const size_t smem = sizeof(sgqa::IndexTcSmem) + 1024;
    // the score kernel addresses a CTA's output rows with 32-bit offsets
    if (static_cast<int64_t>(sgqa::kIdxCols) * G * w.rpad >= INT32_MAX)
      return fail(SGQA_ERR_UNSUPPORTED, "context too long for the index score kernel");
    auto launch_score = [&](int mode, sgqa::ScoreOut o) {
#define SGQA_SCORE(HH, MM)                                                                                       \
  do {                                                                                                           \
    cudaFuncSetAttribute(sgqa::index_score_tc_kernel<HH, MM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    sgqa::index_score_tc_kernel<HH, MM><<<static_cast<unsigned>(grid), sgqa::kScoreTcThreads, smem, st>>>(       \
        km, qm, idx_w, o, nq, G, q0, B, w.rpad);                                                                 \
  } while (0)
      if (H == 8) {
        if (mode == sgqa::kScoreRows) SGQA_SCORE(8, sgqa::kScoreRows);
        else if (mode == sgqa::kScoreSample) SGQA_SCORE(8, sgqa::kScoreSample);
        else SGQA_SCORE(8, sgqa::kScoreFilter);
      } else {
        if (mode == sgqa::kScoreRows) SGQA_SCORE(4, sgqa::kScoreRows);
        else if (mode == sgqa::kScoreSample) SGQA_SCORE(4, sgqa::kScoreSample);
        else SGQA_SCORE(4, sgqa::kScoreFilter);
      }
#undef SGQA_SCORE
    };
    if (w.filtered) {
      // Long rows: sampled threshold, filtered score pass, exact select from the
      // kept lists; rows the filter could not settle are recomputed and
      // radix-selected by the fallback kernel.  No FP32 score row is written.
      const int64_t rows = S * nq * G;
      float* sample = ws_at<float>(ws, w.region_off);
      float* thr = ws_at<float>(ws, w.thr_off);
      uint2* staging = ws_at<uint2>(ws, w.region_off);
      float* slots = ws_at<float>(ws, w.region_off);
      int32_t* staged = ws_at<int32_t>(ws, w.staged_off);
      launch_score(sgqa::kScoreSample, sgqa::ScoreOut{sample, w.f.nsamp, w.f.samp, nullptr, nullptr, nullptr, 0});
      SGQA_LAUNCH_CHECK("index_score_tc_kernel (sample)");
      sgqa::index_threshold_kernel<<<static_cast<unsigned>(rows), sgqa::kThrThreads, 0, st>>>(
          sample, w.f.nsamp, nq, G, q0, B, w.f.samp, w.f.rank, thr);
      SGQA_LAUNCH_CHECK("index_threshold_kernel");
      launch_score(sgqa::kScoreFilter, sgqa::ScoreOut{nullptr, 0, 0, thr, staging, staged, w.f.subcap});
      SGQA_LAUNCH_CHECK("index_score_tc_kernel (filter)");
      cudaError_t e = cudaMemsetAsync(list_count, 0, 4, st);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(list count)");
      if (p->topk <= 512) {
        const int nwords_max = static_cast<int>((rneed + 31) / 32);
        const size_t dsmem = static_cast<size_t>(2 * sgqa::kFilterCap + nwords_max) * 4;
        if (dsmem > 227 * 1024) return fail(SGQA_ERR_UNSUPPORTED, "context too long for the staged top-k kernel");
        cudaFuncSetAttribute(sgqa::topk_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsmem);
        sgqa::topk_staged_kernel<<<static_cast<unsigned>(rows), sgqa::kStagedThreads, dsmem, st>>>(
            staging, staged, nq, G, q0, B, p->topk, w.f.subcap, nwords_max, sel, sel_count, flags, list, list_count);
        SGQA_LAUNCH_CHECK("topk_staged_kernel");
      } else {
        const size_t dsmem = sizeof(sgqa::StagedBigSmem);
        cudaFuncSetAttribute(sgqa::topk_staged_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsmem);
        sgqa::topk_staged_sort_kernel<<<static_cast<unsigned>(rows), sgqa::kStagedBigThreads, dsmem, st>>>(
            staging, staged, nq, G, q0, B, p->topk, w.f.subcap, sel, sel_count, flags, list, list_count);
        SGQA_LAUNCH_CHECK("topk_staged_sort_kernel");
      }
      sgqa::index_fallback_select_kernel<<<static_cast<unsigned>(w.fb_grid), sgqa::kSelThreads, 0, st>>>(
          iq, idx_w, keys, list, list_count, slots, nq, G, H, q0, B, w.rpad, p->topk, sel, sel_count);
      SGQA_LAUNCH_CHECK("index_fallback_select_kernel");
      return SGQA_OK;
    }
    launch_score(sgqa::kScoreRows, sgqa::ScoreOut{scores, w.rpad, 0, nullptr, nullptr, nullptr, 0});
    SGQA_LAUNCH_CHECK("index_score_tc_kernel");
  } else if (rneed > 0 && G == 4 && H == 8) {
    // few queries: the (query, candidate range) CTAs score all four groups from the E4M3 store; two
    // CTAs per SM over the whole launch, each range at least 1024 candidates and a whole number of strips
    const int64_t qrows = S * nq;
    if (qrows > 65535) return fail(SGQA_ERR_UNSUPPORTED, "decode index grid too large");
    float* smax = ws_at<float>(ws, w.region_off + align256(static_cast<size_t>(qrows * G) * w.rpad * 4));
    const int64_t want = std::max<int64_t>(1, (2 * kSmCount) / qrows);
    int64_t per_cta = (rneed + want - 1) / want;
    per_cta = std::max<int64_t>(1024, (per_cta + 15) / 16 * 16);
    dim3 grid(static_cast<unsigned>((rneed + per_cta - 1) / per_cta), static_cast<unsigned>(qrows));
    cudaError_t ea = cudaFuncSetAttribute(sgqa::index_score_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(sgqa::kDecScoreSmem));
    if (ea != cudaSuccess) return cuda_fail(ea, "cudaFuncSetAttribute(index_score_decode_kernel)");
    sgqa::index_score_decode_kernel<<<grid, sgqa::kDecScoreThreads, sgqa::kDecScoreSmem, st>>>(
        iq, idx_w, store, scores, nq, q0, B, w.rpad, cap / B, per_cta, smax, list_count);
    SGQA_LAUNCH_CHECK("index_score_decode_kernel");
    if (rneed <= static_cast<int64_t>(sgqa::kBndSelThreads) * sgqa::kBndSelPer && rneed >= 16 * p->topk + 128) {
      // each row ranked from the bound its strip maxima give; rows with massive ties are listed
      const int64_t rows = S * nq * G;
      sgqa::topk_rows_bound_kernel<<<static_cast<unsigned>(rows), sgqa::kBndSelThreads, 0, st>>>(
          scores, w.rpad, smax, nq, G, q0, B, static_cast<int>(p->topk), sel, sel_count, list, list_count);
      SGQA_LAUNCH_CHECK("topk_rows_bound_kernel");
      sgqa::topk_rows_list_kernel<<<static_cast<unsigned>(std::min<int64_t>(rows, kSmCount)), sgqa::kSelThreads, 0,
                                    st>>>(scores, w.rpad, nq, G, q0, B, p->topk, sel, sel_count, list, list_count);
      SGQA_LAUNCH_CHECK("topk_rows_list_kernel");
      return SGQA_OK;
    }
  } else if (rneed > 0) {
    // few queries: warp-MMA scores straight from the E4M3 store
    const int qpc = 64 / H;
    dim3 grid(static_cast<unsigned>((nq + qpc - 1) / qpc),
              static_cast<unsigned>((rneed + sgqa::kScoreCandPerCta - 1) / sgqa::kScoreCandPerCta),
              static_cast<unsigned>(S * G));
    if (grid.y > 65535 || grid.z > 65535) return fail(SGQA_ERR_UNSUPPORTED, "index grid too large");
    if (H == 8)
      sgqa::index_score_kernel<8, true><<<grid, sgqa::kScoreWarps * 32, 0, st>>>(iq, idx_w, store, scores, nq, G,
                                                                                  q0, B, w.rpad, cap / B);
    else
      sgqa::index_score_kernel<4, true><<<grid, sgqa::kScoreWarps * 32, 0, st>>>(iq, idx_w, store, scores, nq, G,
                                                                                  q0, B, w.rpad, cap / B);
    SGQA_LAUNCH_CHECK("index_score_kernel");
  }
  const int64_t rows = S * nq * G;
  // few long rows (decode): the register-resident select; many rows (prefill):
  // the 512-thread radix select, which keeps more rows in flight per SM
  if (nq <= kDecodeMaxNq && rneed <= sgqa::kRegSelThreads * sgqa::kRegSelPer) {
    sgqa::topk_rows_reg_kernel<<<static_cast<unsigned>(rows), sgqa::kRegSelThreads, 0, st>>>(
        scores, w.rpad, nq, G, q0, B, p->topk, sel, sel_count);
    SGQA_LAUNCH_CHECK("topk_rows_reg_kernel");
    return SGQA_OK;
  }
  const int nwords = static_cast<int>((std::max<int64_t>(rneed, 1) + 31) / 32);
  const size_t ssmem = (static_cast<size_t>(sgqa::kRows2Warps) * sgqa::kRows2Bins / 2 + 2 * sgqa::kRows2Cand + nwords) * 4;
  // Rows of 2048 .. 16384 candidates: a sampled threshold, one pass over the
  // row keeping the survivors, a linear histogram and an exact boundary-bin
  // select over them.  Long rows (>= 32768 candidates): two passes over the
  // row in HBM (histogram, then gather).  Rows either cannot finish
  // (boundary-bin overflow) go to the radix kernel, which also takes the rows
  // in between and short rows (its per-row set-up is smaller).
  if (rneed >= 2048 && rneed <= sgqa::kHistMaxCand && p->topk <= 512) {
    cudaError_t e = cudaMemsetAsync(list_count, 0, 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(list count)");
    sgqa::topk_rows_hist_kernel<<<static_cast<unsigned>(rows), sgqa::kHistThreads, 0, st>>>(
        scores, w.rpad, nq, G, q0, B, p->topk, sel, sel_count, flags, list, list_count);
    SGQA_LAUNCH_CHECK("topk_rows_hist_kernel");
    sgqa::topk_rows_list_kernel<<<static_cast<unsigned>(std::min<int64_t>(rows, 2 * 148)), sgqa::kSelThreads, 0, st>>>(
        scores, w.rpad, nq, G, q0, B, p->topk, sel, sel_count, list, list_count);
    SGQA_LAUNCH_CHECK("topk_rows_list_kernel");
    return SGQA_OK;
  } else if (rneed >= 32768 && ssmem <= 112 * 1024) {
    cudaFuncSetAttribute(sgqa::topk_rows2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
    cudaError_t e = cudaMemsetAsync(list_count, 0, 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(list count)");
    sgqa::topk_rows2_kernel<<<static_cast<unsigned>(rows), sgqa::kRows2Threads, ssmem, st>>>(
        scores, w.rpad, nq, G, q0, B, p->topk, nwords, sel, sel_count, flags, list, list_count);
    SGQA_LAUNCH_CHECK("topk_rows2_kernel");
    sgqa::topk_rows_list_kernel<<<static_cast<unsigned>(std::min<int64_t>(rows, 2 * 148)), sgqa::kSelThreads, 0, st>>>(
        scores, w.rpad, nq, G, q0, B, p->topk, sel, sel_count, list, list_count);
    SGQA_LAUNCH_CHECK("topk_rows_list_kernel");
    return SGQA_OK;
  }
  // the radix kernel takes every row
  sgqa::topk_rows_kernel<false><<<static_cast<unsigned>(rows), sgqa::kSelThreads, 0, st>>>(
      scores, w.rpad, nq, G, q0, B, p->topk, sel, sel_count, nullptr);
  SGQA_LAUNCH_CHECK("topk_rows_kernel");
  return SGQA_OK;
}

template <int B>
sgqa_status launch_attn(const sgqa_params* p, int64_t S, int64_t q0, int64_t nq, const void* q, const KvSource& kv,
                        const int32_t* sel, const int32_t* sel_count, void* out, const void* gate, void* ws,
                        cudaStream_t st) {
  const int G = p->num_kv_groups, k = p->topk;
  const __nv_bfloat16* gb = static_cast<const __nv_bfloat16*>(gate);
  const float scale_log2 = softmax_scale(p) * 1.4426950408889634f;
  const AttnWs w = attn_ws(p, S, nq);
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(kv.k);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(kv.v);
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(out);
  if (nq <= kDecodeMaxNq && B == 8) {
    // TMA-fed gather, the splits of a row combined inside their cluster
    const int64_t rows = S * nq * G;
    CUtensorMap km, vm;
    sgqa_status s;
    if ((s = kv_maps(kv, G, S, &km, &vm)) != SGQA_OK) return s;
    // the splits of a row run as one cluster (combined through distributed shared memory)
    const int nsplit = std::min(decode_splits(rows), sgqa::kDecMaxSplit);
    const size_t smem = sizeof(sgqa::DecSmem) + 1024;
    cudaFuncSetAttribute(sgqa::attn_decode_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows * nsplit));
    cfg.blockDim = dim3(sgqa::kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(nsplit);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, sgqa::attn_decode_tma_kernel, km, vm, qb, sel, sel_count, ob, gb, nq, G,
                                       k, q0, nsplit, scale_log2, kv.page_table, kv.max_pages, kv.num_pages);
    if (e != cudaSuccess) return cuda_fail(e, "attn_decode_tma_kernel launch");
    SGQA_LAUNCH_CHECK("attn_decode_tma_kernel");
    return SGQA_OK;
  }
  if (kv.paged() && B != 8) return fail(SGQA_ERR_UNSUPPORTED, "paged K/V needs block_size 8");
  if (nq <= kDecodeMaxNq) {
    const int64_t rows = S * nq * G;
    const size_t smem = sgqa::kDecWarps * sgqa::kDecStages * 2 * sgqa::kStageElems * 2;
    cudaFuncSetAttribute(sgqa::attn_decode_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    float* po = ws_at<float>(ws, w.po_off);
    float* pml = ws_at<float>(ws, w.pml_off);
    sgqa::attn_decode_kernel<B><<<static_cast<unsigned>(rows * w.nsplit), sgqa::kDecWarps * 32, smem, st>>>(
        qb, kb, vb, sel, sel_count, po, pml, nq, G, k, q0, kv.cap, w.nsplit, scale_log2);
    SGQA_LAUNCH_CHECK("attn_decode_kernel");
    sgqa::attn_combine_kernel<<<static_cast<unsigned>(rows * 16), 64, 0, st>>>(po, pml, ob, gb, rows, w.nsplit);
    SGQA_LAUNCH_CHECK("attn_combine_kernel");
    return SGQA_OK;
  }
  const int64_t units = S * ((nq + 7) / 8) * G;
  const int64_t nbits = std::max<int64_t>((q0 + nq - 1) / B, 1);
  const int nwords = static_cast<int>((nbits + 31) / 32);
  int32_t* ids = ws_at<int32_t>(ws, w.ids_off);
  uint8_t* msk = ws_at<uint8_t>(ws, w.mask_off);
  int32_t* cnt = ws_at<int32_t>(ws, w.cnt_off);
  // bitmap, prefix of every word (or, for wide id ranges, of every eighth), masks
  auto plan_smem = [&](int pshift) {
    return static_cast<size_t>(nwords) * 4 + static_cast<size_t>(((nwords - 1) >> pshift) + 2) * 4 +
           static_cast<size_t>(k) * 8;
  };
  const int pshift = plan_smem(0) <= 96 * 1024 ? 0 : 3;
  const size_t psmem = plan_smem(pshift);
  if (psmem <= 200 * 1024) {
    cudaFuncSetAttribute(sgqa::attn_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem);
    sgqa::attn_plan_kernel<<<static_cast<unsigned>(units), sgqa::kPlanThreads, psmem, st>>>(
        sel, sel_count, nq, G, k, nwords, pshift, q0, B, ids, msk, cnt);
    SGQA_LAUNCH_CHECK("attn_plan_kernel");
  } else {
    const int pow2 = plan_pow2(k);
    const size_t ssmem = static_cast<size_t>(pow2) * 4;
    cudaFuncSetAttribute(sgqa::attn_plan_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
    sgqa::attn_plan_sort_kernel<<<static_cast<unsigned>(units), sgqa::kPlanSortThreads, ssmem, st>>>(
        sel, sel_count, nq, G, k, pow2, q0, B, ids, msk, cnt);
    SGQA_LAUNCH_CHECK("attn_plan_sort_kernel");
  }
  return launch_attn_tc<B>(p, S, q0, nq, q, kv, ids, msk, cnt, out, gate, units, st);
}

sgqa_status do_attn_kv(const sgqa_params* p, int64_t S, int64_t q0, int64_t nq, const void* q, const KvSource& kv,
                       const int32_t* sel, const int32_t* sel_count, void* out, const void* gate, void* ws,
                       cudaStream_t st) {
  switch (p->block_size) {
    case 1: return launch_attn<1>(p, S, q0, nq, q, kv, sel, sel_count, out, gate, ws, st);
    case 2: return launch_attn<2>(p, S, q0, nq, q, kv, sel, sel_count, out, gate, ws, st);
    case 4: return launch_attn<4>(p, S, q0, nq, q, kv, sel, sel_count, out, gate, ws, st);
    default: return launch_attn<8>(p, S, q0, nq, q, kv, sel, sel_count, out, gate, ws, st);
  }
}

sgqa_status do_attn(const sgqa_params* p, int64_t S, int64_t q0, int64_t nq, const void* q,
                    int64_t cap, int64_t clen, const void* kc, const void* vc, const int32_t* sel,
                    const int32_t* sel_count, void* out, const void* gate, void* ws, cudaStream_t st) {
  KvSource kv;
  kv.k = kc;
  kv.v = vc;
  kv.cap = cap;
  kv.clen = clen;
  return do_attn_kv(p, S, q0, nq, q, kv, sel, sel_count, out, gate, ws, st);
}

sgqa_status check_common(const sgqa_params* p, int64_t S, int64_t q0, int64_t nq, int64_t cap) {
  sgqa_status s = check_params(p);
  if (s != SGQA_OK) return s;
  if (S < 1) return fail(SGQA_ERR_INVALID_ARGUMENT, "num_seqs must be >= 1");
  if (q0 < 0) return fail(SGQA_ERR_INVALID_ARGUMENT, "q_pos0 must be >= 0");
  if (nq < 0) return fail(SGQA_ERR_INVALID_ARGUMENT, "nq must be >= 0");
  if (cap < q0 + nq) return fail(SGQA_ERR_INVALID_ARGUMENT, "cache_cap (%lld) < q_pos0 + nq (%lld)",
                                 (long long)cap, (long long)(q0 + nq));
  if (cap > (int64_t(1) << 31) - 1) return fail(SGQA_ERR_UNSUPPORTED, "cache_cap must be < 2^31");
  return SGQA_OK;
}

#define REQUIRE_PTR(ptr, align)                                                                 \
  do {                                                                                          \
    if ((ptr) == nullptr) return fail(SGQA_ERR_INVALID_ARGUMENT, #ptr " is NULL");             \
    if (!aligned((ptr), (align))) return fail(SGQA_ERR_INVALID_ARGUMENT, #ptr " must be %d-byte aligned", (int)(align)); \
  } while (0)

// Scratch for sgqa_sparse_attn_noalloc: a file-scope device array (one per
// device that loads the library).  Host code needs its device address, looked
// up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SGQA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_noalloc_ptr[kMaxDevices];

sgqa_status noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SGQA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_noalloc_ptr[dev].store(p, std::memory_order_release);
  }
  *ptr = p;
  return SGQA_OK;
}

}  // namespace

extern "C" {

const char* sgqa_version(void) { return "sgqa-b200 0.1 (sm_100a)"; }

uint64_t sgqa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* sgqa_last_error(void) { return g_err.c_str(); }

sgqa_status sgqa_workspace_size(const sgqa_params* p, int64_t num_seqs, int64_t nq, int64_t max_ctx,
                                size_t* bytes) {
  g_err.clear();
  sgqa_status s = check_params(p);
  if (s != SGQA_OK) return s;
  if (bytes == nullptr) return fail(SGQA_ERR_INVALID_ARGUMENT, "bytes is NULL");
  if (num_seqs < 1 || nq < 0 || max_ctx < nq) return fail(SGQA_ERR_INVALID_ARGUMENT, "bad sizes");
  const size_t iw = index_ws_bytes_upto(p, num_seqs, nq, std::max<int64_t>(max_ctx, 1));
  const AttnWs aw = attn_ws(p, num_seqs, nq);
  *bytes = std::max(iw, aw.bytes);
  return SGQA_OK;
}

sgqa_status sgqa_merge_blocks(const sgqa_params* p, int64_t num_seqs, int64_t cache_cap,
                              const void* proxy_k, const void* comp_logits, int64_t blk_begin,
                              int64_t blk_end, float* merged_f32, uint8_t* store, void* stream) {
  g_err.clear();
  sgqa_status s = check_params(p);
  if (s != SGQA_OK) return s;
  if (num_seqs < 1 || cache_cap < 0) return fail(SGQA_ERR_INVALID_ARGUMENT, "bad num_seqs/cache_cap");
  if (blk_begin < 0 || blk_end < blk_begin || blk_end * p->block_size > cache_cap)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "block range [%lld, %lld) not complete within cache_cap %lld",
                (long long)blk_begin, (long long)blk_end, (long long)cache_cap);
  if (blk_end == blk_begin) return SGQA_OK;
  REQUIRE_PTR(proxy_k, 16);
  REQUIRE_PTR(comp_logits, 16);
  REQUIRE_PTR(store, 8);
  if (merged_f32 != nullptr && !aligned(merged_f32, 16))
    return fail(SGQA_ERR_INVALID_ARGUMENT, "merged_f32 must be 16-byte aligned");
  return do_merge(p, num_seqs, cache_cap, proxy_k, comp_logits, blk_begin, blk_end, merged_f32, store,
                  static_cast<cudaStream_t>(stream));
}

sgqa_status sgqa_index_topk(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                            const void* idx_q, const float* idx_w, int64_t cache_cap,
                            const uint8_t* store, int32_t* sel, int32_t* sel_count, void* workspace,
                            size_t workspace_bytes, void* stream) {
  g_err.clear();
  sgqa_status s = check_common(p, num_seqs, q_pos0, nq, cache_cap);
  if (s != SGQA_OK) return s;
  if (nq == 0) return SGQA_OK;
  REQUIRE_PTR(idx_q, 16);
  REQUIRE_PTR(idx_w, 8);
  REQUIRE_PTR(store, 16);
  REQUIRE_PTR(sel, 4);
  REQUIRE_PTR(sel_count, 4);
  const IndexWs w = index_ws(p, num_seqs, nq, q_pos0 + nq);
  if ((s = check_ws(workspace, workspace_bytes, w.bytes)) != SGQA_OK) return s;
  return do_index(p, num_seqs, q_pos0, nq, idx_q, idx_w, cache_cap, store, sel, sel_count, workspace,
                  static_cast<cudaStream_t>(stream));
}

static sgqa_status sparse_attn_impl(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                    const void* q, int64_t cache_cap, int64_t cache_len, const void* k_cache,
                                    const void* v_cache, const int32_t* sel, const int32_t* sel_count,
                                    const void* gate, void* out, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  g_err.clear();
  sgqa_status s = check_common(p, num_seqs, q_pos0, nq, cache_cap);
  if (s != SGQA_OK) return s;
  if (cache_len < q_pos0 + nq || cache_len > cache_cap)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "need q_pos0 + nq <= cache_len <= cache_cap");
  if (nq == 0) return SGQA_OK;
  REQUIRE_PTR(q, 16);
  REQUIRE_PTR(k_cache, 16);
  REQUIRE_PTR(v_cache, 16);
  REQUIRE_PTR(sel, 4);
  REQUIRE_PTR(sel_count, 4);
  REQUIRE_PTR(out, 16);
  if (gate != nullptr && !aligned(gate, 2)) return fail(SGQA_ERR_INVALID_ARGUMENT, "gate must be 2-byte aligned");
  const AttnWs w = attn_ws(p, num_seqs, nq);
  if ((s = check_ws(workspace, workspace_bytes, w.bytes)) != SGQA_OK) return s;
  return do_attn(p, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel, sel_count, out, gate,
                 workspace, static_cast<cudaStream_t>(stream));
}

sgqa_status sgqa_sparse_attn(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                             const void* q, int64_t cache_cap, int64_t cache_len, const void* k_cache,
                             const void* v_cache, const int32_t* sel, const int32_t* sel_count,
                             void* out, void* workspace, size_t workspace_bytes, void* stream) {
  return sparse_attn_impl(p, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel, sel_count,
                          nullptr, out, workspace, workspace_bytes, stream);
}

sgqa_status sgqa_sparse_attn_gated(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                   const void* q, int64_t cache_cap, int64_t cache_len, const void* k_cache,
                                   const void* v_cache, const int32_t* sel, const int32_t* sel_count,
                                   const void* gate, void* out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  return sparse_attn_impl(p, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel, sel_count,
                          gate, out, workspace, workspace_bytes, stream);
}

static sgqa_status forward_impl(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                const void* q, const void* idx_q, const float* idx_w, int64_t cache_cap,
                                int64_t cache_len, const void* proxy_k, const void* comp_logits,
                                const void* k_cache, const void* v_cache, float* merged_f32, uint8_t* store,
                                int32_t* sel, int32_t* sel_count, const void* gate, void* out, void* workspace,
                                size_t workspace_bytes, void* stream) {
  g_err.clear();
  sgqa_status s = check_common(p, num_seqs, q_pos0, nq, cache_cap);
  if (s != SGQA_OK) return s;
  if (cache_len < q_pos0 + nq || cache_len > cache_cap)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "need q_pos0 + nq <= cache_len <= cache_cap");
  if (nq == 0) return SGQA_OK;
  REQUIRE_PTR(q, 16);
  REQUIRE_PTR(idx_q, 16);
  REQUIRE_PTR(idx_w, 8);
  REQUIRE_PTR(proxy_k, 16);
  REQUIRE_PTR(comp_logits, 16);
  REQUIRE_PTR(k_cache, 16);
  REQUIRE_PTR(v_cache, 16);
  REQUIRE_PTR(store, 16);
  REQUIRE_PTR(sel, 4);
  REQUIRE_PTR(sel_count, 4);
  REQUIRE_PTR(out, 16);
  if (merged_f32 != nullptr && !aligned(merged_f32, 16))
    return fail(SGQA_ERR_INVALID_ARGUMENT, "merged_f32 must be 16-byte aligned");
  if (gate != nullptr && !aligned(gate, 2)) return fail(SGQA_ERR_INVALID_ARGUMENT, "gate must be 2-byte aligned");
  size_t need = 0;
  if ((s = sgqa_workspace_size(p, num_seqs, nq, q_pos0 + nq, &need)) != SGQA_OK) return s;
  if ((s = check_ws(workspace, workspace_bytes, need)) != SGQA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int B = p->block_size;
  if ((s = do_merge(p, num_seqs, cache_cap, proxy_k, comp_logits, q_pos0 / B, (q_pos0 + nq) / B,
                    merged_f32, store, st)) != SGQA_OK)
    return s;
  if ((s = do_index(p, num_seqs, q_pos0, nq, idx_q, idx_w, cache_cap, store, sel, sel_count, workspace,
                    st)) != SGQA_OK)
    return s;
  return do_attn(p, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel, sel_count, out, gate,
                 workspace, st);
}

sgqa_status sgqa_forward(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                         const void* q, const void* idx_q, const float* idx_w, int64_t cache_cap,
                         int64_t cache_len, const void* proxy_k, const void* comp_logits,
                         const void* k_cache, const void* v_cache, float* merged_f32, uint8_t* store,
                         int32_t* sel, int32_t* sel_count, void* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return forward_impl(p, num_seqs, q_pos0, nq, q, idx_q, idx_w, cache_cap, cache_len, proxy_k, comp_logits, k_cache,
                      v_cache, merged_f32, store, sel, sel_count, nullptr, out, workspace, workspace_bytes, stream);
}

sgqa_status sgqa_forward_gated(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                               const void* q, const void* idx_q, const float* idx_w, int64_t cache_cap,
                               int64_t cache_len, const void* proxy_k, const void* comp_logits,
                               const void* k_cache, const void* v_cache, float* merged_f32, uint8_t* store,
                               int32_t* sel, int32_t* sel_count, const void* gate, void* out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return forward_impl(p, num_seqs, q_pos0, nq, q, idx_q, idx_w, cache_cap, cache_len, proxy_k, comp_logits, k_cache,
                      v_cache, merged_f32, store, sel, sel_count, gate, out, workspace, workspace_bytes, stream);
}

sgqa_status sgqa_sparse_attn_paged(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                   const void* q, const void* k_pool, const void* v_pool, int64_t num_pages,
                                   const int32_t* page_table, int64_t max_pages, int64_t cache_len,
                                   const int32_t* sel, const int32_t* sel_count, const void* gate, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  g_err.clear();
  sgqa_status s = check_params(p);
  if (s != SGQA_OK) return s;
  if (num_seqs < 1) return fail(SGQA_ERR_INVALID_ARGUMENT, "num_seqs must be >= 1");
  if (q_pos0 < 0 || nq < 0) return fail(SGQA_ERR_INVALID_ARGUMENT, "q_pos0 and nq must be >= 0");
  if (nq == 0) return SGQA_OK;
  if (p->block_size != 8) return fail(SGQA_ERR_UNSUPPORTED, "sgqa_sparse_attn_paged needs block_size 8");
  if (cache_len < q_pos0 + nq) return fail(SGQA_ERR_INVALID_ARGUMENT, "need q_pos0 + nq <= cache_len");
  if (max_pages * sgqa::kPageTokens < cache_len)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "max_pages (%lld) pages of %d tokens do not hold cache_len %lld",
                (long long)max_pages, sgqa::kPageTokens, (long long)cache_len);
  if (num_pages < 1 || num_pages * sgqa::kPageTokens > (int64_t(1) << 31) - 1)
    return fail(SGQA_ERR_UNSUPPORTED, "num_pages must be in [1, 2^27)");
  REQUIRE_PTR(q, 16);
  REQUIRE_PTR(k_pool, 16);
  REQUIRE_PTR(v_pool, 16);
  REQUIRE_PTR(page_table, 4);
  REQUIRE_PTR(sel, 4);
  REQUIRE_PTR(sel_count, 4);
  REQUIRE_PTR(out, 16);
  if (gate != nullptr && !aligned(gate, 2)) return fail(SGQA_ERR_INVALID_ARGUMENT, "gate must be 2-byte aligned");
  if (nq > kDecodeMaxNq) {  // the union plan of the prefill kernel lives in the workspace
    const AttnWs w = attn_ws(p, num_seqs, nq);
    if ((s = check_ws(workspace, workspace_bytes, w.bytes)) != SGQA_OK) return s;
  }
  KvSource kv;
  kv.k = k_pool;
  kv.v = v_pool;
  kv.cap = kv.clen = cache_len;
  kv.page_table = page_table;
  kv.max_pages = max_pages;
  kv.num_pages = num_pages;
  return do_attn_kv(p, num_seqs, q_pos0, nq, q, kv, sel, sel_count, out, gate, workspace,
                    static_cast<cudaStream_t>(stream));
}

sgqa_status sgqa_sparse_attn_noalloc(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                     const void* q, int64_t cache_cap, int64_t cache_len, const void* k_cache,
                                     const void* v_cache, const int32_t* sel, const int32_t* sel_count,
                                     void* out, void* stream) {
  g_err.clear();
  sgqa_status s = check_common(p, num_seqs, q_pos0, nq, cache_cap);
  if (s != SGQA_OK) return s;
  if (cache_len < q_pos0 + nq || cache_len > cache_cap)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "need q_pos0 + nq <= cache_len <= cache_cap");
  if (nq == 0) return SGQA_OK;
  if (nq > kDecodeMaxNq)
    return fail(SGQA_ERR_UNSUPPORTED, "sgqa_sparse_attn_noalloc takes at most %d queries per sequence (got %lld)",
                (int)kDecodeMaxNq, (long long)nq);
  REQUIRE_PTR(q, 16);
  REQUIRE_PTR(k_cache, 16);
  REQUIRE_PTR(v_cache, 16);
  REQUIRE_PTR(sel, 4);
  REQUIRE_PTR(sel_count, 4);
  REQUIRE_PTR(out, 16);
  // Block size 8 takes the cluster-combined decode kernel, which keeps its
  // split partials in shared memory: no scratch.  Other block sizes write
  // split partials, which live in the static array.
  void* scratch = nullptr;
  if (p->block_size != 8) {
    const AttnWs w = attn_ws(p, num_seqs, nq);
    if (w.bytes > SGQA_NOALLOC_SCRATCH_BYTES)
      return fail(SGQA_ERR_UNSUPPORTED, "call needs %zu bytes of scratch; the static array holds %u",
                  w.bytes, (unsigned)SGQA_NOALLOC_SCRATCH_BYTES);
    if ((s = noalloc_scratch(&scratch)) != SGQA_OK) return s;
  }
  return do_attn(p, num_seqs, q_pos0, nq, q, cache_cap, cache_len, k_cache, v_cache, sel, sel_count, out, nullptr,
                 scratch, static_cast<cudaStream_t>(stream));
}

sgqa_status sgqa_set_wait_limit_ns(uint64_t ns) {
  g_err.clear();
  if (ns > sgqa::kWaitLimitNs)
    return fail(SGQA_ERR_INVALID_ARGUMENT, "wait limit %llu ns is above the maximum of %llu ns",
                (unsigned long long)ns, (unsigned long long)sgqa::kWaitLimitNs);
  const uint64_t v = ns == 0 ? sgqa::kWaitLimitNs : ns;
  cudaError_t e = cudaMemcpyToSymbol(sgqa::g_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "set wait limit");
  return SGQA_OK;
}

sgqa_status sgqa_check(void* stream) {
  g_err.clear();
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int code = 0;
  e = cudaMemcpyFromSymbol(&code, sgqa::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  if (code == 0) return SGQA_OK;
  const int zero = 0;
  cudaMemcpyToSymbol(sgqa::g_status, &zero, sizeof(int));
  if (code == sgqa::kDevTimeout) return fail(SGQA_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  return fail(SGQA_ERR_DEVICE, "a kernel's device-side check failed (code %d)", code);
}

}  // extern "C"
