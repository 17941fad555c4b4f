/*
 * sgqa.h -- C ABI of the Sparse GQA global-attention hot path (sm_100a).
 *
 * The operation is the one described on the page "Step-5-Preview: Sparse
 * Reads Are Not a Compressed KV Cache" (flozi.net): block-wise merging of
 * proxy keys into a compressed search store, a per-KV-group weighted-ReLU
 * indexer with causal top-k block selection, and exact softmax attention over
 * the selected original K/V plus the query's current block.  Each entry point
 * below cites the section of that page that defines it.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every tensor pointer is a DEVICE pointer owned by the caller.  The library
 *   allocates no device memory: scratch space comes from a caller workspace
 *   whose size sgqa_workspace_size() returns.  Tensors are C-contiguous in the
 *   layouts stated below; "bf16" tensors hold IEEE bfloat16 bit patterns.
 * - S = num_seqs independent sequences of equal length are processed per call.
 *   Per-sequence cache tensors are strided by `cache_cap` tokens (the cache
 *   capacity per sequence, >= cache_len).
 * - G = num_kv_groups, Hg = heads_per_group (query heads per KV group),
 *   D = head_dim, H = idx_heads (indexer heads per group), Di = idx_dim,
 *   B = block_size, k = topk (historical blocks kept per query and group).
 * - Query i of a call sits at absolute position t = q_pos0 + i (zero-based).
 * - `stream` is a cudaStream_t (passed as void*).  Calls only enqueue work on
 *   it and return; results are valid once the stream reaches that point.
 * - Return value: SGQA_OK, or an error code with a message available from
 *   sgqa_last_error() (thread-local).  Invalid arguments are rejected on the
 *   host before anything is enqueued.  No C++ exception crosses the ABI.
 * - Every wait inside the kernels is bounded in time.  A kernel that gives up
 *   sets a device status word and returns; sgqa_check() reports it as
 *   SGQA_ERR_TIMEOUT (or SGQA_ERR_DEVICE for a failed device-side check).
 */
#ifndef SGQA_H
#define SGQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SGQA_OK = 0,
  SGQA_ERR_INVALID_ARGUMENT = 1, /* a pointer, size or layout the call cannot take */
  SGQA_ERR_UNSUPPORTED = 2,      /* a valid shape this build has no kernel for   */
  SGQA_ERR_WORKSPACE = 3,        /* workspace missing, misaligned or too small   */
  SGQA_ERR_CUDA = 4,             /* a CUDA runtime/driver call or launch failed  */
  SGQA_ERR_TIMEOUT = 5,          /* a kernel's bounded wait ran out              */
  SGQA_ERR_DEVICE = 6            /* a kernel's own bounds check failed           */
} sgqa_status;

typedef struct {
  int32_t num_kv_groups;    /* G: KV groups (4 for the global layer)                */
  int32_t heads_per_group;  /* Hg: query heads sharing one KV group and selection  */
  int32_t head_dim;         /* D: main Q/K/V head width (192)                       */
  int32_t idx_heads;        /* H: indexer heads per group (4 or 8)                  */
  int32_t idx_dim;          /* Di: proxy-key / indexer width (64)                   */
  int32_t block_size;       /* B: tokens merged into one summary (8; 1, 2, 4 also)  */
  int32_t topk;             /* k: historical blocks kept per (query, group)         */
  int32_t merge_in_f32;     /* proxy keys / logits dtype: 0 = bf16, 1 = fp32        */
  float scale;              /* softmax scale; <= 0 means 1/sqrt(D)                  */
} sgqa_params;

/* Supported by this build: Hg = 16, D = 192, Di = 64, H in {4, 8},
 * B in {1, 2, 4, 8}, 1 <= k <= 2048, G >= 1.  Other values return
 * SGQA_ERR_UNSUPPORTED. */

/*
 * Bytes of workspace a call with these sizes needs (for sgqa_index_topk,
 * sgqa_sparse_attn and sgqa_forward alike).  nq = queries per sequence per
 * call, max_ctx = the largest q_pos0 + nq the workspace will serve.  The
 * workspace must be 256-byte aligned.  Pure host computation; no CUDA call.
 */
sgqa_status sgqa_workspace_size(const sgqa_params* p, int64_t num_seqs, int64_t nq,
                                int64_t max_ctx, size_t* bytes);

/*
 * Block-wise token merging.  Page section "Eight tokens become one search
 * key, coordinate by coordinate": for every completed block r in
 * [blk_begin, blk_end) and every proxy coordinate d,
 *     merged[r, d] = sum_j softmax_j(c[B r + j, d]) * kp[B r + j, d],
 * the softmax taken over the block's B logits of that coordinate with their
 * maximum subtracted, accumulated in FP32; the stored code is
 *     store[r, d] = E4M3_satfinite(BF16_rne(merged[r, d]))  (OCP FP8 E4M3).
 *
 * proxy_k, comp_logits : [S, cache_cap, Di]   bf16 (or fp32 if merge_in_f32)
 * merged_f32           : [S, cache_cap / B, Di] fp32, or NULL to skip
 * store                : [S, cache_cap / B, Di] uint8 E4M3 codes
 * Blocks must be complete: B * blk_end <= cache_cap.  Rows outside
 * [blk_begin, blk_end) are not touched.
 */
sgqa_status sgqa_merge_blocks(const sgqa_params* p, int64_t num_seqs, int64_t cache_cap,
                              const void* proxy_k, const void* comp_logits,
                              int64_t blk_begin, int64_t blk_end,
                              float* merged_f32, uint8_t* store, void* stream);

/*
 * Indexer score and causal top-k selection.  Page section "Selection is a
 * weighted ReLU score, not attention softmax": for query t, group g and
 * historical block r < floor(t / B),
 *     I[t, g, r] = sum_i w[t, g, i] * max(0, q[t, g, i] . widen(store[r])),
 * with no softmax; the k blocks with the largest I are kept, equal scores
 * going to the smaller block id.  With fewer than k candidates all are kept.
 *
 * idx_q     : [S, nq, G, H, Di] bf16 indexer queries
 * idx_w     : [S, nq, G, H]     fp32 signed head weights (prescale included)
 * store     : [S, cache_cap / B, Di] uint8 E4M3 codes; blocks
 *             [0, floor((q_pos0 + nq - 1) / B)) must be merged already
 * sel       : [S, nq, G, k] int32 out: selected block ids in ascending order,
 *             padded with -1
 * sel_count : [S, nq, G]    int32 out: min(k, floor(t / B))
 */
sgqa_status sgqa_index_topk(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                            const void* idx_q, const float* idx_w,
                            int64_t cache_cap, const uint8_t* store,
                            int32_t* sel, int32_t* sel_count,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sparse attention over the selected original K/V.  Page sections "Main
 * attention still reads original K/V" and "Selection is a weighted ReLU
 * score ...": query head h uses group g = floor(h / Hg); it attends, with
 * plain scaled dot-product scores and an exact softmax, to every token of the
 * blocks in sel[t, g] plus the positions B*floor(t/B) .. t of its current
 * block.  The Hg heads of a group share the selection.  The output is the
 * pre-gate head vector.
 *
 * q        : [S, nq, G*Hg, D] bf16
 * k_cache, v_cache : [S, cache_cap, G, D] bf16; tokens < cache_len are valid and
 *            cache_len >= q_pos0 + nq (the call's own K/V are already written)
 * sel, sel_count   : as produced by sgqa_index_topk (ids ascending, < floor(t/B))
 * out      : [S, nq, G*Hg, D] bf16
 */
sgqa_status sgqa_sparse_attn(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                             const void* q, int64_t cache_cap, int64_t cache_len,
                             const void* k_cache, const void* v_cache,
                             const int32_t* sel, const int32_t* sel_count, void* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * sgqa_sparse_attn followed by the head-wise sigmoid output gate, fused into
 * the attention kernels' final normalisation.  Page section "Main attention
 * still reads original K/V": each head's result is sigmoid-gated before the
 * heads are concatenated and projected; one gate logit per (token, head) (the
 * head-wise gate of the vendor's sibling-model configuration table,
 * "Every architecture field").
 *
 * gate : [S, nq, G*Hg] bf16 gate logits (device, 2-byte aligned), read only;
 *        out[s, t, h, :] = sigmoid(gate[s, t, h]) * attention[s, t, h, :].
 *        NULL makes the call identical to sgqa_sparse_attn.
 * Every other argument, the workspace and the errors as sgqa_sparse_attn;
 * SGQA_ERR_INVALID_ARGUMENT for a misaligned gate.
 */
sgqa_status sgqa_sparse_attn_gated(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                   const void* q, int64_t cache_cap, int64_t cache_len,
                                   const void* k_cache, const void* v_cache,
                                   const int32_t* sel, const int32_t* sel_count, const void* gate,
                                   void* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The whole hot path for one call: merge the blocks that this call's tokens
 * complete (blocks [floor(q_pos0/B), floor((q_pos0+nq)/B))), then
 * sgqa_index_topk, then sgqa_sparse_attn.  Arguments as above; the proxy keys,
 * logits and K/V of positions [q_pos0, q_pos0 + nq) must already be in the
 * caches, and blocks below floor(q_pos0/B) merged by earlier calls.  sel and
 * sel_count are outputs too.  merged_f32 may be NULL.
 */
sgqa_status sgqa_forward(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                         const void* q, const void* idx_q, const float* idx_w,
                         int64_t cache_cap, int64_t cache_len,
                         const void* proxy_k, const void* comp_logits,
                         const void* k_cache, const void* v_cache,
                         float* merged_f32, uint8_t* store,
                         int32_t* sel, int32_t* sel_count, void* out,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * sgqa_forward with the head-wise sigmoid output gate of
 * sgqa_sparse_attn_gated (gate: [S, nq, G*Hg] bf16 logits, or NULL).
 */
sgqa_status sgqa_forward_gated(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                               const void* q, const void* idx_q, const float* idx_w,
                               int64_t cache_cap, int64_t cache_len,
                               const void* proxy_k, const void* comp_logits,
                               const void* k_cache, const void* v_cache,
                               float* merged_f32, uint8_t* store,
                               int32_t* sel, int32_t* sel_count, const void* gate, void* out,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sparse attention for decode-sized calls without a caller workspace.  The
 * pages have no counterpart: this entry point exists for callers that cannot
 * allocate device memory when they call -- a host runtime that fixed its
 * device memory at start-up, or a plugin reached through a plain C interface
 * with no allocator handle -- and cudaMalloc may also synchronise the device,
 * which a latency-bound decode step must avoid.
 *
 * Same computation and arguments as sgqa_sparse_attn, minus the workspace.
 * It takes only calls with nq <= 32 queries per sequence (the split-K decode
 * path); more return SGQA_ERR_UNSUPPORTED.  With block_size 8 the splits of a
 * row combine inside their thread-block cluster and no scratch is used.  With
 * block_size 1, 2 or 4 the split partials (S * nq * G rows, each split 16 x D
 * FP32 values plus a max and a sum per head) live in the library's static
 * scratch array of SGQA_NOALLOC_SCRATCH_BYTES (16 MiB) per device; calls whose
 * partials do not fit return SGQA_ERR_UNSUPPORTED with a message.  The array
 * is a file-scope __device__ variable that every GPU loading the library
 * holds until exit.  The first call on a device that uses the array looks up
 * its device address (set-up); make that first call before any stream
 * capture.  The address is looked up once per device and process: calls
 * after cudaDeviceReset() on that device are not supported.  All calls share
 * the array, so calls that overlap on the GPU (other streams, other host
 * threads) race; order them on one stream.  Nothing in the array needs
 * clearing: every call writes each partial it reads.  No cudaMalloc, cudaFree
 * or allocating routine.
 */
#define SGQA_NOALLOC_SCRATCH_BYTES (16u << 20)
sgqa_status sgqa_sparse_attn_noalloc(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                     const void* q, int64_t cache_cap, int64_t cache_len,
                                     const void* k_cache, const void* v_cache,
                                     const int32_t* sel, const int32_t* sel_count, void* out, void* stream);

/*
 * Sparse attention over a paged K/V cache.  Page section "Cache capacity:
 * 4,104 reads do not mean 4,104 stored tokens": capacity is kept in 16-token
 * pages reached through page tables.  The computation is that of
 * sgqa_sparse_attn_gated; only where the tokens live differs: token j of
 * sequence s is row j % 16 of page page_table[s][j / 16] of the pools.  Each
 * page holds its 16 tokens group by group, so one group's 8-token block is a
 * contiguous 3 KB run (one copy).
 *
 * k_pool, v_pool : [num_pages, G, 16, D] bf16 (physical pages of 16 tokens)
 * page_table     : [S, max_pages] int32, the physical page of each logical
 *                  page; pages [0, ceil(cache_len / 16)) of every sequence
 *                  must be mapped to pages in [0, num_pages)
 * cache_len      : valid tokens of every sequence (q_pos0 + nq <= cache_len)
 * q, sel, sel_count, gate (NULL = no gate), out : as sgqa_sparse_attn_gated
 * workspace      : as sgqa_sparse_attn (sgqa_workspace_size); calls of at
 *                  most 32 queries per sequence need none (NULL, 0)
 *
 * block_size 8 only (others return SGQA_ERR_UNSUPPORTED); any number of
 * queries (decode-sized calls take the split gather, larger ones the
 * tensor-core prefill kernel).  A page-table entry outside [0, num_pages)
 * is never followed: its tokens read as zeros, sgqa_check reports
 * SGQA_ERR_DEVICE, and the outputs of the call are undefined.
 */
sgqa_status sgqa_sparse_attn_paged(const sgqa_params* p, int64_t num_seqs, int64_t q_pos0, int64_t nq,
                                   const void* q, const void* k_pool, const void* v_pool, int64_t num_pages,
                                   const int32_t* page_table, int64_t max_pages, int64_t cache_len,
                                   const int32_t* sel, const int32_t* sel_count, const void* gate, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream` and report the device status word that bounded waits
 * and device-side checks write (then clear it).  Returns SGQA_OK,
 * SGQA_ERR_TIMEOUT, SGQA_ERR_DEVICE or SGQA_ERR_CUDA.
 */
sgqa_status sgqa_check(void* stream);

/*
 * Time limit of the kernels' pipeline waits on the current device (a
 * consumer waiting for its data, a producer for a free buffer slot), in
 * nanoseconds; 0 restores the default and maximum of 2 s.  The pages have no
 * counterpart: this is a diagnostic control.  A wait that runs out makes its
 * kernel stop early (its outputs are then undefined), after it has let the
 * copies and MMAs it already issued complete, and sgqa_check() reports
 * SGQA_ERR_TIMEOUT; later calls run normally once the limit is long enough.
 * A very short limit is how the tests make those waits run out; limits
 * below 1 ms are counted in SM clock cycles (at most the given nanoseconds
 * at clocks up to 2 GHz), since the device's nanosecond timer advances in
 * steps of up to a microsecond.  The new
 * limit applies to waits that start after the call returns; do not call it
 * while kernels of this library run on the device.  Returns
 * SGQA_ERR_INVALID_ARGUMENT above the maximum, SGQA_ERR_CUDA if the device
 * variable cannot be written.
 */
sgqa_status sgqa_set_wait_limit_ns(uint64_t ns);

/* Message of the last failed call on this thread ("" if none).  The pointer
 * stays valid until the next call on this thread. */
const char* sgqa_last_error(void);

/* Library version string. */
const char* sgqa_version(void);

/* Number of kernels the library has launched in this process since it was
 * loaded (all host threads and devices together); a call that fails before a
 * launch adds nothing.  Launches issued while a stream is being captured into
 * a CUDA graph are counted once, at capture: replays of the graph add nothing.
 * Meant for counting GPU work, e.g. kernels per call in a benchmark.  Pure host
 * read; never fails. */
uint64_t sgqa_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* SGQA_H */
