/*
 * dsa.h - C ABI of the B200 (sm_100a) DeepSeek-Sparse-Attention hot path:
 *         lightning indexer -> per-query top-k -> absorbed sparse MLA.
 *
 * What the calls compute (sources: the "Mistral Large 4" concept page,
 * liminalml.com/concepts/mistral-large-4, paragraphs "What to keep",
 * "Where to look", "Cache", "Sparse attention", "Query scaling"; and the
 * DSA paragraph of the reading of the technical report at
 * avisoori1x.github.io/mistral_large_4):
 *
 *   indexer     I[t,s] = sum_{j<32} w[t,j] * max(0, q[t,j,:] . k[s,:])      (128-dim heads)
 *   selection   the k best positions s <= q_pos[t] (ties to the lower position)
 *   attention   z[h,i] = (q_nope[t,h,:] . c_{s_i} + q_pe[t,h,:] . kR_{s_i}) * scale * m[t,h]
 *               o[t,h,:] = sum_i softmax_i(z[h,:]) c_{s_i}       (64 heads, 512-value latent)
 *
 * Conventions shared by every call
 *   - Every tensor argument is a DEVICE pointer owned by the caller (allocated
 *     by PyTorch or cudaMalloc); the library allocates nothing on the hot path
 *     and keeps no state between calls except a per-device error word read by
 *     dsa_check_errors().  Scratch memory is passed in as `workspace`.
 *   - All calls are asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  They only enqueue work; outputs are valid once
 *     the stream reaches that point.
 *   - bf16 tensors are row-major with the innermost dimension contiguous and
 *     every pointer 16-byte aligned.  Row strides are given in elements.
 *   - Sequence description: rows of sequence b occupy
 *     [seq_row_start[b], seq_row_start[b] + length) of EVERY cache buffer
 *     (index keys and latent caches alike); query t belongs to sequence
 *     q_seq[t] and sits at absolute position q_pos[t]; its candidates are the
 *     positions 0..q_pos[t] (its own position included).  Decode: q_pos = L-1.
 *     Prefill chunk: q_pos = P + i.
 *   - T == 0 is a no-op returning DSA_OK.
 *   - Errors: argument problems visible on the host return DSA_ERR_INVALID_ARG
 *     (nothing is launched); a failed launch returns DSA_ERR_CUDA.  Problems
 *     only visible on the device (an index or sequence id out of range, a
 *     query group that mixes sequences, a pipeline wait that gave up) do not
 *     fault: the kernel skips the bad element, sets a bit in the device error
 *     word and finishes; dsa_check_errors() reports and clears it.
 *     dsa_last_error() returns a text for the last failure on this thread.
 *   - Thread safety: calls may be issued from several host threads; calls
 *     that overlap on the GPU only share the device error word.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or stride          */
  DSA_ERR_UNSUPPORTED = 2,   /* a shape this build does not implement                  */
  DSA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed                   */
  DSA_ERR_DEVICE_CHECK = 4,  /* device-side check failed (see dsa_check_errors)        */
  DSA_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up                     */
  DSA_ERR_WORKSPACE = 6      /* workspace too small or misaligned                      */
} dsa_status_t;

/* Device error word bits (returned through dsa_check_errors' out argument). */
#define DSA_DEVERR_BAD_INDEX    0x1u  /* a selected position < 0 (other than -1 padding), past q_pos
                                         when q_pos is given, or outside the cache; or count < 0 or > k */
#define DSA_DEVERR_BAD_SEQ      0x2u  /* q_seq out of range or q_pos >= ld               */
#define DSA_DEVERR_MIXED_GROUP  0x4u  /* q_group > 1 but a group spans several sequences */
#define DSA_DEVERR_TIMEOUT      0x8u  /* a pipeline barrier wait hit its iteration limit */

/* Fixed dimensions of this build (one Mistral Large 4 attention layer). */
#define DSA_IDX_HEADS 32   /* indexer heads                        */
#define DSA_IDX_DIM   128  /* indexer head dimension               */
#define DSA_HEADS     64   /* attention heads                      */
#define DSA_LATENT    512  /* latent c_s per position              */
#define DSA_ROPE      64   /* rotary key kR_s per position (RoPE)  */

/*
 * dsa_index_scores - lightning-indexer scores.
 * Concept page, "Where to look" and "Sparse attention": a scorer with 32 small
 * heads rates every earlier position, 32 x 128 multiply-adds each.
 *
 *   q_idx   bf16 [T, 32, 128]   indexer queries
 *   w       f32  [T, 32]        per-head weights
 *   k_idx   bf16 [n_rows, 128]  index keys, rows located by seq_row_start
 *   seq_row_start int64 [B], q_seq int32 [T], q_pos int32 [T]  (device); B >= 1
 *   q_group 1: no assumption.  4 or 8: the caller guarantees that queries
 *           [q_group g, q_group (g + 1)) share one sequence (several decode
 *           queries of a sequence, e.g. drafted tokens being verified; chunked
 *           prefill); they are then scored together, q_group queries x 32
 *           heads per tensor-core tile, so each key row is read once per group.
 *   scores  f32 [T, ld]: I[t,s] for s <= q_pos[t], -inf for q_pos[t] < s < ld.
 *           ld >= max(q_pos) + 1 and ld % 4 == 0.
 *   hist    uint32 [T, 2048] or NULL (q_group 1 only): overwritten with, for
 *           each query, how many of its scores s <= q_pos[t] fall in each bin of
 *           the top 11 bits of their order-preserving key (the first histogram
 *           of dsa_topk's radix select, which then skips that pass).
 * Returns DSA_ERR_INVALID_ARG for null/misaligned pointers, T < 0, n_rows < 1,
 * n_rows >= 2^31 - 256, ld < 4 or ld % 4, q_group not 1, 4 or 8, hist with q_group > 1.
 */
dsa_status_t dsa_index_scores(const void* q_idx, const float* w, const void* k_idx,
                              int64_t n_rows, const int64_t* seq_row_start, int32_t B,
                              const int32_t* q_seq, const int32_t* q_pos, int32_t T,
                              int32_t q_group, float* scores, int64_t ld, uint32_t* hist, void* stream);

/*
 * dsa_index_scores_fp8 - lightning-indexer scores on FP8 (E4M3) keys and queries.
 * Concept page, "Where to look" and "Sparse attention" (the scorer), and the
 * 1M-token serving scenario (indexer keys kept in FP8, 128 B per position per
 * indexer layer).  The page gives no scale convention; this call takes one fp32
 * scale per key row and per query head:
 *     k[s]   = k_scale[s]   * e4m3(k8[s, :])
 *     q[t,j] = q_scale[t,j] * e4m3(q8[t, j, :])
 * and writes I[t,s] = sum_j w[t,j] * max(0, q[t,j] . k[s]) exactly as
 * dsa_index_scores does for bf16 inputs.
 *
 *   q8      uint8 [T, 32, 128]  E4M3 codes (OCP FP8 E4M3: bias 7, max 448, NaN = S.1111.111)
 *   q_scale f32   [T, 32]       > 0
 *   w       f32   [T, 32]
 *   k8      uint8 [n_rows, 128] E4M3 codes, rows located by seq_row_start
 *   k_scale f32   [n_rows]      > 0
 *   the remaining arguments (hist included), layouts, q_group and errors as
 *   dsa_index_scores; additionally DSA_ERR_INVALID_ARG for a null or misaligned
 *   q_scale / k_scale.
 * Scales must be positive (the ReLU is applied to the unscaled dot product
 * times the scales); codes must not be NaN.
 */
dsa_status_t dsa_index_scores_fp8(const void* q8, const float* q_scale, const float* w, const void* k8,
                                  const float* k_scale, int64_t n_rows, const int64_t* seq_row_start,
                                  int32_t B, const int32_t* q_seq, const int32_t* q_pos, int32_t T,
                                  int32_t q_group, float* scores, int64_t ld, uint32_t* hist, void* stream);

/*
 * dsa_topk - per-query top-k of a score array.
 * Concept page, "Sparse attention" (keeps the top 2,048) and the report's DSA
 * paragraph (chosen per query).  Candidates of query t are columns
 * 0..q_pos[t] of scores[t, :].  Ranking: higher score first; equal scores go to
 * the lower position; -0.0 == +0.0; NaN ranks as -inf.  Writes the best
 * k_eff = min(k, q_pos[t] + 1) positions to idx[t, 0:k_eff] in ascending order,
 * -1 in idx[t, k_eff:k], and k_eff to count[t].  Bit-exact and deterministic.
 *
 *   scores f32 [T, ld] (ld % 4 == 0, 16-byte aligned), q_pos int32 [T],
 *   idx int32 [T, k] (out), count int32 [T] (out), 1 <= k <= 16384.
 *   hist   uint32 [T, 2048] or NULL: the histogram dsa_index_scores wrote for
 *          these scores.  With it, the first radix pass is skipped: rows of at
 *          most 40,960 scores (ld <= 40960) are selected by one thread block
 *          per query from shared memory (no workspace); longer rows are
 *          filtered on every SM and need a workspace of
 *          dsa_topk_workspace_size(T, ld, k) bytes, 256-byte aligned.  The
 *          result is the same (a histogram that does not match the scores is
 *          detected and the row selected without it).  NULL: no workspace.
 */
size_t dsa_topk_workspace_size(int32_t T, int64_t ld, int32_t k);
dsa_status_t dsa_topk(const float* scores, int64_t ld, const int32_t* q_pos, int32_t T,
                      int32_t k, int32_t* idx, int32_t* count, const uint32_t* hist, void* workspace,
                      size_t ws_bytes, void* stream);

/*
 * sparse_mla_attend - absorbed MLA over the selected rows of a latent cache.
 * Concept page, "What to keep" (512-value latent + 64-value rotary key per
 * position shared by all 64 heads), "Sparse attention" (attention normalizes
 * over the selected positions alone, 64 x (512 + 64 + 512) multiply-adds per
 * attended position) and "Query scaling" (a per-head query multiplier).
 *
 *   q_nope bf16 [T, 64, 512]   absorbed no-rope queries (W_UK already applied)
 *   q_pe   bf16 [T, 64, 64]    rotary queries; NULL iff d_rope == 0 (NoPE layer)
 *   qmul   f32  [T, 64]        per-(t, head) query multiplier m[t,h]
 *   softmax_scale              e.g. 1/sqrt(192)
 *   cache  bf16 [n_rows, ld_c] rows [c_s (512) | kR_s (d_rope)]; ld_c >= 512 + d_rope,
 *                              ld_c % 8 == 0;  d_rope in {0, 64}
 *   seq_row_start int64 [B], q_seq int32 [T]; B >= 1
 *   q_pos  int32 [T] or NULL   when given, a selected position s of query t is
 *                              used only if s <= q_pos[t] (the causal bound:
 *                              decode q_pos = L - 1); a position past it is
 *                              skipped and flagged DSA_DEVERR_BAD_INDEX.  With
 *                              NULL only the cache bound is checked.
 *   idx    int32 [T, k] positions (ascending or not; -1 entries are skipped),
 *   count  int32 [T]    number of leading idx entries to use (<= k)
 *   out    bf16 [T, 64, 512]   o[t,h] = sum_i p_i c_{s_i}   (round to nearest even)
 *   lse    f32  [T, 64] or NULL: natural-log log-sum-exp of the logits
 *   count == 0 gives out = 0 and lse = -inf.
 *   workspace: sparse_mla_workspace_size(T, k) bytes, 256-byte aligned (may be
 *              NULL when that size is 0).  The size is 0 when each query is
 *              handled by one thread block, or split over 2-8 blocks that run as
 *              a thread-block cluster and merge their partials in distributed
 *              shared memory (used when every cluster of the call can be
 *              resident at once); otherwise it holds the fp32 split partials.
 *              dsa_plan_attend tells which case a batch size falls in.
 */
size_t sparse_mla_workspace_size(int32_t T, int32_t k);
dsa_status_t sparse_mla_attend(const void* q_nope, const void* q_pe, const float* qmul,
                               float softmax_scale, const void* cache, int64_t n_rows,
                               int32_t ld_c, int32_t d_rope, const int64_t* seq_row_start,
                               int32_t B, const int32_t* q_seq, const int32_t* q_pos,
                               const int32_t* idx, const int32_t* count,
                               int32_t T, int32_t k, void* out, float* lse, void* workspace,
                               size_t ws_bytes, void* stream);

/*
 * sparse_mla_attend_noalloc - sparse_mla_attend for callers that cannot
 * allocate device memory.
 *
 * The pages have no counterpart to this call: it is a convenience of this
 * library.  Some callers are handed only their input and output buffers and
 * may not allocate, for example code running inside another framework's
 * memory pool or an inference-engine plugin, where a cudaMalloc would bypass
 * the pool's accounting and can synchronize the whole device.  This call takes
 * the arguments of sparse_mla_attend without the workspace and computes the
 * same result with the same kernels; when a query's selection is split across
 * several thread blocks, the partial results go to a fixed scratch array
 * inside the library instead of a caller buffer.
 *   - Scratch: a file-scope __device__ array of DSA_NOALLOC_MAX_PARTIALS x 64 x
 *     516 floats (16.9 MB) that every GPU loading the library holds until the
 *     process exits.  The call allocates nothing and calls no allocating routine.
 *   - Limit: a call needs T x n_split partials, where n_split is the number of
 *     blocks each query is split across, unless those blocks merge on chip
 *     (n_split of 2-8 with every cluster resident: no scratch; n_split = 1 once
 *     T reaches the SM count: no scratch).  Calls needing more than
 *     DSA_NOALLOC_MAX_PARTIALS return DSA_ERR_WORKSPACE with a message that
 *     states the limit.  The need is not monotone in T: a smaller batch splits
 *     each query wider, so retrying with fewer queries can be refused again;
 *     dsa_plan_attend(T, 1, k, NULL, &plan) predicts it (plan.workspace_bytes
 *     > 0 means T x plan.n_split partials are needed).
 *   - Set-up: the first call on each device (and again after a device reset)
 *     looks up the array's device address (cudaGetSymbolAddress) with that
 *     device current.  Make that first call before any stream capture.
 *   - Sharing: all calls on a device use the same array, which keeps the last
 *     call's contents.  Each call overwrites every entry it reads, so nothing
 *     needs clearing, but calls that overlap on the GPU (other streams, other
 *     host threads) race on the array: the caller must serialize them.
 */
#define DSA_NOALLOC_MAX_PARTIALS 128
dsa_status_t sparse_mla_attend_noalloc(const void* q_nope, const void* q_pe, const float* qmul,
                                       float softmax_scale, const void* cache, int64_t n_rows,
                                       int32_t ld_c, int32_t d_rope, const int64_t* seq_row_start,
                                       int32_t B, const int32_t* q_seq, const int32_t* q_pos,
                                       const int32_t* idx, const int32_t* count, int32_t T, int32_t k,
                                       void* out, float* lse, void* stream);

/* One attention layer fed by a shared selection (fields as in sparse_mla_attend). */
typedef struct dsa_layer_args {
  const void* q_nope;   /* bf16 [T, 64, 512]                                  */
  const void* q_pe;     /* bf16 [T, 64, 64] or NULL (NoPE)                    */
  const float* qmul;    /* f32 [T, 64]                                        */
  const void* cache;    /* bf16 [n_rows, ld_c], or FP8 rows when cache_fp8 = 1 */
  int32_t ld_c;         /* row stride: elements (bf16) or bytes (FP8 rows)    */
  int32_t d_rope;       /* 64 or 0                                            */
  void* out;            /* bf16 [T, 64, 512], or f32 when out_f32 = 1         */
  float* lse;           /* f32 [T, 64] or NULL                                */
  int32_t out_f32;      /* 1: fp32 output (partials for dsa_lse_combine)      */
  int32_t cache_fp8;    /* 1: the cache holds FP8 latent rows (below)         */
} dsa_layer_args;

/*
 * FP8 latent-cache rows (cache_fp8 = 1).  The report's serving section keeps
 * the KV cache in FP8 natively and its training section runs FP8 with
 * blockwise scales; the pages give no layout.  This library's layout, one row
 * of ld_c bytes per position (ld_c % 16 == 0, the cache 16-byte aligned):
 *   bytes [0, 512 + d_rope)            E4M3 codes (OCP FP8 E4M3) of [c_s | kR_s]
 *   bytes [512 + d_rope, + 4 * nb)     little-endian fp32 scales: one per 128
 *                                      latent values (4) and, on RoPE layers, one
 *                                      for kR_s (nb = 5; NoPE: nb = 4)
 *   then padding (ignored)             minimum ld_c: 608 (RoPE), 528 (NoPE)
 * Column i < 512 is scale[i / 128] * e4m3(code[i]); column 512 + j is
 * scale[4] * e4m3(code[512 + j]).  The attention widens each selected row to
 * bf16 on chip (one rounding of scale * value to bf16) and then computes
 * exactly as on a bf16 cache.  Codes must not be NaN.  Every layer of one call
 * must use the same cache format (DSA_ERR_INVALID_ARG otherwise).
 */

/*
 * sparse_mla_attend_layers - sparse_mla_attend for several layers that share
 * one selection.  Concept page bullet "28 layers reuse the selection made by
 * the most recent layer that ran its indexer": every layer in `layers` (host
 * array of n_layers entries, device pointers inside; RoPE and NoPE layers may
 * be mixed) attends over idx / count.  Up to 8 layers run in one launch whose
 * work units are layers x queries x splits, so a small decode batch still
 * fills the GPU.  The remaining arguments are those of sparse_mla_attend;
 * workspace: sparse_mla_layers_workspace_size(T, n_layers, k) bytes, 256-byte
 * aligned (may be NULL when that size is 0).
 */
size_t sparse_mla_layers_workspace_size(int32_t T, int32_t n_layers, int32_t k);
dsa_status_t sparse_mla_attend_layers(int32_t n_layers, const dsa_layer_args* layers, float softmax_scale,
                                      int64_t n_rows, const int64_t* seq_row_start, int32_t B,
                                      const int32_t* q_seq, const int32_t* q_pos, const int32_t* idx,
                                      const int32_t* count, int32_t T, int32_t k, void* workspace,
                                      size_t ws_bytes, void* stream);

/*
 * dsa_sparse_mla_forward - one selection reused by several layers.
 * Concept page bullet "28 layers reuse the selection made by the most recent
 * layer that ran its indexer": the indexer and top-k run once, then every
 * layer in `layers` (host array of n_layers entries, device pointers inside)
 * attends over that selection.  Up to 8 layers run in one attention launch
 * (work units = layers x queries x splits), so a small decode batch still
 * fills the GPU; RoPE and NoPE layers may be mixed.  Queries are processed in
 * chunks so that the fp32 score rows fit the workspace (chunked prefill);
 * every chunk, the last one included, stays inside the workspace.  The
 * attention launches start copying the layers' queries (q_nope, q_pe) while
 * the call's top-k still runs: like every input, they must be complete before
 * the call in stream order and must not be written while it runs.
 *
 *   idx_out / count_out: optional [T, k] / [T] copies of the selection (NULL = not needed).
 *   workspace: at least dsa_forward_workspace_size(T, ld, k, q_group, n_layers)
 *   bytes for one pass over all queries; a smaller workspace (>= the size for
 *   q_group queries) makes the call process queries in chunks
 *   (dsa_plan_forward shows the chunking and the workspace layout).
 */
size_t dsa_forward_workspace_size(int32_t T, int64_t ld, int32_t k, int32_t q_group, int32_t n_layers);
dsa_status_t dsa_sparse_mla_forward(const void* q_idx, const float* w, const void* k_idx,
                                    int64_t n_rows, const int64_t* seq_row_start, int32_t B,
                                    const int32_t* q_seq, const int32_t* q_pos, int32_t T,
                                    int32_t q_group, int64_t ld, int32_t n_layers,
                                    const dsa_layer_args* layers, float softmax_scale,
                                    int32_t k, int32_t* idx_out, int32_t* count_out,
                                    void* workspace, size_t ws_bytes, void* stream);

/*
 * dsa_sparse_mla_forward_fp8 - dsa_sparse_mla_forward with FP8 (E4M3) index keys.
 * Concept page, 1M-token serving scenario (indexer keys kept in FP8): the
 * indexer scores E4M3 keys and queries with per-row / per-head scales exactly
 * as dsa_index_scores_fp8 does; the selection and every layer's attention are
 * those of dsa_sparse_mla_forward.  q8 uint8 [T, 32, 128], q_scale f32 [T, 32],
 * k8 uint8 [n_rows, 128], k_scale f32 [n_rows]; everything else, the workspace
 * size included, as dsa_sparse_mla_forward.
 */
dsa_status_t dsa_sparse_mla_forward_fp8(const void* q8, const float* q_scale, const float* w, const void* k8,
                                        const float* k_scale, int64_t n_rows, const int64_t* seq_row_start,
                                        int32_t B, const int32_t* q_seq, const int32_t* q_pos, int32_t T,
                                        int32_t q_group, int64_t ld, int32_t n_layers,
                                        const dsa_layer_args* layers, float softmax_scale, int32_t k,
                                        int32_t* idx_out, int32_t* count_out, void* workspace, size_t ws_bytes,
                                        void* stream);

/*
 * Context-parallel decode (report's serving section, Figures 16-17: the
 * positions of a long sequence are split over ranks; each rank scores and
 * selects among its own positions, the candidates are exchanged and merged
 * into the global selection, each rank attends over the selected rows it
 * holds, and the partial outputs are combined).  The exchanges themselves
 * (all-gathers over NCCL) are the caller's; these calls are the steps between.
 *
 * dsa_topk_export: a rank's selection as exchange candidates.  For query t and
 *   i < count[t]: out_score[t, i] = scores[t, idx[t, i]], out_pos[t, i] =
 *   idx[t, i] + pos_offset (the global position); -inf / -1 elsewhere and for
 *   -1 entries.  scores f32 [T, ld], idx int32 [T, k], count int32 [T],
 *   out_score f32 [T, k], out_pos int32 [T, k]; global positions < 2^31.
 *
 * dsa_topk_merge: the global selection from R ranks' candidates
 *   cand_score f32 [R, T, kr], cand_pos int32 [R, T, kr] (-1 = empty slot).
 *   Rank r must hold a contiguous range of positions, ranges in rank order, and
 *   list its candidates in ascending position (dsa_topk's order), so that the
 *   concatenation is in position order.  Same ranking rule as dsa_topk (score
 *   descending, ties to the lower position, -0 == +0, NaN as -inf); writes the
 *   best min(k, valid candidates) positions ascending to idx_global [T, k]
 *   (optional), their number to count [T], and (optional, together) the ones
 *   in this rank's shard [shard_lo, shard_hi) as shard-local positions
 *   (position - shard_lo), ascending and compacted, -1 after them, to
 *   idx_local [T, k], with their number in count_local [T] - the selection
 *   this rank's attention runs over.  R x kr <= 16384.
 *
 * dsa_lse_combine: merges R partial attentions over disjoint parts of one
 *   selection: o_parts f32 [R, T, 64, 512] (each normalised over its part: a
 *   layer run with out_f32 = 1), lse_parts f32 [R, T, 64] (-inf for an empty
 *   part) -> out bf16 [T, 64, 512] = sum_r exp(lse_r - lse) o_r and lse f32
 *   [T, 64] (optional) = log sum_r exp(lse_r).  1 <= R <= 64.
 */
dsa_status_t dsa_topk_export(const float* scores, int64_t ld, const int32_t* idx, const int32_t* count, int32_t T,
                             int32_t k, int64_t pos_offset, float* out_score, int32_t* out_pos, void* stream);
dsa_status_t dsa_topk_merge(const float* cand_score, const int32_t* cand_pos, int32_t R, int32_t T, int32_t kr,
                            int32_t k, int64_t shard_lo, int64_t shard_hi, int32_t* idx_global, int32_t* idx_local,
                            int32_t* count_local, int32_t* count, void* stream);
dsa_status_t dsa_lse_combine(const float* o_parts, const float* lse_parts, int32_t R, int32_t T, void* out,
                             float* lse, void* stream);

/*
 * Launch planning queries (host only: no device work, no allocation).  They
 * return what the calls above will do, from the current device's properties or
 * from `props` when it is non-NULL (then they work without a GPU).
 *
 * dsa_get_device_props: SM count of the current device and, for c = 2..8, how
 * many clusters of c attention blocks it can keep resident at once.
 *
 * dsa_plan_attend: how sparse_mla_attend (n_layers = 1) or one attention
 * launch of dsa_sparse_mla_forward (n_layers <= 8 layers) splits T queries:
 * n_split blocks per (layer, query) of rows_per_split selected rows each;
 * merge = 1 when those blocks form a cluster and merge on chip; and
 * workspace_bytes, the split partials that otherwise go through the workspace.
 * The plan is the split of least estimated time; allow_partials = 0 restricts
 * it to plans without partials (what dsa_sparse_mla_forward uses when its
 * workspace is too tight for partials: dsa_forward_plan.attend_partials = 0).
 *
 * dsa_plan_forward: how dsa_sparse_mla_forward cuts T queries into chunks for
 * a workspace of ws_bytes, and where each region sits in it (byte offsets;
 * SIZE_MAX for idx / count regions replaced by the caller's idx_out /
 * count_out, i.e. has_idx_out / has_count_out != 0; the score histogram and
 * top-k lists exist for decode, q_group = 1).  Returns
 * DSA_ERR_WORKSPACE (chunk = 0) when even q_group queries do not fit.
 */
typedef struct dsa_device_props {
  int32_t sms;                 /* streaming multiprocessors                              */
  int32_t max_clusters[9];     /* [c], c = 2..8: resident clusters of c attention blocks */
} dsa_device_props;

typedef struct dsa_attend_plan {
  int32_t n_split;             /* blocks per (layer, query)                        */
  int32_t rows_per_split;      /* selected rows per block (a multiple of 64)       */
  int32_t merge;               /* 1: the blocks of a (layer, query) merge on chip  */
  int32_t reserved;
  size_t workspace_bytes;      /* split partials in the workspace (0: none)        */
} dsa_attend_plan;

typedef struct dsa_forward_plan {
  int32_t chunk;               /* queries per chunk (a multiple of q_group, or T) */
  int32_t n_chunks;
  int32_t last_chunk;          /* queries in the final chunk                      */
  int32_t attend_partials;     /* 0: attention plans restricted to no partials    */
  size_t idx_offset;           /* [chunk, k] int32 selection (SIZE_MAX: idx_out)  */
  size_t count_offset;         /* [chunk] int32 counts (SIZE_MAX: count_out)      */
  size_t attend_offset;        /* attention split partials                        */
  size_t attend_bytes;         /* the largest need of any chunk's launches        */
  size_t hist_offset;          /* [chunk, 2048] score histogram (SIZE_MAX: none)  */
  size_t topk_offset;          /* top-k candidate lists (SIZE_MAX: none)          */
  size_t topk_bytes;
  size_t scores_offset;        /* [chunk, ld] f32 scores                          */
  size_t end;                  /* bytes used (<= ws_bytes)                        */
} dsa_forward_plan;

dsa_status_t dsa_get_device_props(dsa_device_props* out);
dsa_status_t dsa_plan_attend(int32_t T, int32_t n_layers, int32_t k, int32_t allow_partials,
                             const dsa_device_props* props, dsa_attend_plan* out);
dsa_status_t dsa_plan_forward(int32_t T, int64_t ld, int32_t k, int32_t q_group, int32_t n_layers,
                              int32_t has_idx_out, int32_t has_count_out, size_t ws_bytes,
                              const dsa_device_props* props, dsa_forward_plan* out);

/*
 * dsa_set_fault_test - testing hook for the failure-detection path of the
 * attention kernel (process-wide; affects later launches only).  The pages have
 * no counterpart to it.
 *   wait_limit_ns  limit of the kernel's pipeline waits (0: the default, 4 s)
 *   stall_tile     >= 0: every block skips gathering that 64-row tile, so the
 *                  wait for it runs out after wait_limit_ns; the kernel then
 *                  unwinds (copies drained, MMAs completed, tensor memory
 *                  freed), sets DSA_DEVERR_TIMEOUT and returns, leaving the
 *                  outputs of the affected queries undefined.  -1: off.
 * A call after dsa_set_fault_test(0, -1) behaves normally again.
 */
dsa_status_t dsa_set_fault_test(uint64_t wait_limit_ns, int32_t stall_tile);

/*
 * dsa_check_errors - synchronizes `stream`, returns DSA_ERR_DEVICE_CHECK (or
 * DSA_ERR_TIMEOUT if that bit is set) when any kernel on the current device
 * set a bit of the device error word since the last check, stores the word in
 * *bits (if non-NULL) and clears it.  DSA_OK otherwise.
 */
dsa_status_t dsa_check_errors(void* stream, uint32_t* bits);

/*
 * dsa_launch_count - number of kernels this library has launched in this
 * process so far (all devices, all threads).  Callers difference two readings
 * to count the launches of a region of work.
 */
uint64_t dsa_launch_count(void);

/* Text of the last failure reported on the calling thread ("" if none). */
const char* dsa_last_error(void);

/* ABI version of this library (major * 100 + minor): 201. */
int32_t dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
