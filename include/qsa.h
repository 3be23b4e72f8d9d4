/*
 * qsa.h -- C ABI of libqsa.so, the B200 (sm_100a) hot path of Qwen Sparse
 * Attention (QSA): indexer scores -> exact Top-K over 4-token groups ->
 * expansion to token ids -> GQA attention over only those tokens of a paged
 * KV cache.
 *
 * The method: "Qwen3.8-27B QSA - BF16 source weights" model card, section
 * "QSA in brief" (a learned compressed indexer picks 4-token blocks; a fixed
 * budget plus the current block; all KV stays resident); TensorRT-LLM
 * "QSASparseAttentionConfig" (exact radix Top-K over compressed groups,
 * selections expanded to individual tokens, MTP index sharing); "QSA
 * HiSparse" README (page size 64, FP8 E4M3 KV); the Ascend CANN prefill
 * article "Qwen4-Exp QSA kommt zu Huaweis Ascend", section "Was der Pull
 * Request tatsächlich hinzufügt" (-1 padding, zero output for empty rows,
 * default and explicit softmax scale).
 *
 * Conventions shared by every call
 *  - Memory: every pointer argument is device memory owned by the caller,
 *    aligned to 16 bytes.  The library never allocates or frees.  Calls that
 *    need scratch take a caller-provided workspace and report its size
 *    through a matching *_workspace_size query (a pure host function).
 *  - Streams: every call only enqueues kernels on `stream` (a cudaStream_t;
 *    NULL is the legacy default stream) and never synchronises with the host.
 *  - Errors: argument errors (shapes, dtypes, alignment, workspace size) are
 *    detected on the host and returned before anything is launched; the
 *    message is available from qsa_last_error_string() on the calling
 *    thread.  A launch failure returns QSA_ERR_CUDA.
 *  - Bad data on the device (a page id outside [0, num_pages), a token id
 *    outside the page table, a selected group outside the candidates) is
 *    skipped and ORed into *dev_status as a QSA_DEV_* bit when dev_status is
 *    not NULL.  No kernel traps.  The status word is only ever ORed into;
 *    the caller clears it.  The word is the caller's, one uint32 of device
 *    memory passed to every call; qsa_get_device_status reads it on the host
 *    and turns its bits into QSA_ERR_DEVICE_INDEX or QSA_ERR_TIMEOUT.  (The
 *    "QSA HiSparse" README's offload contract has unsupported configurations
 *    fail at start-up; a kernel cannot return a code, so errors found on the
 *    device go through this word instead of aborting the context.)
 *  - Layouts (row-major, innermost last):
 *      indexer query    q_idx        [T, H_I, D_I]          f32 | bf16
 *      indexer weights  w_idx        [T, H_I]               f32
 *      indexer keys     k_idx_pages  [num_pages, 16, D_I]   f32 | bf16
 *                       (one compressed key per 4-token group; a 64-token
 *                        page holds 16 groups and shares the KV page table)
 *      KV cache         k_pages, v_pages [num_pages, 64, Hkv, D]
 *                                                           f32 | bf16 | fp8 e4m3
 *      page table       page_table   [pt_rows, pt_stride]   int32 physical page ids
 *      query            q            [T, Hq, D]             f32 | bf16
 *      output           out          [T, Hq, D]             f32 | bf16
 *      log-sum-exp      lse          [T, Hq]                f32 (natural log)
 *    Query token t belongs to request q_req[t] (q_req NULL: request t), a row
 *    of the page table (a request id outside [0, pt_rows) skips the row and
 *    sets QSA_DEV_BAD_REQUEST), and sits at absolute position q_pos[t]; its
 *    current block is group c = q_pos[t] / 4 and its candidates are the
 *    complete groups 0..c-1.
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define QSA_API __attribute__((visibility("default")))
#else
#define QSA_API
#endif

typedef struct CUstream_st* qsa_stream_t; /* the same type as cudaStream_t */

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1, /* a null pointer, bad shape, misalignment */
  QSA_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement */
  QSA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
  QSA_ERR_CUDA = 4,        /* a CUDA launch, copy or attribute call failed */
  QSA_ERR_DEVICE_INDEX = 5, /* qsa_get_device_status: a kernel skipped bad data on
                               the device (a page, token, group or request id out
                               of range; any QSA_DEV_* bit but QSA_DEV_TIMEOUT) */
  QSA_ERR_TIMEOUT = 6      /* qsa_get_device_status: a bounded wait inside a kernel
                              ran out (QSA_DEV_TIMEOUT); that launch's outputs are
                              invalid */
} qsa_status_t;

typedef enum { QSA_F32 = 0, QSA_BF16 = 1, QSA_FP8_E4M3 = 2 } qsa_dtype_t;

/* bits ORed into *dev_status by the kernels */
#define QSA_DEV_BAD_PAGE 1u   /* a page-table entry outside [0, num_pages) */
#define QSA_DEV_BAD_TOKEN 2u  /* a token id < -1 or beyond the page table */
#define QSA_DEV_BAD_GROUP 4u  /* a selected group outside the candidates */
#define QSA_DEV_ROW_RANGE 8u  /* a row's candidates exceed score_stride or
                                 its tokens exceed W */
#define QSA_DEV_BAD_REQUEST 16u /* a request id outside [0, pt_rows) */
#define QSA_DEV_TIMEOUT 32u   /* a bounded wait inside a kernel ran out (the
                                 kernel stopped early; its outputs are invalid) */

/* Before stage 1 -- the indexer projection (a reading fixed by this library:
 * "QSA in brief" names a learned indexer, not its layers).  y[t, n] =
 * sum_h x[t, h] * w[n, h] in FP32 for hidden states x [T, H] and weights
 * w [N, H] (each F32 or BF16, 16-byte aligned, H a multiple of 8); y [T, N]
 * FP32, row-major.  Stacking w = [W_q; W_w; W_k] ([H_I*D_I + H_I + D_I, H])
 * gives every token's indexer query (y[t, 0 .. H_I*D_I)), head weights
 * (next H_I) and token key (last D_I) in one call.  A few tokens (decode)
 * take a GEMV that reads w once; BF16 x and w with T >= 128 and H a multiple
 * of 64 take a tcgen05 GEMM (TMA-fed tiles, TMEM accumulators).
 * workspace: none (qsa_indexer_project_workspace_size returns 0). */
QSA_API size_t qsa_indexer_project_workspace_size(int T, int H, int N);
QSA_API qsa_status_t qsa_indexer_project(const void* x, qsa_dtype_t x_dt, const void* w, qsa_dtype_t w_dt, int T,
                                         int H, int N, float* y, uint32_t* dev_status, qsa_stream_t stream);

/* Before stage 1 -- the C4 compressed-key write ("QSA in brief": the indexer
 * keys are compressed over four-token blocks; "QSA HiSparse", entry-point
 * table: the backend's prefill writes; the compression itself is a reading
 * fixed by this library).  For each of n_groups completed groups i, with
 * token keys k_tok[(4*i + j) * tok_stride + e] (j = 0..3 the group's tokens
 * in order, e < D_I; FP32):
 *   khat[d] = bias[d] + sum_{j<4} sum_{e<D_I} wphi[d * 4*D_I + j*D_I + e] * k_tok[...]
 * (wphi [D_I, 4*D_I] FP32; bias [D_I] FP32 or NULL), written to row
 * g_id[i] % 16 of page page_table[g_req[i]][g_id[i] / 16] of k_idx_pages
 * [num_pages, 16, D_I] in k_dt (F32, or BF16 rounded to nearest even).
 * g_req NULL: every group belongs to request 0.  A request id outside
 * [0, pt_rows) sets QSA_DEV_BAD_REQUEST, a group id < 0 or beyond the page
 * table QSA_DEV_BAD_GROUP, a physical page outside [0, num_pages)
 * QSA_DEV_BAD_PAGE; such groups are not written.  Nothing else in
 * k_idx_pages changes.  D_I in {32, 64, 128}.  With tok_stride the rows of
 * qsa_indexer_project's output can be read in place (k_tok = y + H_I*D_I +
 * H_I, tok_stride = N, four consecutive tokens per group).
 * workspace: none (qsa_compress_keys_workspace_size returns 0). */
QSA_API size_t qsa_compress_keys_workspace_size(int n_groups, int D_I);
QSA_API qsa_status_t qsa_compress_keys(const float* k_tok, int tok_stride, int n_groups, const int32_t* g_req,
                                       const int32_t* g_id, const float* wphi, const float* bias, int D_I,
                                       void* k_idx_pages, qsa_dtype_t k_dt, int num_pages,
                                       const int32_t* page_table, int pt_rows, int pt_stride,
                                       uint32_t* dev_status, qsa_stream_t stream);

/* Width of one row of the optional prefix histogram passed from stage 1 to
 * stage 2 (prefix_hist below): one uint32 count per value of the top 12 bits
 * of a score's order key.  The order key of a float is its bit pattern with
 * the sign bit set when the sign is clear, and with every bit flipped when the
 * sign is set (-0.0 counts as +0.0): unsigned key order is score order. */
#define QSA_PREFIX_HIST_BINS 4096

/* Stage 1 -- indexer scores.
 * For every query token t and complete group g < c = q_pos[t]/4 (capped at
 * score_stride):  scores[t*score_stride + g] = sum_h w_idx[t,h] *
 * ReLU(q_idx[t,h,:] . khat[g,:]), computed in FP32.  khat[g] is row g%16 of
 * page page_table[q_req[t]][g/16].  Entries g >= c are either left as they
 * are or set to -inf (the tensor-core pass writes whole tiles).  A group
 * whose page id is out of range scores -inf and sets QSA_DEV_BAD_PAGE.
 * Supported: H_I in {2, 4}, D_I in {32, 64, 128}, q_dt and k_dt F32 or BF16.
 * The score formula is the one this library fixes for the learned compressed
 * indexer ("QSA in brief" names the indexer, not its formula).
 * prefix_hist (optional; NULL = not used): [T, QSA_PREFIX_HIST_BINS] uint32,
 * all zero on entry.  The streaming scan (the pass used unless T >= 256 with
 * BF16 query and keys, H_I = 4, D_I = 128) adds to row t one count per score
 * it writes, in the bin of the score's top 12 order-key bits.  The tensor-core
 * pass leaves the buffer as it is.  Given to the Top-K call that reads these
 * scores, the histogram replaces that call's first radix passes; the Top-K
 * call zeroes it again. */
/* Workspace of qsa_index_scores: 0 bytes for every supported shape (the scan
 * and the tensor-core pass keep their state on chip).  Every stage has such a
 * query so that a caller can size all of them the same way. */
QSA_API size_t qsa_index_scores_workspace_size(int T, int H_I, int D_I, int score_stride);
QSA_API qsa_status_t qsa_index_scores(const void* q_idx, qsa_dtype_t q_dt, const float* w_idx,
                              const void* k_idx_pages, qsa_dtype_t k_dt, int num_pages,
                              const int32_t* page_table, int pt_rows, int pt_stride,
                              const int32_t* q_req, const int32_t* q_pos, int T, int H_I,
                              int D_I, float* scores, int score_stride, uint32_t* prefix_hist,
                              uint32_t* dev_status, qsa_stream_t stream);

/* Stage 2 -- exact Top-K over compressed groups (TensorRT-LLM
 * "QSASparseAttentionConfig", enable_heuristic_topk: the exact radix Top-K).
 * For every row t, keeps n = min(K, c) of the candidates 0..c-1 (c =
 * q_pos[t]/4, capped at score_stride) ranked by score descending, ties to the
 * lower group id (-0.0 ranks equal to +0.0; scores must not be NaN).
 * sel [T, K] receives the kept group ids in ascending order followed by -1;
 * n_sel [T] receives n.  c <= K keeps every candidate (dense fallback).
 * workspace: qsa_topk_groups_workspace_size() bytes (may be 0 / NULL).
 * prefix_hist (optional; NULL = not used): the histogram qsa_index_scores
 * built while writing these scores, unchanged since.  A row whose histogram
 * total equals its candidate count c takes the bin of its n-th largest key
 * from it instead of from radix passes over the scores; any other row runs
 * the full passes.  The outputs are the same either way.  On return rows
 * 0..T-1 of prefix_hist are zero, ready for the next qsa_index_scores. */
QSA_API size_t qsa_topk_groups_workspace_size(int T, int K, int score_stride);
QSA_API qsa_status_t qsa_topk_groups(const float* scores, int score_stride, uint32_t* prefix_hist,
                             const int32_t* q_pos, int T, int K, int32_t* sel, int32_t* n_sel,
                             void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                             qsa_stream_t stream);

/* Stage 2 as a guess-verify-refine Top-K with hint-free self-sampling
 * (TensorRT-LLM "QSASparseAttentionConfig", enable_heuristic_topk: the GVR
 * Top-K, for group budgets of 512, 1,024 and 2,048, falling back to the exact
 * radix Top-K otherwise).  Same inputs, outputs and result as
 * qsa_topk_groups: the exact top-min(K, c) of every row, ties to the lower
 * group id, ascending, -1 padded.  Per row it guesses from a strided sample
 * of the row's own scores where the K-th largest lies, verifies the guess by
 * exact counts, and refines with an exact select among the candidates the
 * guess leaves; a row whose guess fails takes a radix select over the whole
 * row.  The guess is a window of 12-bit key bins around the sample's rank of
 * the K-th key; the counts of the keys above and in it are exact, and the
 * select runs over the window's keys alone.  Rows run as qsa_topk_groups
 * runs them: one CTA per row for many rows (148 or more) of up to 32,768
 * candidates and for rows of up to 8,192, one thread-block cluster per row
 * otherwise (decode).  score_stride at most 262,144.  path (optional, [T]
 * int32) receives per row: 0 dense (c <= K), 1 the guess verified, 3 the
 * radix select over the whole row.
 * For K outside {512, 1024, 2048} the call runs qsa_topk_groups instead (a
 * message on stderr the first time) and leaves path unwritten. */
QSA_API qsa_status_t qsa_topk_groups_gvr(const float* scores, int score_stride, const int32_t* q_pos, int T, int K,
                                         int32_t* sel, int32_t* n_sel, int32_t* path, uint32_t* dev_status,
                                         qsa_stream_t stream);

/* Stage 3 -- expansion of the kept groups to token ids ("QSA in brief": the
 * budget plus the current block; TensorRT-LLM get_indices_block_size: the
 * selections address single tokens; the MTP index-sharing field).
 * Row t of tok [T, W] becomes: tokens 4g..4g+3 of each sel[t, 0..n_sel)
 * entry, then -- when capture_pos is not NULL and p0 = capture_pos[t] <
 * q_pos[t] -- the groups c(p0)..c(p)-1 completed since the capture, then the
 * current block 4c(p)..p, then -1 padding.  n_tok[t] = the used width.  A
 * sel entry outside [0, c(p0)) becomes four -1 slots and sets
 * QSA_DEV_BAD_GROUP; a row wider than W is cut at W and sets
 * QSA_DEV_ROW_RANGE.  W >= 4*K + 4 (+4 per group completed since capture). */
/* Workspace of qsa_expand_select: 0 bytes (one thread per output slot). */
QSA_API size_t qsa_expand_select_workspace_size(int T, int K, int W);
QSA_API qsa_status_t qsa_expand_select(const int32_t* sel, const int32_t* n_sel, int K,
                               const int32_t* q_pos, const int32_t* capture_pos, int T,
                               int32_t* tok, int32_t* n_tok, int W, uint32_t* dev_status,
                               qsa_stream_t stream);

/* Stages 2 and 3 in one launch, for rows without an MTP capture: exactly
 * qsa_topk_groups(scores, score_stride, prefix_hist, q_pos, T, K, sel, n_sel)
 * followed by qsa_expand_select(sel, n_sel, K, q_pos, NULL, T, tok, n_tok, W),
 * with the same outputs, layouts and status bits (prefix_hist as there).  The
 * expansion is not defined by the pages as a separate pass: joining it to the
 * selection saves a launch and a read of sel on the decode path.
 * W >= 4*K + 4. */
QSA_API qsa_status_t qsa_topk_expand(const float* scores, int score_stride, uint32_t* prefix_hist,
                             const int32_t* q_pos, int T, int K, int32_t* sel, int32_t* n_sel,
                             int32_t* tok, int32_t* n_tok, int W, uint32_t* dev_status,
                             qsa_stream_t stream);

/* The sequence-length threshold separating dense and QSA attention
 * (TensorRT-LLM "QSASparseAttentionConfig", seq_len_threshold): `requested`
 * tokens, or the token budget 4*K when requested <= 0; a value below 4*K is
 * raised to 4*K, as it cannot reduce attention work.  Pure host function. */
QSA_API int qsa_seq_len_threshold(int requested, int K);
/* Dense rows of the threshold: every query whose sequence q_pos[t] + 1 is at
 * most `threshold` tokens gets the token list 0 .. q_pos[t] (n_tok =
 * q_pos[t] + 1, -1 padded to W), i.e. dense causal attention; the other rows
 * of tok / n_tok are left as they are (the QSA selection of stage 3).  A
 * dense row longer than W is cut and sets QSA_DEV_ROW_RANGE.  threshold <= 0:
 * nothing is written. */
QSA_API qsa_status_t qsa_dense_select(const int32_t* q_pos, int T, int threshold, int32_t* tok, int32_t* n_tok,
                                      int W, uint32_t* dev_status, qsa_stream_t stream);

/* Stage 4 -- GQA attention over the selected tokens ("QSA in brief": only the
 * selected entries are read; the Ascend article: rows with nothing to attend
 * give exact zeros, the D-based scale is the default).
 * For query t and head h (KV head kv = h / (Hq/Hkv)), over the entries j of
 * tok[t, 0..n_tok[t]) other than -1:
 *   logit_j = scale * q[t,h,:] . K(j),  out[t,h,:] = sum_j softmax(logit)_j V(j),
 *   lse[t,h] = log sum_j exp(logit_j)   (-inf and out = 0 for an empty row)
 * K(j) / V(j) are row (page_table[r][j/64], j%64, kv) of k_pages / v_pages
 * with r = q_req[t]; FP8 values are code * k_scale (or v_scale); the scales
 * are ignored for F32 / BF16 caches.  scale = sm_scale, or 1/sqrt(D) when
 * sm_scale <= 0.  lse may be NULL.
 * Supported: D in {64, 128, 256}, Hq/Hkv <= 16, q_dt F32 or BF16, kv_dt F32,
 * BF16 or FP8_E4M3, out_dt F32 or BF16.
 * _decode with fewer (query, KV head) rows than SMs (the BF16 / FP8 caches,
 * D 128 or 256) splits every row's tokens over several CTAs, one per SM;
 * each CTA leaves its partial (o, max, sum) in the workspace and a second
 * kernel merges a row's partials: qsa_sparse_attn_decode_workspace_size(...,
 * kv_dt) bytes (0 when the rows fill the GPU and nothing is split).
 * _prefill gives each (query, KV head) its own warp and needs no workspace. */
QSA_API size_t qsa_sparse_attn_decode_workspace_size(int T, int Hq, int Hkv, int D, int W,
                                                     qsa_dtype_t kv_dt);
QSA_API qsa_status_t qsa_sparse_attn_decode(const void* q, qsa_dtype_t q_dt, const void* k_pages,
                                    const void* v_pages, qsa_dtype_t kv_dt, float k_scale,
                                    float v_scale, int num_pages, const int32_t* page_table,
                                    int pt_rows, int pt_stride, const int32_t* q_req,
                                    const int32_t* tok,
                                    const int32_t* n_tok, int W, int T, int Hq, int Hkv, int D,
                                    float sm_scale, void* out, qsa_dtype_t out_dt, float* lse,
                                    void* workspace, size_t workspace_bytes,
                                    uint32_t* dev_status, qsa_stream_t stream);

/* Stages 3 and 4 in one call for decode: exactly
 *   qsa_expand_select(sel, n_sel, K, q_pos, capture_pos, T, tok, n_tok, W)
 *   qsa_sparse_attn_decode(..., tok, n_tok, W, ...)
 * with the same out / lse and status bits, without the token lists in
 * between: the decode kernel that spreads few rows over every SM (BF16 / FP8
 * caches, D 128 or 256) lists each chunk's tokens from the selection itself
 * (4 per kept group, then 4*c(p0) .. p, cut at W).  For other shapes the
 * call writes the lists into its workspace first and runs the regular
 * decode.  capture_pos may be NULL (no MTP reuse).  W >= 4*K + 4 (+4 per
 * group completed since the capture).  Workspace:
 * qsa_sparse_attn_decode_sel_workspace_size(...) bytes, 16-byte aligned
 * (0: none needed); pointers as for the two calls it replaces. */
QSA_API size_t qsa_sparse_attn_decode_sel_workspace_size(int T, int Hq, int Hkv, int D, int W,
                                                         qsa_dtype_t kv_dt);
QSA_API qsa_status_t qsa_sparse_attn_decode_sel(const void* q, qsa_dtype_t q_dt, const void* k_pages,
                                                const void* v_pages, qsa_dtype_t kv_dt, float k_scale,
                                                float v_scale, int num_pages, const int32_t* page_table,
                                                int pt_rows, int pt_stride, const int32_t* q_req,
                                                const int32_t* sel, const int32_t* n_sel, int K,
                                                const int32_t* q_pos, const int32_t* capture_pos, int W, int T,
                                                int Hq, int Hkv, int D, float sm_scale, void* out,
                                                qsa_dtype_t out_dt, float* lse, void* workspace,
                                                size_t workspace_bytes, uint32_t* dev_status,
                                                qsa_stream_t stream);

/* Workspace of qsa_sparse_attn_prefill: 0 bytes (each (query, KV head) row is
 * finished by the warps that stream it). */
QSA_API size_t qsa_sparse_attn_prefill_workspace_size(int T, int Hq, int Hkv, int D, int W,
                                                      qsa_dtype_t kv_dt);
QSA_API qsa_status_t qsa_sparse_attn_prefill(const void* q, qsa_dtype_t q_dt, const void* k_pages,
                                     const void* v_pages, qsa_dtype_t kv_dt, float k_scale,
                                     float v_scale, int num_pages, const int32_t* page_table,
                                     int pt_rows, int pt_stride, const int32_t* q_req,
                                     const int32_t* tok,
                                     const int32_t* n_tok, int W, int T, int Hq, int Hkv, int D,
                                     float sm_scale, void* out, qsa_dtype_t out_dt, float* lse,
                                     uint32_t* dev_status, qsa_stream_t stream);

/* qsa_sparse_attn_decode without a workspace argument, for callers that cannot
 * allocate device memory: code recorded into a CUDA graph that must not
 * allocate, code running under a memory pool that is already fully carved up,
 * or a plugin layer that is handed only its input and output buffers.  (The
 * pages have no counterpart: this is a deployment convenience of this
 * library, not part of the method.)
 * Same arguments, results and checks as qsa_sparse_attn_decode.  The split-K
 * scratch lives in a fixed array of QSA_DECODE_NOALLOC_SCRATCH_BYTES inside
 * the library, which every GPU that loads libqsa.so keeps until the process
 * exits; a shape whose scratch (qsa_sparse_attn_decode_workspace_size) is
 * larger is refused with QSA_ERR_WORKSPACE.  The call allocates nothing.
 * The arguments are checked exactly as qsa_sparse_attn_decode checks them,
 * before the scratch size.  The first call on a device looks up that device's
 * copy of the array (cudaGetSymbolAddress, with the device current) and keeps
 * the address: make that first call before any stream capture on the device.
 * The address belongs to the device's primary context; after cudaDeviceReset,
 * or from another context, do not call this entry point again on that device.  Every call shares the one array
 * and every kernel overwrites all the scratch it later reads, so nothing
 * needs clearing; but calls whose kernels overlap on the GPU (two streams, or
 * two host threads) race on it -- serialise them. */
#define QSA_DECODE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
QSA_API qsa_status_t qsa_sparse_attn_decode_noalloc(
    const void* q, qsa_dtype_t q_dt, const void* k_pages, const void* v_pages, qsa_dtype_t kv_dt,
    float k_scale, float v_scale, int num_pages, const int32_t* page_table, int pt_rows,
    int pt_stride, const int32_t* q_req, const int32_t* tok, const int32_t* n_tok, int W, int T,
    int Hq, int Hkv, int D, float sm_scale, void* out, qsa_dtype_t out_dt, float* lse,
    uint32_t* dev_status, qsa_stream_t stream);

/* Sequence-sharded decode (decode context parallelism; the Ascend article's
 * context section names it for the QSA path).  R shards each hold a
 * contiguous range of every request's pages -- shard r the groups
 * [g_lo, g_hi), g_lo a multiple of 16 -- as a slice of the page table over
 * the same (or its own) KV cache and compressed keys.  A decode step:
 *   qsa_dcp_shard_positions  -> q_pos_local (per shard)
 *   qsa_index_scores, qsa_topk_groups on the shard (q_pos_local, its slice)
 *   qsa_dcp_candidates       -> (score, global group id) records [T, K]
 *   all-gather of the records over the shards -> [R, T, K] (shard order)
 *   qsa_dcp_merge_topk       -> the global selection sel [T, K], n_sel [T]
 *   qsa_dcp_expand           -> the shard's token lists (shard-local ids)
 *   qsa_sparse_attn_decode on the shard (F32 out, lse) -> partials
 *   all-gather of the partials -> [R, T, Hq, D], [R, T, Hq]
 *   qsa_dcp_merge_attn       -> out [T, Hq, D], lse [T, Hq]
 * The selection is exactly the one unsharded stage 2 makes from the same
 * scores (each of the global K best is among the K best of its shard), and
 * the merged output is the attention over the same tokens. */
/* q_pos_local[t] = 4 * clamp(q_pos[t] / 4 - g_lo, 0, g_hi - g_lo): the shard's
 * candidate count as a query position, for stages 1 and 2 on the slice. */
QSA_API qsa_status_t qsa_dcp_shard_positions(const int32_t* q_pos, int T, int g_lo, int g_hi,
                                             int32_t* q_pos_local, qsa_stream_t stream);
/* The shard's selection sel/n_sel [T, K] (shard-local ids, ascending, from
 * qsa_topk_groups on its scores [T, score_stride]) as records:
 * cand_id = sel + g_lo, cand_score = that group's score; slots past n_sel
 * get (-inf, -1).  A sel entry outside [0, score_stride) becomes (-inf, -1)
 * and sets QSA_DEV_BAD_GROUP. */
QSA_API qsa_status_t qsa_dcp_candidates(const float* scores, int score_stride, const int32_t* sel,
                                        const int32_t* n_sel, int T, int K, int g_lo, float* cand_score,
                                        int32_t* cand_id, uint32_t* dev_status, qsa_stream_t stream);
/* The global top-K of the gathered records cand_score / cand_id [R, T, K]
 * (shard r's block at r * T * K): n_sel[t] = min(K, real records of row t),
 * sel[t] their ids ranked by (score descending, id ascending), written in
 * ascending id order and padded with -1.  The output order relies on the
 * records ascending by id in (shard, slot) order, which holds for records
 * of shards with ascending group ranges.  R * K <= 16384. */
QSA_API qsa_status_t qsa_dcp_merge_topk(const float* cand_score, const int32_t* cand_id, int R, int T, int K,
                                        int32_t* sel, int32_t* n_sel, qsa_stream_t stream);
/* The shard's part of the global selection sel/n_sel [T, K] (ascending global
 * ids): tokens 4(g - g_lo) .. 4(g - g_lo) + 3 of every selected g in
 * [g_lo, g_hi), then -- when the current block c = q_pos[t] / 4 lies in
 * [g_lo, g_hi) -- its tokens 4(c - g_lo) .. q_pos[t] - 4 g_lo, as shard-local
 * token ids, ascending, -1 padded to W; n_tok[t] the count.  A row wider than
 * W is cut and sets QSA_DEV_ROW_RANGE. */
QSA_API qsa_status_t qsa_dcp_expand(const int32_t* sel, const int32_t* n_sel, int K, const int32_t* q_pos, int T,
                                    int g_lo, int g_hi, int32_t* tok, int32_t* n_tok, int W,
                                    uint32_t* dev_status, qsa_stream_t stream);
/* LSE merge of R partial attentions: o_parts [R, T, Hq, D] (F32, each
 * normalised over its shard's tokens) and lse_parts [R, T, Hq] (natural log,
 * -inf for a shard without tokens): out = sum_r exp(lse_r - LSE) o_r with
 * LSE = log sum_r exp(lse_r); rows where every shard is empty give 0 and
 * -inf.  out_dt F32 or BF16; lse may be NULL. */
QSA_API qsa_status_t qsa_dcp_merge_attn(const float* o_parts, const float* lse_parts, int R, int T, int Hq, int D,
                                        void* out, qsa_dtype_t out_dt, float* lse, qsa_stream_t stream);

/* Device status query (the boundary's error channel for data the kernels
 * check on the device; see "Conventions" above).  Waits for `stream` to finish
 * the work queued so far, reads the caller's status word dev_status and
 * returns:
 *   QSA_ERR_TIMEOUT       when QSA_DEV_TIMEOUT is set (it wins over the rest),
 *   QSA_ERR_DEVICE_INDEX  when any other QSA_DEV_* bit is set,
 *   QSA_OK                when the word is zero,
 *   QSA_ERR_CUDA          when the synchronisation or the copy failed
 *                         (a kernel fault earlier on the stream shows here),
 *   QSA_ERR_INVALID_ARG   when dev_status is NULL or not 4-byte aligned.
 * bits_out (host memory, may be NULL) receives the raw word.  clear != 0 sets
 * the word back to zero after reading it.  Unlike the compute calls, this one
 * synchronises with the host: call it between steps, never inside a stream
 * capture. */
QSA_API qsa_status_t qsa_get_device_status(uint32_t* dev_status, uint32_t* bits_out, int clear,
                                           qsa_stream_t stream);

/* Self-test of the bounded wait that every TMA / tensor-core kernel of this
 * library uses for its mbarrier phases (the error channel above, for a wait
 * that never completes).  One CTA of two warps: warp 0 puts a 16-byte bulk
 * copy in flight on one barrier, then waits on a second barrier that nothing
 * arrives at, with a limit of limit_us microseconds (1 .. 1,000,000); when it
 * runs out the warp sets the CTA's abort flag and ORs QSA_DEV_TIMEOUT into
 * *dev_status.  Warp 1 waits on the same barrier with a limit one second
 * longer and must be released by the abort flag instead.  Warp 0 then drains
 * the bulk copy (bounded too) before the CTA exits.  No fault, trap or hang:
 * the context stays usable.  report (device memory, 6 x uint32, written):
 *   [0] warp 0's wait result (0: timed out), [1] warp 1's wait result
 *   (0: released), [2] warp 0's wait in microseconds, [3] warp 1's,
 *   [4] 1 when the drain saw the copy land, [5] 1 when its 16 bytes match.
 * dev_status must not be NULL.  QSA_ERR_INVALID_ARG for a NULL pointer or a
 * limit out of range. */
QSA_API qsa_status_t qsa_selftest_bounded_wait(uint32_t limit_us, uint32_t* dev_status, uint32_t* report,
                                               qsa_stream_t stream);

/* Human-readable message for the last non-OK status returned on this thread. */
QSA_API const char* qsa_last_error_string(void);
/* Static name of a status code. */
QSA_API const char* qsa_status_name(qsa_status_t s);
/* ABI version: bumped on any change of the entry points (2: the decode
 * workspace query takes the KV dtype; 3: qsa_topk_expand; 4: the prefix_hist
 * argument of qsa_index_scores, qsa_topk_groups and qsa_topk_expand; 5: the
 * status codes QSA_ERR_DEVICE_INDEX / QSA_ERR_TIMEOUT, qsa_get_device_status
 * and a workspace query for every stage; 6: qsa_indexer_project and
 * qsa_compress_keys; 7: the sequence-sharded decode calls qsa_dcp_*; 8:
 * qsa_topk_groups_gvr; 9: qsa_seq_len_threshold and qsa_dense_select; 10:
 * qsa_selftest_bounded_wait; 11: qsa_sparse_attn_decode_sel). */
QSA_API int qsa_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* QSA_H */
