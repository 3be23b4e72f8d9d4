/*
 * qsa_oracle.h -- plain CPU oracle for the Qwen Sparse Attention (QSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (libqsa.so and its Python binding) never calls it and shares no code,
 * header, table or helper with it.
 *
 * What it computes (all four stages of QSA for one layer):
 *   1. indexer scores  s[t,g] = sum_h w[t,h] * ReLU(q_I[t,h,:] . khat[g,:])
 *      over the complete 4-token groups g < c(p) = floor(p/4);
 *   2. the exact top-min(K,c) groups under (score desc, group id asc);
 *   3. the expansion of the kept groups to token ids plus the current block
 *      (tokens 4c..p), with optional multi-token-prediction (MTP) reuse;
 *   4. softmax attention of every query head over exactly those tokens of a
 *      paged KV cache (page size 64), GQA head sharing.
 * Sources: "Qwen3.8-27B QSA - BF16 source weights" model card, section "QSA in
 * brief" (4-token blocks, learned compressed indexer, fixed budget plus the
 * current block, all KV resident); TensorRT-LLM "QSASparseAttentionConfig"
 * (exact radix Top-K over compressed groups, token-level expanded selections,
 * MTP index sharing); "QSA HiSparse" README (page size 64, FP8 E4M3 KV).
 * The score formula itself is not on the pages: this oracle fixes it as above
 * (parity unpinned against the real learned indexer; see the design notes).
 *
 * Arithmetic: every floating-point accumulation is in double precision; BF16
 * and FP8 E4M3FN inputs are decoded bit by bit by this file's own decoders.
 * Scores are rounded once to float.  Nothing is blocked, fused or reordered.
 */
#ifndef QSA_ORACLE_H
#define QSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* dtype codes understood by the oracle */
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8_E4M3 = 2 };

/* tokens per KV page and groups (4 tokens each) per page */
#define ORC_PAGE_TOKENS 64
#define ORC_GROUP_TOKENS 4
#define ORC_PAGE_GROUPS (ORC_PAGE_TOKENS / ORC_GROUP_TOKENS)

double orc_bf16_to_f64(uint16_t bits);
double orc_e4m3_to_f64(uint8_t code);

/* Stage 1.  q_idx [T,H_I,D_I] (q_dt), w_idx [T,H_I] f32,
 * k_idx_pages [num_pages,16,D_I] (k_dt), page_table [*, pt_stride] int32,
 * q_req [T] (NULL: query t belongs to request t), q_pos [T].
 * Writes scores[t*score_stride + g] for g < floor(q_pos[t]/4) and -inf for
 * the rest of the first score_stride entries.  Groups whose page-table entry
 * is out of range score -inf.  Returns the number of such skipped groups, or
 * a negative value on an argument error. */
long orc_index_scores(const void* q_idx, int q_dt, const float* w_idx,
                      const void* k_idx_pages, int k_dt, int num_pages,
                      const int32_t* page_table, int pt_stride,
                      const int32_t* q_req, const int32_t* q_pos,
                      int T, int H_I, int D_I, float* scores, int score_stride);

/* Stage 2.  Exact top-min(K, c) of scores[t, 0..c) with c = floor(q_pos/4),
 * ranked by (score desc, group id asc) after mapping -0 to +0.  sel [T,K]
 * receives the kept ids in ascending order followed by -1 padding; n_sel [T]
 * the count.  Returns 0, or a negative value on an argument error or a NaN
 * candidate score. */
long orc_topk_groups(const float* scores, int score_stride, const int32_t* q_pos,
                     int T, int K, int32_t* sel, int32_t* n_sel);

/* Stage 3.  tok [T,W]: the tokens 4g..4g+3 of each kept group in sel order,
 * then (MTP reuse, capture_pos != NULL) the groups c(p0)..c(p)-1 completed
 * since the capture position p0, then the current block 4c(p)..p; -1 padding.
 * A sel entry outside [0, c(p0)) expands to four -1 slots and is counted.
 * Returns the count of such entries, or a negative value on an argument error
 * (including a row that would not fit in W). */
long orc_expand_select(const int32_t* sel, const int32_t* n_sel, int K,
                       const int32_t* q_pos, const int32_t* capture_pos, int T,
                       int32_t* tok, int32_t* n_tok, int W);

/* Stage 4.  q [T,Hq,D] (q_dt), k_pages/v_pages [num_pages,64,Hkv,D] (kv_dt;
 * FP8 values are code*scale with k_scale / v_scale), tok [T,W] with n_tok [T]
 * used entries (-1 skipped), q_req [T] (NULL: identity).  sm_scale <= 0 means
 * 1/sqrt(D).  out [T,Hq,D] and lse [T,Hq] (natural log) in double; empty rows
 * give out = 0 and lse = -inf.  Returns the number of skipped invalid token
 * entries, or a negative value on an argument error. */
long orc_sparse_attn(const void* q, int q_dt, const void* k_pages,
                     const void* v_pages, int kv_dt, float k_scale, float v_scale,
                     int num_pages, const int32_t* page_table, int pt_stride,
                     const int32_t* q_req, const int32_t* tok,
                     const int32_t* n_tok, int W, int T, int Hq, int Hkv, int D,
                     float sm_scale, double* out, double* lse);

/* Indexer projection (the step before stage 1): y[t][n] = sum_h x[t][h] *
 * w[n][h] for x [T,H] and w [N,H] (F32 or BF16), accumulated in double and
 * rounded once to float.  Rows of w stack the indexer query heads (H_I*D_I),
 * the head weights (H_I) and the token key (D_I).  Returns 0, or a negative
 * value on an argument error. */
long orc_indexer_project(const void* x, int x_dt, const void* w, int w_dt, int T, int H, int N,
                         float* y);

/* C4 compressed-key write (the step before stage 1).  For completed group i
 * (request g_req[i], NULL: request 0; group id g_id[i]) with token keys
 * k_tok[i][0..3][0..D_I) (f32):
 *   khat[d] = bias[d] + sum_{j<4} sum_{e<D_I} wphi[d][j*D_I + e] * k_tok[i][j][e]
 * (wphi [D_I][4*D_I] f32, bias [D_I] f32 or NULL), accumulated in double,
 * rounded once to float (then to bfloat16, round to nearest even, for BF16
 * storage) and written to row g%16 of page page_table[req][g/16] of
 * k_idx_pages [num_pages,16,D_I] (k_dt F32 or BF16).  A group whose request,
 * logical page or physical page is out of range is skipped and counted.
 * Returns the count, or a negative value on an argument error. */
long orc_compress_keys(const float* k_tok, int n_groups, const int32_t* g_req, const int32_t* g_id,
                       const float* wphi, const float* bias, int D_I, void* k_idx_pages, int k_dt,
                       int num_pages, const int32_t* page_table, int pt_rows, int pt_stride);

/* Threads the OpenMP loops over query tokens use for a row count of T. */
int orc_threads_for(int T);
/* Caps the threads of those loops (the host's core count by default); used to
 * time the oracle on one core.  Changes no result. */
void orc_set_max_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
