// qsa_abi.cu -- the extern "C" entry points of libqsa.so (include/qsa.h):
// host-side argument validation, then one launch per stage on the caller's
// stream.  No allocation, no host synchronisation.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include "qsa_internal.cuh"

namespace {

thread_local char g_err[512] = "";

qsa_status_t fail(qsa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

qsa_status_t cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return QSA_OK;
  return fail(QSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

#define REQUIRE(cond, ...) \
  do {                     \
    if (!(cond)) return fail(QSA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)
#define SUPPORT(cond, ...) \
  do {                     \
    if (!(cond)) return fail(QSA_ERR_UNSUPPORTED, __VA_ARGS__); \
  } while (0)

constexpr int kMaxGridY = 65535;
constexpr int kPageGroupsAbi = 16;   // groups per 64-token page

qsa_status_t check_attn(const void* q, qsa_dtype_t q_dt, const void* k_pages, const void* v_pages,
                        qsa_dtype_t kv_dt, int num_pages, const int32_t* page_table, int pt_rows,
                        int pt_stride,
                        const int32_t* tok, const int32_t* n_tok, int W, int T, int Hq, int Hkv,
                        int D, void* out, qsa_dtype_t out_dt, float k_scale, float v_scale) {
  REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  REQUIRE(Hq >= 1 && Hkv >= 1 && Hq % Hkv == 0, "need Hq %% Hkv == 0 (Hq=%d, Hkv=%d)", Hq, Hkv);
  SUPPORT(Hq / Hkv <= 16, "at most 16 query heads per KV head (got %d)", Hq / Hkv);
  SUPPORT(D == 64 || D == 128 || D == 256, "head dim D must be 64, 128 or 256 (got %d)", D);
  REQUIRE(W >= 1, "W must be >= 1 (got %d)", W);
  REQUIRE(num_pages >= 1 && pt_rows >= 1 && pt_stride >= 1,
          "num_pages, pt_rows and pt_stride must be >= 1");
  SUPPORT(num_pages <= (1 << 25), "num_pages = %d exceeds the %d pages (2^31 token rows) a cache may hold",
          num_pages, 1 << 25);
  REQUIRE(q_dt == QSA_F32 || q_dt == QSA_BF16, "q dtype must be F32 or BF16");
  REQUIRE(kv_dt == QSA_F32 || kv_dt == QSA_BF16 || kv_dt == QSA_FP8_E4M3, "bad KV dtype");
  REQUIRE(out_dt == QSA_F32 || out_dt == QSA_BF16, "out dtype must be F32 or BF16");
  if (kv_dt == QSA_FP8_E4M3)
    REQUIRE(isfinite(k_scale) && isfinite(v_scale) && k_scale > 0.f && v_scale > 0.f,
            "FP8 scales must be finite and > 0");
  if (T == 0) return QSA_OK;
  REQUIRE(q && k_pages && v_pages && page_table && tok && n_tok && out, "null pointer argument");
  REQUIRE(aligned16(q) && aligned16(k_pages) && aligned16(v_pages) && aligned16(out),
          "q, k_pages, v_pages and out must be 16-byte aligned");
  return QSA_OK;
}

}  // namespace

void qsa::set_last_error(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }

qsa_status_t qsa::check_attn_args(const void* q, qsa_dtype_t q_dt, const void* k_pages,
                                  const void* v_pages, qsa_dtype_t kv_dt, int num_pages,
                                  const int32_t* page_table, int pt_rows, int pt_stride,
                                  const int32_t* tok, const int32_t* n_tok, int W, int T, int Hq,
                                  int Hkv, int D, void* out, qsa_dtype_t out_dt, float k_scale,
                                  float v_scale) {
  return check_attn(q, q_dt, k_pages, v_pages, kv_dt, num_pages, page_table, pt_rows, pt_stride, tok,
                    n_tok, W, T, Hq, Hkv, D, out, out_dt, k_scale, v_scale);
}

extern "C" {

const char* qsa_last_error_string(void) { return g_err; }

const char* qsa_status_name(qsa_status_t s) {
  switch (s) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_WORKSPACE: return "QSA_ERR_WORKSPACE";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
    case QSA_ERR_DEVICE_INDEX: return "QSA_ERR_DEVICE_INDEX";
    case QSA_ERR_TIMEOUT: return "QSA_ERR_TIMEOUT";
  }
  return "QSA_ERR_UNKNOWN";
}

int qsa_abi_version(void) { return 11; }

size_t qsa_index_scores_workspace_size(int T, int H_I, int D_I, int score_stride) {
  (void)T; (void)H_I; (void)D_I; (void)score_stride;
  return 0;
}

size_t qsa_expand_select_workspace_size(int T, int K, int W) {
  (void)T; (void)K; (void)W;
  return 0;
}

size_t qsa_sparse_attn_prefill_workspace_size(int T, int Hq, int Hkv, int D, int W, qsa_dtype_t kv_dt) {
  (void)T; (void)Hq; (void)Hkv; (void)D; (void)W; (void)kv_dt;
  return 0;
}

qsa_status_t qsa_get_device_status(uint32_t* dev_status, uint32_t* bits_out, int clear,
                                   qsa_stream_t stream) {
  REQUIRE(dev_status != nullptr, "dev_status is NULL");
  REQUIRE(((uintptr_t)dev_status & 3u) == 0, "dev_status must be 4-byte aligned");
  const cudaStream_t s = (cudaStream_t)stream;
  uint32_t bits = 0;
  // the copy is ordered after the work already queued on the stream
  qsa_status_t st = cuda_status(cudaMemcpyAsync(&bits, dev_status, sizeof bits, cudaMemcpyDeviceToHost, s),
                                "qsa_get_device_status: read");
  if (st == QSA_OK && clear)
    st = cuda_status(cudaMemsetAsync(dev_status, 0, sizeof bits, s), "qsa_get_device_status: clear");
  if (st == QSA_OK) st = cuda_status(cudaStreamSynchronize(s), "qsa_get_device_status: stream");
  if (st != QSA_OK) return st;
  if (bits_out) *bits_out = bits;
  if (bits & QSA_DEV_TIMEOUT)
    return fail(QSA_ERR_TIMEOUT, "a bounded wait inside a kernel ran out (device status 0x%x)", bits);
  if (bits)
    return fail(QSA_ERR_DEVICE_INDEX,
                "a kernel skipped out-of-range data on the device (device status 0x%x: %s%s%s%s%s)",
                bits, (bits & QSA_DEV_BAD_PAGE) ? "page " : "", (bits & QSA_DEV_BAD_TOKEN) ? "token " : "",
                (bits & QSA_DEV_BAD_GROUP) ? "group " : "", (bits & QSA_DEV_ROW_RANGE) ? "row-range " : "",
                (bits & QSA_DEV_BAD_REQUEST) ? "request" : "");
  return QSA_OK;
}

qsa_status_t qsa_selftest_bounded_wait(uint32_t limit_us, uint32_t* dev_status, uint32_t* report,
                                       qsa_stream_t stream) {
  REQUIRE(dev_status && report, "null pointer argument");
  REQUIRE(limit_us >= 1 && limit_us <= 1000000, "limit_us must be in 1 .. 1,000,000 (got %u)", limit_us);
  return cuda_status(qsa::launch_selftest_wait(limit_us, dev_status, report, (cudaStream_t)stream),
                     "qsa_selftest_bounded_wait launch");
}

size_t qsa_indexer_project_workspace_size(int T, int H, int N) {
  (void)T; (void)H; (void)N;
  return 0;
}

qsa_status_t qsa_indexer_project(const void* x, qsa_dtype_t x_dt, const void* w, qsa_dtype_t w_dt, int T, int H,
                                 int N, float* y, uint32_t* dev_status, qsa_stream_t stream) {
  REQUIRE(T >= 0 && H >= 1 && N >= 1, "need T >= 0, H >= 1, N >= 1 (got %d, %d, %d)", T, H, N);
  REQUIRE(x_dt == QSA_F32 || x_dt == QSA_BF16, "x dtype must be F32 or BF16");
  REQUIRE(w_dt == QSA_F32 || w_dt == QSA_BF16, "w dtype must be F32 or BF16");
  SUPPORT(H % 8 == 0, "the hidden size H = %d must be a multiple of 8", H);
  if (T == 0) return QSA_OK;
  REQUIRE(x && w && y, "null pointer argument");
  REQUIRE(aligned16(x) && aligned16(w), "x and w must be 16-byte aligned");
  qsa::ProjectArgs a{x, w, T, H, N, y, dev_status};
  return cuda_status(qsa::launch_indexer_project(a, x_dt, w_dt, (cudaStream_t)stream), "qsa_indexer_project launch");
}

size_t qsa_compress_keys_workspace_size(int n_groups, int D_I) {
  (void)n_groups; (void)D_I;
  return 0;
}

qsa_status_t qsa_compress_keys(const float* k_tok, int tok_stride, int n_groups, const int32_t* g_req,
                               const int32_t* g_id, const float* wphi, const float* bias, int D_I,
                               void* k_idx_pages, qsa_dtype_t k_dt, int num_pages, const int32_t* page_table,
                               int pt_rows, int pt_stride, uint32_t* dev_status, qsa_stream_t stream) {
  REQUIRE(n_groups >= 0, "n_groups must be >= 0 (got %d)", n_groups);
  SUPPORT(D_I == 32 || D_I == 64 || D_I == 128, "D_I must be 32, 64 or 128 (got %d)", D_I);
  REQUIRE(tok_stride >= D_I, "tok_stride %d is smaller than D_I %d", tok_stride, D_I);
  REQUIRE(k_dt == QSA_F32 || k_dt == QSA_BF16, "k_idx_pages dtype must be F32 or BF16");
  REQUIRE(num_pages >= 1 && pt_rows >= 1 && pt_stride >= 1, "num_pages, pt_rows and pt_stride must be >= 1");
  SUPPORT(n_groups <= (1 << 30), "n_groups = %d is too large", n_groups);
  if (n_groups == 0) return QSA_OK;
  REQUIRE(k_tok && g_id && wphi && k_idx_pages && page_table, "null pointer argument");
  qsa::CompressArgs c{k_tok, tok_stride, n_groups, g_req, g_id, wphi, bias, D_I, k_idx_pages, num_pages,
                      page_table, pt_rows, pt_stride, dev_status};
  return cuda_status(qsa::launch_compress_keys(c, k_dt, (cudaStream_t)stream), "qsa_compress_keys launch");
}

qsa_status_t qsa_index_scores(const void* q_idx, qsa_dtype_t q_dt, const float* w_idx,
                              const void* k_idx_pages, qsa_dtype_t k_dt, int num_pages,
                              const int32_t* page_table, int pt_rows, int pt_stride,
                              const int32_t* q_req,
                              const int32_t* q_pos, int T, int H_I, int D_I, float* scores,
                              int score_stride, uint32_t* prefix_hist, uint32_t* dev_status,
                              qsa_stream_t stream) {
  REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  SUPPORT((H_I == 2 || H_I == 4) && (D_I == 32 || D_I == 64 || D_I == 128),
          "indexer shape H_I=%d, D_I=%d not built (H_I in {2,4}, D_I in {32,64,128})", H_I, D_I);
  REQUIRE(q_dt == QSA_F32 || q_dt == QSA_BF16, "q_idx dtype must be F32 or BF16");
  REQUIRE(k_dt == QSA_F32 || k_dt == QSA_BF16, "k_idx_pages dtype must be F32 or BF16");
  REQUIRE(score_stride >= 1 && pt_stride >= 1 && pt_rows >= 1 && num_pages >= 1,
          "score_stride, pt_rows, pt_stride and num_pages must be >= 1");
  if (T == 0) return QSA_OK;
  REQUIRE(q_idx && w_idx && k_idx_pages && page_table && q_pos && scores, "null pointer argument");
  REQUIRE(aligned16(q_idx) && aligned16(k_idx_pages), "q_idx and k_idx_pages must be 16-byte aligned");
  REQUIRE(aligned16(prefix_hist), "prefix_hist must be 16-byte aligned");
  qsa::IndexArgs a{q_idx, q_dt, w_idx, k_idx_pages, k_dt, num_pages, page_table, pt_rows, pt_stride,
                   q_req, q_pos, T, H_I, D_I, scores, score_stride, dev_status};
  a.hist = prefix_hist;
  // many queries with BF16 operands (a prefill chunk): the tensor-core GEMM;
  // otherwise the streaming scan
  const cudaError_t e = (T >= 256 && qsa::index_tc_supported(a))
                            ? qsa::launch_index_scores_tc(a, (cudaStream_t)stream)
                            : qsa::launch_index_scores(a, (cudaStream_t)stream);
  return cuda_status(e, "qsa_index_scores launch");
}

qsa_status_t qsa_dcp_shard_positions(const int32_t* q_pos, int T, int g_lo, int g_hi, int32_t* q_pos_local,
                                     qsa_stream_t stream) {
  REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  REQUIRE(g_lo >= 0 && g_hi >= g_lo, "need 0 <= g_lo <= g_hi (got %d, %d)", g_lo, g_hi);
  REQUIRE(g_lo % kPageGroupsAbi == 0, "shard boundaries must fall on pages: g_lo %% 16 == 0 (got %d)", g_lo);
  if (T == 0) return QSA_OK;
  REQUIRE(q_pos && q_pos_local, "null pointer argument");
  return cuda_status(qsa::launch_dcp_positions(q_pos, T, g_lo, g_hi, q_pos_local, (cudaStream_t)stream),
                     "qsa_dcp_shard_positions launch");
}

qsa_status_t qsa_dcp_candidates(const float* scores, int score_stride, const int32_t* sel, const int32_t* n_sel,
                                int T, int K, int g_lo, float* cand_score, int32_t* cand_id, uint32_t* dev_status,
                                qsa_stream_t stream) {
  REQUIRE(T >= 0 && K >= 1 && score_stride >= 1 && g_lo >= 0, "need T >= 0, K >= 1, score_stride >= 1, g_lo >= 0");
  if (T == 0) return QSA_OK;
  REQUIRE(scores && sel && n_sel && cand_score && cand_id, "null pointer argument");
  return cuda_status(qsa::launch_dcp_candidates(scores, score_stride, sel, n_sel, T, K, g_lo, cand_score, cand_id,
                                                dev_status, (cudaStream_t)stream),
                     "qsa_dcp_candidates launch");
}

qsa_status_t qsa_dcp_merge_topk(const float* cand_score, const int32_t* cand_id, int R, int T, int K, int32_t* sel,
                                int32_t* n_sel, qsa_stream_t stream) {
  REQUIRE(T >= 0 && K >= 1 && R >= 1, "need T >= 0, K >= 1, R >= 1 (got %d, %d, %d)", T, K, R);
  SUPPORT((long long)R * K <= qsa::dcp_merge_max_candidates(), "R * K = %lld exceeds the %d candidates a row may merge",
          (long long)R * K, qsa::dcp_merge_max_candidates());
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  if (T == 0) return QSA_OK;
  REQUIRE(cand_score && cand_id && sel && n_sel, "null pointer argument");
  return cuda_status(qsa::launch_dcp_merge_topk(cand_score, cand_id, R, T, K, sel, n_sel, (cudaStream_t)stream),
                     "qsa_dcp_merge_topk launch");
}

qsa_status_t qsa_dcp_expand(const int32_t* sel, const int32_t* n_sel, int K, const int32_t* q_pos, int T, int g_lo,
                            int g_hi, int32_t* tok, int32_t* n_tok, int W, uint32_t* dev_status,
                            qsa_stream_t stream) {
  REQUIRE(T >= 0 && K >= 1 && W >= 1, "need T >= 0, K >= 1, W >= 1");
  REQUIRE(g_lo >= 0 && g_hi >= g_lo, "need 0 <= g_lo <= g_hi (got %d, %d)", g_lo, g_hi);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  if (T == 0) return QSA_OK;
  REQUIRE(sel && n_sel && q_pos && tok && n_tok, "null pointer argument");
  return cuda_status(qsa::launch_dcp_expand(sel, n_sel, K, q_pos, T, g_lo, g_hi, tok, n_tok, W, dev_status,
                                            (cudaStream_t)stream),
                     "qsa_dcp_expand launch");
}

qsa_status_t qsa_dcp_merge_attn(const float* o_parts, const float* lse_parts, int R, int T, int Hq, int D, void* out,
                                qsa_dtype_t out_dt, float* lse, qsa_stream_t stream) {
  REQUIRE(T >= 0 && R >= 1 && Hq >= 1 && D >= 1, "need T >= 0, R, Hq, D >= 1");
  REQUIRE(out_dt == QSA_F32 || out_dt == QSA_BF16, "out dtype must be F32 or BF16");
  SUPPORT((long long)T * Hq <= 0x7fffffffLL, "T * Hq too large");
  if (T == 0) return QSA_OK;
  REQUIRE(o_parts && lse_parts && out, "null pointer argument");
  return cuda_status(qsa::launch_dcp_merge_attn(o_parts, lse_parts, R, T, Hq, D, out, out_dt, lse,
                                                (cudaStream_t)stream),
                     "qsa_dcp_merge_attn launch");
}

size_t qsa_topk_groups_workspace_size(int T, int K, int score_stride) {
  (void)T; (void)K; (void)score_stride;
  return 0;
}

qsa_status_t qsa_topk_groups(const float* scores, int score_stride, uint32_t* prefix_hist,
                             const int32_t* q_pos, int T, int K, int32_t* sel, int32_t* n_sel,
                             void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                             qsa_stream_t stream) {
  (void)workspace; (void)workspace_bytes;
  REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  REQUIRE(K >= 1, "K must be >= 1 (got %d)", K);
  REQUIRE(score_stride >= 1, "score_stride must be >= 1");
  SUPPORT(qsa::topk_cluster_size(score_stride) > 0, "score_stride %d exceeds the %d groups a row may hold",
          score_stride, 8 * 512 * 64);
  if (T == 0) return QSA_OK;
  REQUIRE(scores && q_pos && sel && n_sel, "null pointer argument");
  REQUIRE(aligned16(prefix_hist), "prefix_hist must be 16-byte aligned");
  qsa::TopkArgs a{scores, score_stride, q_pos, T, K, sel, n_sel, dev_status};
  a.hist = prefix_hist;
  return cuda_status(qsa::launch_topk_groups(a, (cudaStream_t)stream), "qsa_topk_groups launch");
}

qsa_status_t qsa_topk_groups_gvr(const float* scores, int score_stride, const int32_t* q_pos, int T, int K,
                                 int32_t* sel, int32_t* n_sel, int32_t* path, uint32_t* dev_status,
                                 qsa_stream_t stream) {
  REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  REQUIRE(K >= 1, "K must be >= 1 (got %d)", K);
  REQUIRE(score_stride >= 1, "score_stride must be >= 1");
  if (!qsa::topk_gvr_budget(K)) {
    // the pages' prerequisite for the self-sampling engine: the exact radix
    // Top-K runs instead, with a warning the first time
    static bool warned = false;
    if (!warned) {
      warned = true;
      fprintf(stderr, "qsa_topk_groups_gvr: budget K = %d is not 512, 1024 or 2048; using the exact radix Top-K\n",
              K);
    }
    return qsa_topk_groups(scores, score_stride, nullptr, q_pos, T, K, sel, n_sel, nullptr, 0, dev_status, stream);
  }
  SUPPORT(qsa::topk_cluster_size(score_stride) > 0, "score_stride %d exceeds the %d groups a row may hold",
          score_stride, 8 * 512 * 64);
  if (T == 0) return QSA_OK;
  REQUIRE(scores && q_pos && sel && n_sel, "null pointer argument");
  // the Top-K kernels of stage 2 with the self-sampled guess in front of
  // their radix passes: one CTA per row (many rows, or short ones), one
  // cluster per row (few long rows)
  qsa::TopkArgs a{scores, score_stride, q_pos, T, K, sel, n_sel, dev_status};
  a.gvr = 1;
  a.path = path;
  return cuda_status(qsa::launch_topk_groups(a, (cudaStream_t)stream), "qsa_topk_groups_gvr launch");
}

qsa_status_t qsa_expand_select(const int32_t* sel, const int32_t* n_sel, int K, const int32_t* q_pos,
                               const int32_t* capture_pos, int T, int32_t* tok, int32_t* n_tok,
                               int W, uint32_t* dev_status, qsa_stream_t stream) {
  REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  REQUIRE(K >= 1, "K must be >= 1 (got %d)", K);
  REQUIRE(W >= 4 * K + 4, "W must be >= 4*K + 4 = %d (got %d)", 4 * K + 4, W);
  if (T == 0) return QSA_OK;
  REQUIRE(sel && n_sel && q_pos && tok && n_tok, "null pointer argument");
  qsa::ExpandArgs a{sel, n_sel, K, q_pos, capture_pos, T, tok, n_tok, W, dev_status};
  return cuda_status(qsa::launch_expand_select(a, (cudaStream_t)stream), "qsa_expand_select launch");
}

int qsa_seq_len_threshold(int requested, int K) {
  const long long budget = 4ll * (K > 0 ? K : 0);   // the budget in tokens
  const long long want = requested > 0 ? requested : budget;
  const long long thr = want > budget ? want : budget;
  return thr > 0x7fffffffLL ? 0x7fffffff : (int)thr;
}

qsa_status_t qsa_dense_select(const int32_t* q_pos, int T, int threshold, int32_t* tok, int32_t* n_tok, int W,
                              uint32_t* dev_status, qsa_stream_t stream) {
  REQUIRE(T >= 0 && W >= 1, "need T >= 0 and W >= 1 (got %d, %d)", T, W);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  if (T == 0 || threshold <= 0) return QSA_OK;
  REQUIRE(q_pos && tok && n_tok, "null pointer argument");
  return cuda_status(qsa::launch_dense_select(q_pos, T, threshold, tok, n_tok, W, dev_status, (cudaStream_t)stream),
                     "qsa_dense_select launch");
}

qsa_status_t qsa_topk_expand(const float* scores, int score_stride, uint32_t* prefix_hist,
                             const int32_t* q_pos, int T, int K, int32_t* sel, int32_t* n_sel,
                             int32_t* tok, int32_t* n_tok, int W, uint32_t* dev_status,
                             qsa_stream_t stream) {
  REQUIRE(T >= 0, "T must be >= 0 (got %d)", T);
  SUPPORT(T <= kMaxGridY, "T = %d exceeds %d query tokens per call", T, kMaxGridY);
  REQUIRE(K >= 1, "K must be >= 1 (got %d)", K);
  REQUIRE(W >= 4 * K + 4, "W must be >= 4*K + 4 = %d (got %d)", 4 * K + 4, W);
  REQUIRE(score_stride >= 1, "score_stride must be >= 1");
  SUPPORT(qsa::topk_cluster_size(score_stride) > 0, "score_stride %d exceeds the %d groups a row may hold",
          score_stride, 8 * 512 * 64);
  if (T == 0) return QSA_OK;
  REQUIRE(scores && q_pos && sel && n_sel && tok && n_tok, "null pointer argument");
  REQUIRE(aligned16(prefix_hist), "prefix_hist must be 16-byte aligned");
  qsa::TopkArgs a{scores, score_stride, q_pos, T, K, sel, n_sel, dev_status, tok, n_tok, W};
  a.hist = prefix_hist;
  return cuda_status(qsa::launch_topk_groups(a, (cudaStream_t)stream), "qsa_topk_expand launch");
}

size_t qsa_sparse_attn_decode_workspace_size(int T, int Hq, int Hkv, int D, int W,
                                             qsa_dtype_t kv_dt) {
  if (T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || W <= 0) return 0;
  return qsa::attn_decode_ws_bytes(T, Hq, D, qsa::attn_decode_plan(T, Hq, Hkv, D, W, kv_dt).s);
}

qsa_status_t qsa_sparse_attn_decode(const void* q, qsa_dtype_t q_dt, const void* k_pages,
                                    const void* v_pages, qsa_dtype_t kv_dt, float k_scale,
                                    float v_scale, int num_pages, const int32_t* page_table,
                                    int pt_rows, int pt_stride, const int32_t* q_req,
                                    const int32_t* tok,
                                    const int32_t* n_tok, int W, int T, int Hq, int Hkv, int D,
                                    float sm_scale, void* out, qsa_dtype_t out_dt, float* lse,
                                    void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                                    qsa_stream_t stream) {
  qsa_status_t st = check_attn(q, q_dt, k_pages, v_pages, kv_dt, num_pages, page_table, pt_rows,
                               pt_stride,
                               tok, n_tok, W, T, Hq, Hkv, D, out, out_dt, k_scale, v_scale);
  if (st != QSA_OK || T == 0) return st;
  const qsa::DecodePlan plan = qsa::attn_decode_plan(T, Hq, Hkv, D, W, kv_dt);
  const size_t need = qsa::attn_decode_ws_bytes(T, Hq, D, plan.s);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return fail(QSA_ERR_WORKSPACE, "decode needs %zu bytes of 16-byte-aligned workspace (got %zu)",
                need, workspace ? workspace_bytes : (size_t)0);
  qsa::AttnArgs a{q, q_dt, k_pages, v_pages, kv_dt, k_scale, v_scale, num_pages, page_table,
                  pt_rows, pt_stride, q_req, tok, n_tok, W, T, Hq, Hkv, D, sm_scale, out, out_dt, lse,
                  dev_status};
  return cuda_status(qsa::launch_sparse_attn(a, plan, workspace, (cudaStream_t)stream, true),
                     "qsa_sparse_attn_decode launch");
}

namespace {
size_t align16z(size_t n) { return (n + 15) & ~(size_t)15; }
// The fused call's workspace: the decode plan's partials, plus -- for plans
// other than the gather kernel's -- the token lists the expansion writes first.
size_t decode_sel_ws(const qsa::DecodePlan& plan, int T, int Hq, int D, int W) {
  const size_t attn = qsa::attn_decode_ws_bytes(T, Hq, D, plan.s);
  if (plan.gather) return attn;
  return align16z(attn) + align16z((size_t)T * W * sizeof(int32_t)) + align16z((size_t)T * sizeof(int32_t));
}
}  // namespace

size_t qsa_sparse_attn_decode_sel_workspace_size(int T, int Hq, int Hkv, int D, int W, qsa_dtype_t kv_dt) {
  if (T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || W <= 0) return 0;
  return decode_sel_ws(qsa::attn_decode_plan(T, Hq, Hkv, D, W, kv_dt), T, Hq, D, W);
}

qsa_status_t qsa_sparse_attn_decode_sel(const void* q, qsa_dtype_t q_dt, const void* k_pages, const void* v_pages,
                                        qsa_dtype_t kv_dt, float k_scale, float v_scale, int num_pages,
                                        const int32_t* page_table, int pt_rows, int pt_stride,
                                        const int32_t* q_req, const int32_t* sel, const int32_t* n_sel, int K,
                                        const int32_t* q_pos, const int32_t* capture_pos, int W, int T, int Hq,
                                        int Hkv, int D, float sm_scale, void* out, qsa_dtype_t out_dt, float* lse,
                                        void* workspace, size_t workspace_bytes, uint32_t* dev_status,
                                        qsa_stream_t stream) {
  REQUIRE(K >= 1, "K must be >= 1 (got %d)", K);
  REQUIRE(W >= 4 * K + 4, "W must be >= 4*K + 4 = %d (got %d)", 4 * K + 4, W);
  // the selection stands in for the token lists in the shared checks
  qsa_status_t st = check_attn(q, q_dt, k_pages, v_pages, kv_dt, num_pages, page_table, pt_rows, pt_stride, sel,
                               n_sel, W, T, Hq, Hkv, D, out, out_dt, k_scale, v_scale);
  if (st != QSA_OK || T == 0) return st;
  REQUIRE(q_pos != nullptr, "null pointer argument");
  const qsa::DecodePlan plan = qsa::attn_decode_plan(T, Hq, Hkv, D, W, kv_dt);
  const size_t need = decode_sel_ws(plan, T, Hq, D, W);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return fail(QSA_ERR_WORKSPACE, "decode needs %zu bytes of 16-byte-aligned workspace (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  qsa::AttnArgs a{q, q_dt, k_pages, v_pages, kv_dt, k_scale, v_scale, num_pages, page_table,
                  pt_rows, pt_stride, q_req, nullptr, nullptr, W, T, Hq, Hkv, D, sm_scale, out, out_dt, lse,
                  dev_status};
  const cudaStream_t s = (cudaStream_t)stream;
  if (plan.gather) {  // the gather kernel lists each chunk's tokens itself
    a.sel = sel;
    a.n_sel = n_sel;
    a.K = K;
    a.q_pos = q_pos;
    a.capture_pos = capture_pos;
    return cuda_status(qsa::launch_sparse_attn(a, plan, workspace, s, true), "qsa_sparse_attn_decode_sel launch");
  }
  // other plans: stage 3 into the workspace, then the decode attention
  unsigned char* base = static_cast<unsigned char*>(workspace);
  int32_t* tok = reinterpret_cast<int32_t*>(base + align16z(qsa::attn_decode_ws_bytes(T, Hq, D, plan.s)));
  int32_t* n_tok = reinterpret_cast<int32_t*>(reinterpret_cast<unsigned char*>(tok) +
                                              align16z((size_t)T * W * sizeof(int32_t)));
  qsa::ExpandArgs e{sel, n_sel, K, q_pos, capture_pos, T, tok, n_tok, W, dev_status};
  st = cuda_status(qsa::launch_expand_select(e, s), "qsa_sparse_attn_decode_sel launch");
  if (st != QSA_OK) return st;
  a.tok = tok;
  a.n_tok = n_tok;
  return cuda_status(qsa::launch_sparse_attn(a, plan, workspace, s, true), "qsa_sparse_attn_decode_sel launch");
}

qsa_status_t qsa_sparse_attn_prefill(const void* q, qsa_dtype_t q_dt, const void* k_pages,
                                     const void* v_pages, qsa_dtype_t kv_dt, float k_scale,
                                     float v_scale, int num_pages, const int32_t* page_table,
                                     int pt_rows, int pt_stride, const int32_t* q_req,
                                     const int32_t* tok,
                                     const int32_t* n_tok, int W, int T, int Hq, int Hkv, int D,
                                     float sm_scale, void* out, qsa_dtype_t out_dt, float* lse,
                                     uint32_t* dev_status, qsa_stream_t stream) {
  qsa_status_t st = check_attn(q, q_dt, k_pages, v_pages, kv_dt, num_pages, page_table, pt_rows,
                               pt_stride,
                               tok, n_tok, W, T, Hq, Hkv, D, out, out_dt, k_scale, v_scale);
  if (st != QSA_OK || T == 0) return st;
  qsa::AttnArgs a{q, q_dt, k_pages, v_pages, kv_dt, k_scale, v_scale, num_pages, page_table,
                  pt_rows, pt_stride, q_req, tok, n_tok, W, T, Hq, Hkv, D, sm_scale, out, out_dt, lse,
                  dev_status};
  return cuda_status(qsa::launch_sparse_attn(a, qsa::DecodePlan{}, nullptr, (cudaStream_t)stream,
                                             false),
                     "qsa_sparse_attn_prefill launch");
}

}  // extern "C"
