/* c_abi_decode.c -- one QSA decode step through the C ABI of libqsa.so alone
 * (include/qsa.h): no Python, no torch.  Stage 1 (indexer scores with the
 * prefix histogram), stages 2 + 3 (qsa_topk_expand) and stage 4
 * (qsa_sparse_attn_decode with its queried workspace), then the device
 * status word, on the legacy default stream.
 *
 *   c_abi_decode IN_DIR OUT_DIR
 *
 * IN_DIR holds dims.txt ("T H_I D_I num_pages pt_rows pt_stride Hq Hkv D K W
 * score_stride q_dt kv_dt out_dt k_scale v_scale", dtypes as qsa_dtype_t
 * codes) and the raw arrays q_idx (F32), w_idx (F32), k_idx (F32),
 * page_table, q_req, q_pos (int32), q (q_dt), k_pages, v_pages (kv_dt).
 * OUT_DIR receives scores, sel, n_sel, tok, n_tok, out, lse as raw arrays.
 * Any status other than QSA_OK prints the library's message and exits 1. */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "qsa.h"

#define CHECK(call)                                                                    \
  do {                                                                                 \
    qsa_status_t st_ = (call);                                                         \
    if (st_ != QSA_OK) {                                                               \
      fprintf(stderr, "%s -> %s: %s\n", #call, qsa_status_name(st_), qsa_last_error_string()); \
      exit(1);                                                                         \
    }                                                                                  \
  } while (0)
#define CUDA(call)                                                                     \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess) {                                                           \
      fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));                      \
      exit(1);                                                                         \
    }                                                                                  \
  } while (0)

static const char* g_in;
static const char* g_out;

static size_t elem_size(int dt) { return dt == QSA_F32 ? 4 : (dt == QSA_BF16 ? 2 : 1); }

/* the whole file IN_DIR/name uploaded to a new device buffer of `bytes` */
static void* upload(const char* name, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", g_in, name);
  FILE* f = fopen(path, "rb");
  if (!f) {
    fprintf(stderr, "cannot open %s\n", path);
    exit(1);
  }
  void* h = malloc(bytes ? bytes : 1);
  if (fread(h, 1, bytes, f) != bytes) {
    fprintf(stderr, "%s: expected %zu bytes\n", path, bytes);
    exit(1);
  }
  fclose(f);
  void* d = NULL;
  CUDA(cudaMalloc(&d, bytes ? bytes : 16));
  CUDA(cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice));
  free(h);
  return d;
}

static void* zeros(size_t bytes) {
  void* d = NULL;
  CUDA(cudaMalloc(&d, bytes ? bytes : 16));
  CUDA(cudaMemset(d, 0, bytes ? bytes : 16));
  return d;
}

static void save(const char* name, const void* d, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s", g_out, name);
  void* h = malloc(bytes ? bytes : 1);
  CUDA(cudaMemcpy(h, d, bytes, cudaMemcpyDeviceToHost));
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(h, 1, bytes, f) != bytes) {
    fprintf(stderr, "cannot write %s\n", path);
    exit(1);
  }
  fclose(f);
  free(h);
}

int main(int argc, char** argv) {
  if (argc != 3) {
    fprintf(stderr, "usage: %s IN_DIR OUT_DIR\n", argv[0]);
    return 2;
  }
  g_in = argv[1];
  g_out = argv[2];
  char path[4096];
  snprintf(path, sizeof path, "%s/dims.txt", g_in);
  FILE* f = fopen(path, "r");
  int T, H_I, D_I, num_pages, pt_rows, pt_stride, Hq, Hkv, D, K, W, stride, q_dt, kv_dt, out_dt;
  float k_scale, v_scale;
  if (!f || fscanf(f, "%d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %f %f", &T, &H_I, &D_I, &num_pages, &pt_rows,
                   &pt_stride, &Hq, &Hkv, &D, &K, &W, &stride, &q_dt, &kv_dt, &out_dt, &k_scale, &v_scale) != 17) {
    fprintf(stderr, "bad %s\n", path);
    return 1;
  }
  fclose(f);
  const size_t kv_bytes = (size_t)num_pages * 64 * Hkv * D * elem_size(kv_dt);
  const float* q_idx = (const float*)upload("q_idx", (size_t)T * H_I * D_I * 4);
  const float* w_idx = (const float*)upload("w_idx", (size_t)T * H_I * 4);
  const float* k_idx = (const float*)upload("k_idx", (size_t)num_pages * 16 * D_I * 4);
  const int32_t* pt = (const int32_t*)upload("page_table", (size_t)pt_rows * pt_stride * 4);
  const int32_t* q_req = (const int32_t*)upload("q_req", (size_t)T * 4);
  const int32_t* q_pos = (const int32_t*)upload("q_pos", (size_t)T * 4);
  const void* q = upload("q", (size_t)T * Hq * D * elem_size(q_dt));
  const void* kp = upload("k_pages", kv_bytes);
  const void* vp = upload("v_pages", kv_bytes);

  float* scores = (float*)zeros((size_t)T * stride * 4);
  uint32_t* hist = (uint32_t*)zeros((size_t)T * QSA_PREFIX_HIST_BINS * 4);  /* zero before first use */
  int32_t* sel = (int32_t*)zeros((size_t)T * K * 4);
  int32_t* n_sel = (int32_t*)zeros((size_t)T * 4);
  int32_t* tok = (int32_t*)zeros((size_t)T * W * 4);
  int32_t* n_tok = (int32_t*)zeros((size_t)T * 4);
  void* out = zeros((size_t)T * Hq * D * elem_size(out_dt));
  float* lse = (float*)zeros((size_t)T * Hq * 4);
  uint32_t* status = (uint32_t*)zeros(4);

  CHECK(qsa_index_scores(q_idx, QSA_F32, w_idx, k_idx, QSA_F32, num_pages, pt, pt_rows, pt_stride, q_req, q_pos,
                         T, H_I, D_I, scores, stride, hist, status, NULL));
  CHECK(qsa_topk_expand(scores, stride, hist, q_pos, T, K, sel, n_sel, tok, n_tok, W, status, NULL));
  const size_t ws_bytes = qsa_sparse_attn_decode_workspace_size(T, Hq, Hkv, D, W, (qsa_dtype_t)kv_dt);
  void* ws = zeros(ws_bytes);
  CHECK(qsa_sparse_attn_decode(q, (qsa_dtype_t)q_dt, kp, vp, (qsa_dtype_t)kv_dt, k_scale, v_scale, num_pages, pt,
                               pt_rows, pt_stride, q_req, tok, n_tok, W, T, Hq, Hkv, D, 0.f, out,
                               (qsa_dtype_t)out_dt, lse, ws, ws_bytes, status, NULL));
  uint32_t bits = 0;
  CHECK(qsa_get_device_status(status, &bits, 0, NULL));

  save("scores", scores, (size_t)T * stride * 4);
  save("sel", sel, (size_t)T * K * 4);
  save("n_sel", n_sel, (size_t)T * 4);
  save("tok", tok, (size_t)T * W * 4);
  save("n_tok", n_tok, (size_t)T * 4);
  save("out", out, (size_t)T * Hq * D * elem_size(out_dt));
  save("lse", lse, (size_t)T * Hq * 4);
  printf("ok abi=%d workspace=%zu\n", qsa_abi_version(), ws_bytes);
  return 0;
}
