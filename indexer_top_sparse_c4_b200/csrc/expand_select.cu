// expand_select.cu -- stage 3 of QSA: kept groups -> token ids.
// "Qwen3.8-27B QSA - BF16 source weights", "QSA in brief": the budget is
// spent on four-token blocks and the current block is always added;
// TensorRT-LLM "QSASparseAttentionConfig": expanded selections address single
// tokens (get_indices_block_size), and in the MTP draft loop the selection
// captured at draft-extend is reused with the groups completed since then
// appended.  Because the kept ids are ascending and every appended group and
// the current block lie above them, a row is: 4 tokens per kept group, then
// the contiguous run 4*c(p0) .. p, then -1 padding.  One thread per slot.
#include "qsa_internal.cuh"

namespace qsa {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) expand_kernel(ExpandArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.y;
  const int p = a.q_pos[t];
  int p0 = a.capture_pos ? a.capture_pos[t] : p;
  if (p0 > p) p0 = p;
  const int c0 = p0 >= 0 ? p0 / kGroupTokens : 0;
  int ns = a.n_sel[t];
  ns = ns < 0 ? 0 : (ns > a.K ? a.K : ns);
  const int head = kGroupTokens * ns;                       // slots of kept groups
  const int tail = p >= 0 ? p - kGroupTokens * c0 + 1 : 0;  // 4*c0 .. p
  const int total = head + tail;
  const int32_t* srow = a.sel + (size_t)t * a.K;
  int32_t* row = a.tok + (size_t)t * a.W;
  for (int i = blockIdx.x * kThreads + threadIdx.x; i < a.W; i += gridDim.x * kThreads) {
    int v = -1;
    if (i < head) {
      const int g = __ldg(srow + i / kGroupTokens);
      if (g >= 0 && g < c0) v = kGroupTokens * g + i % kGroupTokens;
      else if (i % kGroupTokens == 0) flag(a.status, QSA_DEV_BAD_GROUP);
    } else if (i < total) {
      v = kGroupTokens * c0 + (i - head);
    }
    row[i] = v;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.n_tok[t] = total < a.W ? total : a.W;
    if (total > a.W) flag(a.status, QSA_DEV_ROW_RANGE);
  }
}

// Dense rows of the sequence-length threshold ("QSASparseAttentionConfig",
// seq_len_threshold): a query whose sequence (p + 1 tokens) is at most the
// threshold attends to every token 0 .. p; other rows are left as they are.
__global__ void __launch_bounds__(kThreads) dense_select_kernel(const int32_t* q_pos, int threshold, int32_t* tok,
                                                                int32_t* n_tok, int W, uint32_t* status) {
  pdl_wait();
  const int t = blockIdx.y;
  const int p = q_pos[t];
  const int L = p + 1;
  if (p < 0 || L > threshold) return;   // (whole CTA: the row is not dense)
  int32_t* row = tok + (size_t)t * W;
  for (int i = blockIdx.x * kThreads + threadIdx.x; i < W; i += gridDim.x * kThreads) row[i] = i < L ? i : -1;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    n_tok[t] = L < W ? L : W;
    if (L > W) flag(status, QSA_DEV_ROW_RANGE);
  }
}

}  // namespace

cudaError_t launch_dense_select(const int32_t* q_pos, int T, int threshold, int32_t* tok, int32_t* n_tok, int W,
                                uint32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  int bx = (W + kThreads - 1) / kThreads;
  if (bx > 64) bx = 64;
  return launch_k(dense_select_kernel, dim3(bx, T), dim3(kThreads), 0, s, 1, q_pos, threshold, tok, n_tok, W,
                  status);
}

cudaError_t launch_expand_select(const ExpandArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  int bx = (a.W + kThreads - 1) / kThreads;
  if (bx > 64) bx = 64;
  return launch_k(expand_kernel, dim3(bx, a.T), dim3(kThreads), 0, s, 1, a);
}

}  // namespace qsa
