// dcp.cu -- sequence-sharded (decode context parallel) QSA decode: the steps
// that let R shards, each holding a contiguous range of every request's
// pages (its slice of the page table, KV cache and compressed indexer keys),
// run the hot path on their own slice and still select and attend exactly as
// one device would (the Ascend article's context section: decode context
// parallelism for the QSA path).
//
// Shard r owns the groups [g_lo, g_hi) of every request.  Per decode step:
//   1. qsa_dcp_shard_positions: the shard-local query position 4 * c_r,
//      c_r = clamp(c(p) - g_lo, 0, g_hi - g_lo) candidates of the shard, so
//      that qsa_index_scores and qsa_topk_groups run unchanged on the slice;
//   2. qsa_dcp_candidates: the shard's top-K as (score, global group id)
//      records, ascending by id, padded with (-inf, -1);
//   3. an all-gather of the records of every shard ([R, T, K]);
//   4. qsa_dcp_merge_topk: the global top-K of the union, which is the exact
//      top-K of all candidates (each of the global K best is among the K best
//      of its own shard); ties go to the lower group id;
//   5. qsa_dcp_expand: the shard's part of the global selection, as
//      shard-local token ids, plus the current block on the shard that owns it;
//   6. qsa_sparse_attn_decode on the shard: a partial output and its LSE;
//   7. an all-gather of the partials; qsa_dcp_merge_attn: out = sum_r
//      exp(lse_r - LSE) out_r with LSE = log sum_r exp(lse_r).
#include <limits.h>
#include <math.h>

#include "qsa_internal.cuh"

namespace qsa {
namespace {

__global__ void dcp_positions_kernel(const int32_t* q_pos, int T, int g_lo, int g_hi, int32_t* q_pos_local) {
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int p = q_pos[t];
  const int c = p >= 0 ? p / kGroupTokens : 0;
  int cl = c - g_lo;
  cl = cl < 0 ? 0 : (cl > g_hi - g_lo ? g_hi - g_lo : cl);
  q_pos_local[t] = kGroupTokens * cl;
}

__global__ void dcp_candidates_kernel(const float* scores, int score_stride, const int32_t* sel, const int32_t* n_sel,
                                      int T, int K, int g_lo, float* cand_score, int32_t* cand_id, uint32_t* status) {
  pdl_wait();
  const int t = blockIdx.x;
  int ns = n_sel[t];
  ns = ns < 0 ? 0 : (ns > K ? K : ns);
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    const int s = i < ns ? sel[(size_t)t * K + i] : -1;
    const bool ok = s >= 0 && s < score_stride;
    if (i < ns && !ok) flag(status, QSA_DEV_BAD_GROUP);
    cand_id[(size_t)t * K + i] = ok ? s + g_lo : -1;
    cand_score[(size_t)t * K + i] = ok ? scores[(size_t)t * score_stride + s] : -INFINITY;
  }
}

// ---- the merge of the shards' candidates ---------------------------------------
//
// One CTA per row.  Candidate i of the row (shard i / K, slot i % K) gets the
// 64-bit key (order key of its score) << 32 | ~id: unique, and larger for a
// better candidate (score descending, then id ascending); padding gets 0,
// below every real candidate.  A radix select over the keys, 8 bits at a
// time from the top, finds the n-th largest key; the candidates at or above
// it are the selection.  Records arrive ascending by id within a shard and
// the shards own ascending id ranges, so the records in (shard, slot) order
// are ascending by id: a block prefix sum over the selected flags writes
// them out in ascending order without a sort.

constexpr int kMgThreads = 1024;
constexpr int kMgMaxCand = 16384;   // shards x K per row

__device__ __forceinline__ uint64_t cand_key(float s, int32_t id) {
  if (id < 0) return 0ull;
  return ((uint64_t)order_key(s) << 32) | (uint64_t)(~(uint32_t)id);
}

// exclusive block prefix sum of one value per thread (kMgThreads threads)
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kMgThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    warp_sums[lane] = w;   // inclusive sums of the warps
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  if (total) *total = warp_sums[kMgThreads / 32 - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kMgThreads) dcp_merge_topk_kernel(const float* cand_score, const int32_t* cand_id,
                                                                   int R, int T, int K, int32_t* sel, int32_t* n_sel) {
  extern __shared__ __align__(16) uint64_t keys[];   // [R * K]
  __shared__ int hist[256];
  __shared__ int warp_sums[32];
  __shared__ int s_bin, s_need, s_valid;
  pdl_wait();
  const int t = blockIdx.x;
  const int n = R * K;
  const int tid = threadIdx.x;
  int valid = 0;
  for (int i = tid; i < n; i += kMgThreads) {
    const int r = i / K, k = i % K;
    const size_t src = ((size_t)r * T + t) * K + k;
    const uint64_t key = cand_key(cand_score[src], cand_id[src]);
    keys[i] = key;
    valid += key != 0ull;
  }
  if (tid == 0) s_valid = 0;
  __syncthreads();
  atomicAdd(&s_valid, valid);
  __syncthreads();
  const int nv = s_valid;
  const int want = nv < K ? nv : K;

  // radix select of the want-th largest key
  uint64_t prefix = 0ull, mask = 0ull;
  int need = want;
  if (want > 0) {
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int b = tid; b < 256; b += kMgThreads) hist[b] = 0;
      __syncthreads();
      for (int base = 0; base < n; base += kMgThreads) {   // one atomic per bin and warp
        const int i = base + tid;
        int bin = -1;
        if (i < n) {
          const uint64_t k = keys[i];
          if ((k & mask) == prefix) bin = (int)((k >> shift) & 0xFF);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && (tid & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
      }
      __syncthreads();
      find_bin_from_top(hist, need, &s_bin, &s_need);   // the bin of the need-th largest matching key
      __syncthreads();
      prefix |= (uint64_t)s_bin << shift;
      mask |= 0xFFull << shift;
      need = s_need;
      __syncthreads();
    }
  }
  const uint64_t tau = prefix;   // the want-th largest key (keys are unique)

  // write the selection, ascending by id, then the padding
  int total = 0;
  for (int base = 0; base < n; base += kMgThreads) {
    const int i = base + tid;
    const bool take = want > 0 && i < n && keys[i] >= tau && keys[i] != 0ull;
    int cnt;
    const int pos = block_exclusive_scan(take ? 1 : 0, warp_sums, &cnt);
    if (take) sel[(size_t)t * K + total + pos] = (int32_t)~(uint32_t)(keys[i] & 0xFFFFFFFFull);
    total += cnt;
  }
  for (int i = total + tid; i < K; i += kMgThreads) sel[(size_t)t * K + i] = -1;
  if (tid == 0) n_sel[t] = total;
}

// ---- the shard's part of the selection as shard-local token ids -----------------

__global__ void dcp_expand_kernel(const int32_t* sel, const int32_t* n_sel, int K, const int32_t* q_pos, int T,
                                  int g_lo, int g_hi, int32_t* tok, int32_t* n_tok, int W, uint32_t* status) {
  __shared__ int s_a, s_b;
  pdl_wait();
  const int t = blockIdx.x;
  int ns = n_sel[t];
  ns = ns < 0 ? 0 : (ns > K ? K : ns);
  const int32_t* srow = sel + (size_t)t * K;
  if (threadIdx.x == 0) {
    s_a = ns;
    s_b = ns;
  }
  __syncthreads();
  // the selection ascends: the shard's entries are the run [a, b)
  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const int g = srow[i];
    const int gp = i > 0 ? srow[i - 1] : INT_MIN;
    if (g >= g_lo && gp < g_lo) atomicMin(&s_a, i);
    if (g >= g_hi && gp < g_hi) atomicMin(&s_b, i);
  }
  __syncthreads();
  const int a = s_a, b = s_b > s_a ? s_b : s_a;
  const int p = q_pos[t];
  const int c = p >= 0 ? p / kGroupTokens : 0;
  const bool own_block = p >= 0 && c >= g_lo && c < g_hi;   // the current block is on this shard
  const int nblock = own_block ? p - kGroupTokens * c + 1 : 0;
  const int used = kGroupTokens * (b - a) + nblock;
  if (used > W && threadIdx.x == 0) flag(status, QSA_DEV_ROW_RANGE);
  int32_t* trow = tok + (size_t)t * W;
  for (int s = threadIdx.x; s < W; s += blockDim.x) {
    int v = -1;
    if (s < kGroupTokens * (b - a)) v = kGroupTokens * (srow[a + s / kGroupTokens] - g_lo) + s % kGroupTokens;
    else if (s < used) v = kGroupTokens * (c - g_lo) + (s - kGroupTokens * (b - a));
    trow[s] = v;
  }
  if (threadIdx.x == 0) n_tok[t] = used < W ? used : W;
}

// ---- the LSE merge of the shards' partial outputs --------------------------------

template <typename OT>
__global__ void dcp_merge_attn_kernel(const float* o_parts, const float* lse_parts, int R, int TH, int D, void* out,
                                      float* lse) {
  pdl_wait();
  const size_t th = blockIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) M = fmaxf(M, lse_parts[(size_t)r * TH + th]);
  float L = 0.f;
  for (int r = 0; r < R; ++r) {
    const float lr = lse_parts[(size_t)r * TH + th];
    L += lr == -INFINITY ? 0.f : expf(lr - M);
  }
  const float LSE = L > 0.f ? M + logf(L) : -INFINITY;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    if (L > 0.f) {
      for (int r = 0; r < R; ++r) {
        const float lr = lse_parts[(size_t)r * TH + th];
        if (lr == -INFINITY) continue;
        acc = fmaf(expf(lr - LSE), o_parts[((size_t)r * TH + th) * D + d], acc);
      }
    }
    if constexpr (sizeof(OT) == 4) reinterpret_cast<float*>(out)[th * D + d] = acc;
    else reinterpret_cast<__nv_bfloat16*>(out)[th * D + d] = __float2bfloat16_rn(acc);
  }
  if (threadIdx.x == 0 && lse) lse[th] = LSE;
}

}  // namespace

cudaError_t launch_dcp_positions(const int32_t* q_pos, int T, int g_lo, int g_hi, int32_t* q_pos_local,
                                 cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  return launch_k(dcp_positions_kernel, dim3((T + 127) / 128), dim3(128), 0, s, 1, q_pos, T, g_lo, g_hi,
                  q_pos_local);
}

cudaError_t launch_dcp_candidates(const float* scores, int score_stride, const int32_t* sel, const int32_t* n_sel,
                                  int T, int K, int g_lo, float* cand_score, int32_t* cand_id, uint32_t* status,
                                  cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  return launch_k(dcp_candidates_kernel, dim3(T), dim3(256), 0, s, 1, scores, score_stride, sel, n_sel, T, K, g_lo,
                  cand_score, cand_id, status);
}

int dcp_merge_max_candidates() { return kMgMaxCand; }

cudaError_t launch_dcp_merge_topk(const float* cand_score, const int32_t* cand_id, int R, int T, int K, int32_t* sel,
                                  int32_t* n_sel, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const size_t smem = (size_t)R * K * sizeof(uint64_t);
  cudaError_t e = cudaFuncSetAttribute(dcp_merge_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_k(dcp_merge_topk_kernel, dim3(T), dim3(kMgThreads), smem, s, 1, cand_score, cand_id, R, T, K, sel,
                  n_sel);
}

cudaError_t launch_dcp_expand(const int32_t* sel, const int32_t* n_sel, int K, const int32_t* q_pos, int T, int g_lo,
                              int g_hi, int32_t* tok, int32_t* n_tok, int W, uint32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  return launch_k(dcp_expand_kernel, dim3(T), dim3(256), 0, s, 1, sel, n_sel, K, q_pos, T, g_lo, g_hi, tok, n_tok,
                  W, status);
}

cudaError_t launch_dcp_merge_attn(const float* o_parts, const float* lse_parts, int R, int T, int Hq, int D,
                                  void* out, qsa_dtype_t out_dt, float* lse, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int TH = T * Hq;
  if (out_dt == QSA_BF16)
    return launch_k(dcp_merge_attn_kernel<__nv_bfloat16>, dim3(TH), dim3(D < 256 ? D : 256), 0, s, 1, o_parts,
                    lse_parts, R, TH, D, out, lse);
  return launch_k(dcp_merge_attn_kernel<float>, dim3(TH), dim3(D < 256 ? D : 256), 0, s, 1, o_parts, lse_parts, R,
                  TH, D, out, lse);
}

}  // namespace qsa
