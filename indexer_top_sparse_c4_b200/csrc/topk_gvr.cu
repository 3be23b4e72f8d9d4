// topk_gvr.cu -- stage 2 of QSA as a guess-verify-refine (GVR) Top-K with
// hint-free self-sampling (TensorRT-LLM "QSASparseAttentionConfig",
// enable_heuristic_topk: the GVR Top-K for group budgets of 512, 1,024 and
// 2,048, with the exact radix Top-K as the fallback).
//
// One CTA of 1024 threads per row; the result is the exact top-K, ties to
// the lower group id, ascending:
//  * guess: S = 4,096 scores sampled at even strides over the row's c
//    candidates give, by a radix select over the sample, a threshold tau
//    about (1.25 K + 32) / c of the way down the row -- no histogram or
//    other hint from stage 1 is needed;
//  * verify: one pass over the row counts the scores >= tau.  When the count
//    lies in [K, CAP] every one of the K best is among them; otherwise the
//    guess moves (a deeper sample rank when too few, a shallower one when too
//    many) and the count is taken again, up to three times;
//  * refine: the >= tau candidates are gathered into shared memory in id
//    order (a block prefix sum over per-thread counts of contiguous id
//    ranges) and an exact radix select over at most CAP of them finds the
//    K-th key; the kept ones are written ascending by a second prefix sum;
//  * a row whose guesses all fail (e.g. thousands of equal scores) runs the
//    same radix select over the whole row instead.
// path[t] (optional) records what happened: 0 dense (c <= K), 1 the first
// guess verified, 2 a later guess verified, 3 the whole-row radix select.
#include "qsa_internal.cuh"

namespace qsa {
namespace {

constexpr int kGvThreads = 1024;
constexpr int kGvSample = 4096;
constexpr int kGvCap = 12288;      // candidates the refine step holds (96 KiB of key, id pairs)
constexpr int kGvTries = 3;

struct GvShared {
  uint32_t sample[kGvSample];
  uint32_t ckey[kGvCap];
  int32_t cid[kGvCap];
  int hist[256];
  int warp_sums[32];
  int s_bin, s_need, s_count;
};

// exclusive prefix sum over the block of one value per thread; *total gets the sum
__device__ __forceinline__ int gv_scan(int v, GvShared& sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) sh.warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = sh.warp_sums[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    sh.warp_sums[lane] = w;
  }
  __syncthreads();
  const int before = (warp > 0 ? sh.warp_sums[warp - 1] : 0) + x - v;
  *total = sh.warp_sums[31];
  __syncthreads();
  return before;
}

__device__ __forceinline__ int gv_sum(int v, GvShared& sh) {
  int total;
  gv_scan(v, sh, &total);
  return total;
}

// The r-th largest (1-based) of m keys get(i), i < m, by four 8-bit radix
// passes from the top; also returns how many keys are strictly above it.
template <typename Get>
__device__ uint32_t gv_select(Get get, int m, int r, GvShared& sh, int* above) {
  uint32_t prefix = 0u, mask = 0u;
  int need = r;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += kGvThreads) sh.hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < m; i += kGvThreads) {
      const uint32_t k = get(i);
      if ((k & mask) == prefix) atomicAdd(&sh.hist[(k >> shift) & 0xFF], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int acc = 0, b = 255;
      for (; b > 0; --b) {
        if (acc + sh.hist[b] >= need) break;
        acc += sh.hist[b];
      }
      sh.s_bin = b;
      sh.s_need = need - acc;
    }
    __syncthreads();
    prefix |= (uint32_t)sh.s_bin << shift;
    mask |= 0xFFu << shift;
    need = sh.s_need;
    __syncthreads();
  }
  *above = r - need;   // keys strictly greater than the r-th largest
  return prefix;
}

__global__ void __launch_bounds__(kGvThreads, 1)
    topk_gvr_kernel(const float* scores, int score_stride, const int32_t* q_pos, int K, int32_t* sel, int32_t* n_sel,
                    int32_t* path) {
  extern __shared__ __align__(16) unsigned char gv_raw[];
  GvShared& sh = *reinterpret_cast<GvShared*>(gv_raw);
  pdl_wait();
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int p = q_pos[t];
  int c = p >= 0 ? p / kGroupTokens : 0;
  c = c < score_stride ? c : score_stride;
  const float* row = scores + (size_t)t * score_stride;
  int32_t* out = sel + (size_t)t * K;
  auto key_at = [&](int i) { return order_key(row[i]); };

  if (c <= K) {  // dense: every candidate
    for (int i = tid; i < K; i += kGvThreads) out[i] = i < c ? i : -1;
    if (tid == 0) {
      n_sel[t] = c;
      if (path) path[t] = 0;
    }
    return;
  }

  // ---- guess: a threshold from a strided sample of the row itself
  const int S = c < kGvSample ? c : kGvSample;
  for (int s = tid; s < S; s += kGvThreads) sh.sample[s] = key_at((int)((long long)s * c / S));
  __syncthreads();
  int r = (int)(((long long)(K + K / 4 + 32) * S + c - 1) / c);
  r = r < 1 ? 1 : (r > S ? S : r);
  // each thread owns a contiguous range of ids: prefix sums give id order
  const int per = (c + kGvThreads - 1) / kGvThreads;
  const int lo = tid * per < c ? tid * per : c;
  const int hi = lo + per < c ? lo + per : c;

  int count = -1, tries = 0, dummy;
  uint32_t tau = 0u;
  while (tries < kGvTries) {
    tau = gv_select([&](int i) { return sh.sample[i]; }, S, r, sh, &dummy);
    // ---- verify: how many of the row's keys reach the guess
    int mine = 0;
    for (int i = lo; i < hi; ++i) mine += key_at(i) >= tau;
    count = gv_sum(mine, sh);
    ++tries;
    if (count >= K && count <= kGvCap) break;
    if (count < K) {
      if (r == S) { count = -1; break; }     // the whole sample is not enough: give up guessing
      r = r * 2 + 16 < S ? r * 2 + 16 : S;
    } else {
      if (r == 1) { count = -1; break; }
      r = r / 2 > 1 ? r / 2 : 1;
    }
    count = -1;
  }

  if (count >= K && count <= kGvCap) {
    // ---- refine: gather the candidates in id order, then an exact select among them
    int mine = 0;
    for (int i = lo; i < hi; ++i) mine += key_at(i) >= tau;
    int total;
    int pos = gv_scan(mine, sh, &total);
    for (int i = lo; i < hi; ++i) {
      const uint32_t k = key_at(i);
      if (k >= tau) {
        sh.ckey[pos] = k;
        sh.cid[pos] = i;
        ++pos;
      }
    }
    __syncthreads();
    int above;
    const uint32_t tk = gv_select([&](int i) { return sh.ckey[i]; }, total, K, sh, &above);
    const int need = K - above;   // keys equal to tk that are kept: the lowest ids among them
    // kept = key > tk, or key == tk among the first `need` equal keys in id order
    const int per2 = (total + kGvThreads - 1) / kGvThreads;
    const int a0 = tid * per2 < total ? tid * per2 : total;
    const int a1 = a0 + per2 < total ? a0 + per2 : total;
    int eq = 0;
    for (int i = a0; i < a1; ++i) eq += sh.ckey[i] == tk;
    int eq_total;
    int eq_before = gv_scan(eq, sh, &eq_total);
    int kept = 0;
    {
      int e = eq_before;
      for (int i = a0; i < a1; ++i) {
        const uint32_t k = sh.ckey[i];
        if (k > tk || (k == tk && e++ < need)) ++kept;
      }
    }
    int kt;
    int opos = gv_scan(kept, sh, &kt);
    {
      int e = eq_before;
      for (int i = a0; i < a1; ++i) {
        const uint32_t k = sh.ckey[i];
        if (k > tk || (k == tk && e++ < need)) out[opos++] = sh.cid[i];
      }
    }
    if (tid == 0) {
      n_sel[t] = K;
      if (path) path[t] = tries == 1 ? 1 : 2;
    }
  } else {
    // ---- fallback: the exact radix select over the whole row
    int above;
    const uint32_t tk = gv_select(key_at, c, K, sh, &above);
    const int need = K - above;
    int eq = 0;
    for (int i = lo; i < hi; ++i) eq += key_at(i) == tk;
    int eq_total;
    const int eq_before = gv_scan(eq, sh, &eq_total);
    int kept = 0;
    {
      int e = eq_before;
      for (int i = lo; i < hi; ++i) {
        const uint32_t k = key_at(i);
        if (k > tk || (k == tk && e++ < need)) ++kept;
      }
    }
    int kt;
    int opos = gv_scan(kept, sh, &kt);
    {
      int e = eq_before;
      for (int i = lo; i < hi; ++i) {
        const uint32_t k = key_at(i);
        if (k > tk || (k == tk && e++ < need)) out[opos++] = i;
      }
    }
    if (tid == 0) {
      n_sel[t] = K;
      if (path) path[t] = 3;
    }
  }
}

}  // namespace

bool topk_gvr_budget(int K) { return K == 512 || K == 1024 || K == 2048; }

cudaError_t launch_topk_gvr(const float* scores, int score_stride, const int32_t* q_pos, int T, int K, int32_t* sel,
                            int32_t* n_sel, int32_t* path, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const size_t smem = sizeof(GvShared);
  cudaError_t e = cudaFuncSetAttribute(topk_gvr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_k(topk_gvr_kernel, dim3(T), dim3(kGvThreads), smem, s, 1, scores, score_stride, q_pos, K, sel, n_sel,
                  path);
}

}  // namespace qsa
