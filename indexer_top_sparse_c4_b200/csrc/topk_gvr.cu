// topk_gvr.cu -- stage 2 of QSA as a guess-verify-refine (GVR) Top-K with
// hint-free self-sampling (TensorRT-LLM "QSASparseAttentionConfig",
// enable_heuristic_topk: the GVR Top-K for group budgets of 512, 1,024 and
// 2,048, with the exact radix Top-K as the fallback).
//
// This kernel serves calls with many rows (one CTA each).  Few long rows
// (decode) run on a thread-block cluster per row instead: the cluster Top-K of
// topk_groups.cu in its self-sampling mode, whose guess is a window of key
// bins read off a strided sample, verified by exact cluster-wide counts.
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
//    order and an exact radix select over at most CAP of them finds the K-th
//    key; the kept ones are written ascending.  Every pass over ids gives
//    each warp a contiguous range read 32 consecutive scores at a time
//    (coalesced); ballots order a warp's hits, and one prefix sum over the
//    32 warps' counts orders the warps;
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
    // keys of a warp that fall in the same bin are counted with one atomic
    // (the top digits of a row's scores are mostly equal: per-key atomics on
    // one bin would serialise)
    for (int base = 0; base < m; base += kGvThreads) {
      const int i = base + threadIdx.x;
      int bin = -1;
      if (i < m) {
        const uint32_t k = get(i);
        if ((k & mask) == prefix) bin = (int)((k >> shift) & 0xFF);
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && (int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
    }
    __syncthreads();
    find_bin_from_top(sh.hist, need, &sh.s_bin, &sh.s_need);
    __syncthreads();
    prefix |= (uint32_t)sh.s_bin << shift;
    mask |= 0xFFu << shift;
    need = sh.s_need;
    __syncthreads();
  }
  *above = r - need;   // keys strictly greater than the r-th largest
  return prefix;
}

// A warp's contiguous share [lo, hi) of n ids (multiples of 32 wide).
__device__ __forceinline__ void gv_warp_range(int n, int& lo, int& hi) {
  const int warp = threadIdx.x >> 5;
  const int per = ((n + kGvThreads / 32 - 1) / (kGvThreads / 32) + 31) / 32 * 32;
  lo = warp * per < n ? warp * per : n;
  hi = lo + per < n ? lo + per : n;
}

constexpr int kGvUnroll = 8;   // 32-wide steps a warp loads before it tests them

// Ids i in [0, n) whose key get(i) satisfies pred(key), in id order:
// emit(position, i, key).  Returns the total.  Every thread of the block
// calls it.  Each warp loads kGvUnroll steps of 32 consecutive keys before it
// tests them, so a warp has that many loads in flight.
template <typename Get, typename Pred, typename Emit>
__device__ int gv_ordered(int n, Get get, Pred pred, Emit emit, GvShared& sh) {
  const int lane = threadIdx.x & 31;
  int lo, hi;
  gv_warp_range(n, lo, hi);
  int cnt = 0;
  for (int k = lo; k < hi; k += 32 * kGvUnroll) {
    uint32_t v[kGvUnroll];
#pragma unroll
    for (int u = 0; u < kGvUnroll; ++u) {
      const int i = k + 32 * u + lane;
      v[u] = i < hi ? get(i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kGvUnroll; ++u) {
      const int i = k + 32 * u + lane;
      cnt += __popc(__ballot_sync(0xffffffffu, i < hi && pred(v[u])));
    }
  }
  int total;
  // one value per warp enters the block scan (lane 0 carries it)
  int base = gv_scan(lane == 0 ? cnt : 0, sh, &total);
  base = __shfl_sync(0xffffffffu, base, 0);
  const unsigned below = (1u << lane) - 1u;
  for (int k = lo; k < hi; k += 32 * kGvUnroll) {
    uint32_t v[kGvUnroll];
#pragma unroll
    for (int u = 0; u < kGvUnroll; ++u) {
      const int i = k + 32 * u + lane;
      v[u] = i < hi ? get(i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kGvUnroll; ++u) {
      const int i = k + 32 * u + lane;
      const bool f = i < hi && pred(v[u]);
      const unsigned m = __ballot_sync(0xffffffffu, f);
      if (f) emit(base + __popc(m & below), i, v[u]);
      base += __popc(m);
    }
  }
  return total;
}

// How many ids i in [0, n) have pred(get(i)) (coalesced warp ranges).
template <typename Get, typename Pred>
__device__ int gv_count(int n, Get get, Pred pred, GvShared& sh) {
  const int lane = threadIdx.x & 31;
  int lo, hi;
  gv_warp_range(n, lo, hi);
  int cnt = 0;
  for (int k = lo; k < hi; k += 32 * kGvUnroll) {
    uint32_t v[kGvUnroll];
#pragma unroll
    for (int u = 0; u < kGvUnroll; ++u) {
      const int i = k + 32 * u + lane;
      v[u] = i < hi ? get(i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kGvUnroll; ++u) {
      const int i = k + 32 * u + lane;
      cnt += __popc(__ballot_sync(0xffffffffu, i < hi && pred(v[u])));
    }
  }
  return gv_sum(lane == 0 ? cnt : 0, sh);
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

  int count = -1, tries = 0, dummy;
  uint32_t tau = 0u;
  while (tries < kGvTries) {
    tau = gv_select([&](int i) { return sh.sample[i]; }, S, r, sh, &dummy);
    // ---- verify: how many of the row's keys reach the guess
    count = gv_count(c, key_at, [&](uint32_t k) { return k >= tau; }, sh);
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

  int tk_above;
  uint32_t tk;
  bool from_buffer = count >= K && count <= kGvCap;
  if (from_buffer) {
    // ---- refine: gather the candidates in id order, then an exact select among them
    const int total = gv_ordered(c, key_at, [&](uint32_t k) { return k >= tau; },
                                 [&](int pos, int i, uint32_t k) {
                                   sh.ckey[pos] = k;
                                   sh.cid[pos] = i;
                                 },
                                 sh);
    __syncthreads();
    count = total;
    tk = gv_select([&](int i) { return sh.ckey[i]; }, total, K, sh, &tk_above);
  } else {
    // ---- fallback: the exact radix select over the whole row
    tk = gv_select(key_at, c, K, sh, &tk_above);
  }
  // keys equal to tk: the `need` lowest ids among them are kept
  const int need = K - tk_above;
  const int n = from_buffer ? count : c;
  auto key_of = [&](int i) { return from_buffer ? sh.ckey[i] : key_at(i); };
  auto id_of = [&](int i) { return from_buffer ? sh.cid[i] : i; };
  // the rank of each equal key among the equal keys, in id order: the first
  // `need` of them are kept; a first ordered pass records the cut-off id
  if (tid == 0) sh.s_count = 0x7fffffff;
  __syncthreads();
  gv_ordered(n, key_of, [&](uint32_t k) { return k == tk; },
             [&](int pos, int i, uint32_t) {
               if (pos == need - 1) sh.s_count = i;   // the last equal key kept
             },
             sh);
  __syncthreads();
  const int last_eq = sh.s_count;
  // kept: above tk, or equal to it and not past the last equal key kept
  // (equal keys past it are read as 0, below every real key)
  gv_ordered(n, [&](int i) {
               const uint32_t k = key_of(i);
               // keys equal to tk past the cut-off are sent below tk
               return (k == tk && i > last_eq) ? 0u : k;
             },
             [&](uint32_t k) { return k >= tk && k != 0u; },
             [&](int pos, int i, uint32_t) { out[pos] = id_of(i); }, sh);
  if (tid == 0) {
    n_sel[t] = K;
    if (path) path[t] = from_buffer ? (tries == 1 ? 1 : 2) : 3;
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
