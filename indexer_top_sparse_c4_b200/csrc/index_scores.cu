// index_scores.cu -- stage 1 of QSA: the indexer score of every complete
// 4-token group against the query token ("Qwen3.8-27B QSA - BF16 source
// weights", section "QSA in brief": a learned compressed indexer scores the
// context in four-token blocks).  Score fixed by this library:
//   s[t,g] = sum_h w[t,h] * ReLU(q_I[t,h,:] . khat[g,:])      (FP32)
//
// Decode-shaped kernel (few query tokens, long context): the pass is bound by
// HBM reads of the compressed keys (512 B per group at D_I = 128 FP32 against
// 2 FLOP per byte).  One warp owns one 64-token page at a time = 16 groups x
// D_I contiguous values (8 KiB at D_I = 128): lane l loads the 16-byte slice
// [4l, 4l+4) of every group row (16 fully coalesced 512-byte warp loads),
// accumulates the 16 x H_I partial dots of its slice, and a 5-step butterfly
// reduce-scatter leaves lane l holding the finished dots of group l/2 for
// H_I/2 heads; one more shuffle adds the head pair.  Shuffles per group:
// ~H_I, against 5*H_I for a plain per-group warp reduction.
//
// Optionally the scan also counts its scores by the top 12 bits of their
// order keys (the prefix histogram of the row): a shared-memory histogram per
// CTA, added into the row's global one when the CTA ends.  The Top-K stage
// then knows which 12-bit bin holds the n-th largest score without a pass of
// its own over the row.
#include "qsa_internal.cuh"

namespace qsa {
namespace {

// One butterfly step of a warp reduce-scatter: lanes with `upper` set keep
// the upper half of the N-pair window, the others the lower half, and each
// adds the half its partner (lane ^ mask) gave away.
template <int N>
__device__ __forceinline__ void rs_step(float* v, bool upper, int mask) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float send = upper ? v[i] : v[i + N];
    const float keep = upper ? v[i + N] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
  }
}

// After this, v[j] for j < V/32 holds the warp-wide sum of value index
// (V/32)*lane + j.
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float* v, int lane) {
  static_assert(V >= 32 && (V & (V - 1)) == 0, "V must be a power of two >= 32");
  rs_step<V / 2>(v, lane & 16, 16);
  rs_step<V / 4>(v, lane & 8, 8);
  rs_step<V / 8>(v, lane & 4, 4);
  rs_step<V / 16>(v, lane & 2, 2);
  rs_step<V / 32>(v, lane & 1, 1);
}

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// L2 policies: the key stream (twice the L2 at B8 x 262,144 tokens) is read
// once and marked evict-first, so it does not push out what the next stages
// read right after it (the score rows, the page tables, the token lists); the
// page-table entries are marked evict-last.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ int ldg_policy(const int32_t* p, uint64_t pol) {
  int v;
  asm volatile("ld.global.nc.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(v) : "l"(p), "l"(pol));
  return v;
}
// VEC consecutive keys (element index i), widened to float, loaded with an L2 policy.
template <typename KT, int VEC>
__device__ __forceinline__ void ld_keys(const KT* base, size_t i, float* out, uint64_t pol) {
  const void* p = base + i;
  constexpr int B = VEC * (int)sizeof(KT);
  uint32_t w[4];
  if constexpr (B == 16) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.b32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "l"(p), "l"(pol));
  } else if constexpr (B == 8) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.b32 {%0,%1}, [%2], %3;"
                 : "=r"(w[0]), "=r"(w[1]) : "l"(p), "l"(pol));
  } else if constexpr (B == 4) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(w[0]) : "l"(p), "l"(pol));
  } else {
    unsigned short h;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.b16 %0, [%1], %2;" : "=h"(h) : "l"(p), "l"(pol));
    w[0] = h;
  }
  if constexpr (sizeof(KT) == 4) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) out[e] = __uint_as_float(w[e]);
  } else {  // BF16 pairs: the high half of an FP32 pattern
#pragma unroll
    for (int e = 0; e < VEC; ++e)
      out[e] = __uint_as_float((e & 1) ? (w[e / 2] & 0xffff0000u) : (w[e / 2] << 16));
  }
}

template <int H_I, int D_I, typename QT, typename KT>
__device__ __forceinline__ void scan_row(const IndexArgs& a, int t, int c, int npages, int wid, int lane,
                                         int warps_per_row, uint32_t* hist_s) {
  constexpr int VEC = D_I / 32;          // dims per lane
  constexpr int V = kPageGroups * H_I;   // partial dots per lane per page
  constexpr int R = V / 32;              // finished dots per lane (= H_I / 2)
  const int r = a.q_req ? a.q_req[t] : t;
  const bool bad_req = r < 0 || r >= a.pt_rows;  // every group of the row is skipped

  // this lane's slice of every indexer head of the query
  float q[H_I][VEC];
  const QT* qp = reinterpret_cast<const QT*>(a.q_idx) + (size_t)t * H_I * D_I + lane * VEC;
#pragma unroll
  for (int h = 0; h < H_I; ++h) VecLoad<QT, VEC>::get(qp, (size_t)h * D_I, q[h]);
  // weights of the heads whose dots this lane finishes: h = (lane & 1) * R + j
  float w[R];
#pragma unroll
  for (int j = 0; j < R; ++j) w[j] = __ldg(a.w_idx + (size_t)t * H_I + (lane & 1) * R + j);

  const KT* kbase = reinterpret_cast<const KT*>(a.k_idx_pages);
  const uint64_t pol_stream = l2_policy_evict_first(), pol_keep = l2_policy_evict_last();
  const int32_t* pt = a.page_table + (size_t)(bad_req ? 0 : r) * a.pt_stride;
  float* srow = a.scores + (size_t)t * a.score_stride;

  for (int lp = wid; lp < npages; lp += warps_per_row) {
    const int g = lp * kPageGroups + (lane >> 1);
    const int page = (!bad_req && lp < a.pt_stride) ? ldg_policy(pt + lp, pol_keep) : -1;
    if (page < 0 || page >= a.num_pages) {  // warp-uniform
      if (lane == 0) flag(a.status, bad_req ? QSA_DEV_BAD_REQUEST : QSA_DEV_BAD_PAGE);
      if ((lane & 1) == 0 && g < c) {
        srow[g] = -INFINITY;
        if (hist_s) atomicAdd(&hist_s[order_key(-INFINITY) >> kPrefixShift], 1u);
      }
      continue;
    }
    const KT* kp = kbase + (size_t)page * kPageGroups * D_I + lane * VEC;
    float k[kPageGroups][VEC];
#pragma unroll
    for (int gi = 0; gi < kPageGroups; ++gi) ld_keys<KT, VEC>(kp, (size_t)gi * D_I, k[gi], pol_stream);
    float acc[V];
#pragma unroll
    for (int gi = 0; gi < kPageGroups; ++gi) {
#pragma unroll
      for (int h = 0; h < H_I; ++h) {
        float d = q[h][0] * k[gi][0];
#pragma unroll
        for (int j = 1; j < VEC; ++j) d = fmaf(q[h][j], k[gi][j], d);
        acc[gi * H_I + h] = d;
      }
    }
    warp_reduce_scatter<V>(acc, lane);
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < R; ++j) s = fmaf(w[j], fmaxf(acc[j], 0.f), s);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    if ((lane & 1) == 0 && g < c) {
      srow[g] = s;
      if (hist_s) atomicAdd(&hist_s[order_key(s) >> kPrefixShift], 1u);
    }
  }
}

template <int H_I, int D_I, typename QT, typename KT>
__global__ void __launch_bounds__(kThreads) index_scores_kernel(IndexArgs a, int warps_per_row) {
  __shared__ __align__(16) uint32_t hist_s[kPrefixBins];
  const int t = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * kWarps + (threadIdx.x >> 5);
  pdl_wait();
  // (no early trigger: the dependents launch when this grid completes; launched
  // earlier, their CTAs took SMs from this grid's later waves)
  const int p = a.q_pos[t];
  int c = p >= 0 ? p / kGroupTokens : 0;
  if (c > a.score_stride) {
    if (wid == 0 && lane == 0) flag(a.status, QSA_DEV_ROW_RANGE);
    c = a.score_stride;
  }
  const int npages = (c + kPageGroups - 1) / kPageGroups;
  if (blockIdx.x * kWarps >= npages) return;  // (CTA-uniform: before any barrier)
  uint32_t* const hist_g = a.hist ? a.hist + (size_t)t * kPrefixBins : nullptr;
  if (hist_g) {
#pragma unroll
    for (int i = 4 * threadIdx.x; i < kPrefixBins; i += 4 * kThreads)
      *reinterpret_cast<uint4*>(&hist_s[i]) = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
  }
  if (wid < npages) scan_row<H_I, D_I, QT, KT>(a, t, c, npages, wid, lane, warps_per_row,
                                               hist_g ? hist_s : nullptr);
  if (hist_g) {  // the CTA's counts into the row's histogram (few bins are non-zero)
    __syncthreads();
#pragma unroll 4
    for (int i = threadIdx.x; i < kPrefixBins; i += kThreads) {
      const uint32_t v = hist_s[i];
      if (v) atomicAdd(hist_g + i, v);
    }
  }
}

// CTAs of this instantiation that fit on the device at once (SMs x resident
// CTAs per SM), looked up once per device.
template <int H_I, int D_I, typename QT, typename KT>
int resident_ctas() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, index_scores_kernel<H_I, D_I, QT, KT>, kThreads, 0) !=
            cudaSuccess || per_sm < 1)
      per_sm = 1;
    cache[dev] = sms * per_sm;
  }
  return cache[dev];
}

// One wave: every CTA the device holds at once, split evenly over the rows,
// with each warp striding over its row's pages.  (Several waves of shorter
// CTAs left SMs underfed whenever a wave drained: 45.2 us against 41.8 us on
// the B8 x 262,144 scan.)
template <int H_I, int D_I, typename QT, typename KT>
cudaError_t launch_typed(const IndexArgs& a, cudaStream_t s) {
  int cmax = a.score_stride;
  if (cmax > a.pt_stride * kPageGroups) cmax = a.pt_stride * kPageGroups;
  const int npages = (cmax + kPageGroups - 1) / kPageGroups;
  int blocks = resident_ctas<H_I, D_I, QT, KT>() / a.T;   // per row
  const int need = (npages + kWarps - 1) / kWarps;          // more would find no page
  if (blocks > need) blocks = need;
  if (blocks < 1) blocks = 1;
  dim3 grid(blocks, a.T);
  return launch_k(index_scores_kernel<H_I, D_I, QT, KT>, grid, dim3(kThreads), 0, s, 1, a, blocks * kWarps);
}

template <int H_I, int D_I>
cudaError_t launch_dims(const IndexArgs& a, cudaStream_t s) {
  if (a.q_dt == QSA_F32 && a.k_dt == QSA_F32) return launch_typed<H_I, D_I, float, float>(a, s);
  if (a.q_dt == QSA_F32 && a.k_dt == QSA_BF16) return launch_typed<H_I, D_I, float, __nv_bfloat16>(a, s);
  if (a.q_dt == QSA_BF16 && a.k_dt == QSA_F32) return launch_typed<H_I, D_I, __nv_bfloat16, float>(a, s);
  return launch_typed<H_I, D_I, __nv_bfloat16, __nv_bfloat16>(a, s);
}

}  // namespace

cudaError_t launch_index_scores(const IndexArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  switch (a.H_I * 1000 + a.D_I) {
    case 2032: return launch_dims<2, 32>(a, s);
    case 2064: return launch_dims<2, 64>(a, s);
    case 2128: return launch_dims<2, 128>(a, s);
    case 4032: return launch_dims<4, 32>(a, s);
    case 4064: return launch_dims<4, 64>(a, s);
    case 4128: return launch_dims<4, 128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qsa
