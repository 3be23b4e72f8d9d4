// topk_groups.cu -- stage 2 of QSA: the exact Top-K over compressed groups
// (TensorRT-LLM "QSASparseAttentionConfig", field enable_heuristic_topk: the
// exact radix Top-K is the default selector over the compressed-group
// budget).  Ranking: score descending, ties to the lower group id.
//
// Design (sm_100a): one thread-block cluster of CL CTAs x 512 threads per
// query row; thread i of CTA r owns KPT consecutive candidates in registers as
// order-preserving uint32 keys, so the row is read from memory once.
//  * Radix select, 8 bits per pass from the most significant end, finds the
//    exact key tau of the n-th largest candidate.  Each pass histograms only
//    the keys that still match the digits found so far: per-warp shared
//    histograms (no block-wide atomic hot spots), one block reduction, and one
//    distributed-shared-memory add into CTA 0's histogram for the cluster.
//  * Output: every key > tau is kept, plus the first `need` keys == tau in
//    index order.  Because each thread owns a contiguous run of ids, one
//    exclusive scan over threads and one over the cluster's CTAs give every
//    thread the position of its first kept id: the ids come out ascending with
//    no sort.
#include <cooperative_groups.h>

#include "qsa_internal.cuh"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;

struct TopkSmem {
  uint32_t hw[kWarps][kBins];  // per-warp histogram of the current digit
  uint32_t ghist[4][kBins];    // cluster histogram per pass (CTA 0's copy is used)
  int cnt_gt[8], cnt_eq[8];    // per-CTA counts of keys > tau and == tau
  int wa[kWarps], wb[kWarps];  // per-warp scan totals
  int bin, above;
};

// float -> uint32 whose unsigned order equals the float order; -0 maps like +0.
// 0 is below every finite or infinite score: it marks "no candidate".
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <int CL>
__device__ __forceinline__ void csync() {
  if constexpr (CL > 1) cg::this_cluster().sync();
  else __syncthreads();
}

// Exclusive prefix of v over the block's threads (in tid order), and the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += u;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int x = warp_tot[w];
    before += w < warp ? x : 0;
    total += x;
  }
  return before + incl - v;
}

template <int CL, int KPT>
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int rank = 0;
  if constexpr (CL > 1) rank = (int)cg::this_cluster().block_rank();
  const int t = blockIdx.y;
  pdl_wait();
  const int p = a.q_pos[t];
  int c = p >= 0 ? p / kGroupTokens : 0;
  if (c > a.score_stride) {
    if (rank == 0 && tid == 0) flag(a.status, QSA_DEV_ROW_RANGE);
    c = a.score_stride;
  }
  const int K = a.K;
  const int n = c < K ? c : K;
  int32_t* out = a.sel + (size_t)t * K;
  if (c <= K) {  // every candidate is kept: dense fallback (uniform over the cluster)
    pdl_launch_dependents();
    for (int i = rank * kThreads + tid; i < K; i += CL * kThreads) out[i] = i < c ? i : -1;
    if (rank == 0 && tid == 0) a.n_sel[t] = n;
    return;
  }

  // ---- this thread's KPT consecutive candidates, as keys
  const int first = (rank * kThreads + tid) * KPT;
  const float* row = a.scores + (size_t)t * a.score_stride;
  uint32_t keys[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) keys[j] = first + j < c ? order_key(__ldg(row + first + j)) : 0u;
  for (int i = tid; i < 4 * kBins; i += kThreads) (&sm.ghist[0][0])[i] = 0u;
  pdl_launch_dependents();
  csync<CL>();  // every CTA's cluster histograms are zero before anyone adds

  uint32_t* ghist0 = &sm.ghist[0][0];
  if constexpr (CL > 1) ghist0 = cg::this_cluster().map_shared_rank(ghist0, 0);

  // ---- radix select: 4 passes of 8 bits locate tau
  uint32_t prefix = 0;
  int need = n;  // how many keys matching `prefix` are still to be taken
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int b = lane; b < kBins; b += 32) sm.hw[warp][b] = 0u;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const uint32_t k = keys[j];
      const bool match = pass == 0 ? k != 0u : (k >> (shift + 8)) == (prefix >> (shift + 8));
      if (match) atomicAdd(&sm.hw[warp][(k >> shift) & (kBins - 1)], 1u);
    }
    __syncthreads();
    if (tid < kBins) {
      uint32_t v = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += sm.hw[w][tid];
      if constexpr (CL > 1) {
        if (v) atomicAdd(ghist0 + pass * kBins + tid, v);
      } else {
        sm.ghist[pass][tid] = v;
      }
    }
    csync<CL>();
    // the bin holding the need-th largest: thread i looks at bin 255 - i, so
    // an exclusive scan over threads counts the keys in all higher bins
    if (tid < kBins) {
      const int h = (int)ghist0[pass * kBins + (kBins - 1 - tid)];
      int incl = h;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += u;
      }
      if (lane == 31) sm.wa[warp] = incl;
      asm volatile("bar.sync 1, %0;" ::"r"(kBins));  // the 8 warps that scan
      int above = incl - h;
      for (int w = 0; w < warp; ++w) above += sm.wa[w];
      if (above < need && above + h >= need) {
        sm.bin = kBins - 1 - tid;
        sm.above = above;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)sm.bin << shift;
    need -= sm.above;
    __syncthreads();
  }
  const uint32_t tau = prefix;

  // ---- kept ids: all keys > tau, then the first `need` keys == tau by id
  int gt = 0, eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    gt += keys[j] > tau;
    eq += keys[j] == tau;
  }
  int gt_cta, eq_cta;
  const int gt_before = block_exclusive_scan(gt, sm.wa, gt_cta);
  const int eq_before = block_exclusive_scan(eq, sm.wb, eq_cta);
  if (tid == 0) {
    if constexpr (CL > 1) {
      cg::cluster_group cl = cg::this_cluster();
      for (int q = 0; q < CL; ++q) {
        cl.map_shared_rank(sm.cnt_gt, q)[rank] = gt_cta;
        cl.map_shared_rank(sm.cnt_eq, q)[rank] = eq_cta;
      }
    } else {
      sm.cnt_gt[0] = gt_cta;
      sm.cnt_eq[0] = eq_cta;
    }
  }
  csync<CL>();  // last cluster-wide step: from here every access is local
  int off = 0, eq_prev = 0;
  for (int q = 0; q < rank; ++q) {
    const int rem = need - eq_prev;
    off += sm.cnt_gt[q] + (rem <= 0 ? 0 : (rem < sm.cnt_eq[q] ? rem : sm.cnt_eq[q]));
    eq_prev += sm.cnt_eq[q];
  }
  int rem = need - eq_prev;                     // tau-keys still to take at this CTA's start
  rem = rem < 0 ? 0 : rem;
  int pos = off + gt_before + (rem < eq_before ? rem : eq_before);
  int take = rem - eq_before;                   // tau-keys this thread may take
  take = take < 0 ? 0 : take;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const uint32_t k = keys[j];
    bool keep = k > tau;
    if (k == tau && take > 0) {
      keep = true;
      --take;
    }
    if (keep) {
      if (pos < K) out[pos] = first + j;
      ++pos;
    }
  }
  if (rank == 0) {
    for (int i = n + tid; i < K; i += kThreads) out[i] = -1;
    if (tid == 0) a.n_sel[t] = n;
  }
}

template <int CL, int KPT>
cudaError_t launch_cfg(const TopkArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(TopkSmem);
  auto kern = topk_kernel<CL, KPT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_k(kern, dim3(CL, a.T), dim3(kThreads), smem, s, CL, a);
}

template <int KPT>
cudaError_t launch_kpt(const TopkArgs& a, int cl, cudaStream_t s) {
  switch (cl) {
    case 1: return launch_cfg<1, KPT>(a, s);
    case 2: return launch_cfg<2, KPT>(a, s);
    case 4: return launch_cfg<4, KPT>(a, s);
    default: return launch_cfg<8, KPT>(a, s);
  }
}

struct TopkPlan { int cl, kpt; };

// Few rows (decode): spread a row over up to 8 CTAs at 16 keys per thread.
// Many rows (prefill): one CTA per row while 64 keys per thread suffice.
TopkPlan plan_for(int T, int score_stride) {
  const int per_cta16 = kThreads * 16;
  if (T >= 148) {
    for (int kpt = 8; kpt <= 64; kpt <<= 1)
      if (kThreads * kpt >= score_stride) return {1, kpt};
  }
  for (int cl = 1; cl <= 8; cl <<= 1)
    if (cl * per_cta16 >= score_stride) return {cl, 16};
  for (int kpt = 32; kpt <= 64; kpt <<= 1)
    if (8 * kThreads * kpt >= score_stride) return {8, kpt};
  return {0, 0};
}

}  // namespace

int topk_cluster_size(int score_stride) { return plan_for(1, score_stride).cl; }

cudaError_t launch_topk_groups(const TopkArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const TopkPlan p = plan_for(a.T, a.score_stride);
  switch (p.kpt) {
    case 8: return launch_kpt<8>(a, p.cl, s);
    case 16: return launch_kpt<16>(a, p.cl, s);
    case 32: return launch_kpt<32>(a, p.cl, s);
    case 64: return launch_kpt<64>(a, p.cl, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qsa
