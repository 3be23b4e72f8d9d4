// topk_groups.cu -- stage 2 of QSA: the exact Top-K over compressed groups
// (TensorRT-LLM "QSASparseAttentionConfig", field enable_heuristic_topk: the
// exact radix Top-K is the default selector over the compressed-group
// budget).  Ranking: score descending, ties to the lower group id.
//
// Design (sm_100a): one thread-block cluster of CL CTAs per query row.  Each
// CTA stages its contiguous slice of the row in shared memory as
// order-preserving uint32 keys, so the row is read from memory exactly once.
// Three radix passes (11 + 11 + 10 bits, most significant first) find the
// exact key tau of the n-th largest candidate: every CTA histograms its slice,
// the per-CTA histograms are summed through distributed shared memory (CTA q
// reduces bin slice q and pushes the totals into every CTA), and every CTA
// then locates the same bin.  The output pass keeps all keys > tau plus the
// first `need` keys == tau in index order; a ballot/popc block scan writes the
// kept ids in ascending order, each CTA at the offset given by the counts of
// the CTAs before it.
#include <cooperative_groups.h>

#include "qsa_internal.cuh"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;               // bins of the widest digit (11 bits)
constexpr int kMaxChunk = 49152;          // keys per CTA (192 KiB of shared memory)

struct TopkSmem {
  uint32_t hist[kBins];      // this CTA's histogram of the current digit
  uint32_t ghist[kBins];     // cluster-wide histogram (pushed by the reducers)
  int cnt_gt[8], cnt_eq[8];  // per-CTA counts of keys > tau and == tau
  int warp_a[kWarps], warp_b[kWarps];
  int bin, above;
};

// float -> uint32 whose unsigned order equals the float order; -0 maps like +0
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

template <int CL>
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a, int chunk) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkSmem));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int rank = 0;
  if constexpr (CL > 1) rank = (int)cg::this_cluster().block_rank();
  const int t = blockIdx.y;
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
    for (int i = rank * kThreads + tid; i < K; i += CL * kThreads) out[i] = i < c ? i : -1;
    if (rank == 0 && tid == 0) a.n_sel[t] = n;
    return;
  }

  // ---- stage the slice as keys
  const int lo = rank * chunk;
  int m = c - lo;
  m = m < 0 ? 0 : (m > chunk ? chunk : m);
  const float* row = a.scores + (size_t)t * a.score_stride + lo;
  for (int i = tid; i < m; i += kThreads) keys[i] = order_key(__ldg(row + i));

  // ---- three radix passes locate tau, the key of the n-th largest candidate
  uint32_t prefix = 0;
  int need = n;  // how many of the keys that match `prefix` are still to be taken
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + (pass == 2 ? 10 : 11)));
    for (int b = tid; b < nb; b += kThreads) sm.hist[b] = 0;
    __syncthreads();
    for (int i = tid; i < m; i += kThreads) {
      const uint32_t k = keys[i];
      if ((k & hi_mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & (nb - 1)], 1u);
    }
    csync<CL>();
    // cluster-wide histogram: CTA `rank` sums its bin slice and pushes it everywhere
    {
      const int per = nb / CL;
      for (int b = rank * per + tid; b < (rank + 1) * per; b += kThreads) {
        uint32_t tot = 0;
        if constexpr (CL > 1) {
          cg::cluster_group cl = cg::this_cluster();
#pragma unroll
          for (int q = 0; q < CL; ++q) tot += cl.map_shared_rank(sm.hist, q)[b];
#pragma unroll
          for (int q = 0; q < CL; ++q) cl.map_shared_rank(sm.ghist, q)[b] = tot;
        } else {
          sm.ghist[b] = sm.hist[b];
        }
      }
    }
    csync<CL>();
    // locate the bin holding the need-th largest: thread tid owns the bpt bins
    // just below the (tid * bpt)-th bin counted from the top
    const int bpt = nb / kThreads;
    const int top = nb - tid * bpt;  // bins [top - bpt, top)
    int local = 0;
    for (int b = top - bpt; b < top; ++b) local += (int)sm.ghist[b];
    // exclusive scan of `local` over tid: the count in all higher bins
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) sm.warp_a[warp] = incl;
    __syncthreads();
    int above = incl - local;
    for (int w = 0; w < warp; ++w) above += sm.warp_a[w];
    if (above < need && above + local >= need) {
      int acc = above;
      for (int b = top - 1; b >= top - bpt; --b) {
        const int h = (int)sm.ghist[b];
        if (acc + h >= need) { sm.bin = b; sm.above = acc; break; }
        acc += h;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)sm.bin << shift;
    need -= sm.above;
    __syncthreads();
  }
  const uint32_t tau = prefix;

  // ---- counts of keys above / equal to tau in every CTA
  {
    int gt = 0, eq = 0;
    for (int i = tid; i < m; i += kThreads) {
      const uint32_t k = keys[i];
      gt += k > tau;
      eq += k == tau;
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, d);
      eq += __shfl_xor_sync(0xffffffffu, eq, d);
    }
    if (lane == 0) { sm.warp_a[warp] = gt; sm.warp_b[warp] = eq; }
    __syncthreads();
    if (tid == 0) {
      int g2 = 0, e2 = 0;
      for (int w = 0; w < kWarps; ++w) { g2 += sm.warp_a[w]; e2 += sm.warp_b[w]; }
      if constexpr (CL > 1) {
        cg::cluster_group cl = cg::this_cluster();
        for (int q = 0; q < CL; ++q) {
          cl.map_shared_rank(sm.cnt_gt, q)[rank] = g2;
          cl.map_shared_rank(sm.cnt_eq, q)[rank] = e2;
        }
      } else {
        sm.cnt_gt[0] = g2;
        sm.cnt_eq[0] = e2;
      }
    }
    csync<CL>();
  }
  // ---- where this CTA's kept ids start, and how many tau-keys it keeps
  int off = 0, eq_before = 0;
  for (int q = 0; q < rank; ++q) {
    int take = need - eq_before;
    take = take < 0 ? 0 : (take > sm.cnt_eq[q] ? sm.cnt_eq[q] : take);
    off += sm.cnt_gt[q] + take;
    eq_before += sm.cnt_eq[q];
  }
  int take_eq = need - eq_before;
  take_eq = take_eq < 0 ? 0 : (take_eq > sm.cnt_eq[rank] ? sm.cnt_eq[rank] : take_eq);

  // ---- ordered write: ballot/popc scan over tiles of kThreads keys
  const unsigned lt_mask = (1u << lane) - 1u;
  int eq_run = 0, pos_run = off;
  for (int base = 0; base < m; base += kThreads) {
    const int i = base + tid;
    const uint32_t k = i < m ? keys[i] : 0u;
    const bool is_eq = i < m && k == tau;
    const bool is_gt = i < m && k > tau;
    const unsigned be = __ballot_sync(0xffffffffu, is_eq);
    if (lane == 0) sm.warp_a[warp] = __popc(be);
    __syncthreads();
    int eq_rank = eq_run + __popc(be & lt_mask), eq_tile = 0;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) eq_rank += sm.warp_a[w];
      eq_tile += sm.warp_a[w];
    }
    const bool keep = is_gt || (is_eq && eq_rank < take_eq);
    const unsigned bk = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) sm.warp_b[warp] = __popc(bk);
    __syncthreads();
    int pos = pos_run + __popc(bk & lt_mask), keep_tile = 0;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) pos += sm.warp_b[w];
      keep_tile += sm.warp_b[w];
    }
    if (keep && pos < K) out[pos] = lo + i;
    eq_run += eq_tile;
    pos_run += keep_tile;
    __syncthreads();
  }
  if (rank == 0) {
    for (int i = n + tid; i < K; i += kThreads) out[i] = -1;
    if (tid == 0) a.n_sel[t] = n;
  }
}

template <int CL>
cudaError_t launch_cl(const TopkArgs& a, cudaStream_t s) {
  int chunk = (a.score_stride + CL - 1) / CL;
  chunk = (chunk + 3) & ~3;
  if (chunk < 4) chunk = 4;
  const size_t smem = sizeof(TopkSmem) + (size_t)chunk * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel<CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, a.T, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_kernel<CL>, a, chunk);
}

}  // namespace

// Smallest cluster whose per-CTA slice stays small; large row counts prefer
// one CTA per row (more rows in flight), small ones spread a row over up to 8.
int topk_cluster_size(int score_stride) {
  for (int cl = 1; cl <= 8; cl <<= 1) {
    const int chunk = (score_stride + cl - 1) / cl;
    if (chunk <= 8192) return cl;
  }
  return (score_stride + 7) / 8 <= kMaxChunk ? 8 : 0;
}

cudaError_t launch_topk_groups(const TopkArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  int cl = topk_cluster_size(a.score_stride);
  // many rows: one CTA per row while its slice fits comfortably
  if (a.T >= 148 && a.score_stride <= 16384) cl = 1;
  switch (cl) {
    case 1: return launch_cl<1>(a, s);
    case 2: return launch_cl<2>(a, s);
    case 4: return launch_cl<4>(a, s);
    case 8: return launch_cl<8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qsa
