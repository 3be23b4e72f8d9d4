// topk_groups.cu -- stage 2 of QSA: the exact Top-K over compressed groups
// (TensorRT-LLM "QSASparseAttentionConfig", field enable_heuristic_topk: the
// exact radix Top-K is the default selector over the compressed-group
// budget).  Ranking: score descending, ties to the lower group id.
//
// Design (sm_100a): one thread-block cluster of CL CTAs x 512 threads per
// query row; thread i of CTA r owns KPT consecutive candidates in registers as
// order-preserving uint32 keys, so the row is read from memory once (16-byte
// loads where the row is aligned).
//  * Radix select, 8 bits per pass from the most significant end, finds the
//    exact key tau of the n-th largest candidate.  Each pass histograms only
//    the keys that still match the digits found so far: per-warp shared
//    histograms (no block-wide atomic hot spots), one block reduction, and
//    then every CTA WRITES its 256 counts into its own slot of that pass's
//    table in every CTA of the cluster.  After one cluster barrier each CTA
//    adds the CL slots locally and finds the digit itself: one barrier per
//    pass, no remote reads, no zeroing.
//  * Output: every key > tau is kept, plus the first `need` keys == tau in
//    index order.  Because each thread owns a contiguous run of ids, one
//    exclusive scan over threads gives every thread the position of its first
//    kept id within its CTA; the counts of the CTAs before it come from the
//    histogram tables every CTA already holds (keys above tau are the keys
//    above the chosen digit in some pass), so no further exchange is needed
//    and the ids come out ascending with no sort.
#include <cooperative_groups.h>

#include "qsa_internal.cuh"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;
constexpr int kMaxCL = 8;

constexpr int kCandCap = 2048;  // candidates gathered after two passes (else four cluster passes)
constexpr int kRankCap = 512;   // up to this many candidates are ranked directly

struct TopkSmem {
  uint32_t hw[kWarps][kBins];            // per-warp histogram of the current digit
  uint32_t hall[4][kMaxCL][kBins];       // per pass: slot q = CTA q's histogram
  uint2 cand[kCandCap];                  // (key, id) of every candidate of the cluster
  int wsum[kWarps][kMaxCL];              // block reduction of the per-CTA counts above tau
  int ccnt[2 * kMaxCL];                  // per CTA: candidates above tau, equal to tau
  int wa[kWarps];                        // per-warp scan totals
  int bin[4], above[4];
  uint32_t tau;
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

// Threads 0..255 (warps 0..7) hold the counts h of the bins 255 - tid, i.e.
// from the top: the thread whose bin holds the need-th largest key writes the
// bin and the count of keys in all higher bins.
__device__ __forceinline__ void find_bin(int h, int need, int my_bin, int* bin_out, int* above_out, int* wa) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = h;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += u;
  }
  if (lane == 31) wa[warp] = incl;
  asm volatile("bar.sync 1, %0;" ::"r"(kBins));  // the 8 warps that scan
  int above = incl - h;
  for (int w = 0; w < warp; ++w) above += wa[w];
  if (above < need && above + h >= need) {
    *bin_out = my_bin;
    *above_out = above;
  }
}

template <int CL, int KPT>
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a, int vec, int tvec) {
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
  // the expanded row (when asked for): 4 tokens per kept group, then the
  // current block 4*c(p) .. p, then -1
  int32_t* trow = a.tok ? a.tok + (size_t)t * a.W : nullptr;
  const int cb = p >= 0 ? p - kGroupTokens * (p / kGroupTokens) + 1 : 0;  // current-block tokens
  if (c <= K) {  // every candidate is kept: dense fallback (uniform over the cluster)
    pdl_launch_dependents();
    for (int i = rank * kThreads + tid; i < K; i += CL * kThreads) out[i] = i < c ? i : -1;
    if (trow) {  // tokens 0 .. p (the kept groups and the current block are contiguous)
      const int total = kGroupTokens * n + cb;
      for (int i = rank * kThreads + tid; i < a.W; i += CL * kThreads)
        trow[i] = i < total ? (i < kGroupTokens * n ? i : kGroupTokens * (p / kGroupTokens) + i - kGroupTokens * n) : -1;
      if (rank == 0 && tid == 0) {
        a.n_tok[t] = total < a.W ? total : a.W;
        if (total > a.W) flag(a.status, QSA_DEV_ROW_RANGE);
      }
    }
    if (rank == 0 && tid == 0) a.n_sel[t] = n;
    return;
  }

  // ---- this thread's KPT consecutive candidates, as keys
  const int first = (rank * kThreads + tid) * KPT;
  const float* row = a.scores + (size_t)t * a.score_stride;
  uint32_t keys[KPT];
#pragma unroll
  for (int j = 0; j < KPT; j += 4) {
    if (vec && first + j + 3 < c) {  // 16-byte aligned when the row stride is a multiple of 4
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + first + j));
      keys[j] = order_key(v.x);
      keys[j + 1] = order_key(v.y);
      keys[j + 2] = order_key(v.z);
      keys[j + 3] = order_key(v.w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) keys[j + e] = first + j + e < c ? order_key(__ldg(row + first + j + e)) : 0u;
    }
  }
  // (dependents launch when this grid completes: launched earlier, their CTAs
  // compete for the SMs this kernel still needs)

  // ---- radix select: passes of 8 bits from the top locate tau.  After two
  // cluster passes the keys that still match (the candidates) are usually a
  // few dozen; then every CTA receives all of them and finishes the last two
  // digits on its own, without further cluster barriers.
  uint32_t prefix = 0;
  int need = n;  // how many keys matching `prefix` are still to be taken
  int npass = 4;  // cluster passes whose tables count the keys above tau
  int ncand = 0;
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
        cg::cluster_group cl = cg::this_cluster();
#pragma unroll
        for (int q = 0; q < CL; ++q) cl.map_shared_rank(&sm.hall[pass][rank][tid], q)[0] = v;
      } else {
        sm.hall[pass][0][tid] = v;
      }
    }
    csync<CL>();  // every CTA's counts are in every CTA's table
    if (tid < kBins) {
      int h = 0;
#pragma unroll
      for (int q = 0; q < CL; ++q) h += (int)sm.hall[pass][q][kBins - 1 - tid];
      find_bin(h, need, kBins - 1 - tid, &sm.bin[pass], &sm.above[pass], sm.wa);
    }
    __syncthreads();
    prefix |= (uint32_t)sm.bin[pass] << shift;
    need -= sm.above[pass];
    if (CL > 1 && pass == 1) {  // (a one-CTA row keeps its four passes)
      int total = 0;
#pragma unroll
      for (int q = 0; q < CL; ++q) total += (int)sm.hall[1][q][sm.bin[1]];
      if (total <= kCandCap) {  // the same decision in every CTA
        npass = 2;
        ncand = total;
        break;
      }
    }
  }

  if constexpr (CL > 1) if (npass == 2) {
    // ---- candidates: every CTA writes its keys matching the 16-bit prefix,
    // with their ids, into every CTA's list (CTA q's block starts after the
    // candidates of CTAs 0 .. q-1, whose counts pass 1's table holds)
    int mine = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) mine += (keys[j] >> 16) == (prefix >> 16);
    int cta_total;
    int pos = block_exclusive_scan(mine, sm.wa, cta_total);
    for (int q = 0; q < rank; ++q) pos += (int)sm.hall[1][q][sm.bin[1]];
    if (mine) {
      cg::cluster_group cl = cg::this_cluster();
#pragma unroll
      for (int j = 0; j < KPT; ++j) {
        if ((keys[j] >> 16) == (prefix >> 16)) {
          const uint2 e = make_uint2(keys[j], (uint32_t)(first + j));
          for (int q = 0; q < CL; ++q) *cl.map_shared_rank(&sm.cand[pos], q) = e;
          ++pos;
        }
      }
    }
    if (tid < 2 * kMaxCL) sm.ccnt[tid] = 0;
    csync<CL>();  // the lists are complete; from here every access is local
    if (ncand <= kRankCap) {
      // ---- few candidates: the rank of each under (key desc, id asc) is a
      // direct count; the candidate of rank need-1 is tau
      if (tid < ncand) {
        const uint2 me = sm.cand[tid];
        int r = 0, r_key = 0;  // rank, and candidates with a larger key
        for (int i = 0; i < ncand; ++i) {
          const uint2 o = sm.cand[i];
          r += o.x > me.x || (o.x == me.x && o.y < me.y);
          r_key += o.x > me.x;
        }
        if (r == need - 1) {
          sm.tau = me.x;
          sm.above[2] = r_key;  // candidates above tau
        }
      }
      __syncthreads();
      prefix = sm.tau;
      need -= sm.above[2];
    } else {
      // ---- the last two digits, over the candidates only
#pragma unroll
      for (int pass = 2; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        if (tid < kBins) sm.hw[0][tid] = 0u;
        __syncthreads();
        for (int i = tid; i < ncand; i += kThreads) {
          const uint32_t k = sm.cand[i].x;
          if ((k >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&sm.hw[0][(k >> shift) & (kBins - 1)], 1u);
        }
        __syncthreads();
        if (tid < kBins)
          find_bin((int)sm.hw[0][kBins - 1 - tid], need, kBins - 1 - tid, &sm.bin[pass], &sm.above[pass], sm.wa);
        __syncthreads();
        prefix |= (uint32_t)sm.bin[pass] << shift;
        need -= sm.above[pass];
      }
    }
    // per-CTA counts of candidates above and equal to tau (the CTA owning an id)
    for (int i = tid; i < ncand; i += kThreads) {
      const uint2 e = sm.cand[i];
      const int q = (int)(e.y / (uint32_t)(kThreads * KPT));
      if (e.x > prefix) atomicAdd(&sm.ccnt[q], 1);
      else if (e.x == prefix) atomicAdd(&sm.ccnt[kMaxCL + q], 1);
    }
  }
  const uint32_t tau = prefix;

  // ---- keys above tau in each CTA: a key is above tau when, in the first
  // pass where its digit differs from tau's, its digit is the larger one, and
  // that pass's table counted it under that digit in its CTA's slot (on the
  // candidate path the last two passes are counted from the candidate list)
  if (tid < kBins) {
    int x[kMaxCL];
#pragma unroll
    for (int q = 0; q < CL; ++q) x[q] = 0;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      if (pass < npass && tid > sm.bin[pass]) {
#pragma unroll
        for (int q = 0; q < CL; ++q) x[q] += (int)sm.hall[pass][q][tid];
      }
    }
#pragma unroll
    for (int q = 0; q < CL; ++q) {
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) x[q] += __shfl_xor_sync(0xffffffffu, x[q], d);
      if (lane == 0) sm.wsum[warp][q] = x[q];
    }
  }

  // ---- kept ids: all keys > tau, then the first `need` keys == tau by id
  int gt = 0, eq = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    gt += keys[j] > tau;
    eq += keys[j] == tau;
  }
  int both;  // one scan of gt (low 16 bits) and eq (high): per-CTA counts stay below 2^16
  const int before = block_exclusive_scan(gt | (eq << 16), sm.wa, both);  // syncs: wsum, ccnt visible
  const int gt_before = before & 0xffff, eq_before = before >> 16;
  // the CTAs before this one: lane q of every warp takes CTA q's counts, and a
  // warp prefix over q gives the offsets (no serial loop, no extra barrier)
  int off = 0, eq_prev = 0;
  if constexpr (CL > 1) {
    int gt_q = 0, eq_q = 0;
    if (lane < CL) {
      gt_q = npass == 2 ? sm.ccnt[lane] : 0;
#pragma unroll
      for (int w = 0; w < kBins / 32; ++w) gt_q += sm.wsum[w][lane];
      eq_q = npass == 2 ? sm.ccnt[kMaxCL + lane] : (int)sm.hall[3][lane][sm.bin[3]];
    }
    // exclusive prefix over lanes q < rank of the kept count: gt_q plus the
    // tau-keys CTA q takes, which depends on the tau-keys before it
    int eq_incl = eq_q;
#pragma unroll
    for (int d = 1; d < kMaxCL; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, eq_incl, d);
      if (lane >= d) eq_incl += u;
    }
    const int eq_before_q = eq_incl - eq_q;
    const int rem_q = need - eq_before_q;
    int kept_q = lane < rank ? gt_q + (rem_q <= 0 ? 0 : (rem_q < eq_q ? rem_q : eq_q)) : 0;
#pragma unroll
    for (int d = 1; d < kMaxCL; d <<= 1) kept_q += __shfl_xor_sync(0xffffffffu, kept_q, d);
    off = __shfl_sync(0xffffffffu, kept_q, 0);
    eq_prev = __shfl_sync(0xffffffffu, eq_before_q, rank);
  }
  int rem = need - eq_prev;                     // tau-keys still to take at this CTA's start
  rem = rem < 0 ? 0 : rem;
  int pos = off + gt_before + (rem < eq_before ? rem : eq_before);
  int take = rem - eq_before;                   // tau-keys this thread may take
  take = take < 0 ? 0 : take;
  if (gt > 0 || take > 0)  // (most threads keep nothing)
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const uint32_t k = keys[j];
    bool keep = k > tau;
    if (k == tau && take > 0) {
      keep = true;
      --take;
    }
    if (keep) {
      if (pos < K) {
        const int g = first + j;
        out[pos] = g;
        if (trow) {
          if (tvec) {
            *reinterpret_cast<int4*>(trow + kGroupTokens * pos) =
                make_int4(kGroupTokens * g, kGroupTokens * g + 1, kGroupTokens * g + 2, kGroupTokens * g + 3);
          } else {
#pragma unroll
            for (int e = 0; e < kGroupTokens; ++e) trow[kGroupTokens * pos + e] = kGroupTokens * g + e;
          }
        }
      }
      ++pos;
    }
  }
  if (rank == 0) {
    for (int i = n + tid; i < K; i += kThreads) out[i] = -1;
    if (tid == 0) a.n_sel[t] = n;
    if (trow) {  // the current block, then padding
      const int head = kGroupTokens * n, total = head + cb;
      for (int i = head + tid; i < a.W; i += kThreads)
        trow[i] = i < total ? kGroupTokens * (p / kGroupTokens) + (i - head) : -1;
      if (tid == 0) {
        a.n_tok[t] = total < a.W ? total : a.W;
        if (total > a.W) flag(a.status, QSA_DEV_ROW_RANGE);
      }
    }
  }
}

template <int CL, int KPT>
cudaError_t launch_cfg(const TopkArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(TopkSmem);
  auto kern = topk_kernel<CL, KPT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int vec = (a.score_stride % 4 == 0) && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0;
  const int tvec = a.tok && a.W % 4 == 0 && (reinterpret_cast<uintptr_t>(a.tok) & 15u) == 0;
  return launch_k(kern, dim3(CL, a.T), dim3(kThreads), smem, s, CL, a, vec, tvec);
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
