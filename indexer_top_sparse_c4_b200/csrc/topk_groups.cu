// topk_groups.cu -- stage 2 of QSA: the exact Top-K over compressed groups
// (TensorRT-LLM "QSASparseAttentionConfig", field enable_heuristic_topk: the
// exact radix Top-K is the default selector over the compressed-group
// budget).  Ranking: score descending, ties to the lower group id.
//
// Candidates become order-preserving uint32 keys; thread i of a CTA owns KPT
// consecutive ids, so the row is read from memory once (16-byte loads where
// the row is aligned).  Radix select over 8-bit digits from the most
// significant end finds the exact key tau of the n-th largest candidate; the
// output keeps every key > tau plus the first `need` keys == tau in id order.
// Because each thread owns a contiguous run of ids, one exclusive scan over
// the threads places every kept id, and the ids come out ascending without a
// sort.
//
// Two kernels:
//  * topk_row_kernel (many rows, e.g. a prefill chunk): one CTA per row, keys
//    in registers, four block-local passes.  Many CTAs per SM keep the code
//    hot in the instruction caches.  In its guess-verify-refine mode (no
//    hint) the passes over the whole row give way to a self-sampled guess:
//    a histogram of the top 12 key bits of every (KPT/4)-th key gives a
//    window of bins around the n-th key's sample rank, one pass counts the
//    keys above and in it, and when the counts confirm it the digit passes
//    run over the window's keys alone.
//  * topk_cluster_kernel (few long rows, decode): one thread-block cluster of
//    CL CTAs per row.  Each code path runs once per launch, so the kernel is
//    written for a small instruction footprint: keys live in shared memory
//    ([j][thread], conflict-free) and the loops over them stay rolled.
//    - With the prefix histogram the scan built (counts of the top 12 key
//      bits of the row), every CTA finds the 12-bit bin of the n-th largest
//      key directly.  Each CTA lists its keys in that bin (a few hundred per
//      row here) in its own shared memory and sends every CTA its counts in
//      and above the bin; after one cluster barrier each CTA checks the
//      histogram's answer against those exact counts, pulls all lists into
//      registers with independent DSMEM loads, and finds the low 20 bits
//      with three block-local digit passes.  A histogram that does not match
//      (or an overfull bin) sends the row to the cluster passes below: it is
//      a hint, and the result never depends on it.
//    - Cluster passes: per pass, per-warp shared histograms, one block
//      reduction, and every CTA writes its 256 counts into its own slot of
//      that pass's table in every CTA; after one cluster barrier each CTA
//      adds the slots and finds the digit itself.  After two passes the keys
//      that still match the 16-bit prefix (usually a few dozen) are pushed
//      into every CTA, which finishes the last two digits locally.
//    - Guess-verify-refine with self-sampling (no histogram): every CTA reads
//      the same strided sample of 2,048 of the row's scores and takes, from a
//      histogram of their top 12 key bits, the window of bins between the
//      sample ranks n*2048/c -+ (3 sigma + 1).  The keys in the window are the
//      candidates and the exact counts verify the guess as above; after the
//      pull, one 256-bin pass over the window finds the exact bin and the
//      digit passes go on.  A failed guess takes the cluster passes.
//    - The counts of the CTAs before a CTA come from data every CTA already
//      holds (the pass tables, or the exchanged counts), so the output needs
//      no further exchange.
#include <cooperative_groups.h>

#include "qsa_internal.cuh"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;
constexpr int kMaxCL = 8;

constexpr int kCandCap = 2048;  // candidates gathered by a cluster (else more cluster passes)
constexpr int kListCapG = 4096; // self-sampling window path: candidates listed by a cluster
constexpr int kSampleN = 2048;  // self-sampling guess: scores sampled per row
constexpr int kRankCap = 512;   // up to this many candidates are ranked directly
constexpr int kKeptCap = kWarps * kBins;  // kept ids a CTA stages for its coalesced output

template <int CAP>
struct __align__(16) TopkSmemT {
  uint32_t hw[kWarps][kBins];            // per-warp histogram of the current digit
  uint32_t hall[4][kMaxCL][kBins];       // per pass: slot q = CTA q's histogram
  uint2 cand[CAP];                       // (key, id) candidates
  int wsum[kWarps][kMaxCL];              // block reduction of the per-CTA counts above tau
  int ccnt[2 * kMaxCL];                  // per CTA: candidates above tau, equal to tau
  int wa[kWarps];                        // per-warp scan totals
  int bin[4], above[4];
  uint32_t tau;
  // prefix-histogram path: the bin of the n-th largest key (from the
  // histogram), and per source CTA its keys in and above that bin
  int pbin, pbin_lo;                     // the guessed window of 12-bit bins (one bin: equal)
  int scnt[kMaxCL], sgt[kMaxCL];
  uint2 fin[kRankCap];                   // candidates left after the first local digit
  int nfin;
};
static_assert(kThreads * 8 == kPrefixBins, "each thread reads 8 bins of the prefix histogram");
static_assert(kWarps * kBins == kPrefixBins && kSampleN % kThreads == 0 && 4 * kMaxCL >= kWarps,
              "the sample histogram reuses hw, 8 bins per thread");
using TopkSmem = TopkSmemT<kCandCap>;   // the histogram / plain paths
using TopkSmemG = TopkSmemT<kListCapG>; // the self-sampling path
static_assert(sizeof(TopkSmem) % 16 == 0 && sizeof(TopkSmemG) % 16 == 0,
              "the key array after the shared struct starts on 16 bytes");

// A thread's KPT keys.  RegKeys: in registers (loops over them fully
// unrolled).  SmemKeys: in shared memory, key j of thread i at [j][i], so
// loops over them can stay rolled (kUnroll keys per iteration).
template <int KPT>
struct RegKeys {
  static constexpr int kUnroll = KPT;
  uint32_t v[KPT];
  __device__ __forceinline__ uint32_t get(int j) const { return v[j]; }
  __device__ __forceinline__ void set(int j, uint32_t k) { v[j] = k; }
};
template <int KPT>
struct SmemKeys {
  static constexpr int kUnroll = 4;
  uint32_t* col;  // this thread's column of the [KPT][kThreads] array
  __device__ __forceinline__ uint32_t get(int j) const { return col[j * kThreads]; }
  __device__ __forceinline__ void set(int j, uint32_t k) { col[j * kThreads] = k; }
};

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
#pragma unroll
  for (int w = 0; w < kBins / 32; ++w) above += w < warp ? wa[w] : 0;
  if (above < need && above + h >= need) {
    *bin_out = my_bin;
    *above_out = above;
  }
}

// CTA `rank`'s share of a row of the prefix histogram back to zero.
template <int CL>
__device__ __forceinline__ void zero_hist_share(uint32_t* hrow, int rank) {
  constexpr int per = kPrefixBins / CL;
  for (int i = rank * per + 4 * (int)threadIdx.x; i < (rank + 1) * per; i += 4 * kThreads)
    *reinterpret_cast<uint4*>(hrow + i) = make_uint4(0u, 0u, 0u, 0u);
}

// What a CTA knows about its row before any pass.
struct Row {
  int p, c, K, n;       // query position, candidates, budget, kept count
  int cb;               // tokens of the current block (4*c(p) .. p)
  int32_t* out;         // sel row
  int32_t* trow;        // expanded row, or nullptr
  uint32_t* hrow;       // prefix-histogram row, or nullptr
};

__device__ __forceinline__ Row row_of(const TopkArgs& a, int t, bool leader) {
  Row r;
  r.p = a.q_pos[t];
  r.c = r.p >= 0 ? r.p / kGroupTokens : 0;
  if (r.c > a.score_stride) {
    if (leader) flag(a.status, QSA_DEV_ROW_RANGE);
    r.c = a.score_stride;
  }
  r.K = a.K;
  r.n = r.c < r.K ? r.c : r.K;
  r.cb = r.p >= 0 ? r.p - kGroupTokens * (r.p / kGroupTokens) + 1 : 0;
  r.out = a.sel + (size_t)t * r.K;
  // the expanded row (when asked for): 4 tokens per kept group, then the
  // current block 4*c(p) .. p, then -1
  r.trow = a.tok ? a.tok + (size_t)t * a.W : nullptr;
  r.hrow = a.hist ? a.hist + (size_t)t * kPrefixBins : nullptr;
  return r;
}

// c <= K: every candidate is kept (dense fallback), CTA `rank` of CL writes
// its share of the outputs.
template <int CL>
__device__ __forceinline__ void dense_row(const TopkArgs& a, const Row& r, int t, int rank) {
  const int tid = threadIdx.x;
  if (r.hrow) zero_hist_share<CL>(r.hrow, rank);  // (not read on this path)
  for (int i = rank * kThreads + tid; i < r.K; i += CL * kThreads) r.out[i] = i < r.c ? i : -1;
  if (r.trow) {  // tokens 0 .. p (the kept groups and the current block are contiguous)
    const int head = kGroupTokens * r.n, total = head + r.cb;
    for (int i = rank * kThreads + tid; i < a.W; i += CL * kThreads)
      r.trow[i] = i < total ? (i < head ? i : kGroupTokens * (r.p / kGroupTokens) + i - head) : -1;
    if (rank == 0 && tid == 0) {
      a.n_tok[t] = total < a.W ? total : a.W;
      if (total > a.W) flag(a.status, QSA_DEV_ROW_RANGE);
    }
  }
  if (rank == 0 && tid == 0) {
    a.n_sel[t] = r.n;
    if (a.path) a.path[t] = 0;
  }
}

// The thread's KPT consecutive candidates from `first`, as keys (0 past c).
template <int KPT, typename Keys>
__device__ __forceinline__ void load_keys(Keys& keys, const float* row, int first, int c, int vec) {
  constexpr int U = Keys::kUnroll / 4 > 0 ? Keys::kUnroll / 4 : 1;
#pragma unroll U
  for (int j = 0; j < KPT; j += 4) {
    if (vec && first + j + 3 < c) {  // 16-byte aligned when the row stride is a multiple of 4
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + first + j));
      keys.set(j, order_key(v.x));
      keys.set(j + 1, order_key(v.y));
      keys.set(j + 2, order_key(v.z));
      keys.set(j + 3, order_key(v.w));
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) keys.set(j + e, first + j + e < c ? order_key(__ldg(row + first + j + e)) : 0u);
    }
  }
}

// Writes this CTA's kept ids (and their tokens) at positions off ..: every
// key > tau, and tau-keys while `rem` (those still to take at the CTA's
// start) lasts.  gt/eq: this thread's counts; *_before: the threads' before
// it; cta_*: the CTA's totals.  MASKED: only the keys flagged in above_mask
// (certainly kept) and cand_mask (compared with tau) are visited; otherwise
// all KPT.  The ids are staged in shared memory (the per-warp histograms,
// whose last use came before the block scan that gave the positions) and
// written with coalesced stores.
template <int KPT, bool MASKED, typename Keys, typename SM>
__device__ __forceinline__ void emit_kept(SM& sm, const Keys& keys, uint64_t above_mask, uint64_t cand_mask,
                                          int first, uint32_t tau, int gt, int gt_before, int eq_before, int cta_gt,
                                          int cta_eq, int rem, int off, const Row& r, int tvec) {
  constexpr int U = Keys::kUnroll;
  const int tid = threadIdx.x;
  int pos = gt_before + (rem < eq_before ? rem : eq_before);  // within the CTA's kept ids
  int take = rem - eq_before;                                 // tau-keys this thread may take
  take = take < 0 ? 0 : take;
  int* const kept = reinterpret_cast<int*>(&sm.hw[0][0]);
  const int cta_kept = cta_gt + (rem < cta_eq ? rem : cta_eq);
  const bool staged = cta_kept <= kKeptCap;  // (CTA-uniform)
  auto visit = [&](int j, bool above) {
    bool keep = above;
    if (!above) {
      const uint32_t k = keys.get(j);
      keep = k > tau;
      if (k == tau && take > 0) {
        keep = true;
        --take;
      }
    }
    if (keep) {
      const int g = first + j;
      if (staged) {
        kept[pos] = g;
      } else if (off + pos < r.K) {
        r.out[off + pos] = g;
        if (r.trow) {
#pragma unroll
          for (int e = 0; e < kGroupTokens; ++e) r.trow[kGroupTokens * (off + pos) + e] = kGroupTokens * g + e;
        }
      }
      ++pos;
    }
  };
  if (gt > 0 || take > 0) {  // (most threads keep nothing)
    if constexpr (MASKED) {
      for (uint64_t m = above_mask | cand_mask; m; m &= m - 1) {
        const int j = __ffsll((long long)m) - 1;
        visit(j, (above_mask >> j) & 1u);
      }
    } else {
#pragma unroll U
      for (int j = 0; j < KPT; ++j) visit(j, false);
    }
  }
  if (staged) {
    __syncthreads();
    const int lim = cta_kept < r.K - off ? cta_kept : r.K - off;
    for (int i = tid; i < lim; i += kThreads) {
      const int g = kept[i];
      r.out[off + i] = g;
      if (r.trow) {
        if (tvec) {
          *reinterpret_cast<int4*>(r.trow + kGroupTokens * (off + i)) =
              make_int4(kGroupTokens * g, kGroupTokens * g + 1, kGroupTokens * g + 2, kGroupTokens * g + 3);
        } else {
#pragma unroll
          for (int e = 0; e < kGroupTokens; ++e) r.trow[kGroupTokens * (off + i) + e] = kGroupTokens * g + e;
        }
      }
    }
  }
}

// CTA 0's part of every row: -1 after the n kept ids, the current block and
// the padding of the expanded row, the counts.
__device__ __forceinline__ void write_tail(const TopkArgs& a, const Row& r, int t) {
  const int tid = threadIdx.x;
  for (int i = r.n + tid; i < r.K; i += kThreads) r.out[i] = -1;
  if (tid == 0) a.n_sel[t] = r.n;
  if (r.trow) {
    const int head = kGroupTokens * r.n, total = head + r.cb;
    for (int i = head + tid; i < a.W; i += kThreads)
      r.trow[i] = i < total ? kGroupTokens * (r.p / kGroupTokens) + (i - head) : -1;
    if (tid == 0) {
      a.n_tok[t] = total < a.W ? total : a.W;
      if (total > a.W) flag(a.status, QSA_DEV_ROW_RANGE);
    }
  }
}

// gt (low 16 bits) and eq (high) counts of a thread's keys against tau.
template <int KPT, typename Keys>
__device__ __forceinline__ int count_vs(const Keys& keys, uint32_t tau) {
  constexpr int U = Keys::kUnroll;
  int gt = 0, eq = 0;
#pragma unroll U
  for (int j = 0; j < KPT; ++j) {
    const uint32_t k = keys.get(j);
    gt += k > tau;
    eq += k == tau;
  }
  return gt | (eq << 16);
}

// Guess-verify-refine for one CTA's row, keys in registers: the key tau of the
// n-th largest candidate and how many keys equal to tau are kept, without the
// four radix passes over the whole row.  Thread i samples its keys 0, KPT/4,
// KPT/2, 3KPT/4, i.e. every (KPT/4)-th id of the row; a histogram of their
// top 12 key bits gives the window of bins between the sample ranks
// n ns / c -+ (3 sigma + 1).  One pass counts the keys above the window and
// in it; when those exact counts put the n-th key inside the window (and the
// window holds at most kListCapG keys), the window's keys are listed with their
// ids and four digit passes over them alone find tau (the window bin, then
// bits 12..19, 4..11 and 0..3).  The output then needs no pass over the keys:
// the masks of keys above and in the window, with the list, say which are kept.
// Returns false, with nothing written, when the guess fails; the caller then
// runs the radix passes.  (Block-uniform.)
struct RowGuess {
  uint32_t tau;        // the key of the n-th largest candidate
  int need;            // keys equal to tau that are kept (the lowest ids first)
  uint64_t above;      // this thread's keys above the window (all kept)
  uint64_t cand;       // this thread's keys in the window
  int pos0;            // where this thread's window keys start in the list
};

// A thread's window keys, read back from the window list (key j of the
// thread is list entry pos0 + the number of window keys before it).
struct ListKeys {
  static constexpr int kUnroll = 1;
  const uint2* list;
  int pos0;
  uint64_t cand;
  __device__ __forceinline__ uint32_t get(int j) const {
    return list[pos0 + __popcll((long long)(cand & ((1ull << j) - 1ull)))].x;
  }
};

template <int KPT>
__device__ __forceinline__ bool row_guess(TopkSmemG& sm, const RegKeys<KPT>& keys, const float* row, int first,
                                          int c, int n, RowGuess& g) {
  static_assert(KPT <= 64, "key masks are 64 bits");
  static_assert(KPT % 4 == 0 && kThreads * 8 == kPrefixBins, "4 samples per thread, 8 bins per thread");
  constexpr int SS = KPT / 4;  // sample stride
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* const sh = &sm.hw[0][0];  // the 4,096-bin sample histogram (flat)
#pragma unroll
  for (int j = 0; j < 8; ++j) sh[8 * tid + j] = 0u;
  if (tid == 0) {
    sm.pbin = kPrefixBins - 1;
    sm.pbin_lo = 0;
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < 4; ++m)
    if (first + m * SS < c) atomicAdd(&sh[keys.get(m * SS) >> kPrefixShift], 1u);
  __syncthreads();
  const int ns = (c + SS - 1) / SS;  // sampled ids: the multiples of SS below c
  int hs = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) hs += (int)sh[kPrefixBins - 1 - 8 * tid - j];
  int htotal;
  const int hbefore = block_exclusive_scan(hs, sm.wa, htotal);
  const float e = (float)n * (float)ns / (float)c, sd = sqrtf(e);
  const int r_hi = max(1, (int)floorf(e - 3.f * sd - 1.f));
  const int r_lo = min(ns, (int)ceilf(e + 3.f * sd + 1.f));
  int ab = hbefore;
#pragma unroll
  for (int j = 0; j < 8; ++j) {  // (the counts are read again: fewer registers live across the scan)
    const int b = kPrefixBins - 1 - 8 * tid - j;
    const int h = (int)sh[b];
    if (ab < r_hi && ab + h >= r_hi) sm.pbin = b;
    if (ab < r_lo && ab + h >= r_lo) sm.pbin_lo = b;
    ab += h;
  }
  __syncthreads();
  const uint32_t pb = (uint32_t)sm.pbin, pb_lo = (uint32_t)sm.pbin_lo;
  if (pb - pb_lo >= (uint32_t)kBins) return false;  // the window does not fit one 256-bin pass

  // ---- verify: exact counts above the window and in it (and which keys)
  uint64_t am = 0, cm = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const uint32_t b = keys.get(j) >> kPrefixShift;
    const bool valid = first + j < c;
    if (valid && b > pb) am |= 1ull << j;
    if (valid && b <= pb && b >= pb_lo) cm |= 1ull << j;
  }
  int tot;  // candidates (low 16 bits; c <= 32,768) and keys above the window (high)
  int pos = block_exclusive_scan(__popcll((long long)cm) | (__popcll((long long)am) << 16), sm.wa, tot) & 0xffff;
  const int in_win = tot & 0xffff, above_all = tot >> 16;
  if (!(above_all < n && above_all + in_win >= n && in_win <= kListCapG)) return false;
  g.above = am;
  g.cand = cm;
  g.pos0 = pos;

  // ---- refine: the window's keys with their ids, in id order (each key read
  // again from the row, an L1 hit, so that the loop indexes no register array)
  for (uint64_t m = cm; m; m &= m - 1) {
    const int j = __ffsll((long long)m) - 1;
    sm.cand[pos++] = make_uint2(order_key(__ldg(row + first + j)), (uint32_t)(first + j));
  }
  __syncthreads();
  uint32_t pre = 0;
  int nd = n - above_all;  // the nd-th largest in the window is the n-th of the row
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    // pass 0: the window bin (offset from pb_lo); then bits 12..19, 4..11, 0..3
    const int shift = pass == 0 ? kPrefixShift : (pass == 1 ? 12 : (pass == 2 ? 4 : 0));
    const int fixed = pass == 1 ? kPrefixShift : (pass == 2 ? 12 : 4);  // bits above `shift` already known
    const uint32_t dmask = pass == 3 ? 0xFu : 0xFFu;
#pragma unroll
    for (int b = lane; b < kBins; b += 32) sm.hw[warp][b] = 0u;
    __syncwarp();
    for (int i = tid; i < in_win; i += kThreads) {
      const uint32_t k = sm.cand[i].x;
      if (pass == 0) atomicAdd(&sm.hw[warp][(k >> kPrefixShift) - pb_lo], 1u);
      else if ((k >> fixed) == (pre >> fixed)) atomicAdd(&sm.hw[warp][(k >> shift) & dmask], 1u);
    }
    __syncthreads();
    if (tid < kBins) {
      uint32_t v = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += sm.hw[w][kBins - 1 - tid];
      find_bin((int)v, nd, kBins - 1 - tid, &sm.bin[pass], &sm.above[pass], sm.wa);
    }
    __syncthreads();
    const uint32_t d = (uint32_t)sm.bin[pass];
    pre |= pass == 0 ? (pb_lo + d) << kPrefixShift : d << shift;
    nd -= sm.above[pass];
  }
  g.tau = pre;
  g.need = nd;
  return true;
}

// ---- many rows: one CTA per row, keys in registers --------------------------------
// GVR: first the self-sampled guess of row_guess (guess-verify-refine), the
// radix passes only when it fails.
template <int KPT, bool GVR>
__global__ void __launch_bounds__(kThreads, 2) topk_row_kernel(TopkArgs a, int vec, int tvec) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  using SMT = TopkSmemT<GVR ? kListCapG : kCandCap>;
  SMT& sm = *reinterpret_cast<SMT*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int t = blockIdx.y;
  pdl_wait();
  const Row r = row_of(a, t, tid == 0);
  if (r.c <= r.K) {
    dense_row<1>(a, r, t, 0);
    return;
  }
  if (r.hrow) zero_hist_share<1>(r.hrow, 0);  // (not read by this kernel)
  const int first = tid * KPT;
  const float* const row = a.scores + (size_t)t * a.score_stride;
  RegKeys<KPT> keys;
  load_keys<KPT>(keys, row, first, r.c, vec);
  // (dependents launch when this grid completes: launched earlier, their CTAs
  // compete for the SMs this kernel still needs)

  if constexpr (GVR) {
    RowGuess g;
    if (row_guess<KPT>(sm, keys, row, first, r.c, r.n, g)) {
      // kept: the keys above the window, then the window's keys > tau and the
      // first g.need == tau by id (this thread's are list entries pos0 ..)
      int gt = __popcll((long long)g.above), eq = 0;
      const int end = g.pos0 + __popcll((long long)g.cand);
      for (int i = g.pos0; i < end; ++i) {
        const uint32_t k = sm.cand[i].x;
        gt += k > g.tau;
        eq += k == g.tau;
      }
      int both;
      const int before = block_exclusive_scan(gt | (eq << 16), sm.wa, both);
      const ListKeys lk{sm.cand, g.pos0, g.cand};
      emit_kept<KPT, true>(sm, lk, g.above, g.cand, first, g.tau, gt, before & 0xffff, before >> 16,
                           both & 0xffff, both >> 16, g.need, 0, r, tvec);
      write_tail(a, r, t);
      if (tid == 0 && a.path) a.path[t] = 1;
      return;
    }
  }

  // ---- radix select: four passes of 8 bits from the top
  uint32_t prefix = 0;
  int need = r.n;  // how many keys matching `prefix` are still to be taken
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int b = threadIdx.x & 31; b < kBins; b += 32) sm.hw[warp][b] = 0u;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const uint32_t k = keys.get(j);
      const bool match = pass == 0 ? k != 0u : (k >> (shift + 8)) == (prefix >> (shift + 8));
      if (match) atomicAdd(&sm.hw[warp][(k >> shift) & (kBins - 1)], 1u);
    }
    __syncthreads();
    if (tid < kBins) {
      uint32_t v = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += sm.hw[w][kBins - 1 - tid];
      find_bin((int)v, need, kBins - 1 - tid, &sm.bin[pass], &sm.above[pass], sm.wa);
    }
    __syncthreads();
    prefix |= (uint32_t)sm.bin[pass] << shift;
    need -= sm.above[pass];
  }
  const uint32_t tau = prefix;

  // ---- kept ids: all keys > tau, then the first `need` keys == tau by id
  const int ge = count_vs<KPT>(keys, tau);
  int both;
  const int before = block_exclusive_scan(ge, sm.wa, both);
  emit_kept<KPT, false>(sm, keys, 0, 0, first, tau, ge & 0xffff, before & 0xffff, before >> 16, both & 0xffff,
                        both >> 16, need, 0, r, tvec);
  write_tail(a, r, t);
  if (GVR && tid == 0 && a.path) a.path[t] = 3;
}

// ---- few long rows: one cluster per row, keys in shared memory ------------------
template <int CL, int KPT, bool GVR>
__global__ void __launch_bounds__(kThreads, 1) topk_cluster_kernel(TopkArgs a, int vec, int tvec) {
  static_assert(CL > 1, "one-CTA rows use topk_row_kernel");
  static_assert(KPT <= 64, "key masks are 64 bits");
  using SMT = TopkSmemT<GVR ? kListCapG : kCandCap>;
  constexpr int U = SmemKeys<KPT>::kUnroll;
  constexpr int kCap = GVR ? kListCapG : kCandCap;
  constexpr int kSeg = kCap / CL;           // bin / window path: list capacity per CTA
  constexpr int kSlots = kCap / kThreads;   // bin / window path: list entries per thread
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SMT& sm = *reinterpret_cast<SMT*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int t = blockIdx.y;
  pdl_wait();
  const Row r = row_of(a, t, rank == 0 && tid == 0);
  if (r.c <= r.K) {  // (uniform over the cluster)
    dense_row<CL>(a, r, t, rank);
    return;
  }
  const int c = r.c, n = r.n;

  // ---- loads: this thread's KPT consecutive scores, then the prefix
  // histogram (8 bins per thread, from the top)
  const int first = (rank * kThreads + tid) * KPT;
  const float* row = a.scores + (size_t)t * a.score_stride;
  float sc[KPT];
#pragma unroll
  for (int j = 0; j < KPT; j += 4) {
    if (vec && first + j + 3 < c) {  // 16-byte aligned when the row stride is a multiple of 4
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + first + j));
      sc[j] = v.x;
      sc[j + 1] = v.y;
      sc[j + 2] = v.z;
      sc[j + 3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[j + e] = first + j + e < c ? __ldg(row + first + j + e) : 0.f;
    }
  }
  uint4 hv0 = make_uint4(0u, 0u, 0u, 0u), hv1 = hv0;
  if (!GVR && r.hrow) {
    hv0 = __ldcg(reinterpret_cast<const uint4*>(r.hrow + kPrefixBins - 8 - 8 * tid));
    hv1 = __ldcg(reinterpret_cast<const uint4*>(r.hrow + kPrefixBins - 4 - 8 * tid));
  }
  // self-sampling guess: sample i of ns is candidate i * c / ns -- the same
  // positions in every CTA of the cluster (every candidate when c <= kSampleN)
  const int ns = c < kSampleN ? c : kSampleN;
  float smp[kSampleN / kThreads];
  if constexpr (GVR) {
#pragma unroll
    for (int k = 0; k < kSampleN / kThreads; ++k) {
      const int i = tid + k * kThreads;
      smp[k] = i < ns ? __ldg(row + (int)(((long long)i * c) / ns)) : 0.f;
    }
  }

  // ---- the bin of the n-th largest key, from the histogram
  bool hist_ok = false;  // (the same in every CTA: they read the same histogram)
  uint32_t pb = 0;
  if (!GVR && r.hrow) {
    const uint32_t hb[8] = {hv1.w, hv1.z, hv1.y, hv1.x, hv0.w, hv0.z, hv0.y, hv0.x};
    int hs = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) hs += (int)hb[j];
    int htotal;
    const int hbefore = block_exclusive_scan(hs, sm.wa, htotal);
    if (htotal == c) {
      if (hbefore < n && hbefore + hs >= n) {
        int ab = hbefore;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (ab < n && ab + (int)hb[j] >= n) sm.pbin = kPrefixBins - 1 - 8 * tid - j;
          ab += (int)hb[j];
        }
      }
      __syncthreads();
      pb = (uint32_t)sm.pbin;
      hist_ok = true;
    }
  }

  uint32_t pb_lo = pb;  // the window of bins [pb_lo, pb] (one bin on the histogram path)
  if constexpr (GVR) {
    // ---- guess: a histogram of the sample's top 12 key bits (in hw, which
    // only this CTA writes: the cluster passes write the other CTAs' hall, and
    // a peer may start them before this CTA is done here); the window spans
    // the bins of the sample ranks n ns / c -+ (3 sigma + 1): the n-th largest key of the row
    // lies between them unless the sample is far off, which the exact counts
    // below catch
    uint32_t* sh = &sm.hw[0][0];
#pragma unroll
    for (int j = 0; j < 8; ++j) sh[8 * tid + j] = 0u;
    if (tid == 0) {
      sm.pbin = kPrefixBins - 1;
      sm.pbin_lo = 0;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kSampleN / kThreads; ++k)
      if (tid + k * kThreads < ns) atomicAdd(&sh[order_key(smp[k]) >> kPrefixShift], 1u);
    __syncthreads();
    uint32_t hb[8];
    int hs = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      hb[j] = sh[kPrefixBins - 1 - 8 * tid - j];
      hs += (int)hb[j];
    }
    int htotal;
    const int hbefore = block_exclusive_scan(hs, sm.wa, htotal);
    const float e = (float)n * (float)ns / (float)c, sd = sqrtf(e);
    const int r_hi = max(1, (int)floorf(e - 3.f * sd - 1.f));
    const int r_lo = min(ns, (int)ceilf(e + 3.f * sd + 1.f));
    int ab = hbefore;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int b = kPrefixBins - 1 - 8 * tid - j;
      if (ab < r_hi && ab + (int)hb[j] >= r_hi) sm.pbin = b;
      if (ab < r_lo && ab + (int)hb[j] >= r_lo) sm.pbin_lo = b;
      ab += (int)hb[j];
    }
    __syncthreads();
    pb = (uint32_t)sm.pbin;
    pb_lo = (uint32_t)sm.pbin_lo;
    hist_ok = pb - pb_lo < (uint32_t)kBins;  // the exact bin is then found with one 256-bin pass
  }

  // ---- keys into shared memory; on the histogram (or window) path, which of
  // them lie above the bin (kept for sure) and in it (the candidates)
  SmemKeys<KPT> keys{reinterpret_cast<uint32_t*>(smem_raw + sizeof(SMT)) + tid};
  uint64_t above_mask = 0, cand_mask = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const bool valid = first + j < c;
    const uint32_t k = valid ? order_key(sc[j]) : 0u;
    keys.set(j, k);
    if (valid && (k >> kPrefixShift) > pb) above_mask |= 1ull << j;
    if constexpr (GVR) {
      if (valid && (k >> kPrefixShift) <= pb && (k >> kPrefixShift) >= pb_lo) cand_mask |= 1ull << j;
    } else {
      if (valid && (k >> kPrefixShift) == pb) cand_mask |= 1ull << j;
    }
  }

  uint32_t prefix = 0;
  int need = n;    // how many keys matching `prefix` are still to be taken
  int mode = 0;    // how tau was found: 0 four cluster passes, 1 two passes and
                   // the gathered candidates, 2 the prefix histogram
  int ncand = 0;

  if (hist_ok) {
    // this CTA's candidates are listed (with their ids) in its own shared
    // memory; its counts in and above the bin go to every CTA
    const int mine = __popcll((long long)cand_mask), above_pb = __popcll((long long)above_mask);
    int cta2;  // one scan: candidates (low 16 bits), keys above the bin (high)
    int pos = block_exclusive_scan(mine | (above_pb << 16), sm.wa, cta2) & 0xffff;
    for (uint64_t m = cand_mask; m; m &= m - 1) {
      const int j = __ffsll((long long)m) - 1;
      if (pos < kSeg) sm.cand[pos] = make_uint2(keys.get(j), (uint32_t)(first + j));
      ++pos;
    }
    if (tid < CL) {  // thread q tells CTA q
      *cl.map_shared_rank(&sm.scnt[rank], tid) = cta2 & 0xffff;
      *cl.map_shared_rank(&sm.sgt[rank], tid) = cta2 >> 16;
    }
    if (tid < kBins) {
      sm.hw[0][tid] = 0u;
      sm.hw[1][tid] = 0u;
      sm.hw[2][tid] = 0u;
    }
    if (tid < 2 * kMaxCL) sm.ccnt[tid] = 0;
    if (tid == 0) sm.nfin = 0;
    csync<CL>();  // lists and counts complete; every CTA has read the histogram
    // (the histogram is zeroed below while the DSMEM pulls are in flight, or in cluster pass 0)
    // the histogram's bin is taken only when the exact counts confirm it
    int in_bin = 0, above_bin = 0;
    bool over = false;
#pragma unroll
    for (int q = 0; q < CL; ++q) {
      in_bin += sm.scnt[q];
      above_bin += sm.sgt[q];
      over |= sm.scnt[q] > kSeg;
    }
    if (!over && above_bin < n && above_bin + in_bin >= n) {
      mode = 2;
      need = n - above_bin;
      // ---- pull every CTA's list into registers (independent DSMEM loads):
      // slot s of thread tid is entry (tid + s*kThreads) % kSeg of CTA
      // (tid + s*kThreads) / kSeg; then release the lists for their CTAs' exit
      uint2 ck[kSlots];
      uint32_t valid = 0;
#pragma unroll
      for (int s = 0; s < kSlots; ++s) {
        const int e = tid + s * kThreads, q = e / kSeg, i = e % kSeg;
        ck[s] = make_uint2(0u, 0u);
        if (i < sm.scnt[q]) {
          ck[s] = *cl.map_shared_rank(&sm.cand[i], q);
          valid |= 1u << s;
        }
      }
      if (r.hrow) zero_hist_share<CL>(r.hrow, rank);
      asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
      const uint32_t valid_all = valid;  // every listed candidate (the per-CTA counts below)
      if (GVR && pb != pb_lo) {
        // ---- the window: the exact 12-bit bin of the need-th largest among
        // its candidates; only those in that bin go on to the digit passes.
        // The candidates crowd into a few bins: per-warp histograms (in hall,
        // which no peer writes on this path) keep the atomics apart
        uint32_t* const hflat = &sm.hall[0][0][0];   // [kWarps][kBins] of the [4][kMaxCL][kBins] array
        uint32_t* wh = hflat + warp * kBins;
#pragma unroll
        for (int b = lane; b < kBins; b += 32) wh[b] = 0u;
        __syncwarp();
#pragma unroll
        for (int s = 0; s < kSlots; ++s)
          if ((valid >> s) & 1u) atomicAdd(&wh[(ck[s].x >> kPrefixShift) - pb_lo], 1u);
        __syncthreads();
        if (tid < kBins) {
          int h = 0;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) h += (int)hflat[w * kBins + kBins - 1 - tid];
          find_bin(h, need, kBins - 1 - tid, &sm.bin[3], &sm.above[3], sm.wa);
        }
        __syncthreads();
        pb = pb_lo + (uint32_t)sm.bin[3];
        need -= sm.above[3];
#pragma unroll
        for (int s = 0; s < kSlots; ++s)
          if ((ck[s].x >> kPrefixShift) != pb) valid &= ~(1u << s);
      }
      prefix = pb << kPrefixShift;
      // ---- key bits 12..19 over the candidates
#pragma unroll
      for (int s = 0; s < kSlots; ++s)
        if ((valid >> s) & 1u) atomicAdd(&sm.hw[0][(ck[s].x >> 12) & 255u], 1u);
      __syncthreads();
      if (tid < kBins)
        find_bin((int)sm.hw[0][kBins - 1 - tid], need, kBins - 1 - tid, &sm.bin[0], &sm.above[0], sm.wa);
      __syncthreads();
      prefix |= (uint32_t)sm.bin[0] << 12;
      need -= sm.above[0];
      const int m20 = (int)sm.hw[0][sm.bin[0]];  // candidates matching the 20-bit prefix
      if (m20 <= kRankCap) {
        // ---- those few, gathered, are ranked directly under (key desc, id
        // asc): the one of rank need-1 is tau
#pragma unroll
        for (int s = 0; s < kSlots; ++s)
          if (((valid >> s) & 1u) && (ck[s].x >> 12) == (prefix >> 12)) sm.fin[atomicAdd(&sm.nfin, 1)] = ck[s];
        __syncthreads();
        if (tid < m20) {
          const uint2 me = sm.fin[tid];
          int rk = 0, r_key = 0;  // rank, and candidates with a larger key
          for (int i = 0; i < m20; ++i) {
            const uint2 o = sm.fin[i];
            rk += o.x > me.x || (o.x == me.x && o.y < me.y);
            r_key += o.x > me.x;
          }
          if (rk == need - 1) {
            sm.tau = me.x;
            sm.above[2] = r_key;
          }
        }
        __syncthreads();
        prefix = sm.tau;
        need -= sm.above[2];
      } else {
        // ---- many ties in the bin: key bits 4..11, then 0..3
#pragma unroll 1
        for (int L = 1; L < 3; ++L) {
          const int shift = L == 1 ? 4 : 0, hi = L == 1 ? 12 : 4;
          const uint32_t dmask = L == 2 ? 15u : 255u;
#pragma unroll
          for (int s = 0; s < kSlots; ++s)
            if (((valid >> s) & 1u) && (ck[s].x >> hi) == (prefix >> hi))
              atomicAdd(&sm.hw[L][(ck[s].x >> shift) & dmask], 1u);
          __syncthreads();
          if (tid < kBins)
            find_bin((int)sm.hw[L][kBins - 1 - tid], need, kBins - 1 - tid, &sm.bin[L], &sm.above[L], sm.wa);
          __syncthreads();
          prefix |= (uint32_t)sm.bin[L] << shift;
          need -= sm.above[L];
        }
      }
      // per source CTA: candidates above and equal to tau
#pragma unroll
      for (int s = 0; s < kSlots; ++s) {
        if ((valid_all >> s) & 1u) {
          const int q = (tid + s * kThreads) / kSeg;
          if (ck[s].x > prefix) atomicAdd(&sm.ccnt[q], 1);
          else if (ck[s].x == prefix) atomicAdd(&sm.ccnt[kMaxCL + q], 1);
        }
      }
    }
  }

  if (mode != 2) {
    // ---- cluster passes of 8 bits from the top.  After two, the keys that
    // still match (the candidates) are usually a few dozen; then every CTA
    // receives all of them and finishes the last two digits on its own.
    mode = 0;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
#pragma unroll
      for (int b = lane; b < kBins; b += 32) sm.hw[warp][b] = 0u;
      __syncwarp();
#pragma unroll U
      for (int j = 0; j < KPT; ++j) {
        const uint32_t k = keys.get(j);
        const bool match = pass == 0 ? k != 0u : (k >> (shift + 8)) == (prefix >> (shift + 8));
        if (match) atomicAdd(&sm.hw[warp][(k >> shift) & (kBins - 1)], 1u);
      }
      __syncthreads();
      if (tid < kBins) {
        uint32_t v = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += sm.hw[w][tid];
#pragma unroll
        for (int q = 0; q < CL; ++q) cl.map_shared_rank(&sm.hall[pass][rank][tid], q)[0] = v;
      }
      csync<CL>();  // every CTA's counts are in every CTA's table
      if (pass == 0 && r.hrow && mode != 2) zero_hist_share<CL>(r.hrow, rank);
      if (tid < kBins) {
        int h = 0;
#pragma unroll
        for (int q = 0; q < CL; ++q) h += (int)sm.hall[pass][q][kBins - 1 - tid];
        find_bin(h, need, kBins - 1 - tid, &sm.bin[pass], &sm.above[pass], sm.wa);
      }
      __syncthreads();
      prefix |= (uint32_t)sm.bin[pass] << shift;
      need -= sm.above[pass];
      if (pass == 1) {
        int total = 0;
#pragma unroll
        for (int q = 0; q < CL; ++q) total += (int)sm.hall[1][q][sm.bin[1]];
        if (total <= kCandCap) {  // the same decision in every CTA
          mode = 1;
          ncand = total;
          break;
        }
      }
    }
  }

  if (mode == 1) {
    // ---- candidates: every CTA writes its keys matching the 16-bit prefix,
    // with their ids, into every CTA's list (CTA q's block starts after the
    // candidates of CTAs 0 .. q-1, whose counts pass 1's table holds)
    int mine = 0;
#pragma unroll U
    for (int j = 0; j < KPT; ++j) mine += (keys.get(j) >> 16) == (prefix >> 16);
    int cta_total;
    int pos = block_exclusive_scan(mine, sm.wa, cta_total);
#pragma unroll
    for (int q = 0; q < CL; ++q) pos += q < rank ? (int)sm.hall[1][q][sm.bin[1]] : 0;
    if (mine) {
#pragma unroll U
      for (int j = 0; j < KPT; ++j) {
        const uint32_t k = keys.get(j);
        if ((k >> 16) == (prefix >> 16)) {
          const uint2 e = make_uint2(k, (uint32_t)(first + j));
#pragma unroll
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
        int rk = 0, r_key = 0;  // rank, and candidates with a larger key
        for (int i = 0; i < ncand; ++i) {
          const uint2 o = sm.cand[i];
          rk += o.x > me.x || (o.x == me.x && o.y < me.y);
          r_key += o.x > me.x;
        }
        if (rk == need - 1) {
          sm.tau = me.x;
          sm.above[2] = r_key;  // candidates above tau
        }
      }
      __syncthreads();
      prefix = sm.tau;
      need -= sm.above[2];
    } else {
      // ---- the last two digits, over the candidates only
#pragma unroll 1
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

  // ---- keys above tau in each CTA, on the table paths: a key is above tau
  // when, in the first pass where its digit differs from tau's, its digit is
  // the larger one, and that pass's table counted it under that digit in its
  // CTA's slot (after two passes the candidate list counts the rest)
  if (mode != 2 && tid < kBins) {
    const int npass = mode == 1 ? 2 : 4;
    int x[CL];
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

  // ---- kept ids: all keys > tau, then the first `need` keys == tau by id.
  // This thread's counts: on the histogram path from its masks (the keys
  // above the bin, then its few candidates against tau), else from its keys.
  int gt = 0, eq = 0;
  if (mode == 2) {
    gt = __popcll((long long)above_mask);
    for (uint64_t m = cand_mask; m; m &= m - 1) {
      const uint32_t k = keys.get(__ffsll((long long)m) - 1);
      gt += k > tau;
      eq += k == tau;
    }
  } else {
    const int ge = count_vs<KPT>(keys, tau);
    gt = ge & 0xffff;
    eq = ge >> 16;
  }
  int both;  // per-CTA counts stay below 2^16
  const int before = block_exclusive_scan(gt | (eq << 16), sm.wa, both);  // syncs: wsum, ccnt visible
  // the CTAs before this one: lane q of every warp takes CTA q's counts, and a
  // warp prefix over q gives the offsets (no serial loop, no extra barrier)
  int gt_q = 0, eq_q = 0;
  if (lane < CL) {
    if (mode == 2) {  // keys above the bin, plus candidates above tau
      gt_q = sm.sgt[lane] + sm.ccnt[lane];
      eq_q = sm.ccnt[kMaxCL + lane];
    } else {
      gt_q = mode == 1 ? sm.ccnt[lane] : 0;
#pragma unroll
      for (int w = 0; w < kBins / 32; ++w) gt_q += sm.wsum[w][lane];
      eq_q = mode == 1 ? sm.ccnt[kMaxCL + lane] : (int)sm.hall[3][lane][sm.bin[3]];
    }
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
  const int off = __shfl_sync(0xffffffffu, kept_q, 0);
  const int eq_prev = __shfl_sync(0xffffffffu, eq_before_q, rank);
  int rem = need - eq_prev;  // tau-keys still to take at this CTA's start
  rem = rem < 0 ? 0 : rem;
  if (mode == 2)
    emit_kept<KPT, true>(sm, keys, above_mask, cand_mask, first, tau, gt, before & 0xffff, before >> 16,
                         both & 0xffff, both >> 16, rem, off, r, tvec);
  else
    emit_kept<KPT, false>(sm, keys, 0, 0, first, tau, gt, before & 0xffff, before >> 16, both & 0xffff,
                          both >> 16, rem, off, r, tvec);
  if (rank == 0) write_tail(a, r, t);
  if (GVR && rank == 0 && tid == 0 && a.path) a.path[t] = mode == 2 ? 1 : 3;
  // the other CTAs read this CTA's candidate list: stay until they have
  if (mode == 2) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int CL, int KPT>
cudaError_t launch_cfg(const TopkArgs& a, cudaStream_t s) {
  static_assert(CL >= 1, "cluster size");
  const int vec = (a.score_stride % 4 == 0) && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0;
  const int tvec = a.tok && a.W % 4 == 0 && (reinterpret_cast<uintptr_t>(a.tok) & 15u) == 0;
  if constexpr (CL == 1) {
    const size_t smem = a.gvr ? sizeof(TopkSmemG) : sizeof(TopkSmem);
    auto kern = a.gvr ? topk_row_kernel<KPT, true> : topk_row_kernel<KPT, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(1, a.T), dim3(kThreads), smem, s, 1, a, vec, tvec);
  } else {
    auto go = [&](auto kern, size_t base) -> cudaError_t {
      const size_t smem = base + (size_t)KPT * kThreads * sizeof(uint32_t);
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      return launch_k(kern, dim3(CL, a.T), dim3(kThreads), smem, s, CL, a, vec, tvec);
    };
    return a.gvr ? go(topk_cluster_kernel<CL, KPT, true>, sizeof(TopkSmemG))
                 : go(topk_cluster_kernel<CL, KPT, false>, sizeof(TopkSmem));
  }
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

bool topk_gvr_budget(int K) { return K == 512 || K == 1024 || K == 2048; }

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
