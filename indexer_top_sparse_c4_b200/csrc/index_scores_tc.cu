// index_scores_tc.cu -- stage 1 of QSA for prefill chunks on the 5th-generation
// tensor cores.  "Qwen3.8-27B QSA - BF16 source weights", "QSA in brief": a
// learned compressed indexer scores every 4-token group for every query; with
// thousands of queries of one request the pass is a dense contraction
//   acc_h[t, g] = q_I[t,h,:] . khat[g,:]     (M = queries, N = groups, K = D_I)
// for each indexer head h, followed by  s[t,g] = sum_h w[t,h] * ReLU(acc_h[t,g]).
//
// sm_100a design (BF16 indexer query and keys, H_I = 4, D_I = 128):
//  * tile: M = 128 queries (one TMEM lane each), N = 64 groups (4 pages of 16),
//    K = 128; per N tile 4 heads x 8 tcgen05.mma kind::f16 (K = 16), head h
//    accumulating into its own 64 TMEM columns, so a thread of the epilogue
//    holds all four heads of its query and the head sum needs no shuffles;
//  * one persistent CTA per SM with warp roles: warp 0 issues TMA loads (the
//    query tile once per M tile, 128 KiB; a ring of key tiles, each page of
//    16 keys fetched through the page table as two SWIZZLE_128B boxes), warp
//    1 owns TMEM and issues the MMAs (one elected thread), warps 2..9 read the
//    FP32 accumulators (tcgen05.ld), apply ReLU * w_h, add the heads, stage the
//    32 x 32 score block of each warp in shared memory in the 128-byte swizzle
//    and write it with one TMA store;
//  * two accumulator sets (2 x 4 heads x 64 columns = all 512 TMEM columns)
//    so the epilogue of one N tile overlaps the MMAs of the next;
//  * the (M tile, N tile) space is cut into one contiguous range per CTA, so
//    every SM has work even when there are fewer M tiles than SMs;
//  * every mbarrier wait is bounded: on time-out the kernel sets
//    QSA_DEV_TIMEOUT, all roles stop, in-flight copies and MMAs are waited for
//    (with their own bound), and the CTA releases TMEM and exits.
// An M tile whose queries belong to several requests is processed once per
// run of consecutive queries of one request: every run gets the MMAs of all
// 128 rows against its own request's keys, and the epilogue keeps only the
// run's rows.  Scores of groups g >= c(p_t) inside a written tile are -inf.
#include <cuda.h>

#include "mbarrier.cuh"

namespace qsa {
namespace {

using namespace mbar;

constexpr int kQ = 128;                    // queries per M tile (TMEM lanes)
constexpr int kH = 4;                      // indexer heads
constexpr int kN = 64;                     // groups per N tile
constexpr int kNPages = kN / kPageGroups;  // 4 pages per N tile
constexpr int kDI = 128;                   // indexer head dim
constexpr int kKB = 2;                     // 64-column (128-byte) k-blocks per row
constexpr int kStages = 3;                 // key-tile ring depth
constexpr int kEpiWarps = 8;               // 2 per TMEM lane quarter, 32 columns each
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kABlock = kQ * 128;          // one head, one k-block: 16 KiB
constexpr int kABytes = kH * kKB * kABlock;
constexpr int kBBlock = kN * 128;          // one k-block of a key tile: 8 KiB
constexpr int kBBytes = kKB * kBBlock;
constexpr int kOutBytes = 32 * 32 * 4;     // a warp's 32 x 32 FP32 score block
constexpr uint32_t kAccCols = kH * kN;     // 256 columns per accumulator set
constexpr uint32_t kTmemCols = 2 * kAccCols;

struct TcSmem {
  alignas(1024) unsigned char a[kABytes];
  alignas(1024) unsigned char b[kStages][kBBytes];
  alignas(1024) unsigned char out[kEpiWarps][kOutBytes];
  alignas(8) uint64_t a_full, a_empty;
  uint64_t b_full[kStages], b_empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(saddr(dst)), "l"(map), "r"(saddr(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(map), "r"(saddr(src)), "r"(x), "r"(y)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// K-major SWIZZLE_128B UMMA shared-memory descriptor: 8-row atoms of 128-byte
// rows, atoms 1024 bytes apart (SBO), version 1 (sm_100), layout type 2.
__device__ __forceinline__ uint64_t umma_desc(uint32_t smem_byte_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_byte_addr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;              // LBO (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;    // SBO
  d |= (uint64_t)1 << 46;              // version
  d |= (uint64_t)2 << 61;              // SWIZZLE_128B
  return d;
}

// kind::f16 instruction descriptor: F32 accumulate, BF16 A and B, both K-major,
// M = 128, N = 64.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                            ((uint32_t)(kQ >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(acc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(bar))
               : "memory");
}
// 16 consecutive FP32 columns of this thread's TMEM lane (completion awaited
// separately with tcgen05.wait::ld).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ int cand_count(const IndexArgs& a, int t) {
  const int p = a.q_pos[t];
  const int c = p >= 0 ? p / kGroupTokens : 0;
  return c < a.score_stride ? c : a.score_stride;
}

// A run: the rows [rb, re) of an M tile that belong to one request.  Every
// role derives the same runs, in the same order, from global memory (a whole
// warp calls this).
struct Run {
  int re, req, ntiles;
  bool bad;
};
__device__ __forceinline__ Run find_run(const IndexArgs& a, int t0, int nq, int rb) {
  const int lane = threadIdx.x & 31;
  Run r;
  r.req = a.q_req[t0 + rb];
  r.re = nq;
  for (int base = rb + 1; base < nq; base += 32) {
    const int row = base + lane;
    const unsigned m = __ballot_sync(0xffffffffu, row < nq && a.q_req[t0 + row] != r.req);
    if (m) {
      r.re = base + __ffs(m) - 1;
      break;
    }
  }
  int c = 0;
  for (int row = rb + lane; row < r.re; row += 32) c = max(c, cand_count(a, t0 + row));
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) c = max(c, __shfl_xor_sync(0xffffffffu, c, d));
  r.bad = r.req < 0 || r.req >= a.pt_rows;
  r.ntiles = (c + kN - 1) / kN;
  return r;
}

// The CTA's contiguous share [u0, u1) of the (M tile, N tile) space, walked
// one M tile at a time as segments [nt_lo, nt_hi) of that tile's N tiles.
struct Share {
  long long u, u1;
  int nmax;
  int mt, nt_lo, nt_hi;
  __device__ __forceinline__ bool next() {
    if (u >= u1) return false;
    mt = (int)(u / nmax);
    nt_lo = (int)(u % nmax);
    nt_hi = (int)min((long long)nmax, nt_lo + (u1 - u));
    u += nt_hi - nt_lo;
    return true;
  }
};
__device__ __forceinline__ Share my_share(const IndexArgs& a) {
  Share s;
  s.nmax = (a.score_stride + kN - 1) / kN;
  const long long total = (long long)((a.T + kQ - 1) / kQ) * s.nmax;
  s.u = total * blockIdx.x / gridDim.x;
  s.u1 = total * (blockIdx.x + 1) / gridDim.x;
  return s;
}

__global__ void __launch_bounds__(kThreads, 1)
    index_scores_tc_kernel(IndexArgs a, const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_s,
                           int tma_store) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>(
      smem_raw + ((1024 - ((uintptr_t)smem_raw & 1023)) & 1023));  // 1 KiB alignment for SWIZZLE_128B
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sm.a_full, 1);
    mbar_init(&sm.a_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.b_full[s], 1);
      mbar_init(&sm.b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.acc_full[s], 1);
      mbar_init(&sm.acc_empty[s], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // TMEM: two sets of four 64-column FP32 accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();
  pdl_launch_dependents();  // dependents wait for this grid's completion before reading scores
  Share sh = my_share(a);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // "empty" barriers are waited with the parity of their previous phase: the
    // first wait on a fresh barrier passes, later ones wait for the consumer
    uint32_t stage = 0, bphase = 0, a_empty_par = 1;
    bool a_armed = false;
    while (!*abort_flag && sh.next()) {
      const int t0 = sh.mt * kQ, nq = min(kQ, a.T - t0);
      bool a_loaded = false;
      for (int rb = 0; rb < nq && !*abort_flag;) {
        const Run run = find_run(a, t0, nq, rb);
        rb = run.re;
        const int hi = min(sh.nt_hi, run.ntiles);
        if (run.bad || sh.nt_lo >= hi) continue;
        if (!a_loaded) {
          // the whole warp waits; one lane issues
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.a_empty, a_empty_par, abort_flag, a.status));
          if (lane == 0) {
            if (ok) {
              mbar_arrive_tx(&sm.a_full, kABytes);
              for (int h = 0; h < kH; ++h)
                for (int kb = 0; kb < kKB; ++kb)
                  tma_load_2d(sm.a + (h * kKB + kb) * kABlock, &tmap_q, &sm.a_full, h * kDI + kb * 64, t0);
            }
          }
          if (!ok) break;
          a_armed = true;
          a_empty_par ^= 1;
          a_loaded = true;
        }
        const int32_t* pt = a.page_table + (size_t)run.req * a.pt_stride;
        for (int nt = sh.nt_lo; nt < hi; ++nt) {
          // lanes 0..3 look up the tile's 4 pages; an unusable page is pointed
          // past the end of the key tensor (TMA fills zeros; the epilogue writes -inf)
          int page = -1;
          if (lane < kNPages) {
            const int lp = nt * kNPages + lane;
            page = lp < a.pt_stride ? __ldg(pt + lp) : -1;
            if (page < 0 || page >= a.num_pages) page = a.num_pages;
          }
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.b_empty[stage], bphase ^ 1, abort_flag, a.status));
          if (!ok) break;
          if (lane == 0) mbar_arrive_tx(&sm.b_full[stage], kBBytes);
          __syncwarp();
          if (lane < kNPages) {
            for (int kb = 0; kb < kKB; ++kb)
              tma_load_2d(sm.b[stage] + kb * kBBlock + lane * kPageGroups * 128, &tmap_k, &sm.b_full[stage],
                          kb * 64, page * kPageGroups);
          }
          if (++stage == kStages) {
            stage = 0;
            bphase ^= 1;
          }
        }
      }
    }
    if (*abort_flag && lane == 0) {
      // The last armed phase of a_full has the parity a_empty_par now holds;
      // stages below `stage` were last armed in the current round (parity
      // bphase), the others in the previous round (or never: a wait on the
      // parity before a fresh barrier's first phase passes at once).
      if (a_armed) mbar_drain(&sm.a_full, a_empty_par);
      for (int s = 0; s < kStages; ++s) mbar_drain(&sm.b_full[s], s < (int)stage ? bphase : bphase ^ 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    uint32_t stage = 0, bphase = 0, aphase = 0, abuf = 0, accphase = 0;
    bool issued = false, ok = true;
    while (ok && !*abort_flag && sh.next()) {
      const int t0 = sh.mt * kQ, nq = min(kQ, a.T - t0);
      bool a_ready = false;
      for (int rb = 0; rb < nq && ok;) {
        const Run run = find_run(a, t0, nq, rb);
        rb = run.re;
        const int hi = min(sh.nt_hi, run.ntiles);
        if (run.bad || sh.nt_lo >= hi) continue;
        if (!a_ready) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.a_full, aphase, abort_flag, a.status));
          if (!ok) break;
          aphase ^= 1;
          a_ready = true;
        }
        for (int nt = sh.nt_lo; nt < hi; ++nt) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_empty[abuf], accphase ^ 1, abort_flag, a.status) &&
                                           mbar_wait(&sm.b_full[stage], bphase, abort_flag, a.status));
          if (lane == 0) {
            if (ok) {
              asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
              const uint32_t bbase = saddr(sm.b[stage]);
              const uint32_t abase = saddr(sm.a);
#pragma unroll
              for (int h = 0; h < kH; ++h) {
                const uint32_t d = tmem + abuf * kAccCols + h * kN;
#pragma unroll
                for (int kb = 0; kb < kKB; ++kb) {
#pragma unroll
                  for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = umma_desc(abase + (h * kKB + kb) * kABlock + ks * 32);
                    const uint64_t bd = umma_desc(bbase + kb * kBBlock + ks * 32);
                    umma_bf16(d, ad, bd, (kb | ks) != 0);
                  }
                }
              }
              umma_commit(&sm.b_empty[stage]);  // the key stage is free once these MMAs finish
              umma_commit(&sm.acc_full[abuf]);  // the accumulator set is ready
              issued = true;
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (++stage == kStages) {
            stage = 0;
            bphase ^= 1;
          }
          if (++abuf == 2) {
            abuf = 0;
            accphase ^= 1;
          }
        }
      }
      if (ok && a_ready && lane == 0) umma_commit(&sm.a_empty);  // A may be replaced once these MMAs finish
    }
    if (*abort_flag && lane == 0 && issued) {
      umma_commit(&sm.drain);  // arrives once every MMA this thread issued is done
      mbar_drain(&sm.drain, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int ew = warp - 2;
    const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
    const int half = ew >> 2;                      // columns 32*half .. +31 of an N tile
    const int row = 32 * quarter + lane;           // accumulator row = query of the tile
    unsigned char* stage_out = sm.out[ew];
    const uint32_t sbase = saddr(stage_out) + lane * 128;
    uint32_t abuf = 0, accphase = 0;
    bool store_pending = false, ok = true;
    while (ok && !*abort_flag && sh.next()) {
      const int t0 = sh.mt * kQ, nq = min(kQ, a.T - t0);
      for (int rb = 0; rb < nq && ok;) {
        const int run_b = rb;
        const Run run = find_run(a, t0, nq, rb);
        rb = run.re;
        const int hi = min(sh.nt_hi, run.ntiles);
        if (sh.nt_lo >= hi) continue;
        const bool live = row >= run_b && row < run.re;  // row < re <= nq
        const int t = t0 + (live ? row : run_b);
        int c = 0;
        float w[kH] = {0.f, 0.f, 0.f, 0.f};
        if (live) {
          c = cand_count(a, t);
          if (sh.nt_lo == 0 && half == 0 && a.q_pos[t] / kGroupTokens > a.score_stride)
            flag(a.status, QSA_DEV_ROW_RANGE);
          const float4 wv = __ldg(reinterpret_cast<const float4*>(a.w_idx) + t);
          w[0] = wv.x, w[1] = wv.y, w[2] = wv.z, w[3] = wv.w;
        }
        if (run.bad) {  // no keys to read: every candidate of the run's rows is -inf
          if (live) {
            float* srow = a.scores + (size_t)t * a.score_stride;
            for (int nt = sh.nt_lo; nt < hi; ++nt)
              for (int j = 0; j < 32; ++j) {
                const int g = nt * kN + half * 32 + j;
                if (g < c) srow[g] = -INFINITY;
              }
            if (half == 0 && sh.nt_lo * kN < c) flag(a.status, QSA_DEV_BAD_REQUEST);
          }
          continue;
        }
        // the TMA store writes all 32 rows of the warp's block: only when they
        // all belong to this run (rows past the last query are clipped)
        const bool whole =
            tma_store && run_b <= 32 * quarter && (run.re >= 32 * quarter + 32 || run.re == nq);
        const int32_t* pt = a.page_table + (size_t)run.req * a.pt_stride;
        for (int nt = sh.nt_lo; nt < hi; ++nt) {
          const int g0 = nt * kN + half * 32;
          // the two pages of this warp's 32 columns
          const int lp = nt * kNPages + half * 2 + (lane & 1);
          const int pg = lp < a.pt_stride ? __ldg(pt + lp) : -1;
          const unsigned bad2 = __ballot_sync(0xffffffffu, pg < 0 || pg >= a.num_pages) & 3u;
          // when every row's candidates reach past these columns, no mask is needed
          const bool unmasked = __all_sync(0xffffffffu, !live || g0 + 32 <= c);
          ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full[abuf], accphase, abort_flag, a.status));
          if (!ok) break;
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          // the previous TMA store must have read the staging block
          if (store_pending) {
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();
            store_pending = false;
          }
          const uint32_t tbase = tmem + ((uint32_t)(32 * quarter) << 16) + abuf * kAccCols + half * 32;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t r[kH][16];
#pragma unroll
            for (int h = 0; h < kH; ++h) tmem_ld16(tbase + h * kN + ch * 16, r[h]);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            float s[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float x = w[0] * fmaxf(__uint_as_float(r[0][j]), 0.f);
              x = fmaf(w[1], fmaxf(__uint_as_float(r[1][j]), 0.f), x);
              x = fmaf(w[2], fmaxf(__uint_as_float(r[2][j]), 0.f), x);
              s[j] = fmaf(w[3], fmaxf(__uint_as_float(r[3][j]), 0.f), x);
            }
            if (!unmasked) {
#pragma unroll
              for (int j = 0; j < 16; ++j) s[j] = g0 + ch * 16 + j < c ? s[j] : -INFINITY;
            }
            if (bad2 & (1u << ch)) {  // these 16 columns are an unusable page
#pragma unroll
              for (int j = 0; j < 16; ++j) s[j] = -INFINITY;
            }
            // 128-byte swizzle: 16-byte chunk k of row `lane` sits at chunk k ^ (lane & 7)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              st_shared_v4(sbase + (((ch * 4 + k) ^ (lane & 7)) << 4), s[4 * k], s[4 * k + 1], s[4 * k + 2],
                           s[4 * k + 3]);
          }
          asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.acc_empty[abuf]);
          if (live && (((bad2 & 1u) && g0 < c) || ((bad2 & 2u) && g0 + kPageGroups < c)))
            flag(a.status, QSA_DEV_BAD_PAGE);
          if (whole) {
            // (a block wholly past the last query or the last column is skipped)
            if (32 * quarter < nq && g0 < a.score_stride) {
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              __syncwarp();
              if (lane == 0) tma_store_2d(&tmap_s, stage_out, g0, t0 + 32 * quarter);
              store_pending = true;
            }
          } else {
            // rows of other runs share the block: write this run's rows one by one
            __syncwarp();
            const int g = g0 + lane;
            for (int rr = 0; rr < 32; ++rr) {
              const int rrow = 32 * quarter + rr;
              if (rrow < run_b || rrow >= run.re) continue;  // warp-uniform
              const float v = *reinterpret_cast<const float*>(stage_out + rr * 128 +
                                                              (((lane >> 2) ^ (rr & 7)) << 4) + (lane & 3) * 4);
              if (g < a.score_stride) a.scores[(size_t)(t0 + rrow) * a.score_stride + g] = v;
            }
            __syncwarp();
          }
          if (++abuf == 2) {
            abuf = 0;
            accphase ^= 1;
          }
        }
      }
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  // ---- teardown: every role is done issuing; release TMEM
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over a row-major [rows, cols] array, SWIZZLE_128B, box
// (box_cols x box_rows) with box_cols x element size = 128 bytes.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool index_tc_supported(const IndexArgs& a) {
  // without q_req every query is its own request (one-row runs): the
  // streaming scan's shape, not this kernel's
  return a.q_dt == QSA_BF16 && a.k_dt == QSA_BF16 && a.H_I == kH && a.D_I == kDI && a.q_req != nullptr &&
         a.T >= 1 && (reinterpret_cast<uintptr_t>(a.w_idx) & 15u) == 0 && encode_fn() != nullptr;
}

cudaError_t launch_index_scores_tc(const IndexArgs& a, cudaStream_t s) {
  CUtensorMap mq, mk, ms;
  if (!make_map(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.q_idx, kH * kDI, (uint64_t)a.T, 64, kQ) ||
      !make_map(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.k_idx_pages, kDI, (uint64_t)a.num_pages * kPageGroups,
                64, kPageGroups))
    return cudaErrorInvalidValue;
  // the score blocks go out by TMA when every row starts on 16 bytes
  int tma_store = (a.score_stride % 4 == 0) && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0;
  if (tma_store)
    tma_store = make_map(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.scores, (uint64_t)a.score_stride,
                         (uint64_t)a.T, 32, 32);
  if (!tma_store) ms = mq;  // not read by the kernel
  const size_t smem = sizeof(TcSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(index_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = (long long)((a.T + kQ - 1) / kQ) * ((a.score_stride + kN - 1) / kN);
  const int grid = units < sms ? (int)units : sms;
  return launch_k(index_scores_tc_kernel, dim3(grid), dim3(kThreads), smem, s, 1, a, mq, mk, ms, tma_store);
}

}  // namespace qsa
