// index_scores_tc.cu -- stage 1 of QSA for prefill chunks on the 5th-generation
// tensor cores.  "Qwen3.8-27B QSA - BF16 source weights", "QSA in brief": a
// learned compressed indexer scores every 4-token group for every query; with
// thousands of queries of one request the pass is a dense contraction
//   acc[(t,h), g] = q_I[t,h,:] . khat[g,:]   (M = 4 T, N = groups, K = D_I)
// followed by  s[t,g] = sum_h w[t,h] * ReLU(acc[(t,h), g]).
//
// sm_100a design (BF16 indexer query and keys, H_I = 4, D_I = 128):
//  * tile: M = 128 rows = 32 queries x 4 heads (row 4q + h), N = 128 groups
//    (8 pages of 16 groups), K = 128 = 8 x tcgen05.mma kind::f16 (K = 16);
//  * a persistent CTA per SM with warp roles: warp 0 issues TMA loads (one A
//    tile per 32 queries; a 4-stage ring of B tiles, each page of 16 keys
//    fetched through the page table as two 64-column SWIZZLE_128B boxes),
//    warp 1 owns TMEM and issues the MMAs (one elected thread), warps 2..5
//    read the FP32 accumulator from TMEM (tcgen05.ld), apply ReLU * w_h, add
//    the four heads of a query across a lane quad and store the scores;
//  * two 128-column accumulators in TMEM so the epilogue of one tile overlaps
//    the MMAs of the next;
//  * every mbarrier wait is bounded: on time-out the kernel sets
//    QSA_DEV_TIMEOUT, all roles stop, and the CTA releases TMEM and exits.
// A tile whose 32 queries do not all belong to one request cannot share its
// key tiles; its scores are computed by the epilogue warps on CUDA cores.
#include <cuda.h>

#include "qsa_internal.cuh"

namespace qsa {
namespace {

constexpr int kQ = 32;             // queries per M tile
constexpr int kM = 128;            // rows per M tile (kQ x 4 heads)
constexpr int kN = 128;            // groups per N tile
constexpr int kNPages = kN / kPageGroups;  // 8 pages per N tile
constexpr int kDI = 128;           // indexer head dim
constexpr int kKB = 2;             // 64-column (128-byte) k-blocks per row
constexpr int kStages = 4;         // B ring depth
constexpr int kThreads = 192;      // 6 warps
constexpr int kABytes = kKB * kM * 128;   // 32 KiB
constexpr int kBBytes = kKB * kN * 128;   // 32 KiB
constexpr uint32_t kTmemCols = 256;       // two 128-column accumulators
constexpr unsigned long long kWaitLimitNs = 200ull * 1000 * 1000;  // 200 ms per wait

struct TcSmem {
  alignas(1024) unsigned char a[kABytes];
  alignas(1024) unsigned char b[kStages][kBBytes];
  alignas(8) uint64_t a_full, a_empty;
  uint64_t b_full[kStages], b_empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity; false (and the abort flag
// set, QSA_DEV_TIMEOUT raised) when it does not come.
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  const unsigned long long t0 = gtimer();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(b, parity)) return true;
    if (*abort_flag) return false;
    if ((i & 255u) == 255u && gtimer() - t0 > kWaitLimitNs) break;
  }
  *abort_flag = 1;
  flag(status, QSA_DEV_TIMEOUT);
  return false;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(saddr(dst)), "l"(map), "r"(saddr(bar)), "r"(x), "r"(y)
      : "memory");
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

// kind::f16 instruction descriptor: F32 accumulate, BF16 A and B, both K-major.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                            ((uint32_t)(kM >> 4) << 24);

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
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Per M tile facts every role derives identically from global memory.
struct TileInfo {
  int t0, nq, req, ntiles;
  bool mixed;
};
__device__ __forceinline__ TileInfo tile_info(const IndexArgs& a, int mt) {
  const int lane = threadIdx.x & 31;
  TileInfo ti;
  ti.t0 = mt * kQ;
  ti.nq = a.T - ti.t0 < kQ ? a.T - ti.t0 : kQ;
  const int t = ti.t0 + (lane < ti.nq ? lane : 0);
  const int r = a.q_req ? a.q_req[t] : t;
  int c = a.q_pos[t];
  c = c >= 0 ? c / kGroupTokens : 0;
  if (c > a.score_stride) c = a.score_stride;
  const int r0 = __shfl_sync(0xffffffffu, r, 0);
  ti.mixed = !__all_sync(0xffffffffu, r == r0) || r0 < 0 || r0 >= a.pt_rows;
  ti.req = r0;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) c = max(c, __shfl_xor_sync(0xffffffffu, c, d));
  ti.ntiles = ti.mixed ? 0 : (c + kN - 1) / kN;
  return ti;
}

__global__ void __launch_bounds__(kThreads, 1)
    index_scores_tc_kernel(IndexArgs a, const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>(
      smem_raw + ((1024 - ((uintptr_t)smem_raw & 1023)) & 1023));  // 1 KiB alignment for SWIZZLE_128B
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mtiles = (a.T + kQ - 1) / kQ;
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
      mbar_init(&sm.acc_empty[s], 4);  // one arrival per epilogue warp
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // TMEM: two 128-column FP32 accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // "empty" barriers are waited with the parity of their previous phase: the
    // first wait on a fresh barrier passes, later ones wait for the consumer
    uint32_t stage = 0, bphase = 0, a_empty_par = 1;
    for (int mt = blockIdx.x; mt < n_mtiles && !*abort_flag; mt += gridDim.x) {
      const TileInfo ti = tile_info(a, mt);
      if (ti.ntiles == 0) continue;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(&sm.a_empty, a_empty_par, abort_flag, a.status);
        if (ok) {
          mbar_arrive_tx(&sm.a_full, kABytes);
          for (int kb = 0; kb < kKB; ++kb)
            tma_load_2d(sm.a + kb * kM * 128, &tmap_q, &sm.a_full, kb * 64, ti.t0 * 4);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      a_empty_par ^= 1;
      const int32_t* pt = a.page_table + (size_t)ti.req * a.pt_stride;
      for (int nt = 0; nt < ti.ntiles && !*abort_flag; ++nt) {
        // lanes 0..7 look up the tile's 8 pages; an unusable page is pointed
        // past the end of the key tensor (TMA fills zeros; the epilogue writes -inf)
        int page = -1;
        if (lane < kNPages) {
          const int lp = nt * kNPages + lane;
          page = lp < a.pt_stride ? __ldg(pt + lp) : -1;
          if (page < 0 || page >= a.num_pages) page = a.num_pages;
        }
        if (lane == 0 && !mbar_wait(&sm.b_empty[stage], bphase ^ 1, abort_flag, a.status)) {}
        __syncwarp();
        if (*abort_flag) break;
        if (lane == 0) mbar_arrive_tx(&sm.b_full[stage], kBBytes);
        __syncwarp();
        if (lane < kNPages) {
          for (int kb = 0; kb < kKB; ++kb)
            tma_load_2d(sm.b[stage] + kb * kN * 128 + lane * kPageGroups * 128, &tmap_k, &sm.b_full[stage],
                        kb * 64, page * kPageGroups);
        }
        if (++stage == kStages) {
          stage = 0;
          bphase ^= 1;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    uint32_t stage = 0, bphase = 0, aphase = 0, abuf = 0, accphase = 0;
    for (int mt = blockIdx.x; mt < n_mtiles && !*abort_flag; mt += gridDim.x) {
      const TileInfo ti = tile_info(a, mt);
      if (ti.ntiles == 0) continue;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&sm.a_full, aphase, abort_flag, a.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      aphase ^= 1;
      for (int nt = 0; nt < ti.ntiles; ++nt) {
        if (lane == 0) {
          ok = mbar_wait(&sm.acc_empty[abuf], accphase ^ 1, abort_flag, a.status) &&
               mbar_wait(&sm.b_full[stage], bphase, abort_flag, a.status);
          if (ok) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t d = tmem + abuf * kN;
#pragma unroll
            for (int kb = 0; kb < kKB; ++kb) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = umma_desc(saddr(sm.a + kb * kM * 128) + ks * 32);
                const uint64_t bd = umma_desc(saddr(sm.b[stage] + kb * kN * 128) + ks * 32);
                umma_bf16(d, ad, bd, (kb | ks) != 0);
              }
            }
            umma_commit(&sm.b_empty[stage]);   // the B stage is free once these MMAs finish
            umma_commit(&sm.acc_full[abuf]);   // the accumulator is ready
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
      if (!ok) break;
      if (lane == 0) umma_commit(&sm.a_empty);  // A may be replaced once this tile's MMAs finish
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
    const int row = 32 * quarter + lane;        // accumulator row = 4 q + h
    const int ql = row >> 2, h = row & 3;
    uint32_t abuf = 0, accphase = 0;
    for (int mt = blockIdx.x; mt < n_mtiles && !*abort_flag; mt += gridDim.x) {
      const TileInfo ti = tile_info(a, mt);
      const int t = ti.t0 + ql;
      const bool live = ql < ti.nq;
      int c = 0;
      float wh = 0.f;
      if (live) {
        c = a.q_pos[t];
        c = c >= 0 ? c / kGroupTokens : 0;
        if (c > a.score_stride) c = a.score_stride;
        wh = __ldg(a.w_idx + (size_t)t * 4 + h);
      }
      float* srow = a.scores + (size_t)(live ? t : 0) * a.score_stride;
      if (ti.mixed) {
        // queries of several requests share this tile: score it on CUDA cores.
        // The loop runs to the warp's largest candidate count so that every
        // lane takes part in the head-sum shuffles.
        int cw = live ? c : 0;
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) cw = max(cw, __shfl_xor_sync(0xffffffffu, cw, d));
        const int r = live ? (a.q_req ? a.q_req[t] : t) : -1;
        const bool rok = r >= 0 && r < a.pt_rows;
        const __nv_bfloat16* qv = reinterpret_cast<const __nv_bfloat16*>(a.q_idx) + ((size_t)(live ? t : 0) * 4 + h) * kDI;
        const __nv_bfloat16* kp = reinterpret_cast<const __nv_bfloat16*>(a.k_idx_pages);
        const int32_t* prow = a.page_table + (size_t)(rok ? r : 0) * a.pt_stride;
        bool any_bad = false;
        for (int g = 0; g < cw; ++g) {
          float s = 0.f;
          bool bad = false;
          if (live && g < c) {
            const int lp = g / kPageGroups;
            const int page = (rok && lp < a.pt_stride) ? __ldg(prow + lp) : -1;
            if (page < 0 || page >= a.num_pages) {
              bad = true;
            } else {
              const __nv_bfloat16* kr = kp + ((size_t)page * kPageGroups + g % kPageGroups) * kDI;
              float dot = 0.f;
              for (int d = 0; d < kDI; ++d) dot = fmaf(__bfloat162float(qv[d]), __bfloat162float(kr[d]), dot);
              s = wh * fmaxf(dot, 0.f);
            }
          }
          s += __shfl_xor_sync(0xffffffffu, s, 1);  // the four heads: lanes 4q .. 4q+3
          s += __shfl_xor_sync(0xffffffffu, s, 2);
          if (h == 0 && live && g < c) srow[g] = bad ? -INFINITY : s;
          any_bad |= bad;
        }
        if (any_bad) flag(a.status, rok ? QSA_DEV_BAD_PAGE : QSA_DEV_BAD_REQUEST);
        continue;
      }
      const int32_t* pt = a.page_table + (size_t)ti.req * a.pt_stride;
      for (int nt = 0; nt < ti.ntiles; ++nt) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&sm.acc_full[abuf], accphase, abort_flag, a.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        float v[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + abuf * kN + 32 * ch, v[ch]);
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.acc_empty[abuf]);
        // groups of an unusable page score -inf
        const int mypage_lp = nt * kNPages + (lane & 7);
        int mypage = mypage_lp < a.pt_stride ? __ldg(pt + mypage_lp) : -1;
        const bool bad_page = mypage < 0 || mypage >= a.num_pages;
        const unsigned bad_mask = __ballot_sync(0xffffffffu, bad_page) & 0xFFu;
        bool wrote_bad = false;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float x = wh * fmaxf(v[ch][i], 0.f);
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            v[ch][i] = x;
          }
          // lane h of the quad stores columns 4j + h of this 32-column chunk
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int col = 32 * ch + 4 * j + h;
            const int g = nt * kN + col;
            if (live && g < c) {
              const bool bad = (bad_mask >> (col / kPageGroups)) & 1u;
              float x = v[ch][4 * j];
              if (h == 1) x = v[ch][4 * j + 1];
              if (h == 2) x = v[ch][4 * j + 2];
              if (h == 3) x = v[ch][4 * j + 3];
              srow[g] = bad ? -INFINITY : x;
              wrote_bad |= bad;
            }
          }
        }
        if (wrote_bad) flag(a.status, QSA_DEV_BAD_PAGE);
        if (++abuf == 2) {
          abuf = 0;
          accphase ^= 1;
        }
      }
    }
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

// 2-D BF16 map over [rows, 128] with a (64 columns x box_rows) SWIZZLE_128B box.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDI * 2};
  const cuuint32_t box[2] = {64u, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool index_tc_supported(const IndexArgs& a) {
  return a.q_dt == QSA_BF16 && a.k_dt == QSA_BF16 && a.H_I == 4 && a.D_I == kDI && a.T >= kQ &&
         encode_fn() != nullptr;
}

cudaError_t launch_index_scores_tc(const IndexArgs& a, cudaStream_t s) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, a.q_idx, (uint64_t)a.T * 4, kM) ||
      !make_map(&mk, a.k_idx_pages, (uint64_t)a.num_pages * kPageGroups, kPageGroups))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(TcSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(index_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_mtiles = (a.T + kQ - 1) / kQ;
  const int grid = n_mtiles < sms ? n_mtiles : sms;
  return launch_k(index_scores_tc_kernel, dim3(grid), dim3(kThreads), smem, s, 1, a, mq, mk);
}

}  // namespace qsa
