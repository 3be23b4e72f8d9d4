// indexer_write.cu -- the steps that produce stage 1's inputs: the indexer
// projection of the hidden states and the C4 compressed-key write
// ("Qwen3.8-27B QSA - BF16 source weights", "QSA in brief": a learned,
// compressed indexer over four-token blocks; "QSA HiSparse", entry-point
// table: the backend's prefill writes).
//
// Projection  y[t, n] = sum_h x[t, h] w[n, h]: the rows of w stack the
// indexer query heads, the head weights and the token key, so one call gives
// q_I, w and k of every token.
//  * decode (a handful of tokens): a GEMV that streams each row of w once
//    from HBM -- four rows per CTA with every 16-byte load of a chunk of the
//    row in flight at once, the tokens staged in shared memory by cp.async,
//    every token's dot product from the same loaded values;
//  * prefill (hundreds of tokens or more, BF16): a tcgen05 GEMM.  Tiles of
//    128 tokens x 128 rows of w x 64 (128 B, SWIZZLE_128B) arrive by TMA
//    through a 4-stage ring; one elected thread issues 128 x 128 x 16 MMAs
//    into one of two TMEM accumulators, so the epilogue of one tile overlaps
//    the MMAs of the next; four epilogue warps read the accumulators with
//    tcgen05.ld and store FP32 rows.  Every mbarrier wait is bounded.
//
// Compressed-key write  khat_g = W_phi [k_4g; k_4g+1; k_4g+2; k_4g+3] + b_phi
// for each completed group g, written to row g % 16 of page
// page_table[r][g / 16] (FP32 or BF16).  A CTA of 128 threads takes 16 groups:
// their token keys in shared memory, W_phi streamed through shared memory 64
// columns at a time (double-buffered, each column loaded once per CTA,
// coalesced), each thread accumulating a register tile of 4 groups x D_I / 32
// output dims in FP32.
#include "qsa_internal.cuh"
#include "umma.cuh"

namespace qsa {
namespace {

using namespace mbar;

// ---------------------------------------------------------------------------
// projection, decode form.  A CTA of 256 threads owns kGvRows rows of w and
// walks the hidden dimension in chunks: per chunk every thread issues all its
// 16-byte loads of w (one 8-column vector per row and per 256-vector stride)
// into registers, while cp.async stages the chunk of the (up to 8) tokens'
// hidden states in shared memory; one wait, then every loaded w value meets
// every token.  A warp's 32 partial sums (4 rows x 8 tokens) are reduced in
// 31 shuffles by a butterfly that halves the set each step, leaving lane L
// with the sum of value L; the 8 warps' sums meet in shared memory.

constexpr int kGvThreads = 256;
constexpr int kGvRows = 4;                      // rows of w per CTA
constexpr int kGvTok = 8;                       // tokens per pass
static_assert(kGvRows * kGvTok == 32, "one reduced value per lane");

template <typename T> struct RawVec8;           // 8 elements as raw 16-byte words
template <> struct RawVec8<__nv_bfloat16> { uint4 v; };
template <> struct RawVec8<float> { uint4 v[2]; };

template <typename T>
__device__ __forceinline__ RawVec8<T> ld_raw8(const T* p) {
  RawVec8<T> r;
  if constexpr (sizeof(T) == 2) {
    r.v = __ldg(reinterpret_cast<const uint4*>(p));
  } else {
    r.v[0] = __ldg(reinterpret_cast<const uint4*>(p));
    r.v[1] = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  }
  return r;
}
template <typename T>
__device__ __forceinline__ void unpack8(const RawVec8<T>& r, float (&o)[8]) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w[4] = {r.v.x, r.v.y, r.v.z, r.v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] = __uint_as_float(w[j] << 16);
      o[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      o[4 * h + 0] = __uint_as_float(r.v[h].x); o[4 * h + 1] = __uint_as_float(r.v[h].y);
      o[4 * h + 2] = __uint_as_float(r.v[h].z); o[4 * h + 3] = __uint_as_float(r.v[h].w);
    }
  }
}

__device__ __forceinline__ void cp_async16_g(void* smem, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr(smem)), "l"(g) : "memory");
}

// 8-column vectors of a row per thread per chunk: three for BF16 w, two for FP32
template <typename WT> __host__ __device__ constexpr int gv_jv() { return sizeof(WT) == 2 ? 3 : 2; }
template <typename WT> __host__ __device__ constexpr int gv_chunk() { return gv_jv<WT>() * 8 * kGvThreads; }

template <typename XT, typename WT>
__global__ void __launch_bounds__(kGvThreads, 2) project_gemv_kernel(ProjectArgs a) {
  constexpr int JV = gv_jv<WT>(), HC = gv_chunk<WT>();
  extern __shared__ __align__(16) unsigned char gv_smem[];
  XT* xs = reinterpret_cast<XT*>(gv_smem);                                 // [kGvTok][HC]
  float* red = reinterpret_cast<float*>(gv_smem + (size_t)kGvTok * HC * sizeof(XT));  // [8 warps][32]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kGvRows;
  const XT* x = reinterpret_cast<const XT*>(a.x);
  const WT* w = reinterpret_cast<const WT*>(a.w);
  pdl_wait();
  for (int t0 = 0; t0 < a.T; t0 += kGvTok) {
    const int nt = a.T - t0 < kGvTok ? a.T - t0 : kGvTok;
    float acc[kGvRows][kGvTok];
#pragma unroll
    for (int r = 0; r < kGvRows; ++r)
#pragma unroll
      for (int i = 0; i < kGvTok; ++i) acc[r][i] = 0.f;
    for (int c0 = 0; c0 < a.H; c0 += HC) {
      const int hc = a.H - c0 < HC ? a.H - c0 : HC;
      // this chunk's w vectors, all in flight
      RawVec8<WT> wr[kGvRows][JV];
#pragma unroll
      for (int r = 0; r < kGvRows; ++r)
#pragma unroll
        for (int j = 0; j < JV; ++j) {
          const int col = 8 * (tid + kGvThreads * j);
          if (n0 + r < a.N && col < hc) wr[r][j] = ld_raw8(w + (size_t)(n0 + r) * a.H + c0 + col);
          else wr[r][j] = RawVec8<WT>{};
        }
      // the tokens' chunk of x into shared memory
      constexpr int XV = 16 / sizeof(XT);        // elements per 16-byte copy
      const int per_row = hc / XV;
      for (int q = tid; q < nt * per_row; q += kGvThreads) {
        const int i = q / per_row, e = (q - i * per_row) * XV;
        cp_async16_g(xs + (size_t)i * HC + e, x + (size_t)(t0 + i) * a.H + c0 + e);
      }
      asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
      __syncthreads();
#pragma unroll
      for (int j = 0; j < JV; ++j) {
        const int col = 8 * (tid + kGvThreads * j);
        if (col < hc) {
          float wv[kGvRows][8];
#pragma unroll
          for (int r = 0; r < kGvRows; ++r) unpack8(wr[r][j], wv[r]);
#pragma unroll
          for (int i = 0; i < kGvTok; ++i) {
            if (i < nt) {
              float xv[8];
              if constexpr (sizeof(XT) == 2) {
                RawVec8<XT> xr;
                xr.v = *reinterpret_cast<const uint4*>(xs + (size_t)i * HC + col);
                unpack8(xr, xv);
              } else {
                const float4 p = *reinterpret_cast<const float4*>(xs + (size_t)i * HC + col);
                const float4 q = *reinterpret_cast<const float4*>(xs + (size_t)i * HC + col + 4);
                xv[0] = p.x; xv[1] = p.y; xv[2] = p.z; xv[3] = p.w;
                xv[4] = q.x; xv[5] = q.y; xv[6] = q.z; xv[7] = q.w;
              }
#pragma unroll
              for (int r = 0; r < kGvRows; ++r)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[r][i] = fmaf(xv[e], wv[r][e], acc[r][i]);
            }
          }
        }
      }
      __syncthreads();   // xs is free for the next chunk
    }
    // butterfly: value index r * 8 + i; after the step of width d a lane keeps
    // the upper half of its set when (lane & d) != 0, so lane L ends with value L
    float v[32];
#pragma unroll
    for (int r = 0; r < kGvRows; ++r)
#pragma unroll
      for (int i = 0; i < kGvTok; ++i) v[r * kGvTok + i] = acc[r][i];
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
      const bool up = (lane & d) != 0;
#pragma unroll
      for (int k = 0; k < d; ++k) {
        const float send = up ? v[k] : v[k + d];
        const float keep = up ? v[k + d] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, d);
      }
    }
    red[warp * 32 + lane] = v[0];
    __syncthreads();
    if (warp == 0) {
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < kGvThreads / 32; ++q) sum += red[q * 32 + lane];
      const int r = lane / kGvTok, i = lane % kGvTok;
      if (i < nt && n0 + r < a.N) a.y[(size_t)(t0 + i) * a.N + n0 + r] = sum;
    }
    __syncthreads();   // red is free for the next pass
  }
}

// ---------------------------------------------------------------------------
// projection, prefill form: tcgen05 GEMM

constexpr int kPM = 128;                      // tokens per tile (TMEM lanes)
constexpr int kPN = 128;                      // rows of w per tile (TMEM columns)
constexpr int kPStages = 4;                   // k-block ring depth
constexpr int kPEpiWarps = 4;
constexpr int kPThreads = 64 + 32 * kPEpiWarps;
constexpr int kPABytes = kPM * 128;           // one 64-column k-block of x: 16 KiB
constexpr int kPBBytes = kPN * 128;           // one k-block of w: 16 KiB
constexpr uint32_t kPTmemCols = 2 * kPN;      // two accumulators
constexpr uint32_t kPIdesc = umma::idesc_bf16(kPM, kPN);

struct ProjSmem {
  alignas(1024) unsigned char a[kPStages][kPABytes];
  alignas(1024) unsigned char b[kPStages][kPBBytes];
  alignas(8) uint64_t full[kPStages], empty[kPStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kPThreads, 1)
    project_tc_kernel(ProjectArgs a, const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mw) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ProjSmem& sm = *reinterpret_cast<ProjSmem*>(smem_raw + ((1024 - ((uintptr_t)smem_raw & 1023)) & 1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.acc_full[s], 1);
      mbar_init(&sm.acc_empty[s], kPEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&sm.tmem_base)),
                 "r"(kPTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();

  const int ntn = (a.N + kPN - 1) / kPN;
  const int total = ((a.T + kPM - 1) / kPM) * ntn;
  const int nkb = a.H / 64;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // "empty" barriers are waited with the parity of their previous phase: the
    // first wait on a fresh barrier passes, later ones wait for the MMAs
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < total && !*abort_flag; u += gridDim.x) {
      const int mt = u / ntn, nt = u % ntn;
      for (int kb = 0; kb < nkb; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.empty[stage], phase ^ 1, abort_flag, a.status));
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_tx(&sm.full[stage], kPABytes + kPBBytes);
          umma::tma_load_2d(sm.a[stage], &mx, &sm.full[stage], kb * 64, mt * kPM);
          umma::tma_load_2d(sm.b[stage], &mw, &sm.full[stage], kb * 64, nt * kPN);
        }
        __syncwarp();
        if (++stage == kPStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (*abort_flag && lane == 0) {
      // stages below `stage` were last armed in this round (parity `phase`),
      // the others in the previous one (or never: that wait passes at once)
      for (int s = 0; s < kPStages; ++s) mbar_drain(&sm.full[s], s < (int)stage ? phase : phase ^ 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    uint32_t stage = 0, phase = 0, abuf = 0, accphase = 0;
    bool ok = true, issued = false;
    for (int u = blockIdx.x; ok && u < total && !*abort_flag; u += gridDim.x) {
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_empty[abuf], accphase ^ 1, abort_flag, a.status));
      if (!ok) break;
      const uint32_t d = tmem + abuf * kPN;
      for (int kb = 0; kb < nkb; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[stage], phase, abort_flag, a.status));
        if (!ok) break;
        if (lane == 0) {
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t abase = saddr(sm.a[stage]), bbase = saddr(sm.b[stage]);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma::mma_bf16(d, umma::smem_desc(abase + ks * 32), umma::smem_desc(bbase + ks * 32), kPIdesc,
                           (kb | ks) != 0);
          umma::commit(&sm.empty[stage]);  // the stage is free once these MMAs finish
          issued = true;
        }
        __syncwarp();
        if (++stage == kPStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (lane == 0) umma::commit(&sm.acc_full[abuf]);  // the accumulator is complete
      __syncwarp();
      if (++abuf == 2) {
        abuf = 0;
        accphase ^= 1;
      }
    }
    if (*abort_flag && lane == 0 && issued) {
      umma::commit(&sm.drain);  // arrives once every MMA this thread issued is done
      mbar_drain(&sm.drain, 0);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31 (the warp's own quarter)
    const int row = 32 * quarter + lane;    // token row of the tile
    const bool vec = (a.N % 4) == 0 && (reinterpret_cast<uintptr_t>(a.y) & 15u) == 0;
    uint32_t abuf = 0, accphase = 0;
    for (int u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
      const int mt = u / ntn, nt = u % ntn;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full[abuf], accphase, abort_flag, a.status));
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int t = mt * kPM + row;
      float* yrow = a.y + (size_t)(t < a.T ? t : 0) * a.N;
      const uint32_t tbase = tmem + ((uint32_t)(32 * quarter) << 16) + abuf * kPN;
#pragma unroll 1
      for (int c = 0; c < kPN / 16; ++c) {
        uint32_t r[16];
        umma::tmem_ld16(tbase + c * 16, r);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const int n0 = nt * kPN + c * 16;
        if (t < a.T) {
          if (vec) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (n0 + 4 * q < a.N)
                *reinterpret_cast<float4*>(yrow + n0 + 4 * q) =
                    make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (n0 + j < a.N) yrow[n0 + j] = __uint_as_float(r[j]);
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[abuf]);
      if (++abuf == 2) {
        abuf = 0;
        accphase ^= 1;
      }
    }
  }

  // ---- teardown: every role is done issuing; release TMEM
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPTmemCols));
  }
}

// ---------------------------------------------------------------------------
// compressed-key write.  A CTA of 4 warps takes 16 groups; warp q computes
// groups 4q..4q+3 and lane l output dims l, l + 32, ... (D_I / 32 of them), so
// each thread holds a 4 x D_I/32 register tile.  The groups' concatenated
// token keys are staged in shared memory once (every lane of a warp reads the
// same key words: broadcasts); W_phi passes through shared memory in slabs
// of 64 columns, double-buffered by cp.async, rows padded to 68 floats so the
// lanes' 16-byte reads of 32 different rows fall on distinct banks.  Every
// output accumulates its 4 D_I products in column order.

constexpr int kCGroups = 16;                    // groups per CTA
constexpr int kCThreads = 128;
constexpr int kCSlab = 64;                      // columns of W_phi per slab
constexpr int kCRow = kCSlab + 4;               // padded slab row, floats

__device__ __forceinline__ void cp_async4_g(void* smem, const void* g) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(saddr(smem)), "l"(g) : "memory");
}

template <typename KT, int D>
__global__ void __launch_bounds__(kCThreads) compress_keys_kernel(CompressArgs c) {
  constexpr int W4 = kGroupTokens * D;          // columns of W_phi
  constexpr int DJ = D / 32;                    // output dims per lane
  constexpr int NSLAB = W4 / kCSlab;
  static_assert(W4 % kCSlab == 0, "whole slabs");
  extern __shared__ __align__(16) float cs[];
  float* kcat = cs;                                         // [kCGroups][W4]
  float* ws = cs + kCGroups * W4;                           // [2][D][kCRow]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = blockIdx.x * kCGroups;
  const int ng = c.n - i0 < kCGroups ? c.n - i0 : kCGroups;
  const bool w16 = (reinterpret_cast<uintptr_t>(c.wphi) & 15) == 0;
  const bool k16 = (reinterpret_cast<uintptr_t>(c.k_tok) & 15) == 0 && (c.tok_stride & 3) == 0;
  pdl_wait();
  auto stage_slab = [&](int sl) {
    float* dst = ws + (sl & 1) * D * kCRow;
    const float* src = c.wphi + sl * kCSlab;
    if (w16) {
      for (int q = tid; q < D * (kCSlab / 4); q += kCThreads) {
        const int r = q / (kCSlab / 4), e = 4 * (q % (kCSlab / 4));
        cp_async16_g(dst + r * kCRow + e, src + (size_t)r * W4 + e);
      }
    } else {
      for (int q = tid; q < D * kCSlab; q += kCThreads) {
        const int r = q / kCSlab, e = q % kCSlab;
        cp_async4_g(dst + r * kCRow + e, src + (size_t)r * W4 + e);
      }
    }
  };
  // the groups' keys: group g, token j, dim e at kcat[g][j * D + e]
  if (k16) {
    for (int q = tid; q < ng * (W4 / 4); q += kCThreads) {
      const int g = q / (W4 / 4), e = 4 * (q % (W4 / 4));
      cp_async16_g(kcat + g * W4 + e, c.k_tok + ((size_t)(i0 + g) * kGroupTokens + e / D) * c.tok_stride + e % D);
    }
  } else {
    for (int q = tid; q < ng * W4; q += kCThreads) {
      const int g = q / W4, e = q % W4;
      cp_async4_g(kcat + g * W4 + e, c.k_tok + ((size_t)(i0 + g) * kGroupTokens + e / D) * c.tok_stride + e % D);
    }
  }
  stage_slab(0);
  asm volatile("cp.async.commit_group;" ::: "memory");
  if (NSLAB > 1) stage_slab(1);
  asm volatile("cp.async.commit_group;" ::: "memory");

  float acc[4][DJ];
#pragma unroll
  for (int j = 0; j < DJ; ++j) {
    const float b = c.bias ? __ldg(c.bias + lane + 32 * j) : 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) acc[g][j] = b;
  }
  const float* kw = kcat + (4 * warp) * W4;
  for (int sl = 0; sl < NSLAB; ++sl) {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const float* wsl = ws + (sl & 1) * D * kCRow;
#pragma unroll 4
    for (int kk = 0; kk < kCSlab; kk += 4) {
      float4 wv[DJ], xv[4];
#pragma unroll
      for (int j = 0; j < DJ; ++j) wv[j] = *reinterpret_cast<const float4*>(wsl + (lane + 32 * j) * kCRow + kk);
#pragma unroll
      for (int g = 0; g < 4; ++g) xv[g] = *reinterpret_cast<const float4*>(kw + g * W4 + sl * kCSlab + kk);
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int j = 0; j < DJ; ++j) {
          acc[g][j] = fmaf(wv[j].x, xv[g].x, acc[g][j]);
          acc[g][j] = fmaf(wv[j].y, xv[g].y, acc[g][j]);
          acc[g][j] = fmaf(wv[j].z, xv[g].z, acc[g][j]);
          acc[g][j] = fmaf(wv[j].w, xv[g].w, acc[g][j]);
        }
    }
    __syncthreads();   // this slab's buffer is consumed
    if (sl + 2 < NSLAB) stage_slab(sl + 2);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  KT* out = reinterpret_cast<KT*>(c.k_idx_pages);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int gl = 4 * warp + g;
    if (gl >= ng) break;
    const int i = i0 + gl;
    const int r = c.g_req ? __ldg(c.g_req + i) : 0;
    const int gid = __ldg(c.g_id + i);
    if (r < 0 || r >= c.pt_rows) {
      if (lane == 0) flag(c.status, QSA_DEV_BAD_REQUEST);
      continue;
    }
    if (gid < 0 || gid / kPageGroups >= c.pt_stride) {
      if (lane == 0) flag(c.status, QSA_DEV_BAD_GROUP);
      continue;
    }
    const int page = __ldg(c.page_table + (size_t)r * c.pt_stride + gid / kPageGroups);
    if (page < 0 || page >= c.num_pages) {
      if (lane == 0) flag(c.status, QSA_DEV_BAD_PAGE);
      continue;
    }
    const size_t o = ((size_t)page * kPageGroups + gid % kPageGroups) * D;
#pragma unroll
    for (int j = 0; j < DJ; ++j) {
      if constexpr (sizeof(KT) == 4) out[o + lane + 32 * j] = acc[g][j];
      else out[o + lane + 32 * j] = __float2bfloat16_rn(acc[g][j]);
    }
  }
}

template <typename XT, typename WT>
cudaError_t launch_gemv(const ProjectArgs& a, cudaStream_t s) {
  const dim3 grid((a.N + kGvRows - 1) / kGvRows);
  const size_t smem = (size_t)kGvTok * gv_chunk<WT>() * sizeof(XT) + (kGvThreads / 32) * 32 * sizeof(float);
  auto kern = project_gemv_kernel<XT, WT>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return e != cudaSuccess ? e : launch_k(kern, grid, dim3(kGvThreads), smem, s, 1, a);
}

}  // namespace

bool project_tc_supported(const ProjectArgs& a, qsa_dtype_t x_dt, qsa_dtype_t w_dt) {
  return x_dt == QSA_BF16 && w_dt == QSA_BF16 && a.T >= 128 && a.H % 64 == 0 && umma::encode_fn() != nullptr;
}

cudaError_t launch_indexer_project(const ProjectArgs& a, qsa_dtype_t x_dt, qsa_dtype_t w_dt, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  if (project_tc_supported(a, x_dt, w_dt)) {
    CUtensorMap mx, mw;
    if (!umma::make_map_bf16(&mx, a.x, (uint64_t)a.H, (uint64_t)a.T, kPM) ||
        !umma::make_map_bf16(&mw, a.w, (uint64_t)a.H, (uint64_t)a.N, kPN))
      return cudaErrorInvalidValue;
    const size_t smem = sizeof(ProjSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(project_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long tiles = (long long)((a.T + kPM - 1) / kPM) * ((a.N + kPN - 1) / kPN);
    const int grid = tiles < sms ? (int)tiles : sms;
    return launch_k(project_tc_kernel, dim3(grid), dim3(kPThreads), smem, s, 1, a, mx, mw);
  }
  if (x_dt == QSA_BF16)
    return w_dt == QSA_BF16 ? launch_gemv<__nv_bfloat16, __nv_bfloat16>(a, s) : launch_gemv<__nv_bfloat16, float>(a, s);
  return w_dt == QSA_BF16 ? launch_gemv<float, __nv_bfloat16>(a, s) : launch_gemv<float, float>(a, s);
}

template <typename KT, int D>
cudaError_t launch_compress_d(const CompressArgs& c, cudaStream_t s) {
  const size_t smem = ((size_t)kCGroups * kGroupTokens * D + 2 * (size_t)D * kCRow) * sizeof(float);
  const dim3 grid((c.n + kCGroups - 1) / kCGroups);
  auto kern = compress_keys_kernel<KT, D>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return e != cudaSuccess ? e : launch_k(kern, grid, dim3(kCThreads), smem, s, 1, c);
}

template <typename KT>
cudaError_t launch_compress_t(const CompressArgs& c, cudaStream_t s) {
  if (c.D_I == 32) return launch_compress_d<KT, 32>(c, s);
  if (c.D_I == 64) return launch_compress_d<KT, 64>(c, s);
  return launch_compress_d<KT, 128>(c, s);
}

cudaError_t launch_compress_keys(const CompressArgs& c, qsa_dtype_t k_dt, cudaStream_t s) {
  if (c.n == 0) return cudaSuccess;
  return k_dt == QSA_BF16 ? launch_compress_t<__nv_bfloat16>(c, s) : launch_compress_t<float>(c, s);
}

}  // namespace qsa
