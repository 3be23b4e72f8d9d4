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
//    from HBM -- one warp per row, 16-byte loads, every token's dot product
//    from the same loaded values, a warp reduction at the end;
//  * prefill (hundreds of tokens or more, BF16): a tcgen05 GEMM.  Tiles of
//    128 tokens x 128 rows of w x 64 (128 B, SWIZZLE_128B) arrive by TMA
//    through a 4-stage ring; one elected thread issues 128 x 128 x 16 MMAs
//    into one of two TMEM accumulators, so the epilogue of one tile overlaps
//    the MMAs of the next; four epilogue warps read the accumulators with
//    tcgen05.ld and store FP32 rows.  Every mbarrier wait is bounded.
//
// Compressed-key write  khat_g = W_phi [k_4g; k_4g+1; k_4g+2; k_4g+3] + b_phi
// for each completed group g, written to row g % 16 of page
// page_table[r][g / 16] (FP32 or BF16).  A CTA of D_I threads takes 16 groups:
// their token keys in shared memory, W_phi streamed through shared memory 64
// columns at a time (each column loaded once per CTA, coalesced), thread d
// accumulating output dim d of the 16 groups.
#include "qsa_internal.cuh"
#include "umma.cuh"

namespace qsa {
namespace {

using namespace mbar;

// ---------------------------------------------------------------------------
// projection, decode form: one warp per row of w, up to 8 tokens per pass

constexpr int kGvWarps = 4;
constexpr int kGvTok = 8;

template <typename XT, typename WT>
__global__ void __launch_bounds__(kGvWarps * 32) project_gemv_kernel(ProjectArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kGvWarps + warp;
  pdl_wait();
  if (n >= a.N) return;   // (whole warp; no block-wide barrier in this kernel)
  const WT* wrow = reinterpret_cast<const WT*>(a.w) + (size_t)n * a.H;
  const XT* x = reinterpret_cast<const XT*>(a.x);
  for (int t0 = 0; t0 < a.T; t0 += kGvTok) {
    const int nt = a.T - t0 < kGvTok ? a.T - t0 : kGvTok;
    float acc[kGvTok];
#pragma unroll
    for (int i = 0; i < kGvTok; ++i) acc[i] = 0.f;
    for (int h = 8 * lane; h < a.H; h += 256) {
      float wv[8];
      VecLoad<WT, 8>::get(wrow, (size_t)h, wv);
#pragma unroll
      for (int i = 0; i < kGvTok; ++i) {
        if (i < nt) {
          float xv[8];
          VecLoad<XT, 8>::get(x, (size_t)(t0 + i) * a.H + h, xv);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[i] = fmaf(xv[e], wv[e], acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kGvTok; ++i) {
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], d);
    }
    // lane i writes token t0 + i
    float v = acc[0];
#pragma unroll
    for (int i = 1; i < kGvTok; ++i) v = lane == i ? acc[i] : v;
    if (lane < nt) a.y[(size_t)(t0 + lane) * a.N + n] = v;
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
// compressed-key write

constexpr int kCGroups = 16;   // groups per CTA
constexpr int kCSlab = 64;     // columns of W_phi staged at a time

template <typename KT>
__global__ void __launch_bounds__(128) compress_keys_kernel(CompressArgs c) {
  const int D = c.D_I;          // == blockDim.x
  const int d = threadIdx.x;
  extern __shared__ __align__(16) float cs[];
  float* kcat = cs;                                   // [kCGroups][4 * D]
  float* ws = cs + kCGroups * kGroupTokens * D;       // [D][kCSlab + 1]
  const int i0 = blockIdx.x * kCGroups;
  const int ng = c.n - i0 < kCGroups ? c.n - i0 : kCGroups;
  const int W4 = kGroupTokens * D;
  pdl_wait();
  // the groups' token keys: group g, token j, dim e at kcat[g][j * D + e]
  for (int idx = d; idx < ng * W4; idx += D) {
    const int g = idx / W4, j = (idx / D) % kGroupTokens, e = idx % D;
    kcat[idx] = __ldg(c.k_tok + ((size_t)(i0 + g) * kGroupTokens + j) * c.tok_stride + e);
  }
  float acc[kCGroups];
  const float b = c.bias ? __ldg(c.bias + d) : 0.f;
#pragma unroll
  for (int g = 0; g < kCGroups; ++g) acc[g] = b;
  for (int j0 = 0; j0 < W4; j0 += kCSlab) {
    __syncthreads();  // the previous slab is consumed (and the keys are in place)
    for (int idx = d; idx < D * kCSlab; idx += D) {
      const int r = idx / kCSlab, col = idx % kCSlab;
      ws[r * (kCSlab + 1) + col] = __ldg(c.wphi + (size_t)r * W4 + j0 + col);
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < kCSlab; ++jj) {
      const float w = ws[d * (kCSlab + 1) + jj];   // row stride 65: the warp's rows fall on distinct banks
#pragma unroll
      for (int g = 0; g < kCGroups; ++g) acc[g] = fmaf(w, kcat[g * W4 + j0 + jj], acc[g]);
    }
  }
  KT* out = reinterpret_cast<KT*>(c.k_idx_pages);
#pragma unroll
  for (int g = 0; g < kCGroups; ++g) {
    if (g >= ng) break;
    const int i = i0 + g;
    const int r = c.g_req ? __ldg(c.g_req + i) : 0;
    const int gid = __ldg(c.g_id + i);
    if (r < 0 || r >= c.pt_rows) {
      if (d == 0) flag(c.status, QSA_DEV_BAD_REQUEST);
      continue;
    }
    if (gid < 0 || gid / kPageGroups >= c.pt_stride) {
      if (d == 0) flag(c.status, QSA_DEV_BAD_GROUP);
      continue;
    }
    const int page = __ldg(c.page_table + (size_t)r * c.pt_stride + gid / kPageGroups);
    if (page < 0 || page >= c.num_pages) {
      if (d == 0) flag(c.status, QSA_DEV_BAD_PAGE);
      continue;
    }
    const size_t o = ((size_t)page * kPageGroups + gid % kPageGroups) * D + d;
    if constexpr (sizeof(KT) == 4) out[o] = acc[g];
    else out[o] = __float2bfloat16_rn(acc[g]);
  }
}

template <typename XT>
cudaError_t launch_gemv_x(const ProjectArgs& a, qsa_dtype_t w_dt, cudaStream_t s) {
  const dim3 grid((a.N + kGvWarps - 1) / kGvWarps);
  if (w_dt == QSA_BF16) return launch_k(project_gemv_kernel<XT, __nv_bfloat16>, grid, dim3(kGvWarps * 32), 0, s, 1, a);
  return launch_k(project_gemv_kernel<XT, float>, grid, dim3(kGvWarps * 32), 0, s, 1, a);
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
  if (x_dt == QSA_BF16) return launch_gemv_x<__nv_bfloat16>(a, w_dt, s);
  return launch_gemv_x<float>(a, w_dt, s);
}

cudaError_t launch_compress_keys(const CompressArgs& c, qsa_dtype_t k_dt, cudaStream_t s) {
  if (c.n == 0) return cudaSuccess;
  const size_t smem = ((size_t)kCGroups * kGroupTokens * c.D_I + (size_t)c.D_I * (kCSlab + 1)) * sizeof(float);
  const dim3 grid((c.n + kCGroups - 1) / kCGroups);
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e != cudaSuccess ? e : launch_k(kern, grid, dim3(c.D_I), smem, s, 1, c);
  };
  if (k_dt == QSA_BF16) return go(compress_keys_kernel<__nv_bfloat16>);
  return go(compress_keys_kernel<float>);
}

}  // namespace qsa
