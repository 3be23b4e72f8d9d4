// sparse_attn_prefill.cu -- stage 4 of QSA for many rows (prefill chunks, big
// decode batches): GQA attention of every query over its own selected tokens
// of a paged BF16 / FP8-E4M3 KV cache ("Qwen3.8-27B QSA - BF16 source
// weights", "QSA in brief": only the selected cache entries are read).
//
// Every query selects its own ~2K tokens, so the K/V rows a query reads are
// gathered for it alone: 1 KiB per token and KV head at D = 256 BF16, about
// 34 GB for an 8,192-query chunk, served mostly from L2.  The kernel is built
// to move those bytes once and keep many of them in flight:
//  * each (query, KV head) row gathers every K/V row once for ALL query
//    heads of the KV head: one warp per n8 tile of heads (two warps for 9-16
//    heads), sharing the row's staged tiles.  Two warps of ~130 registers
//    instead of one of 255 double the warps an SM holds to hide latency;
//  * the row's warps stream its 16-token tiles through a ring of S
//    shared-memory stages with 16-byte cp.async (each warp copies its share
//    of the rows; no registers held while in flight; S - 1 tiles in flight
//    while one is computed), meeting at one named barrier per tile.  The 16-byte chunk
//    c of staged row r sits at chunk position c ^ sw(r), sw(r) = (r & 7) ^
//    4 (r & 1): the K reads (rows g, g+1 in a quarter-warp) and the V reads
//    (rows 2tq) then fall on distinct banks;
//  * per tile: S^T = K.Q^T on m16n8k16 (tokens as M, heads as N), an
//    online softmax per head in base 2, and O^T += V^T.P^T with V rows
//    paired by byte permutes;
//  * rows run KV head by KV head, so the cache lines being gathered at any
//    time belong to one KV head: half the cache (64 MB for the 65,536-token
//    BF16 chunk), which stays in L2 while every query of the chunk reads it;
//  * each warp writes its heads of the row's output: no merge, no workspace.
#include <math.h>

#include <type_traits>

#include "attn_common.cuh"

namespace qsa {
namespace {

using namespace attn;

// (query, KV head) rows per CTA: 7 rows of one warp, or 6 rows of two warps
// (12 warps of up to 168 registers; 14 would cap them at 128 and spill)
template <int NT>
constexpr int pf_rows() {
  return NT > 1 ? 6 : 7;
}
constexpr int kPfRingBytes = 224 * 1024;    // per CTA

__device__ __forceinline__ void cp_async16_pf(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit_pf() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_pf() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// swizzle of the 16-byte chunks of staged row r (see the file comment)
__device__ __forceinline__ int pf_sw(int r) { return (r & 7) ^ ((r & 1) << 2); }

template <bool FP8, int D, int NT>
constexpr int pf_stages() {
  constexpr int stage = 32 * Geo<FP8, D>::ROWB;  // 16 K rows + 16 V rows
  constexpr int s = kPfRingBytes / pf_rows<NT>() / stage;
  return s > 8 ? 8 : s;
}

// grid: ceil(T * Hkv / R) CTAs of R = pf_rows<NT>() row slots.  The NT warps of
// slot j of CTA b take row b * R + j = kvh * T + t (query t, KV head
// kvh); warp u of a row computes head tile u (heads 8u .. 8u+7 of the G of
// the KV head) and stages tokens 16/NT * u .. of every tile.
template <bool FP8, int D, typename QT, typename OT, int NT>
__global__ void __launch_bounds__(pf_rows<NT>() * NT * 32, 1) attn_prefill_kernel(AttnArgs a, float qk_scale, float vmul,
                                                                           int rows) {
  using G_ = Geo<FP8, D>;
  constexpr int CH = G_::CH, NCH = G_::NCH, KJ = G_::KJ, KS = G_::KS, NKS = G_::NKS, VJ = G_::VJ, MT = G_::MT,
                MTJ = G_::MTJ, ROWB = G_::ROWB;
  constexpr int R = pf_rows<NT>();
  constexpr int S = pf_stages<FP8, D, NT>();
  constexpr int STAGE = 32 * ROWB;
  static_assert(S >= 2, "at least two stages");
  constexpr int TPW = 16 / NT;    // token rows of a tile each warp of the row stages
  constexpr int RPP = 32 / NCH;   // rows a lane pass covers when staging
  static_assert(NCH >= 8 && 32 % NCH == 0 && TPW % RPP == 0, "row chunks must swizzle over 8 and tile a warp");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t valid_s[R][8][NT];  // per stage and warp: bit i = token slot i of the tile is real
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slot = warp / NT, u = warp % NT;
  const int g = lane >> 2, tq = lane & 3;
  const int row = blockIdx.x * R + slot;
  pdl_wait();
  if (row >= rows) return;  // (every warp of the row)
  // KV-head-major order: while the first half of the grid runs, only KV head
  // 0's cache lines are gathered (half the cache, which fits in L2)
  const int kvh = row / a.T, t = row % a.T;
  const int G = a.Hq / a.Hkv;
  const int h0 = kvh * G;

  int r = a.q_req ? a.q_req[t] : t;
  int nt = a.n_tok[t];
  nt = nt < 0 ? 0 : (nt > a.W ? a.W : nt);
  if (r < 0 || r >= a.pt_rows) {
    if (lane == 0 && kvh == 0 && u == 0) flag(a.status, QSA_DEV_BAD_REQUEST);
    r = 0;
    nt = 0;
  }
  const int32_t* trow = a.tok + (size_t)t * a.W;
  const int32_t* pt = a.page_table + (size_t)r * a.pt_stride;
  const size_t row_bytes = (size_t)a.Hkv * ROWB;
  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_pages);
  const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_pages);
  unsigned char* ring = smem + (size_t)slot * S * STAGE;
  const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
  const int ntiles = (nt + 15) / 16;
  // the row's warps meet once per tile: every warp's copies of the tile have
  // landed, and every warp is done with the stage the next copies refill
  auto row_sync = [&]() {
    if constexpr (NT > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + slot), "r"(NT * 32) : "memory");
    else __syncwarp();
  };

  // stage this warp's TPW token rows of tile i: lanes 0..TPW-1 look the rows
  // up, then lane l copies chunk l % NCH of rows l / NCH, l / NCH + RPP, ...
  // of K and V (a warp instruction moves whole 512-byte stretches of a row)
  auto issue = [&](int i) {
    if (i < ntiles) {
      const long long off =
          lane < TPW ? row_offset(a, trow, pt, 16 * i + TPW * u + lane, nt, kvh, row_bytes, ROWB) : -1;
      const unsigned vm = __ballot_sync(0xffffffffu, off >= 0) & ((1u << TPW) - 1u);
      if (lane == 0) valid_s[slot][i % S][u] = vm << (TPW * u);
      const uint32_t sb = ring_s + (uint32_t)((i % S) * STAGE);
      const int c = lane % NCH;
#pragma unroll
      for (int r0 = 0; r0 < TPW; r0 += RPP) {
        const int lr = r0 + lane / NCH;  // row within this warp's share
        const int rr = TPW * u + lr;     // row within the tile
        const long long o = __shfl_sync(0xffffffffu, off, lr);
        const uint32_t pos = (uint32_t)(((c ^ pf_sw(rr)) * 16));
        const uint32_t dk = sb + rr * ROWB + pos, dv = sb + (16 + rr) * ROWB + pos;
        if (o >= 0) {
          cp_async16_pf(dk, kbase + o + c * 16);
          cp_async16_pf(dv, vbase + o + c * 16);
        } else {
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(dk), "r"(0) : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(dv), "r"(0) : "memory");
        }
      }
    }
    cp_async_commit_pf();  // one group per tile (empty groups keep the count)
  };
#pragma unroll
  for (int i = 0; i < S - 1; ++i) issue(i);

  // Q^T B fragments of heads h0 + 8u + g (zero past G), head dim permuted like K
  uint32_t qb[NKS][2];
  {
    const int hg = 8 * u + g;
    const QT* qrow = reinterpret_cast<const QT*>(a.q) + ((size_t)t * a.Hq + h0 + (hg < G ? hg : 0)) * D;
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
#pragma unroll
      for (int q4 = 0; q4 < KS; ++q4) {
        const int d0 = CH * (4 * j + tq) + 4 * q4;
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = hg < G ? Elem<QT>::get(qrow, d0 + e) : 0.f;
        qb[j * KS + q4][0] = pack2<FP8>(v[0], v[1]);
        qb[j * KS + q4][1] = pack2<FP8>(v[2], v[3]);
      }
    }
  }
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, o[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  for (int i = 0; i < ntiles; ++i) {
    cp_async_wait_pf<S - 2>();      // this warp's copies of tile i have landed
    row_sync();                     // ... and every warp's; all are done with tile i - 1
    issue(i + S - 1);               // into the stage tile i - 1 used
    const unsigned char* ks = ring + (size_t)(i % S) * STAGE;
    const unsigned char* vs = ks + 16 * ROWB;
    unsigned vmask = 0;
#pragma unroll
    for (int w = 0; w < NT; ++w) vmask |= valid_s[slot][i % S][w];
    const bool ok0 = (vmask >> g) & 1u, ok1 = (vmask >> (g + 8)) & 1u;

    // ---- S^T = K . Q^T for this warp's head tile (rows g and g+8 share a swizzle)
    // four independent accumulator chains (k-step kk feeds chain kk % 4): the
    // MMAs of a chain wait on each other, the chains do not
    float scc[4][4] = {};
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
      const int pc = ((4 * j + tq) ^ pf_sw(g)) * 16;
      const uint4 k0 = lds16(ks + g * ROWB + pc);
      const uint4 k1 = lds16(ks + (g + 8) * ROWB + pc);
      const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
      const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
      for (int q4 = 0; q4 < KS; ++q4) {
        const int kk = j * KS + q4;
        uint32_t af[4];
        if constexpr (FP8) {  // one word = 4 codes = dims 4q4..4q4+3 of the chunk
          e4m3x4_to_f16x2x2(w0[q4], af[0], af[2]);
          e4m3x4_to_f16x2x2(w1[q4], af[1], af[3]);
          mma_f16(scc[kk & 3], af, qb[kk][0], qb[kk][1]);
        } else {              // two words = 4 bf16 = dims 4q4..4q4+3 of the chunk
          af[0] = w0[2 * q4];
          af[1] = w1[2 * q4];
          af[2] = w0[2 * q4 + 1];
          af[3] = w1[2 * q4 + 1];
          mma_bf16(scc[kk & 3], af, qb[kk][0], qb[kk][1]);
        }
      }
    }

    float sc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[e] = (scc[0][e] + scc[1][e]) + (scc[2][e] + scc[3][e]);

    // ---- online softmax, heads 8u + 2tq (s0, s2) and 8u + 2tq + 1 (s1, s3)
    uint32_t pb[2];
    {
      const float s0 = ok0 ? sc[0] * qk_scale : -INFINITY;
      const float s1 = ok0 ? sc[1] * qk_scale : -INFINITY;
      const float s2 = ok1 ? sc[2] * qk_scale : -INFINITY;
      const float s3 = ok1 ? sc[3] * qk_scale : -INFINITY;
      float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
      for (int d = 4; d <= 16; d <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, d));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, d));
      }
      // the base moves only when the max grows by more than 8 (log2 units): p
      // stays below 2^8 and the FP32 sums keep their accuracy, while most tiles
      // skip the rescale of the accumulators
      const float mn0 = mx0 > m0 + 8.f ? mx0 : m0;
      const float mn1 = mx1 > m1 + 8.f ? mx1 : m1;
      const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - b0);
      const float al1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - b1);
      const float p0 = fast_exp2(s0 - b0), p1 = fast_exp2(s1 - b1), p2 = fast_exp2(s2 - b0), p3 = fast_exp2(s3 - b1);
      m0 = mn0;
      m1 = mn1;
      l0 = l0 * al0 + p0 + p2;
      l1 = l1 * al1 + p1 + p3;
      if (!__all_sync(0xffffffffu, al0 == 1.f && al1 == 1.f)) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[mt][0] *= al0; o[mt][1] *= al1; o[mt][2] *= al0; o[mt][3] *= al1;
        }
      }
      pb[0] = movmatrix_trans(pack2<FP8>(p0, p1));  // tokens 0..7
      pb[1] = movmatrix_trans(pack2<FP8>(p2, p3));  // tokens 8..15
    }

    // ---- O^T += V^T . P^T; staged V rows 2tq, 2tq+1, 2tq+8, 2tq+9 have the
    // swizzles of rows 2tq, 2tq+1, 2tq, 2tq+1
#pragma unroll
    for (int j = 0; j < VJ; ++j) {
      const int c = g + 8 * j;
      const int sa = pf_sw(2 * tq), sb = pf_sw(2 * tq + 1);
      const uint4 A = lds16(vs + (2 * tq) * ROWB + ((c ^ sa) * 16));
      const uint4 B = lds16(vs + (2 * tq + 1) * ROWB + ((c ^ sb) * 16));
      const uint4 C = lds16(vs + (2 * tq + 8) * ROWB + ((c ^ sa) * 16));
      const uint4 E = lds16(vs + (2 * tq + 9) * ROWB + ((c ^ sb) * 16));
      const uint32_t va[4] = {A.x, A.y, A.z, A.w};  // token 2tq
      const uint32_t vb[4] = {B.x, B.y, B.z, B.w};  // token 2tq+1
      const uint32_t vc[4] = {C.x, C.y, C.z, C.w};  // token 2tq+8
      const uint32_t vd[4] = {E.x, E.y, E.z, E.w};  // token 2tq+9
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        if constexpr (FP8) {
          const uint32_t lo01 = __byte_perm(va[wd], vb[wd], 0x5140);
          const uint32_t hi01 = __byte_perm(va[wd], vb[wd], 0x7362);
          const uint32_t lo89 = __byte_perm(vc[wd], vd[wd], 0x5140);
          const uint32_t hi89 = __byte_perm(vc[wd], vd[wd], 0x7362);
          const int mt = j * MTJ + 2 * wd;
          uint32_t af[4], ag[4];
          e4m3x4_to_f16x2x2(lo01, af[0], af[1]);
          e4m3x4_to_f16x2x2(lo89, af[2], af[3]);
          e4m3x4_to_f16x2x2(hi01, ag[0], ag[1]);
          e4m3x4_to_f16x2x2(hi89, ag[2], ag[3]);
          mma_f16(o[mt], af, pb[0], pb[1]);
          mma_f16(o[mt + 1], ag, pb[0], pb[1]);
        } else {
          const int mt = j * MTJ + wd;
          uint32_t af[4];
          af[0] = __byte_perm(va[wd], vb[wd], 0x5410);
          af[1] = __byte_perm(va[wd], vb[wd], 0x7632);
          af[2] = __byte_perm(vc[wd], vd[wd], 0x5410);
          af[3] = __byte_perm(vc[wd], vd[wd], 0x7632);
          mma_bf16(o[mt], af, pb[0], pb[1]);
        }
      }
    }
  }
  cp_async_wait_pf<0>();
  pdl_launch_dependents();

  // ---- this warp's heads of the row's output: heads 8u + 2tq (c0, c2) and
  // 8u + 2tq + 1 (c1, c3); rows g / g+8 of m-tile mt are dims d_lo / d_lo + 1
  const size_t th0 = (size_t)t * a.Hq + h0;
#pragma unroll
  for (int d = 4; d <= 16; d <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, d);
    l1 += __shfl_xor_sync(0xffffffffu, l1, d);
  }
  const float inv0 = l0 > 0.f ? vmul / l0 : 0.f, inv1 = l1 > 0.f ? vmul / l1 : 0.f;
  const int ha = 8 * u + 2 * tq, hb = ha + 1;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int d_lo = CH * (g + 8 * (mt / MTJ)) + 2 * (mt % MTJ);
    if (ha < G) {
      OT* op = reinterpret_cast<OT*>(a.out) + (th0 + ha) * D + d_lo;
      if constexpr (sizeof(OT) == 4) *reinterpret_cast<float2*>(op) = make_float2(o[mt][0] * inv0, o[mt][2] * inv0);
      else *reinterpret_cast<__nv_bfloat162*>(op) = __floats2bfloat162_rn(o[mt][0] * inv0, o[mt][2] * inv0);
    }
    if (hb < G) {
      OT* op = reinterpret_cast<OT*>(a.out) + (th0 + hb) * D + d_lo;
      if constexpr (sizeof(OT) == 4) *reinterpret_cast<float2*>(op) = make_float2(o[mt][1] * inv1, o[mt][3] * inv1);
      else *reinterpret_cast<__nv_bfloat162*>(op) = __floats2bfloat162_rn(o[mt][1] * inv1, o[mt][3] * inv1);
    }
  }
  if (a.lse && g == 0) {
    if (ha < G) a.lse[th0 + ha] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
    if (hb < G) a.lse[th0 + hb] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
  }
}

template <bool FP8, int D, typename QT, typename OT>
cudaError_t launch_pf_typed(const AttnArgs& a, float qk, float vmul, cudaStream_t s) {
  const int rows = a.T * a.Hkv;
  const int G = a.Hq / a.Hkv;
  auto go = [&](auto kern, auto nt_tag) {
    constexpr int NT = decltype(nt_tag)::value, R = pf_rows<NT>();
    const size_t smem = (size_t)R * pf_stages<FP8, D, NT>() * 32 * Geo<FP8, D>::ROWB;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e != cudaSuccess ? e
                            : launch_k(kern, dim3((rows + R - 1) / R), dim3(R * NT * 32), smem, s, 1, a, qk, vmul,
                                       rows);
  };
  return G > 8 ? go(attn_prefill_kernel<FP8, D, QT, OT, 2>, std::integral_constant<int, 2>())
               : go(attn_prefill_kernel<FP8, D, QT, OT, 1>, std::integral_constant<int, 1>());
}

template <bool FP8, int D>
cudaError_t launch_pf_q(const AttnArgs& a, float qk, float vmul, cudaStream_t s) {
  if (a.q_dt == QSA_BF16) {
    if (a.out_dt == QSA_BF16) return launch_pf_typed<FP8, D, __nv_bfloat16, __nv_bfloat16>(a, qk, vmul, s);
    return launch_pf_typed<FP8, D, __nv_bfloat16, float>(a, qk, vmul, s);
  }
  if (a.out_dt == QSA_BF16) return launch_pf_typed<FP8, D, float, __nv_bfloat16>(a, qk, vmul, s);
  return launch_pf_typed<FP8, D, float, float>(a, qk, vmul, s);
}

}  // namespace

cudaError_t launch_sparse_attn_prefill_rows(const AttnArgs& a, float qk, float vmul, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  if (a.D == 256) return fp8 ? launch_pf_q<true, 256>(a, qk, vmul, s) : launch_pf_q<false, 256>(a, qk, vmul, s);
  if (a.D == 128) return fp8 ? launch_pf_q<true, 128>(a, qk, vmul, s) : launch_pf_q<false, 128>(a, qk, vmul, s);
  return cudaErrorInvalidValue;
}

}  // namespace qsa
