// sparse_attn_mma.cu -- stage 4 of QSA for decode rows too long for one
// thread-block cluster: GQA attention over the selected tokens of a paged
// BF16 or FP8-E4M3 KV cache ("Qwen3.8-27B QSA - BF16 source weights", "QSA
// in brief": only the selected cache entries are read), split over CTAs of
// 64 token slots whose partials the combine kernel merges.
//
// The contraction is tiny in N (the <= 8 query heads of one KV head), so it
// runs on the warp-level m16n8k16 MMA with the TOKENS as the M dimension:
//
//   S^T[16 tok x 8 heads]  = K[16 tok x D]   . Q^T[D x 8 heads]
//   O^T[D x 8 heads]      += V^T[D x 16 tok] . P^T[16 tok x 8 heads]
//
// * K A fragments: the dot product may visit the head dimension in any order,
//   so thread (g, t) of a row takes whole 16-byte chunks t, t+4, t+8, ... of
//   it; Q's B fragments use the same permutation.
// * The S fragment (rows = tokens, cols = heads) is exactly the 8x8 b16 layout
//   of movmatrix; its transpose is the P^T B fragment of the PV MMA.
// * V^T's A fragment pairs two tokens per register: thread (g, t) loads the
//   16-byte chunks g, g+8, ... of tokens 2t, 2t+1, 2t+8, 2t+9 and byte-permutes
//   them into token pairs; which output dims a thread accumulates is again a
//   free permutation, undone when the output is written.
// * FP8 codes become f16 pairs with cvt.e4m3x2 (exact) and run on the f16 MMA;
//   the K scale and the softmax scale are applied to S in FP32, the V scale to
//   the final output.  BF16 caches use the bf16 MMA directly.
#include <math.h>

#include <cooperative_groups.h>

#include "attn_common.cuh"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

using namespace attn;

// ---- decode: one 16-token tile per warp ---------------------------------------
//
// A kernel that streams a whole row through one CTA keeps one or two warps per
// SM sub-partition busy with a long dependent instruction chain per round; at
// decode sizes that chain, not HBM, sets the time.  Here every warp owns
// exactly ONE tile, so a CTA of 4 warps covers one 64-token chunk and there is
// no softmax state to carry between tiles: K and V go straight into registers,
// the Q fragments sit
// pre-permuted in shared memory, and each output accumulator is written out
// right after its single MMA.  That keeps the kernel small enough for four
// CTAs (16 warps) per SM, which hides the latencies.  Partials are merged per
// CTA, then across a cluster of CL CTAs through distributed shared memory, and
// cluster groups (S > 1) through the workspace and the combine kernel.
constexpr int kTileWarps = 4;
constexpr int kTileTokens = 16 * kTileWarps;  // token slots per CTA

template <bool FP8, int D, typename QT, typename OT, int CL>
__global__ void __launch_bounds__(kTileWarps * 32, 4) attn_tile_kernel(AttnArgs a, float qk_scale,
                                                                      float vmul, int S,
                                                                      float* ws_o, float* ws_ml) {
  using G_ = Geo<FP8, D>;
  constexpr int CH = G_::CH, KJ = G_::KJ, KS = G_::KS, NKS = G_::NKS, VJ = G_::VJ, MT = G_::MT,
                MTJ = G_::MTJ, ROWB = G_::ROWB;
  constexpr int NT = kTileWarps * 32;
  __shared__ __align__(16) uint32_t qf_s[NKS][32][2];  // Q^T B fragments, per k-step and lane
  __shared__ __align__(16) float wo[kTileWarps][8][D];  // per-warp O; [0] reused for the CTA
  __shared__ float wml[kTileWarps][8][2];               // per-warp (max, sum)
  __shared__ float cml[8][2];                            // CTA (max, sum)
  const int x = blockIdx.x, t = blockIdx.z;
  // more than 8 query heads per KV head: two CTAs, 8 heads each (the second
  // read of the same rows hits in L2)
  const int GQ = a.Hq / a.Hkv;
  const int halves = GQ > 8 ? 2 : 1;
  const int kvh = blockIdx.y / halves, half = blockIdx.y % halves;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int G = GQ - 8 * half < 8 ? GQ - 8 * half : 8;  // this CTA's query heads
  const int h0 = kvh * GQ + 8 * half;

  pdl_wait();

  int r = a.q_req ? a.q_req[t] : t;
  int nt = a.n_tok[t];
  nt = nt < 0 ? 0 : (nt > a.W ? a.W : nt);
  if (r < 0 || r >= a.pt_rows) {
    if (tid == 0 && x == 0) flag(a.status, QSA_DEV_BAD_REQUEST);
    r = 0;
    nt = 0;
  }
  const int32_t* trow = a.tok + (size_t)t * a.W;
  const int32_t* pt = a.page_table + (size_t)r * a.pt_stride;
  const size_t row_bytes = (size_t)a.Hkv * ROWB;
  const int base = x * kTileTokens + 16 * warp;  // this warp's 16 token slots

  // ---- Q^T B fragments into shared memory: warp w builds k-steps w, w+4, ...;
  // the Q loads are issued first so they overlap the token -> page lookups
  constexpr int QPW = (NKS + kTileWarps - 1) / kTileWarps;  // k-steps per warp
  float qv[QPW][4];
  {
    const QT* qrow = reinterpret_cast<const QT*>(a.q) + ((size_t)t * a.Hq + h0 + (g < G ? g : 0)) * D;
#pragma unroll
    for (int i = 0; i < QPW; ++i) {
      const int ks = warp + kTileWarps * i;
      const int j = ks / KS, q4 = ks % KS;
      const int d0 = CH * (4 * j + tq) + 4 * q4;
#pragma unroll
      for (int e = 0; e < 4; ++e) qv[i][e] = (g < G && ks < NKS) ? Elem<QT>::get(qrow, d0 + e) : 0.f;
    }
  }
  // row offsets of the tile's tokens (lanes 0..15)
  const long long off = lane < 16 ? row_offset(a, trow, pt, base + lane, nt, kvh, row_bytes, ROWB) : -1;
#pragma unroll
  for (int i = 0; i < QPW; ++i) {
    const int ks = warp + kTileWarps * i;
    if (ks < NKS) {
      qf_s[ks][lane][0] = pack2<FP8>(qv[i][0], qv[i][1]);
      qf_s[ks][lane][1] = pack2<FP8>(qv[i][2], qv[i][3]);
    }
  }

  // ---- K rows g, g+8 (chunks 4j+tq) and V tokens 2tq, 2tq+1, 2tq+8, 2tq+9 (chunks g+8j)
  const long long offK0 = __shfl_sync(0xffffffffu, off, g);
  const long long offK1 = __shfl_sync(0xffffffffu, off, g + 8);
  const long long offV0 = __shfl_sync(0xffffffffu, off, 2 * tq);
  const long long offV1 = __shfl_sync(0xffffffffu, off, 2 * tq + 1);
  const long long offV2 = __shfl_sync(0xffffffffu, off, 2 * tq + 8);
  const long long offV3 = __shfl_sync(0xffffffffu, off, 2 * tq + 9);
  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_pages);
  const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_pages);
  const uint4 z = make_uint4(0, 0, 0, 0);
  uint4 kr0[KJ], kr1[KJ], vr[4][VJ];
#pragma unroll
  for (int j = 0; j < KJ; ++j) {
    const int cb = (4 * j + tq) * 16;
    kr0[j] = offK0 >= 0 ? ldg16(kbase + offK0 + cb) : z;
    kr1[j] = offK1 >= 0 ? ldg16(kbase + offK1 + cb) : z;
  }
#pragma unroll
  for (int j = 0; j < VJ; ++j) {
    const int cb = (g + 8 * j) * 16;
    vr[0][j] = offV0 >= 0 ? ldg16(vbase + offV0 + cb) : z;
    vr[1][j] = offV1 >= 0 ? ldg16(vbase + offV1 + cb) : z;
    vr[2][j] = offV2 >= 0 ? ldg16(vbase + offV2 + cb) : z;
    vr[3][j] = offV3 >= 0 ? ldg16(vbase + offV3 + cb) : z;
  }
  __syncthreads();  // Q fragments visible
  pdl_launch_dependents();

  // ---- S^T = K . Q^T, two independent accumulation chains
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < KJ; ++j) {
    const uint32_t w0[4] = {kr0[j].x, kr0[j].y, kr0[j].z, kr0[j].w};
    const uint32_t w1[4] = {kr1[j].x, kr1[j].y, kr1[j].z, kr1[j].w};
#pragma unroll
    for (int q4 = 0; q4 < KS; ++q4) {
      const int ks = j * KS + q4;
      const uint2 qb = *reinterpret_cast<const uint2*>(&qf_s[ks][lane][0]);
      uint32_t af[4];
      if constexpr (FP8) {
        af[0] = e4m3x2_to_f16x2(w0[q4]);
        af[1] = e4m3x2_to_f16x2(w1[q4]);
        af[2] = e4m3x2_to_f16x2(w0[q4] >> 16);
        af[3] = e4m3x2_to_f16x2(w1[q4] >> 16);
        if (ks & 1) mma_f16(sb, af, qb.x, qb.y); else mma_f16(sa, af, qb.x, qb.y);
      } else {
        af[0] = w0[2 * q4];
        af[1] = w1[2 * q4];
        af[2] = w0[2 * q4 + 1];
        af[3] = w1[2 * q4 + 1];
        if (ks & 1) mma_bf16(sb, af, qb.x, qb.y); else mma_bf16(sa, af, qb.x, qb.y);
      }
    }
  }
  const bool ok0 = offK0 >= 0, ok1 = offK1 >= 0;
  const float s0 = ok0 ? (sa[0] + sb[0]) * qk_scale : -INFINITY;  // token g, head 2tq
  const float s1 = ok0 ? (sa[1] + sb[1]) * qk_scale : -INFINITY;  // token g, head 2tq+1
  const float s2 = ok1 ? (sa[2] + sb[2]) * qk_scale : -INFINITY;  // token g+8, head 2tq
  const float s3 = ok1 ? (sa[3] + sb[3]) * qk_scale : -INFINITY;  // token g+8, head 2tq+1
  // ---- softmax over the tile, heads 2tq (s0, s2) and 2tq+1 (s1, s3)
  float m0 = fmaxf(s0, s2), m1 = fmaxf(s1, s3);
#pragma unroll
  for (int d = 4; d <= 16; d <<= 1) {
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, d));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, d));
  }
  const float b0 = m0 == -INFINITY ? 0.f : m0, b1 = m1 == -INFINITY ? 0.f : m1;
  const float p0 = exp2f(s0 - b0), p1 = exp2f(s1 - b1), p2 = exp2f(s2 - b0), p3 = exp2f(s3 - b1);
  float l0 = p0 + p2, l1 = p1 + p3;
#pragma unroll
  for (int d = 4; d <= 16; d <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, d);
    l1 += __shfl_xor_sync(0xffffffffu, l1, d);
  }
  if (g == 0) {
    wml[warp][2 * tq][0] = m0;
    wml[warp][2 * tq][1] = l0;
    wml[warp][2 * tq + 1][0] = m1;
    wml[warp][2 * tq + 1][1] = l1;
  }
  const uint32_t pb0 = movmatrix_trans(pack2<FP8>(p0, p1));  // tokens 0..7
  const uint32_t pb1 = movmatrix_trans(pack2<FP8>(p2, p3));  // tokens 8..15

  // ---- O^T = V^T . P^T, each m-tile's accumulator stored as soon as it is done
  float* wow = &wo[warp][0][0];
#pragma unroll
  for (int j = 0; j < VJ; ++j) {
    const uint32_t va[4] = {vr[0][j].x, vr[0][j].y, vr[0][j].z, vr[0][j].w};  // token 2tq
    const uint32_t vb[4] = {vr[1][j].x, vr[1][j].y, vr[1][j].z, vr[1][j].w};  // token 2tq+1
    const uint32_t vc[4] = {vr[2][j].x, vr[2][j].y, vr[2][j].z, vr[2][j].w};  // token 2tq+8
    const uint32_t vd[4] = {vr[3][j].x, vr[3][j].y, vr[3][j].z, vr[3][j].w};  // token 2tq+9
    const int c = g + 8 * j;
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      if constexpr (FP8) {
        const uint32_t lo01 = __byte_perm(va[wd], vb[wd], 0x5140);
        const uint32_t hi01 = __byte_perm(va[wd], vb[wd], 0x7362);
        const uint32_t lo89 = __byte_perm(vc[wd], vd[wd], 0x5140);
        const uint32_t hi89 = __byte_perm(vc[wd], vd[wd], 0x7362);
        const int mt = j * MTJ + 2 * wd;
        float oa[4] = {0.f, 0.f, 0.f, 0.f}, ob[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t af[4];
        af[0] = e4m3x2_to_f16x2(lo01);
        af[1] = e4m3x2_to_f16x2(lo01 >> 16);
        af[2] = e4m3x2_to_f16x2(lo89);
        af[3] = e4m3x2_to_f16x2(lo89 >> 16);
        mma_f16(oa, af, pb0, pb1);
        af[0] = e4m3x2_to_f16x2(hi01);
        af[1] = e4m3x2_to_f16x2(hi01 >> 16);
        af[2] = e4m3x2_to_f16x2(hi89);
        af[3] = e4m3x2_to_f16x2(hi89 >> 16);
        mma_f16(ob, af, pb0, pb1);
        const int da = CH * c + 2 * (mt % MTJ), db = CH * c + 2 * ((mt + 1) % MTJ);
        *reinterpret_cast<float2*>(wow + (2 * tq) * D + da) = make_float2(oa[0], oa[2]);
        *reinterpret_cast<float2*>(wow + (2 * tq + 1) * D + da) = make_float2(oa[1], oa[3]);
        *reinterpret_cast<float2*>(wow + (2 * tq) * D + db) = make_float2(ob[0], ob[2]);
        *reinterpret_cast<float2*>(wow + (2 * tq + 1) * D + db) = make_float2(ob[1], ob[3]);
      } else {
        const int mt = j * MTJ + wd;
        float oa[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t af[4];
        af[0] = __byte_perm(va[wd], vb[wd], 0x5410);
        af[1] = __byte_perm(va[wd], vb[wd], 0x7632);
        af[2] = __byte_perm(vc[wd], vd[wd], 0x5410);
        af[3] = __byte_perm(vc[wd], vd[wd], 0x7632);
        mma_bf16(oa, af, pb0, pb1);
        const int da = CH * c + 2 * (mt % MTJ);
        *reinterpret_cast<float2*>(wow + (2 * tq) * D + da) = make_float2(oa[0], oa[2]);
        *reinterpret_cast<float2*>(wow + (2 * tq + 1) * D + da) = make_float2(oa[1], oa[3]);
      }
    }
  }
  (void)MT;
  __syncthreads();

  // ---- merge the warps: thread -> (head, 4 consecutive dims)
  const size_t th0 = (size_t)t * a.Hq + h0;
  for (int idx = tid; idx < G * (D / 4); idx += NT) {
    const int h = idx / (D / 4), d = 4 * (idx % (D / 4));
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kTileWarps; ++w) M = fmaxf(M, wml[w][h][0]);
    float L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kTileWarps; ++w) {
        const float mw = wml[w][h][0];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
        L = fmaf(wml[w][h][1], f, L);
        const float4 v = *reinterpret_cast<const float4*>(&wo[w][h][d]);
        O.x = fmaf(v.x, f, O.x); O.y = fmaf(v.y, f, O.y); O.z = fmaf(v.z, f, O.z); O.w = fmaf(v.w, f, O.w);
      }
    }
    if constexpr (CL == 1) {
      const size_t th = th0 + h;
      if (S == 1) {
        const float inv = L > 0.f ? vmul / L : 0.f;
        const float Ov[4] = {O.x, O.y, O.z, O.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (sizeof(OT) == 4) reinterpret_cast<float*>(a.out)[th * D + d + e] = Ov[e] * inv;
          else reinterpret_cast<__nv_bfloat16*>(a.out)[th * D + d + e] = __float2bfloat16_rn(Ov[e] * inv);
        }
        if (d == 0 && a.lse) a.lse[th] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
      } else {
        *reinterpret_cast<float4*>(ws_o + (th * S + x) * D + d) = O;
        if (d == 0) {
          ws_ml[(th * S + x) * 2] = M;
          ws_ml[(th * S + x) * 2 + 1] = L;
        }
      }
    } else {
      *reinterpret_cast<float4*>(&wo[0][h][d]) = O;  // read above only by this thread
      if (d == 0) {
        cml[h][0] = M;
        cml[h][1] = L;
      }
    }
  }
  if constexpr (CL > 1) {
    // ---- merge the CL CTAs of the cluster; CTA `rank` finishes 1/CL of the outputs
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    const int rank = (int)cl.block_rank();
    const int sg = x / CL;
    const int items = G * (D / 4);
    const int per = (items + CL - 1) / CL;
    const int lo = rank * per;
    const int hi = lo + per < items ? lo + per : items;
    for (int idx = lo + tid; idx < hi; idx += NT) {
      const int h = idx / (D / 4), d = 4 * (idx % (D / 4));
      float mq[CL];
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < CL; ++q) {
        mq[q] = cl.map_shared_rank(&cml[0][0], q)[h * 2];
        M = fmaxf(M, mq[q]);
      }
      float L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M != -INFINITY) {
#pragma unroll
        for (int q = 0; q < CL; ++q) {
          const float f = mq[q] == -INFINITY ? 0.f : exp2f(mq[q] - M);
          L = fmaf(cl.map_shared_rank(&cml[0][0], q)[h * 2 + 1], f, L);
          const float4 v = *reinterpret_cast<const float4*>(cl.map_shared_rank(&wo[0][h][d], q));
          O.x = fmaf(v.x, f, O.x); O.y = fmaf(v.y, f, O.y); O.z = fmaf(v.z, f, O.z); O.w = fmaf(v.w, f, O.w);
        }
      }
      const size_t th = th0 + h;
      if (S == 1) {
        const float inv = L > 0.f ? vmul / L : 0.f;
        const float Ov[4] = {O.x, O.y, O.z, O.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (sizeof(OT) == 4) reinterpret_cast<float*>(a.out)[th * D + d + e] = Ov[e] * inv;
          else reinterpret_cast<__nv_bfloat16*>(a.out)[th * D + d + e] = __float2bfloat16_rn(Ov[e] * inv);
        }
        if (d == 0 && a.lse) a.lse[th] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
      } else {
        *reinterpret_cast<float4*>(ws_o + (th * S + sg) * D + d) = O;
        if (d == 0) {
          ws_ml[(th * S + sg) * 2] = M;
          ws_ml[(th * S + sg) * 2 + 1] = L;
        }
      }
    }
    cl.sync();  // peers may still read this CTA's shared memory until here
  }
}

template <bool FP8, int D, typename QT, typename OT>
cudaError_t launch_tile_typed(const AttnArgs& a, float qk, float vmul, int CL, int S, void* ws,
                              cudaStream_t s) {
  float* ws_o = reinterpret_cast<float*>(ws);
  float* ws_ml = ws_o ? ws_o + (size_t)a.T * a.Hq * S * D : nullptr;
  const dim3 grid(CL * S, a.Hkv * (a.Hq / a.Hkv > 8 ? 2 : 1), a.T);
  const dim3 block(kTileWarps * 32);
  switch (CL) {
    case 1: return launch_k(attn_tile_kernel<FP8, D, QT, OT, 1>, grid, block, 0, s, 1, a, qk, vmul, S, ws_o, ws_ml);
    case 2: return launch_k(attn_tile_kernel<FP8, D, QT, OT, 2>, grid, block, 0, s, 2, a, qk, vmul, S, ws_o, ws_ml);
    case 4: return launch_k(attn_tile_kernel<FP8, D, QT, OT, 4>, grid, block, 0, s, 4, a, qk, vmul, S, ws_o, ws_ml);
    default: return launch_k(attn_tile_kernel<FP8, D, QT, OT, 8>, grid, block, 0, s, 8, a, qk, vmul, S, ws_o, ws_ml);
  }
}

template <bool FP8, int D>
cudaError_t launch_tile_q(const AttnArgs& a, float qk, float vmul, int CL, int S, void* ws, cudaStream_t s) {
  if (a.q_dt == QSA_BF16) {
    if (a.out_dt == QSA_BF16) return launch_tile_typed<FP8, D, __nv_bfloat16, __nv_bfloat16>(a, qk, vmul, CL, S, ws, s);
    return launch_tile_typed<FP8, D, __nv_bfloat16, float>(a, qk, vmul, CL, S, ws, s);
  }
  if (a.out_dt == QSA_BF16) return launch_tile_typed<FP8, D, float, __nv_bfloat16>(a, qk, vmul, CL, S, ws, s);
  return launch_tile_typed<FP8, D, float, float>(a, qk, vmul, CL, S, ws, s);
}

}  // namespace

bool attn_mma_supported(const AttnArgs& a) {
  return (a.kv_dt == QSA_BF16 || a.kv_dt == QSA_FP8_E4M3) && (a.D == 128 || a.D == 256) &&
         a.Hq / a.Hkv <= 16;
}

int attn_tile_tokens() { return kTileTokens; }

// Decode: grid (CL * S) x Hkv x T of 64-token CTAs (one tile per warp).
cudaError_t launch_sparse_attn_tile(const AttnArgs& a, float qk, float vmul, int CL, int S, void* ws,
                                    cudaStream_t s) {
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  if (fp8) return a.D == 256 ? launch_tile_q<true, 256>(a, qk, vmul, CL, S, ws, s)
                             : launch_tile_q<true, 128>(a, qk, vmul, CL, S, ws, s);
  return a.D == 256 ? launch_tile_q<false, 256>(a, qk, vmul, CL, S, ws, s)
                    : launch_tile_q<false, 128>(a, qk, vmul, CL, S, ws, s);
}

}  // namespace qsa
