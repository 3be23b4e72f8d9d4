// sparse_attn_mma.cu -- stage 4 of QSA on tensor cores: GQA attention over the
// selected tokens of a paged BF16 or FP8-E4M3 KV cache ("Qwen3.8-27B QSA - BF16
// source weights", "QSA in brief": only the selected cache entries are read).
//
// Why tensor cores for a bandwidth-bound decode: with FP8 KV every 512-byte
// K+V row of a KV head feeds 8 query heads x 2 x 256 x 2 = 8 KFLOP, i.e. 16
// FLOP per byte -- above what FP32 FMA sustains at full HBM bandwidth.  The
// contraction is tiny in N (the <= 8 query heads of one KV head), so it runs
// on the warp-level m16n8k16 MMA with the TOKENS as the M dimension:
//
//   S^T[16 tok x 8 heads]  = K[16 tok x D]   . Q^T[D x 8 heads]     (16 MMAs)
//   O^T[D x 8 heads]      += V^T[D x 16 tok] . P^T[16 tok x 8 heads] (D/16 MMAs)
//
// * Gather: a CTA looks up the cache rows of a round of 16*NW selected tokens
//   (token id -> page table -> row) and copies them, K and V, into shared
//   memory with 16-byte cp.async; two rounds are in flight while the previous
//   one computes, so a CTA keeps up to 128 KB of loads outstanding.  The
//   16-byte chunk c of staged row r sits at chunk position c ^ (r & 7), which
//   makes the fragment reads below bank-conflict-free.
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
// Online softmax in base 2 per head; a split's partial (o, max, sum) goes to
// the workspace exactly as for the general kernel, and the same combine
// kernel finishes.
#include <math.h>

#include <cooperative_groups.h>

#include "attn_common.cuh"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

using namespace attn;

// grid (CL * S, Hkv, T), clusters of CL CTAs along x, NW warps per CTA.  CTA
// x covers token slots [x * chunk, (x + 1) * chunk) of its (query, KV head) in
// rounds of 16 * NW slots; the CL CTAs of a cluster merge through distributed
// shared memory; with S > 1 cluster groups each group's merged partial goes to
// the workspace for the combine kernel.
template <bool FP8, int D, typename QT, typename OT, int CL>
__global__ void __launch_bounds__(Geo<FP8, D>::NW * 32) attn_mma_kernel(AttnArgs a, float qk_scale,
                                                                       float vmul, int S, int chunk,
                                                                       float* ws_o, float* ws_ml) {
  using G_ = Geo<FP8, D>;
  constexpr int EB = G_::EB, CH = G_::CH, NCH = G_::NCH, KJ = G_::KJ, KS = G_::KS, NKS = G_::NKS,
                VJ = G_::VJ, MT = G_::MT, MTJ = G_::MTJ, ROWB = G_::ROWB, NW = G_::NW,
                ROUND = G_::ROUND, STAGE = G_::STAGE;
  constexpr int NT = NW * 32;
  extern __shared__ __align__(128) unsigned char smem[];
  // [NSTAGE stages of K rows | V rows] while streaming, reused for the merge;
  // then the row offsets of the current batch of token slots
  constexpr int NSTAGE = G_::NSTAGE, OFFCAP = G_::OFFCAP;
  long long* off_s = reinterpret_cast<long long*>(smem + NSTAGE * STAGE);  // [OFFCAP]
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
  const int beg = x * chunk;
  const int end = nt < beg + chunk ? nt : beg + chunk;
  const int32_t* trow = a.tok + (size_t)t * a.W;
  const int32_t* pt = a.page_table + (size_t)r * a.pt_stride;
  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_pages);
  const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_pages);
  const size_t row_bytes = (size_t)a.Hkv * ROWB;  // one token's row across KV heads
  const uint32_t smem_base = (uint32_t)__cvta_generic_to_shared(smem);

  // copy the K and V rows of the round starting at batch slot `slot0` into
  // stage st; rows of padding / invalid slots are zero-filled
  auto issue_round = [&](int st, int slot0) {
    const uint32_t sb = smem_base + st * STAGE;
    for (int i = tid; i < 2 * ROUND * NCH; i += NT) {
      const int row = i / NCH, c = i % NCH;
      const long long off = off_s[slot0 + (row % ROUND)];
      const uint32_t dst = sb + row * ROWB + ((c ^ (row & 7)) * 16);
      if (off >= 0) {
        cp_async16(dst, (row < ROUND ? kbase : vbase) + off + c * 16);
      } else {
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(dst), "r"(0) : "memory");
      }
    }
  };

  // ---- Q^T B fragments, head g (zero for heads >= G), permuted like K
  uint32_t qb[NKS][2];
  {
    const QT* qrow = reinterpret_cast<const QT*>(a.q) + ((size_t)t * a.Hq + h0 + (g < G ? g : 0)) * D;
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
#pragma unroll
      for (int q4 = 0; q4 < KS; ++q4) {
        const int d0 = CH * (4 * j + tq) + 4 * q4;
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = g < G ? Elem<QT>::get(qrow, d0 + e) : 0.f;
        qb[j * KS + q4][0] = pack2<FP8>(v[0], v[1]);
        qb[j * KS + q4][1] = pack2<FP8>(v[2], v[3]);
      }
    }
  }

  float m0 = -INFINITY, m1 = -INFINITY;  // running max of heads 2tq, 2tq+1 (log2 units)
  float l0 = 0.f, l1 = 0.f;              // this thread's share of the running sums
  float o[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  // ---- batches of up to OFFCAP token slots: look every row up once, then
  // stream the batch's rounds through an NSTAGE-deep cp.async ring
  for (int bstart = beg; bstart < end; bstart += OFFCAP) {
    const int bend = bstart + OFFCAP < end ? bstart + OFFCAP : end;
    const int nrounds = (bend - bstart + ROUND - 1) / ROUND;
    __syncthreads();  // the previous batch is done with off_s and the stages
    for (int i = tid; i < nrounds * ROUND; i += NT)
      off_s[i] = row_offset(a, trow, pt, bstart + i, bend, kvh, row_bytes, ROWB);
    __syncthreads();
#pragma unroll
    for (int rd = 0; rd < NSTAGE - 1; ++rd) {
      if (rd < nrounds) issue_round(rd, rd * ROUND);
      cp_async_commit();
    }
    for (int rd = 0; rd < nrounds; ++rd) {
      const int st = rd % NSTAGE;
      cp_async_wait<NSTAGE - 2>();  // round rd has landed
      __syncthreads();              // ... for every thread; stage (rd-1) % NSTAGE is free
      if (rd + NSTAGE - 1 < nrounds) issue_round((rd + NSTAGE - 1) % NSTAGE, (rd + NSTAGE - 1) * ROUND);
      cp_async_commit();

      if (bstart + rd * ROUND + 16 * warp < bend) {
        const unsigned char* ks = smem + st * STAGE + (16 * warp) * ROWB;  // this warp's 16 K rows
        const unsigned char* vs = ks + ROUND * ROWB;                        // and V rows
        const bool ok0 = off_s[rd * ROUND + 16 * warp + g] >= 0;
        const bool ok1 = off_s[rd * ROUND + 16 * warp + g + 8] >= 0;
        // ---- S^T = K . Q^T (rows g, g+8 of the tile; both have row & 7 == g)
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < KJ; ++j) {
          const int pc = ((4 * j + tq) ^ g) * 16;
          const uint4 k0 = lds16(ks + g * ROWB + pc);
          const uint4 k1 = lds16(ks + (g + 8) * ROWB + pc);
          const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
          const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
          for (int q4 = 0; q4 < KS; ++q4) {
            uint32_t af[4];
            if constexpr (FP8) {  // one word = 4 codes = dims 4q4..4q4+3 of the chunk
              af[0] = e4m3x2_to_f16x2(w0[q4]);
              af[1] = e4m3x2_to_f16x2(w1[q4]);
              af[2] = e4m3x2_to_f16x2(w0[q4] >> 16);
              af[3] = e4m3x2_to_f16x2(w1[q4] >> 16);
              mma_f16(sc, af, qb[j * KS + q4][0], qb[j * KS + q4][1]);
            } else {              // two words = 4 bf16 = dims 4q4..4q4+3 of the chunk
              af[0] = w0[2 * q4];
              af[1] = w1[2 * q4];
              af[2] = w0[2 * q4 + 1];
              af[3] = w1[2 * q4 + 1];
              mma_bf16(sc, af, qb[j * KS + q4][0], qb[j * KS + q4][1]);
            }
          }
        }
        // sc[0], sc[1]: token g, heads 2tq, 2tq+1; sc[2], sc[3]: token g+8
        const float s0 = ok0 ? sc[0] * qk_scale : -INFINITY;
        const float s1 = ok0 ? sc[1] * qk_scale : -INFINITY;
        const float s2 = ok1 ? sc[2] * qk_scale : -INFINITY;
        const float s3 = ok1 ? sc[3] * qk_scale : -INFINITY;
        // ---- online softmax, heads 2tq (s0, s2) and 2tq+1 (s1, s3)
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int d = 4; d <= 16; d <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, d));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, d));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float base0 = mn0 == -INFINITY ? 0.f : mn0;  // all -inf so far: nothing to rescale
        const float base1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = exp2f(m0 - base0), al1 = exp2f(m1 - base1);
        const float p0 = exp2f(s0 - base0), p1 = exp2f(s1 - base1);
        const float p2 = exp2f(s2 - base0), p3 = exp2f(s3 - base1);
        m0 = mn0;
        m1 = mn1;
        l0 = l0 * al0 + p0 + p2;
        l1 = l1 * al1 + p1 + p3;
        if (!__all_sync(0xffffffffu, al0 == 1.f && al1 == 1.f)) {
#pragma unroll
          for (int i = 0; i < MT; ++i) {
            o[i][0] *= al0; o[i][1] *= al1; o[i][2] *= al0; o[i][3] *= al1;
          }
        }
        // ---- P^T B fragments: transpose the two 8x8 halves of the S fragment
        const uint32_t pb0 = movmatrix_trans(pack2<FP8>(p0, p1));  // tokens 0..7
        const uint32_t pb1 = movmatrix_trans(pack2<FP8>(p2, p3));  // tokens 8..15

        // ---- O^T += V^T . P^T; staged V rows 2tq, 2tq+1, 2tq+8, 2tq+9 have
        // row & 7 == 2tq, 2tq+1, 2tq, 2tq+1
#pragma unroll
        for (int j = 0; j < VJ; ++j) {
          const int c = g + 8 * j;
          const uint4 A = lds16(vs + (2 * tq) * ROWB + ((c ^ (2 * tq)) * 16));
          const uint4 B = lds16(vs + (2 * tq + 1) * ROWB + ((c ^ (2 * tq + 1)) * 16));
          const uint4 C = lds16(vs + (2 * tq + 8) * ROWB + ((c ^ (2 * tq)) * 16));
          const uint4 E = lds16(vs + (2 * tq + 9) * ROWB + ((c ^ (2 * tq + 1)) * 16));
          const uint32_t va[4] = {A.x, A.y, A.z, A.w};  // token 2tq
          const uint32_t vb[4] = {B.x, B.y, B.z, B.w};  // token 2tq+1
          const uint32_t vc[4] = {C.x, C.y, C.z, C.w};  // token 2tq+8
          const uint32_t vd[4] = {E.x, E.y, E.z, E.w};  // token 2tq+9
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) {
            if constexpr (FP8) {
              // word wd holds elements 4wd..4wd+3: m-tiles j*MTJ + 2wd (+1), rows g / g+8
              const uint32_t lo01 = __byte_perm(va[wd], vb[wd], 0x5140);  // e0 pair, e1 pair
              const uint32_t hi01 = __byte_perm(va[wd], vb[wd], 0x7362);  // e2 pair, e3 pair
              const uint32_t lo89 = __byte_perm(vc[wd], vd[wd], 0x5140);
              const uint32_t hi89 = __byte_perm(vc[wd], vd[wd], 0x7362);
              const int mt = j * MTJ + 2 * wd;
              uint32_t af[4];
              af[0] = e4m3x2_to_f16x2(lo01);
              af[1] = e4m3x2_to_f16x2(lo01 >> 16);
              af[2] = e4m3x2_to_f16x2(lo89);
              af[3] = e4m3x2_to_f16x2(lo89 >> 16);
              mma_f16(o[mt], af, pb0, pb1);
              af[0] = e4m3x2_to_f16x2(hi01);
              af[1] = e4m3x2_to_f16x2(hi01 >> 16);
              af[2] = e4m3x2_to_f16x2(hi89);
              af[3] = e4m3x2_to_f16x2(hi89 >> 16);
              mma_f16(o[mt + 1], af, pb0, pb1);
            } else {
              // word wd holds elements 2wd (row g) and 2wd+1 (row g+8) of m-tile j*MTJ + wd
              const int mt = j * MTJ + wd;
              uint32_t af[4];
              af[0] = __byte_perm(va[wd], vb[wd], 0x5410);
              af[1] = __byte_perm(va[wd], vb[wd], 0x7632);
              af[2] = __byte_perm(vc[wd], vd[wd], 0x5410);
              af[3] = __byte_perm(vc[wd], vd[wd], 0x7632);
              mma_bf16(o[mt], af, pb0, pb1);
            }
          }
        }
      }
    }
    cp_async_wait<0>();
  }
  pdl_launch_dependents();

  // ---- finish the warp: full row sums, publish (m, l) and O to shared memory
  float* wo = reinterpret_cast<float*>(smem);  // [NW][8][D] per-warp O; [0] reused for the CTA
  float* wml = wo + NW * 8 * D;                // [NW][8][2] per-warp (max, sum)
  float* cml = wml + NW * 8 * 2;               // [8][2] CTA (max, sum)
  __syncthreads();  // the stages are dead: reuse them
#pragma unroll
  for (int d = 4; d <= 16; d <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, d);
    l1 += __shfl_xor_sync(0xffffffffu, l1, d);
  }
  if (g == 0) {
    wml[(warp * 8 + 2 * tq) * 2] = m0;
    wml[(warp * 8 + 2 * tq) * 2 + 1] = l0;
    wml[(warp * 8 + 2 * tq + 1) * 2] = m1;
    wml[(warp * 8 + 2 * tq + 1) * 2 + 1] = l1;
  }
  float* wow = wo + warp * 8 * D;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int c = g + 8 * (mt / MTJ);
    const int d_lo = CH * c + 2 * (mt % MTJ);  // row g; row g+8 is the next dim
    *reinterpret_cast<float2*>(wow + (2 * tq) * D + d_lo) = make_float2(o[mt][0], o[mt][2]);
    *reinterpret_cast<float2*>(wow + (2 * tq + 1) * D + d_lo) = make_float2(o[mt][1], o[mt][3]);
  }
  __syncthreads();

  // ---- merge the warps into this CTA's partial (kept in wo[0] and cml):
  // thread -> (head, 4 consecutive dims)
  const size_t th0 = (size_t)t * a.Hq + h0;
  for (int idx = tid; idx < G * (D / 4); idx += NT) {
    const int h = idx / (D / 4), d = 4 * (idx % (D / 4));
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wml[(w * 8 + h) * 2]);
    float L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = wml[(w * 8 + h) * 2];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
        L = fmaf(wml[(w * 8 + h) * 2 + 1], f, L);
        const float4 v = *reinterpret_cast<const float4*>(wo + (w * 8 + h) * D + d);
        O.x = fmaf(v.x, f, O.x); O.y = fmaf(v.y, f, O.y); O.z = fmaf(v.z, f, O.z); O.w = fmaf(v.w, f, O.w);
      }
    }
    const float Ov[4] = {O.x, O.y, O.z, O.w};
    if constexpr (CL == 1) {
      const size_t th = th0 + h;
      if (S == 1) {
        const float inv = L > 0.f ? vmul / L : 0.f;
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
      *reinterpret_cast<float4*>(wo + h * D + d) = O;  // read above only by this thread
      if (d == 0) {
        cml[h * 2] = M;
        cml[h * 2 + 1] = L;
      }
    }
  }
  if constexpr (CL > 1) {
    // ---- merge the CL CTAs of the cluster through distributed shared memory;
    // CTA `rank` finishes a 1/CL slice of the (head, dim) outputs
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    const int rank = (int)cl.block_rank();
    const int sg = x / CL;
    const int per = (G * D + CL - 1) / CL;
    const int lo = rank * per;
    const int hi = lo + per < G * D ? lo + per : G * D;
    for (int idx = lo + tid; idx < hi; idx += NT) {
      const int h = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < CL; ++q) M = fmaxf(M, cl.map_shared_rank(cml, q)[h * 2]);
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int q = 0; q < CL; ++q) {
          const float mq = cl.map_shared_rank(cml, q)[h * 2];
          if (mq == -INFINITY) continue;
          const float f = exp2f(mq - M);
          L = fmaf(cl.map_shared_rank(cml, q)[h * 2 + 1], f, L);
          O = fmaf(cl.map_shared_rank(wo, q)[h * D + d], f, O);
        }
      }
      const size_t th = th0 + h;
      if (S == 1) {
        const float v = L > 0.f ? O / L * vmul : 0.f;
        if constexpr (sizeof(OT) == 4) reinterpret_cast<float*>(a.out)[th * D + d] = v;
        else reinterpret_cast<__nv_bfloat16*>(a.out)[th * D + d] = __float2bfloat16_rn(v);
        if (d == 0 && a.lse) a.lse[th] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
      } else {
        ws_o[(th * S + sg) * D + d] = O;
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
cudaError_t launch_typed(const AttnArgs& a, float qk, float vmul, int CL, int S, void* ws, cudaStream_t s) {
  using G_ = Geo<FP8, D>;
  const int ctas = CL * S;
  const int chunk = (((a.W + ctas - 1) / ctas) + 15) / 16 * 16;
  float* ws_o = reinterpret_cast<float*>(ws);
  float* ws_ml = ws_o ? ws_o + (size_t)a.T * a.Hq * S * D : nullptr;
  const size_t stream_bytes = (size_t)G_::NSTAGE * G_::STAGE + (size_t)G_::OFFCAP * 8;
  const size_t merge_bytes = ((size_t)G_::NW * 8 * D + G_::NW * 8 * 2 + 8 * 2) * sizeof(float);
  const size_t smem = stream_bytes > merge_bytes ? stream_bytes : merge_bytes;
  const dim3 grid(ctas, a.Hkv * (a.Hq / a.Hkv > 8 ? 2 : 1), a.T);
  auto run = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_k(kern, grid, dim3(G_::NW * 32), smem, s, CL, a, qk, vmul, S, chunk, ws_o, ws_ml);
  };
  switch (CL) {
    case 1: return run(attn_mma_kernel<FP8, D, QT, OT, 1>);
    case 2: return run(attn_mma_kernel<FP8, D, QT, OT, 2>);
    case 4: return run(attn_mma_kernel<FP8, D, QT, OT, 4>);
    default: return run(attn_mma_kernel<FP8, D, QT, OT, 8>);
  }
}

template <bool FP8, int D>
cudaError_t launch_q(const AttnArgs& a, float qk, float vmul, int CL, int S, void* ws, cudaStream_t s) {
  if (a.q_dt == QSA_BF16) {
    if (a.out_dt == QSA_BF16) return launch_typed<FP8, D, __nv_bfloat16, __nv_bfloat16>(a, qk, vmul, CL, S, ws, s);
    return launch_typed<FP8, D, __nv_bfloat16, float>(a, qk, vmul, CL, S, ws, s);
  }
  if (a.out_dt == QSA_BF16) return launch_typed<FP8, D, float, __nv_bfloat16>(a, qk, vmul, CL, S, ws, s);
  return launch_typed<FP8, D, float, float>(a, qk, vmul, CL, S, ws, s);
}

// ---- decode: one 16-token tile per warp ---------------------------------------
//
// The streaming kernel above keeps one or two warps per SM sub-partition busy
// with a long dependent instruction chain per round; at decode sizes that
// chain, not HBM, sets the time.  Here every warp owns exactly ONE tile, so a
// CTA of 4 warps covers one 64-token chunk and there is no softmax state to
// carry between tiles: K and V go straight into registers, the Q fragments sit
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

// ---- many rows (prefill): one warp streams one whole row --------------------
//
// With thousands of (query, KV head) rows there is no need to split a row: a
// warp walks all of its row's 16-token tiles with an online softmax and writes
// the row's output itself, so there is no merge and no workspace.  The K / V
// tile goes straight into registers; the next tile's token -> row lookups are
// issued before the current tile computes.  Throughput comes from the many
// independent warps resident on every SM.
constexpr int kRowWarps = 2;

template <bool FP8, int D, typename QT, typename OT>
__global__ void __launch_bounds__(kRowWarps * 32) attn_rowwarp_kernel(AttnArgs a, float qk_scale,
                                                                      float vmul, int rows) {
  using G_ = Geo<FP8, D>;
  constexpr int CH = G_::CH, KJ = G_::KJ, KS = G_::KS, NKS = G_::NKS, VJ = G_::VJ, MT = G_::MT,
                MTJ = G_::MTJ, ROWB = G_::ROWB;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);  // (t, KV head, head half)
  pdl_wait();
  if (row >= rows) return;
  const int GQ = a.Hq / a.Hkv;
  const int halves = GQ > 8 ? 2 : 1;
  const int t = row / (a.Hkv * halves);
  const int rem = row % (a.Hkv * halves);
  const int kvh = rem / halves, half = rem % halves;
  const int G = GQ - 8 * half < 8 ? GQ - 8 * half : 8;
  const int h0 = kvh * GQ + 8 * half;
  const int g = lane >> 2, tq = lane & 3;

  int r = a.q_req ? a.q_req[t] : t;
  int nt = a.n_tok[t];
  nt = nt < 0 ? 0 : (nt > a.W ? a.W : nt);
  if (r < 0 || r >= a.pt_rows) {
    if (lane == 0 && kvh == 0 && half == 0) flag(a.status, QSA_DEV_BAD_REQUEST);
    r = 0;
    nt = 0;
  }
  const int32_t* trow = a.tok + (size_t)t * a.W;
  const int32_t* pt = a.page_table + (size_t)r * a.pt_stride;
  const size_t row_bytes = (size_t)a.Hkv * ROWB;
  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_pages);
  const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_pages);

  // Q^T B fragments of heads h0 + g (zero beyond G), permuted like K
  uint32_t qb[NKS][2];
  {
    const QT* qrow = reinterpret_cast<const QT*>(a.q) + ((size_t)t * a.Hq + h0 + (g < G ? g : 0)) * D;
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
#pragma unroll
      for (int q4 = 0; q4 < KS; ++q4) {
        const int d0 = CH * (4 * j + tq) + 4 * q4;
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = g < G ? Elem<QT>::get(qrow, d0 + e) : 0.f;
        qb[j * KS + q4][0] = pack2<FP8>(v[0], v[1]);
        qb[j * KS + q4][1] = pack2<FP8>(v[2], v[3]);
      }
    }
  }
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  long long off = lane < 16 ? row_offset(a, trow, pt, lane, nt, kvh, row_bytes, ROWB) : -1;
  for (int base = 0; base < nt; base += 16) {
    const long long offK0 = __shfl_sync(0xffffffffu, off, g);
    const long long offK1 = __shfl_sync(0xffffffffu, off, g + 8);
    const long long offV0 = __shfl_sync(0xffffffffu, off, 2 * tq);
    const long long offV1 = __shfl_sync(0xffffffffu, off, 2 * tq + 1);
    const long long offV2 = __shfl_sync(0xffffffffu, off, 2 * tq + 8);
    const long long offV3 = __shfl_sync(0xffffffffu, off, 2 * tq + 9);
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
    off = (lane < 16 && base + 16 < nt) ? row_offset(a, trow, pt, base + 16 + lane, nt, kvh, row_bytes, ROWB) : -1;

    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
      const uint32_t w0[4] = {kr0[j].x, kr0[j].y, kr0[j].z, kr0[j].w};
      const uint32_t w1[4] = {kr1[j].x, kr1[j].y, kr1[j].z, kr1[j].w};
#pragma unroll
      for (int q4 = 0; q4 < KS; ++q4) {
        const int ks = j * KS + q4;
        uint32_t af[4];
        if constexpr (FP8) {
          af[0] = e4m3x2_to_f16x2(w0[q4]);
          af[1] = e4m3x2_to_f16x2(w1[q4]);
          af[2] = e4m3x2_to_f16x2(w0[q4] >> 16);
          af[3] = e4m3x2_to_f16x2(w1[q4] >> 16);
          if (ks & 1) mma_f16(sb, af, qb[ks][0], qb[ks][1]); else mma_f16(sa, af, qb[ks][0], qb[ks][1]);
        } else {
          af[0] = w0[2 * q4];
          af[1] = w1[2 * q4];
          af[2] = w0[2 * q4 + 1];
          af[3] = w1[2 * q4 + 1];
          if (ks & 1) mma_bf16(sb, af, qb[ks][0], qb[ks][1]); else mma_bf16(sa, af, qb[ks][0], qb[ks][1]);
        }
      }
    }
    const bool ok0 = offK0 >= 0, ok1 = offK1 >= 0;
    const float s0 = ok0 ? (sa[0] + sb[0]) * qk_scale : -INFINITY;
    const float s1 = ok0 ? (sa[1] + sb[1]) * qk_scale : -INFINITY;
    const float s2 = ok1 ? (sa[2] + sb[2]) * qk_scale : -INFINITY;
    const float s3 = ok1 ? (sa[3] + sb[3]) * qk_scale : -INFINITY;
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
    for (int d = 4; d <= 16; d <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, d));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, d));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = exp2f(m0 - b0), al1 = exp2f(m1 - b1);
    const float p0 = exp2f(s0 - b0), p1 = exp2f(s1 - b1), p2 = exp2f(s2 - b0), p3 = exp2f(s3 - b1);
    m0 = mn0;
    m1 = mn1;
    l0 = l0 * al0 + p0 + p2;
    l1 = l1 * al1 + p1 + p3;
    if (!__all_sync(0xffffffffu, al0 == 1.f && al1 == 1.f)) {
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        o[i][0] *= al0; o[i][1] *= al1; o[i][2] *= al0; o[i][3] *= al1;
      }
    }
    const uint32_t pb0 = movmatrix_trans(pack2<FP8>(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack2<FP8>(p2, p3));
#pragma unroll
    for (int j = 0; j < VJ; ++j) {
      const uint32_t va[4] = {vr[0][j].x, vr[0][j].y, vr[0][j].z, vr[0][j].w};
      const uint32_t vb[4] = {vr[1][j].x, vr[1][j].y, vr[1][j].z, vr[1][j].w};
      const uint32_t vc[4] = {vr[2][j].x, vr[2][j].y, vr[2][j].z, vr[2][j].w};
      const uint32_t vd[4] = {vr[3][j].x, vr[3][j].y, vr[3][j].z, vr[3][j].w};
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        if constexpr (FP8) {
          const uint32_t lo01 = __byte_perm(va[wd], vb[wd], 0x5140);
          const uint32_t hi01 = __byte_perm(va[wd], vb[wd], 0x7362);
          const uint32_t lo89 = __byte_perm(vc[wd], vd[wd], 0x5140);
          const uint32_t hi89 = __byte_perm(vc[wd], vd[wd], 0x7362);
          const int mt = j * MTJ + 2 * wd;
          uint32_t af[4];
          af[0] = e4m3x2_to_f16x2(lo01);
          af[1] = e4m3x2_to_f16x2(lo01 >> 16);
          af[2] = e4m3x2_to_f16x2(lo89);
          af[3] = e4m3x2_to_f16x2(lo89 >> 16);
          mma_f16(o[mt], af, pb0, pb1);
          af[0] = e4m3x2_to_f16x2(hi01);
          af[1] = e4m3x2_to_f16x2(hi01 >> 16);
          af[2] = e4m3x2_to_f16x2(hi89);
          af[3] = e4m3x2_to_f16x2(hi89 >> 16);
          mma_f16(o[mt + 1], af, pb0, pb1);
        } else {
          const int mt = j * MTJ + wd;
          uint32_t af[4];
          af[0] = __byte_perm(va[wd], vb[wd], 0x5410);
          af[1] = __byte_perm(va[wd], vb[wd], 0x7632);
          af[2] = __byte_perm(vc[wd], vd[wd], 0x5410);
          af[3] = __byte_perm(vc[wd], vd[wd], 0x7632);
          mma_bf16(o[mt], af, pb0, pb1);
        }
      }
    }
  }
  pdl_launch_dependents();
#pragma unroll
  for (int d = 4; d <= 16; d <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, d);
    l1 += __shfl_xor_sync(0xffffffffu, l1, d);
  }
  // heads 2tq (c0, c2) and 2tq+1 (c1, c3); rows g / g+8 are dims d_lo / d_lo+1
  const float inv0 = l0 > 0.f ? vmul / l0 : 0.f, inv1 = l1 > 0.f ? vmul / l1 : 0.f;
  const size_t th0 = (size_t)t * a.Hq + h0;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int d_lo = CH * (g + 8 * (mt / MTJ)) + 2 * (mt % MTJ);
    if (2 * tq < G) {
      OT* op = reinterpret_cast<OT*>(a.out) + (th0 + 2 * tq) * D + d_lo;
      if constexpr (sizeof(OT) == 4) {
        *reinterpret_cast<float2*>(op) = make_float2(o[mt][0] * inv0, o[mt][2] * inv0);
      } else {
        *reinterpret_cast<__nv_bfloat162*>(op) = __floats2bfloat162_rn(o[mt][0] * inv0, o[mt][2] * inv0);
      }
    }
    if (2 * tq + 1 < G) {
      OT* op = reinterpret_cast<OT*>(a.out) + (th0 + 2 * tq + 1) * D + d_lo;
      if constexpr (sizeof(OT) == 4) {
        *reinterpret_cast<float2*>(op) = make_float2(o[mt][1] * inv1, o[mt][3] * inv1);
      } else {
        *reinterpret_cast<__nv_bfloat162*>(op) = __floats2bfloat162_rn(o[mt][1] * inv1, o[mt][3] * inv1);
      }
    }
  }
  if (a.lse && g == 0) {
    if (2 * tq < G) a.lse[th0 + 2 * tq] = l0 > 0.f ? (m0 + log2f(l0)) * kLn2 : -INFINITY;
    if (2 * tq + 1 < G) a.lse[th0 + 2 * tq + 1] = l1 > 0.f ? (m1 + log2f(l1)) * kLn2 : -INFINITY;
  }
}

template <bool FP8, int D, typename QT, typename OT>
cudaError_t launch_rowwarp_typed(const AttnArgs& a, float qk, float vmul, cudaStream_t s) {
  const int rows = a.T * a.Hkv * (a.Hq / a.Hkv > 8 ? 2 : 1);
  const dim3 grid((rows + kRowWarps - 1) / kRowWarps);
  return launch_k(attn_rowwarp_kernel<FP8, D, QT, OT>, grid, dim3(kRowWarps * 32), 0, s, 1, a, qk,
                  vmul, rows);
}

template <bool FP8, int D>
cudaError_t launch_rowwarp_q(const AttnArgs& a, float qk, float vmul, cudaStream_t s) {
  if (a.q_dt == QSA_BF16) {
    if (a.out_dt == QSA_BF16) return launch_rowwarp_typed<FP8, D, __nv_bfloat16, __nv_bfloat16>(a, qk, vmul, s);
    return launch_rowwarp_typed<FP8, D, __nv_bfloat16, float>(a, qk, vmul, s);
  }
  if (a.out_dt == QSA_BF16) return launch_rowwarp_typed<FP8, D, float, __nv_bfloat16>(a, qk, vmul, s);
  return launch_rowwarp_typed<FP8, D, float, float>(a, qk, vmul, s);
}

}  // namespace

bool attn_mma_supported(const AttnArgs& a) {
  return (a.kv_dt == QSA_BF16 || a.kv_dt == QSA_FP8_E4M3) && (a.D == 128 || a.D == 256) &&
         a.Hq / a.Hkv <= 16;
}

int attn_tile_tokens() { return kTileTokens; }

// Many rows: one warp streams each (query, KV head, head half) row.
cudaError_t launch_sparse_attn_rowwarp(const AttnArgs& a, float qk, float vmul, cudaStream_t s) {
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  if (fp8) return a.D == 256 ? launch_rowwarp_q<true, 256>(a, qk, vmul, s) : launch_rowwarp_q<true, 128>(a, qk, vmul, s);
  return a.D == 256 ? launch_rowwarp_q<false, 256>(a, qk, vmul, s) : launch_rowwarp_q<false, 128>(a, qk, vmul, s);
}

// Decode: grid (CL * S) x Hkv x T of 64-token CTAs (one tile per warp).
cudaError_t launch_sparse_attn_tile(const AttnArgs& a, float qk, float vmul, int CL, int S, void* ws,
                                    cudaStream_t s) {
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  if (fp8) return a.D == 256 ? launch_tile_q<true, 256>(a, qk, vmul, CL, S, ws, s)
                             : launch_tile_q<true, 128>(a, qk, vmul, CL, S, ws, s);
  return a.D == 256 ? launch_tile_q<false, 256>(a, qk, vmul, CL, S, ws, s)
                    : launch_tile_q<false, 128>(a, qk, vmul, CL, S, ws, s);
}

// S == 1: the cluster writes out / lse; S > 1: one partial per cluster group
// for the combine kernel (workspace of attn_decode_ws_bytes(T, Hq, D, S)).
cudaError_t launch_sparse_attn_mma(const AttnArgs& a, float qk, float vmul, int CL, int S, void* ws,
                                   cudaStream_t s) {
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  if (fp8) return a.D == 256 ? launch_q<true, 256>(a, qk, vmul, CL, S, ws, s)
                             : launch_q<true, 128>(a, qk, vmul, CL, S, ws, s);
  return a.D == 256 ? launch_q<false, 256>(a, qk, vmul, CL, S, ws, s)
                    : launch_q<false, 128>(a, qk, vmul, CL, S, ws, s);
}

}  // namespace qsa
