// sparse_attn_cluster.cu -- stage 4 of QSA for decode batches: GQA attention
// over the selected tokens of a paged BF16 / FP8-E4M3 KV cache, one
// thread-block cluster per (query, KV head) row ("Qwen3.8-27B QSA - BF16
// source weights", "QSA in brief": only the selected cache entries are read).
//
// A decode step has few rows (8 queries x 2 KV heads at B8) and ~2K selected
// tokens per row, so the time is latency: token id -> page -> K/V row from
// HBM -> two small MMAs -> a merge.  This kernel keeps that chain to one pass:
//  * a cluster of CL CTAs (one per SM) covers the WHOLE row, so no partial
//    goes through global memory and no second kernel merges them;
//  * warp w of CTA r owns the 16-token tiles r*NW + w + k*CL*NW; it looks up
//    TP tiles' rows at once (lanes 0..15 the first tile, 16..31 the second) and
//    loads their K and V into registers together, so a warp with two tiles
//    waits for HBM once;
//  * per step the warp computes S^T = K.Q^T on the m16n8k16 MMA (tokens as M,
//    the <= 8 query heads of the KV head as N), one softmax over the step's
//    tokens, and O^T = V^T.P^T accumulated over the step's tiles; each output
//    m-tile goes to the warp's slot in shared memory right away (rescaled into
//    the previous steps' sum when the warp has more than one step);
//  * the warps of a CTA merge in shared memory, the CTAs of the cluster
//    through distributed shared memory, and the cluster writes the output.
// Fragment layouts are those of the other MMA kernels of this library: K
// chunks 4j+tq of rows g, g+8; V chunks g+8j of tokens 2tq, 2tq+1, 2tq+8,
// 2tq+9 paired by byte permutes; P^T from S by movmatrix.
#include <math.h>

#include <cooperative_groups.h>

#include "attn_common.cuh"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

using namespace attn;

// warps per CTA, one CTA per SM.  Each SM sub-partition holds 16K registers,
// so 12 warps (3 per sub-partition) leave 168 registers a thread.
constexpr int kClWarps = 12;

// tiles a warp holds at once: two for FP8 (64 registers of K and V each),
// one for BF16 rows at D = 256
template <bool FP8, int D>
constexpr int tiles_per_step() {
  return (FP8 || D <= 128) ? 2 : 1;
}

// 32-bit word k of a 16-byte chunk (k constant after unrolling)
__device__ __forceinline__ uint32_t word(const uint4& v, int k) {
  return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}

// Per-warp O slots in shared memory: head h of a slot starts at h * (D + 4)
// floats and dim d sits at o_pos(d) = d ^ 2 * ((d >> SH) & 7), SH = 5 for
// 16-value chunks (FP8) and 4 for 8-value chunks (BF16).  The MMA epilogue's
// float2 stores (lane (g, tq): heads 2tq, 2tq+1, dims 16g + c or 8g + c) then
// fall on distinct banks; the plain [head][D] layout put 16 of them on one.
// The XOR moves only bits 1..3 of d, so an aligned group of four dims stays
// one aligned group, with its halves swapped when bit 1 of the XOR is set.
template <int D>
constexpr int o_stride() {
  return D + 4;
}
template <int SH>
__device__ __forceinline__ int o_pos(int d) {
  return d ^ (2 * ((d >> SH) & 7));
}
template <int SH>
__device__ __forceinline__ float4 ld_o4(const float* head_base, int d) {
  const int x = 2 * ((d >> SH) & 7);
  const float4 v = *reinterpret_cast<const float4*>(head_base + (d ^ (x & ~3)));
  return (x & 2) ? make_float4(v.z, v.w, v.x, v.y) : v;
}
template <int SH>
__device__ __forceinline__ void st_o4(float* head_base, int d, float4 v) {
  const int x = 2 * ((d >> SH) & 7);
  *reinterpret_cast<float4*>(head_base + (d ^ (x & ~3))) = (x & 2) ? make_float4(v.z, v.w, v.x, v.y) : v;
}

// Final output of (query, head) row th, dims d..d+3: O / L times the V scale,
// and the natural-log LSE; a row with nothing to attend gives zeros and -inf.
template <typename OT, int D>
__device__ __forceinline__ void write_out(const AttnArgs& a, size_t th, int d, float4 O, float M, float L,
                                          float vmul) {
  const float inv = L > 0.f ? vmul / L : 0.f;
  const float Ov[4] = {O.x, O.y, O.z, O.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if constexpr (sizeof(OT) == 4) reinterpret_cast<float*>(a.out)[th * D + d + e] = Ov[e] * inv;
    else reinterpret_cast<__nv_bfloat16*>(a.out)[th * D + d + e] = __float2bfloat16_rn(Ov[e] * inv);
  }
  if (d == 0 && a.lse) a.lse[th] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

template <bool FP8, int D, typename QT, typename OT, int CL>
__global__ void __launch_bounds__(kClWarps * 32, 1)
    attn_cluster_kernel(AttnArgs a, float qk_scale, float vmul) {
  using G_ = Geo<FP8, D>;
  constexpr int CH = G_::CH, KJ = G_::KJ, KS = G_::KS, NKS = G_::NKS, VJ = G_::VJ, MTJ = G_::MTJ,
                ROWB = G_::ROWB;
  constexpr int NW = kClWarps, NT = NW * 32, TP = tiles_per_step<FP8, D>();
  constexpr int OS = o_stride<D>(), SH = CH == 16 ? 5 : 4;
  __shared__ __align__(16) uint32_t qf_s[NKS][32][2];  // Q^T B fragments, per k-step and lane
  extern __shared__ __align__(16) float wo_dyn[];      // [NW][8][OS] per-warp O; warp 0's reused for the CTA
  __shared__ float wml[NW][8][2];                        // per-warp (max, sum)
  cg::cluster_group cl = cg::this_cluster();
  const int rank = CL > 1 ? (int)cl.block_rank() : 0;
  const int t = blockIdx.z;
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
    if (tid == 0 && rank == 0) flag(a.status, QSA_DEV_BAD_REQUEST);
    r = 0;
    nt = 0;
  }
  const int32_t* trow = a.tok + (size_t)t * a.W;
  const int32_t* pt = a.page_table + (size_t)r * a.pt_stride;
  const size_t row_bytes = (size_t)a.Hkv * ROWB;
  const int ntiles = (nt + 15) / 16;
  const int wid = rank * NW + warp;   // this warp's first tile
  constexpr int WSTRIDE = CL * NW;    // tiles between a warp's consecutive tiles

  // Token slot a lane looks up in step k0 (lanes 16i .. 16i+15: tile i of the step),
  // and the row offset of a token id (-1: padding, or an id / page outside the cache).
  auto slot_of = [&](int k0) { return 16 * (wid + (k0 + (lane >> 4)) * WSTRIDE) + (lane & 15); };
  auto offset_of = [&](int j) -> long long {
    if (j == -1) return -1;
    if (j < -1 || j / kPageTokens >= a.pt_stride) {
      flag(a.status, QSA_DEV_BAD_TOKEN);
      return -1;
    }
    const int page = __ldg(pt + j / kPageTokens);
    if (page < 0 || page >= a.num_pages) {
      flag(a.status, QSA_DEV_BAD_PAGE);
      return -1;
    }
    return (long long)(((size_t)page * kPageTokens + (j % kPageTokens)) * row_bytes + (size_t)kvh * ROWB);
  };
  // the first step's token ids go out before the Q loads, their pages right after
  const bool act0 = (lane >> 4) < TP && slot_of(0) < nt;
  const int j0 = act0 ? __ldg(trow + slot_of(0)) : -1;

  // ---- Q^T B fragments into shared memory: warp w builds k-steps w, w+NW, ...
  {
    const QT* qrow = reinterpret_cast<const QT*>(a.q) + ((size_t)t * a.Hq + h0 + (g < G ? g : 0)) * D;
    for (int ks = warp; ks < NKS; ks += NW) {
      const int j = ks / KS, q4 = ks % KS;
      const int d0 = CH * (4 * j + tq) + 4 * q4;
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = g < G ? Elem<QT>::get(qrow, d0 + e) : 0.f;
      qf_s[ks][lane][0] = pack2<FP8>(v[0], v[1]);
      qf_s[ks][lane][1] = pack2<FP8>(v[2], v[3]);
    }
  }
  const long long off0 = act0 ? offset_of(j0) : -1;
  __syncthreads();  // Q fragments visible

  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_pages);
  const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_pages);
  const uint4 z = make_uint4(0, 0, 0, 0);
  float m0 = -INFINITY, m1 = -INFINITY;  // running max of heads 2tq, 2tq+1 (log2 units)
  float l0 = 0.f, l1 = 0.f;              // running sums (complete over the warp's tokens)
  float* wow = wo_dyn + (size_t)warp * 8 * OS;
  bool first = true;

  for (int k0 = 0; wid + k0 * WSTRIDE < ntiles; k0 += TP) {
    // ---- row offsets: lanes 16i .. 16i+15 look up tile i of this step
    long long off = off0;
    if (k0 > 0) {
      const bool act = (lane >> 4) < TP && slot_of(k0) < nt;
      off = act ? offset_of(__ldg(trow + slot_of(k0))) : -1;
    }
    // ---- K rows g, g+8 and V tokens 2tq, 2tq+1, 2tq+8, 2tq+9 of every tile
    uint4 kr0[TP][KJ], kr1[TP][KJ], vr[TP][4][VJ];
    long long oK0[TP], oK1[TP];
#pragma unroll
    for (int i = 0; i < TP; ++i) {
      oK0[i] = __shfl_sync(0xffffffffu, off, 16 * i + g);
      oK1[i] = __shfl_sync(0xffffffffu, off, 16 * i + g + 8);
      const long long oV[4] = {__shfl_sync(0xffffffffu, off, 16 * i + 2 * tq),
                               __shfl_sync(0xffffffffu, off, 16 * i + 2 * tq + 1),
                               __shfl_sync(0xffffffffu, off, 16 * i + 2 * tq + 8),
                               __shfl_sync(0xffffffffu, off, 16 * i + 2 * tq + 9)};
#pragma unroll
      for (int j = 0; j < KJ; ++j) {
        const int cb = (4 * j + tq) * 16;
        kr0[i][j] = oK0[i] >= 0 ? ldg16(kbase + oK0[i] + cb) : z;
        kr1[i][j] = oK1[i] >= 0 ? ldg16(kbase + oK1[i] + cb) : z;
      }
#pragma unroll
      for (int j = 0; j < VJ; ++j) {
        const int cb = (g + 8 * j) * 16;
#pragma unroll
        for (int u = 0; u < 4; ++u) vr[i][u][j] = oV[u] >= 0 ? ldg16(vbase + oV[u] + cb) : z;
      }
    }

    // ---- S^T = K . Q^T per tile: s[i][0], s[i][1] token g, heads 2tq, 2tq+1;
    // s[i][2], s[i][3] token g+8
    float s[TP][4];
#pragma unroll
    for (int i = 0; i < TP; ++i) {
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < KJ; ++j) {
        const uint32_t w0[4] = {kr0[i][j].x, kr0[i][j].y, kr0[i][j].z, kr0[i][j].w};
        const uint32_t w1[4] = {kr1[i][j].x, kr1[i][j].y, kr1[i][j].z, kr1[i][j].w};
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
      const bool ok0 = oK0[i] >= 0, ok1 = oK1[i] >= 0;
      s[i][0] = ok0 ? (sa[0] + sb[0]) * qk_scale : -INFINITY;
      s[i][1] = ok0 ? (sa[1] + sb[1]) * qk_scale : -INFINITY;
      s[i][2] = ok1 ? (sa[2] + sb[2]) * qk_scale : -INFINITY;
      s[i][3] = ok1 ? (sa[3] + sb[3]) * qk_scale : -INFINITY;
    }

    // ---- online softmax over the step's tokens, heads 2tq and 2tq+1
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int i = 0; i < TP; ++i) {
      mx0 = fmaxf(mx0, fmaxf(s[i][0], s[i][2]));
      mx1 = fmaxf(mx1, fmaxf(s[i][1], s[i][3]));
    }
#pragma unroll
    for (int d = 4; d <= 16; d <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, d));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, d));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
    // factors for what earlier steps accumulated (nothing when their max is -inf)
    const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - b0);
    const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - b1);
    m0 = mn0;
    m1 = mn1;
    uint32_t pb[TP][2];
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int i = 0; i < TP; ++i) {
      const float p0 = exp2f(s[i][0] - b0), p1 = exp2f(s[i][1] - b1);
      const float p2 = exp2f(s[i][2] - b0), p3 = exp2f(s[i][3] - b1);
      ls0 += p0 + p2;
      ls1 += p1 + p3;
      pb[i][0] = movmatrix_trans(pack2<FP8>(p0, p1));  // tokens 0..7 of tile i
      pb[i][1] = movmatrix_trans(pack2<FP8>(p2, p3));  // tokens 8..15
    }
#pragma unroll
    for (int d = 4; d <= 16; d <<= 1) {
      ls0 += __shfl_xor_sync(0xffffffffu, ls0, d);
      ls1 += __shfl_xor_sync(0xffffffffu, ls1, d);
    }
    l0 = l0 * f0 + ls0;
    l1 = l1 * f1 + ls1;

    // ---- O^T = V^T . P^T summed over the step's tiles; each m-tile is added
    // into the warp's slot as soon as it is done
#pragma unroll
    for (int j = 0; j < VJ; ++j) {
      const int c = g + 8 * j;
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        float oa[4] = {0.f, 0.f, 0.f, 0.f}, ob[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < TP; ++i) {
          const uint32_t va = word(vr[i][0][j], wd), vb = word(vr[i][1][j], wd);  // tokens 2tq, 2tq+1
          const uint32_t vc = word(vr[i][2][j], wd), vd = word(vr[i][3][j], wd);  // tokens 2tq+8, 2tq+9
          uint32_t af[4];
          if constexpr (FP8) {
            const uint32_t lo01 = __byte_perm(va, vb, 0x5140), hi01 = __byte_perm(va, vb, 0x7362);
            const uint32_t lo89 = __byte_perm(vc, vd, 0x5140), hi89 = __byte_perm(vc, vd, 0x7362);
            af[0] = e4m3x2_to_f16x2(lo01);
            af[1] = e4m3x2_to_f16x2(lo01 >> 16);
            af[2] = e4m3x2_to_f16x2(lo89);
            af[3] = e4m3x2_to_f16x2(lo89 >> 16);
            mma_f16(oa, af, pb[i][0], pb[i][1]);
            af[0] = e4m3x2_to_f16x2(hi01);
            af[1] = e4m3x2_to_f16x2(hi01 >> 16);
            af[2] = e4m3x2_to_f16x2(hi89);
            af[3] = e4m3x2_to_f16x2(hi89 >> 16);
            mma_f16(ob, af, pb[i][0], pb[i][1]);
          } else {
            af[0] = __byte_perm(va, vb, 0x5410);
            af[1] = __byte_perm(va, vb, 0x7632);
            af[2] = __byte_perm(vc, vd, 0x5410);
            af[3] = __byte_perm(vc, vd, 0x7632);
            mma_bf16(oa, af, pb[i][0], pb[i][1]);
          }
        }
        // output dims of this m-tile (and of the second one for FP8)
        const int mt = FP8 ? j * MTJ + 2 * wd : j * MTJ + wd;
        const int da = CH * c + 2 * (mt % MTJ);
        float2* pa0 = reinterpret_cast<float2*>(wow + (2 * tq) * OS + o_pos<SH>(da));
        float2* pa1 = reinterpret_cast<float2*>(wow + (2 * tq + 1) * OS + o_pos<SH>(da));
        if (first) {
          *pa0 = make_float2(oa[0], oa[2]);
          *pa1 = make_float2(oa[1], oa[3]);
        } else {
          const float2 u0 = *pa0, u1 = *pa1;
          *pa0 = make_float2(fmaf(u0.x, f0, oa[0]), fmaf(u0.y, f0, oa[2]));
          *pa1 = make_float2(fmaf(u1.x, f1, oa[1]), fmaf(u1.y, f1, oa[3]));
        }
        if constexpr (FP8) {
          const int db = CH * c + 2 * ((mt + 1) % MTJ);
          float2* pb0 = reinterpret_cast<float2*>(wow + (2 * tq) * OS + o_pos<SH>(db));
          float2* pb1 = reinterpret_cast<float2*>(wow + (2 * tq + 1) * OS + o_pos<SH>(db));
          if (first) {
            *pb0 = make_float2(ob[0], ob[2]);
            *pb1 = make_float2(ob[1], ob[3]);
          } else {
            const float2 u0 = *pb0, u1 = *pb1;
            *pb0 = make_float2(fmaf(u0.x, f0, ob[0]), fmaf(u0.y, f0, ob[2]));
            *pb1 = make_float2(fmaf(u1.x, f1, ob[1]), fmaf(u1.y, f1, ob[3]));
          }
        }
      }
    }
    first = false;
  }
  if (first) {  // a warp without tiles: its slot holds zeros, so merges need no branch
    for (int i = lane; i < 8 * OS / 4; i += 32) reinterpret_cast<float4*>(wow)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (g == 0) {
    wml[warp][2 * tq][0] = m0;  // -inf (and a slot never written) when the warp had no tokens
    wml[warp][2 * tq][1] = l0;
    wml[warp][2 * tq + 1][0] = m1;
    wml[warp][2 * tq + 1][1] = l1;
  }
  __syncthreads();

  // ---- merge the warps.  Every thread merges its items (head h, dims d..d+3)
  // itself: the head's max over the warps and each warp's rescale factor come
  // from the warps' (max, sum), so no per-head pass and no extra barrier.
  // The cluster's outputs are split among its CTAs: CTA r finishes items
  // [r * PER, (r + 1) * PER).  Every CTA pushes its share of item i (and its
  // per-head max and sum) into the owner's receive slots before ONE cluster
  // barrier; after it each CTA reads only its own shared memory.
  constexpr int ITEMS8 = 8 * (D / 4);
  constexpr int PER = (ITEMS8 + CL - 1) / CL;
  __shared__ float4 recv_o[CL][PER];
  __shared__ float recv_ml[CL][8][2];
  const size_t th0 = (size_t)t * a.Hq + h0;
  const int items = G * (D / 4);
  for (int idx = tid; idx < items; idx += NT) {
    const int h = idx / (D / 4), d = 4 * (idx % (D / 4));
    // every slot is written (zeros for warps without tiles): all loads go out at once
    float4 v[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) v[w] = ld_o4<SH>(wo_dyn + (w * 8 + h) * OS, d);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wml[w][h][0]);
    float L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = wml[w][h][0];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);  // -inf: the warp had no tokens
      L = fmaf(wml[w][h][1], f, L);
      O.x = fmaf(v[w].x, f, O.x); O.y = fmaf(v[w].y, f, O.y); O.z = fmaf(v[w].z, f, O.z); O.w = fmaf(v[w].w, f, O.w);
    }
    if constexpr (CL == 1) {
      write_out<OT, D>(a, th0 + h, d, O, M, L, vmul);
    } else {
      const int owner = idx / PER;
      *cl.map_shared_rank(&recv_o[rank][idx - owner * PER], owner) = O;
      if (d == 0) {  // the CTA's (max, sum) of head h, to every CTA
#pragma unroll
        for (int q = 0; q < CL; ++q) {
          float* dst = cl.map_shared_rank(&recv_ml[rank][h][0], q);
          dst[0] = M;
          dst[1] = L;
        }
      }
    }
  }
  if constexpr (CL > 1) {
    cl.sync();  // every push has landed; from here every access is local
    const int lo = rank * PER;
    const int hi = lo + PER < items ? lo + PER : items;
    for (int idx = lo + tid; idx < hi; idx += NT) {
      const int h = idx / (D / 4), d = 4 * (idx % (D / 4));
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < CL; ++q) M = fmaxf(M, recv_ml[q][h][0]);
      float L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < CL; ++q) {
        const float mq = recv_ml[q][h][0];
        const float f = mq == -INFINITY ? 0.f : exp2f(mq - M);
        L = fmaf(recv_ml[q][h][1], f, L);
        const float4 v = recv_o[q][idx - lo];
        O.x = fmaf(v.x, f, O.x); O.y = fmaf(v.y, f, O.y); O.z = fmaf(v.z, f, O.z); O.w = fmaf(v.w, f, O.w);
      }
      write_out<OT, D>(a, th0 + h, d, O, M, L, vmul);
    }
  }
}

// Clusters of CL CTAs of this instantiation that can be resident at once (the
// hardware places a cluster inside one GPC; with one CTA per SM not every GPC
// holds a whole number of clusters).  Cached per instantiation.
template <bool FP8, int D, typename QT, typename OT, int CL>
int max_active_clusters(size_t smem) {
  static int cached = -1;
  if (cached < 0) {
    auto kern = attn_cluster_kernel<FP8, D, QT, OT, CL>;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(CL, 1, 1);
      cfg.blockDim = dim3(kClWarps * 32);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = CL;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();  // a failed query leaves no sticky error behind
    cached = n;
  }
  return cached;
}

template <bool FP8, int D, typename QT, typename OT>
cudaError_t launch_cl_typed(const AttnArgs& a, float qk, float vmul, int max_cl, cudaStream_t s) {
  const int ys = a.Hkv * (a.Hq / a.Hkv > 8 ? 2 : 1);
  const int rows = ys * a.T;
  const dim3 block(kClWarps * 32);
  const size_t smem = (size_t)kClWarps * 8 * o_stride<D>() * sizeof(float);
  auto go = [&](auto kern, int cl) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e != cudaSuccess ? e : launch_k(kern, dim3(cl, ys, a.T), block, smem, s, cl, a, qk, vmul);
  };
  // the largest cluster (up to max_cl) for which every row's cluster is resident at once
  if (max_cl >= 8 && max_active_clusters<FP8, D, QT, OT, 8>(smem) >= rows)
    return go(attn_cluster_kernel<FP8, D, QT, OT, 8>, 8);
  if (max_cl >= 7 && max_active_clusters<FP8, D, QT, OT, 7>(smem) >= rows)
    return go(attn_cluster_kernel<FP8, D, QT, OT, 7>, 7);
  if (max_cl >= 6 && max_active_clusters<FP8, D, QT, OT, 6>(smem) >= rows)
    return go(attn_cluster_kernel<FP8, D, QT, OT, 6>, 6);
  if (max_cl >= 4 && max_active_clusters<FP8, D, QT, OT, 4>(smem) >= rows)
    return go(attn_cluster_kernel<FP8, D, QT, OT, 4>, 4);
  if (max_cl >= 2 && max_active_clusters<FP8, D, QT, OT, 2>(smem) >= rows)
    return go(attn_cluster_kernel<FP8, D, QT, OT, 2>, 2);
  return go(attn_cluster_kernel<FP8, D, QT, OT, 1>, 1);
}

template <bool FP8, int D>
cudaError_t launch_cl_q(const AttnArgs& a, float qk, float vmul, int CL, cudaStream_t s) {
  if (a.q_dt == QSA_BF16) {
    if (a.out_dt == QSA_BF16) return launch_cl_typed<FP8, D, __nv_bfloat16, __nv_bfloat16>(a, qk, vmul, CL, s);
    return launch_cl_typed<FP8, D, __nv_bfloat16, float>(a, qk, vmul, CL, s);
  }
  if (a.out_dt == QSA_BF16) return launch_cl_typed<FP8, D, float, __nv_bfloat16>(a, qk, vmul, CL, s);
  return launch_cl_typed<FP8, D, float, float>(a, qk, vmul, CL, s);
}

}  // namespace

int attn_cluster_tokens_per_round(qsa_dtype_t kv_dt, int D, int cl) {
  const bool two = kv_dt == QSA_FP8_E4M3 || D <= 128;
  return 16 * kClWarps * cl * (two ? 2 : 1);
}

cudaError_t launch_sparse_attn_cluster(const AttnArgs& a, float qk, float vmul, int cl, cudaStream_t s) {
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  if (a.D == 256) return fp8 ? launch_cl_q<true, 256>(a, qk, vmul, cl, s) : launch_cl_q<false, 256>(a, qk, vmul, cl, s);
  if (a.D == 128) return fp8 ? launch_cl_q<true, 128>(a, qk, vmul, cl, s) : launch_cl_q<false, 128>(a, qk, vmul, cl, s);
  return cudaErrorInvalidValue;
}

}  // namespace qsa
