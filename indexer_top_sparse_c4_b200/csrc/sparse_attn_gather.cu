// sparse_attn_gather.cu -- stage 4 of QSA for decode batches: GQA attention
// over the selected tokens of a paged BF16 / FP8-E4M3 KV cache, every
// (query, KV head) row spread over several CTAs so that the batch fills all
// SMs in one wave ("Qwen3.8-27B QSA - BF16 source weights", "QSA in brief":
// only the selected cache entries are read, the cache itself is not
// compressed).
//
// A decode step has few (query, KV head) rows -- 16 at B8 -- each with 2K to
// 8K selected tokens scattered over a cache many times larger than L2.  The
// work is a gather: 512 B (FP8) or 1 KiB (BF16) of K and V per token and KV
// head, against 16 or 32 FLOP per byte of math.  What decides the time is how
// early and how many of those gathers are in flight, so the kernel is built
// around them:
//  * a row is cut into S chunks of token slots, one CTA each, and the grid
//    is one wave of one CTA per SM (S = 9 for the 16 rows of B8); each CTA
//    writes its partial (o, max, sum) to the workspace and the combine
//    kernel merges the S partials of a row;
//  * a CTA first turns its chunk's token ids into cache row indices (token id
//    -> page through the page table), one pass over the chunk, so the
//    dependent id -> page -> row lookups happen once and not per tile;
//  * SL slots of NT warps each (NT = 2 for 9-16 query heads per KV head, one
//    warp per n8 head tile) take the chunk's 16-token tiles in turn; each slot
//    streams its tiles through its own ring of shared-memory stages with
//    16-byte cp.async -- 192 KiB of stages per SM, most of them in flight --
//    and keeps its output accumulators in registers;
//  * per tile, the tensor-core arithmetic of the prefill kernel: S^T = K.Q^T
//    on m16n8k16 (tokens as M, heads as N), an online softmax in base 2 with
//    a lazy rescale, O^T += V^T.P^T (FP8 codes become f16 exactly);
//  * the slots merge in shared memory and the CTA writes its partial (or,
//    with one chunk per row, the output).
// Thread-block clusters would merge a row's CTAs on chip, but at one CTA per
// SM the GPU holds only 15 clusters of 8 (and 7 of 16) at once, too few for
// the 16 rows of B8 to use every SM in one wave.
// The 16-byte chunk c of staged row r sits at chunk c ^ sw(r), sw(r) =
// 2((r >> 1) & 3) ^ 4(r & 1): the K fragment reads (rows g, g+1 of a
// quarter-warp, chunks 4j..4j+3) and the V reads (rows 2tq + {0, 1, 8, 9},
// chunks g + 8j) then fall on eight distinct bank groups.
#include <math.h>

#include <type_traits>

#include "attn_common.cuh"

namespace qsa {
namespace {

using namespace attn;

constexpr int kGaMaxChunk = 1024;         // token slots one CTA resolves at most
constexpr int kGaSMs = 148;               // B200
constexpr int kGaRingBytes = 192 * 1024;  // stages per CTA (one CTA per SM)

__device__ __forceinline__ int ga_sw(int r) { return (((r >> 1) & 3) << 1) ^ ((r & 1) << 2); }

// slots per CTA: eight single-warp slots for FP8 rows of up to 8 heads per
// KV head, four otherwise (BF16 stages are twice the size; two-warp slots)
constexpr int ga_slots(bool fp8, int nt) { return fp8 && nt == 1 ? 8 : 4; }
template <bool FP8, int D, int NT>
constexpr int ga_stages() {
  constexpr int stage = 32 * Geo<FP8, D>::ROWB;  // 16 K rows + 16 V rows
  constexpr int s = kGaRingBytes / (ga_slots(FP8, NT) * stage);
  return s > 6 ? 6 : s;
}

// O slots of the slot merge: head h of slot s at [s][h][D + 4] floats, dim d
// at d ^ 2((d >> SH) & 7) (the float2 stores of one MMA m-tile fall on
// distinct banks; an aligned group of four dims stays one group)
template <int SH>
__device__ __forceinline__ int ga_opos(int d) {
  return d ^ (2 * ((d >> SH) & 7));
}
template <int SH>
__device__ __forceinline__ float4 ga_ld_o4(const float* head_base, int d) {
  const int x = 2 * ((d >> SH) & 7);
  const float4 v = *reinterpret_cast<const float4*>(head_base + (d ^ (x & ~3)));
  return (x & 2) ? make_float4(v.z, v.w, v.x, v.y) : v;
}

// Shared memory of one CTA (dynamic): the slot rings, reused by the slot
// merge once every slot is done, then the chunk's row-index table.
template <bool FP8, int D, int NT>
struct GaSmem {
  static constexpr int SL = ga_slots(FP8, NT);
  static constexpr int GM = 8 * NT;                        // query heads per CTA, padded
  static constexpr int STAGE = 32 * Geo<FP8, D>::ROWB;
  static constexpr int NS = ga_stages<FP8, D, NT>();
  static constexpr int RING = SL * NS * STAGE;
  static constexpr int MERGE = SL * GM * (D + 4) * 4 + SL * GM * 2 * 4;
  static constexpr int BODY = RING > MERGE ? RING : MERGE;
  static constexpr int off_tbl = BODY;
  static constexpr int bytes = off_tbl + kGaMaxChunk * 4;
  static_assert(NS >= 2, "at least two stages");
};

// grid: rows * S CTAs, row = blockIdx.x / S (row = t * Hkv + kvh), chunk
// s = blockIdx.x % S covering the token slots [s * C, s * C + C) of the row's
// list.  S > 1: the CTA's partial goes to ws_o [T * Hq][S][D] / ws_ml
// [T * Hq][S][2] for the combine kernel; S == 1: the CTA writes the output.
template <bool FP8, int D, typename QT, typename OT, int NT>
__global__ void __launch_bounds__(ga_slots(FP8, NT) * NT * 32, 1)
    attn_gather_kernel(AttnArgs a, float qk_scale, float vmul, int S, int C, float* ws_o, float* ws_ml) {
  using G_ = Geo<FP8, D>;
  using SM_ = GaSmem<FP8, D, NT>;
  constexpr int CH = G_::CH, NCH = G_::NCH, KJ = G_::KJ, KS = G_::KS, NKS = G_::NKS, VJ = G_::VJ,
                MT = G_::MT, MTJ = G_::MTJ, ROWB = G_::ROWB;
  constexpr int SL = SM_::SL, NS = SM_::NS, STAGE = SM_::STAGE, GM = SM_::GM;
  constexpr int NTHR = SL * NT * 32;
  constexpr int TPW = 16 / NT;    // token rows of a tile each warp of a slot stages
  constexpr int RPP = 32 / NCH;   // rows one lane pass covers when staging
  constexpr int OS = D + 4, SH = CH == 16 ? 5 : 4;
  static_assert(NCH >= 8 && 32 % NCH == 0 && TPW % RPP == 0, "row chunks must swizzle over 8 and tile a warp");
  extern __shared__ __align__(128) unsigned char smem[];
  int32_t* tbl = reinterpret_cast<int32_t*>(smem + SM_::off_tbl);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slot = warp / NT, u = warp % NT;
  const int g = lane >> 2, tq = lane & 3;
  const int row = blockIdx.x / S, s = blockIdx.x % S;
  const int t = row / a.Hkv, kvh = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int h0 = kvh * G;
  const int cbeg = s * C;

  pdl_wait();
  // ---- the chunk's cache rows: token id -> page -> row index (-1: skipped).
  // The ids, the row's length and its request are loaded together.
  int r = a.q_req ? __ldg(a.q_req + t) : t;
  constexpr int IPT = (kGaMaxChunk + NTHR - 1) / NTHR;  // ids per thread at most
  int jv[IPT];
  int nt;
  if (a.sel) {
    // selection mode: slot i of the row is token 4 g + i % 4 of kept group
    // g = sel[i / 4] while i < 4 n_sel, then 4 c(p0) + (i - 4 n_sel) up to p
    const int p = __ldg(a.q_pos + t);
    int p0 = a.capture_pos ? __ldg(a.capture_pos + t) : p;
    p0 = p0 > p ? p : p0;
    const int c0 = p0 >= 0 ? p0 / kGroupTokens : 0;
    int ns = __ldg(a.n_sel + t);
    ns = ns < 0 ? 0 : (ns > a.K ? a.K : ns);
    const int head = kGroupTokens * ns, total = head + (p >= 0 ? p - kGroupTokens * c0 + 1 : 0);
    nt = total < a.W ? total : a.W;
    if (total > a.W && s == 0 && kvh == 0 && tid == 0) flag(a.status, QSA_DEV_ROW_RANGE);
    const int32_t* srow = a.sel + (size_t)t * a.K;
#pragma unroll
    for (int k = 0; k < IPT; ++k) {
      const int i = tid + k * NTHR, ks = cbeg + i;
      int v = -1;
      if (i < C && ks < nt) {
        if (ks < head) {
          const int g = __ldg(srow + ks / kGroupTokens);
          if (g >= 0 && g < c0) v = kGroupTokens * g + ks % kGroupTokens;
          else if (ks % kGroupTokens == 0 && kvh == 0) flag(a.status, QSA_DEV_BAD_GROUP);
        } else {
          v = kGroupTokens * c0 + (ks - head);
        }
      }
      jv[k] = v;
    }
  } else {
    const int32_t* trow = a.tok + (size_t)t * a.W;
    nt = __ldg(a.n_tok + t);
#pragma unroll
    for (int k = 0; k < IPT; ++k) {
      const int i = tid + k * NTHR;
      jv[k] = (i < C && cbeg + i < a.W) ? __ldg(trow + cbeg + i) : -1;
    }
  }
  nt = nt < 0 ? 0 : (nt > a.W ? a.W : nt);
  if (r < 0 || r >= a.pt_rows) {
    if (tid == 0 && s == 0 && kvh == 0) flag(a.status, QSA_DEV_BAD_REQUEST);
    r = 0;
    nt = 0;
  }
  const int32_t* pt = a.page_table + (size_t)r * a.pt_stride;
  // the chunk slots [lo, hi) of the row-index table: token id -> page -> row
  auto resolve = [&](int lo, int hi) {
#pragma unroll
  for (int k = 0; k < IPT; ++k) {
    const int i = tid + k * NTHR;
    if (i >= lo && i < hi) {
      const int j = cbeg + i < nt ? jv[k] : -1;
      int ri = -1;
      if (j < -1 || (j >= 0 && j / kPageTokens >= a.pt_stride)) {
        if (kvh == 0) flag(a.status, QSA_DEV_BAD_TOKEN);
      } else if (j >= 0) {
        const int page = __ldg(pt + j / kPageTokens);
        if (page < 0 || page >= a.num_pages) {
          if (kvh == 0) flag(a.status, QSA_DEV_BAD_PAGE);
        } else {
          ri = page * kPageTokens + (j % kPageTokens);
        }
      }
      tbl[i] = ri;
    }
  }
  };
  // first the slots of every slot's first NS - 1 tiles (those are issued
  // before the loop); the rest while their copies are in flight
  const int c_first = C < 16 * SL * (NS - 1) ? C : 16 * SL * (NS - 1);
  resolve(0, c_first);

  // ---- Q^T B fragments of heads h0 + 8u + g (zero past G), head dim permuted
  // like K: k-steps j * KS .. j * KS + KS - 1 take dims CH (4j + tq) + 0..CH-1,
  // one contiguous run of the query row, read with vector loads
  uint32_t qb[NKS][2];
  {
    const int hg = 8 * u + g;
    const QT* qrow = reinterpret_cast<const QT*>(a.q) + ((size_t)t * a.Hq + h0 + (hg < G ? hg : 0)) * D;
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
#pragma unroll
      for (int h8 = 0; h8 < CH / 8; ++h8) {
        float v[8];
        if (hg < G) {
          VecLoad<QT, 8>::get(qrow, (size_t)(CH * (4 * j + tq) + 8 * h8), v);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {  // k-step j * KS + 2 h8 + q: elements 4q .. 4q + 3 of the eight
          qb[j * KS + 2 * h8 + q][0] = pack2<FP8>(v[4 * q], v[4 * q + 1]);
          qb[j * KS + 2 * h8 + q][1] = pack2<FP8>(v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
  }
  __syncthreads();  // the first tiles' rows are in the table

  const int clen = nt - cbeg < C ? nt - cbeg : C;             // slots of this chunk in the list
  const int ntiles = clen > 0 ? (clen + 15) / 16 : 0;          // tiles of the chunk
  const int myt = ntiles > slot ? (ntiles - slot + SL - 1) / SL : 0;  // this slot's tiles
  const size_t row_bytes = (size_t)a.Hkv * ROWB;
  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(a.k_pages) + (size_t)kvh * ROWB;
  const unsigned char* vbase = reinterpret_cast<const unsigned char*>(a.v_pages) + (size_t)kvh * ROWB;
  unsigned char* ring = smem + (size_t)slot * NS * STAGE;
  const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
  auto slot_sync = [&]() {
    if constexpr (NT > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + slot), "r"(NT * 32) : "memory");
    else __syncwarp();
  };

  // stage this warp's TPW rows of the slot's i-th tile (chunk tile slot + i * SL):
  // lane l copies chunk l % NCH of rows l / NCH, l / NCH + RPP, ... of K and V
  auto issue = [&](int i) {
    if (i < myt) {
      const int tb = 16 * (slot + i * SL);
      const uint32_t sb = ring_s + (uint32_t)((i % NS) * STAGE);
      const int c = lane % NCH;
#pragma unroll
      for (int r0 = 0; r0 < TPW; r0 += RPP) {
        const int rr = TPW * u + r0 + lane / NCH;  // row within the tile
        const int ri = tbl[tb + rr];               // tb + rr < 16 * ntiles <= C (+ 15)
        const uint32_t pos = (uint32_t)((c ^ ga_sw(rr)) * 16);
        const uint32_t dk = sb + rr * ROWB + pos, dv = sb + (16 + rr) * ROWB + pos;
        if (ri >= 0) {
          const size_t o = (size_t)ri * row_bytes + c * 16;
          cp_async16(dk, kbase + o);
          cp_async16(dv, vbase + o);
        } else {
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(dk), "r"(0) : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(dv), "r"(0) : "memory");
        }
      }
    }
    cp_async_commit();  // one group per tile (empty groups keep the count)
  };
#pragma unroll
  for (int i = 0; i < NS - 1; ++i) issue(i);
  if (c_first < C) {
    resolve(c_first, C);
    __syncthreads();  // the rest of the table is complete
  }

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, o[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  for (int i = 0; i < myt; ++i) {
    cp_async_wait<NS - 2>();   // this warp's copies of tile i have landed
    slot_sync();               // ... and the slot's other warp's; both are done with tile i - 1
    issue(i + NS - 1);         // into the stage tile i - 1 used
    const unsigned char* ks = ring + (size_t)(i % NS) * STAGE;
    const unsigned char* vs = ks + 16 * ROWB;
    const int tb = 16 * (slot + i * SL);
    const bool ok0 = tbl[tb + g] >= 0, ok1 = tbl[tb + g + 8] >= 0;

    // ---- S^T = K . Q^T for this warp's head tile (rows g and g+8 share a swizzle)
    // four independent accumulator chains (k-step kk feeds chain kk % 4): the
    // MMAs of a chain wait on each other, the chains do not
    float scc[4][4] = {};
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
      const int pc = ((4 * j + tq) ^ ga_sw(g)) * 16;
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
      const int sa = ga_sw(2 * tq), sb = ga_sw(2 * tq + 1);
      const uint4 A = lds16(vs + (2 * tq) * ROWB + ((c ^ sa) * 16));
      const uint4 B = lds16(vs + (2 * tq + 1) * ROWB + ((c ^ sb) * 16));
      const uint4 Cc = lds16(vs + (2 * tq + 8) * ROWB + ((c ^ sa) * 16));
      const uint4 E = lds16(vs + (2 * tq + 9) * ROWB + ((c ^ sb) * 16));
      const uint32_t va[4] = {A.x, A.y, A.z, A.w};      // token 2tq
      const uint32_t vb[4] = {B.x, B.y, B.z, B.w};      // token 2tq+1
      const uint32_t vc[4] = {Cc.x, Cc.y, Cc.z, Cc.w};  // token 2tq+8
      const uint32_t vd[4] = {E.x, E.y, E.z, E.w};      // token 2tq+9
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
  cp_async_wait<0>();
#pragma unroll
  for (int d = 4; d <= 16; d <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, d);
    l1 += __shfl_xor_sync(0xffffffffu, l1, d);
  }
  __syncthreads();  // every slot is done with its ring: the merge area reuses it

  // ---- the slots' partials into the merge area: O of head 8u + 2tq (c0, c2)
  // and 8u + 2tq + 1 (c1, c3); rows g / g+8 of m-tile mt are dims d_lo, d_lo+1
  float* mo = reinterpret_cast<float*>(smem);                              // [SL][GM][OS]
  float* mml = reinterpret_cast<float*>(smem + (size_t)SL * GM * OS * 4);    // [SL][GM][2]
  {
    const int ha = 8 * u + 2 * tq, hb = ha + 1;
    float* oa = mo + ((size_t)slot * GM + ha) * OS;
    float* ob = mo + ((size_t)slot * GM + hb) * OS;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int d_lo = CH * (g + 8 * (mt / MTJ)) + 2 * (mt % MTJ);
      *reinterpret_cast<float2*>(oa + ga_opos<SH>(d_lo)) = make_float2(o[mt][0], o[mt][2]);
      *reinterpret_cast<float2*>(ob + ga_opos<SH>(d_lo)) = make_float2(o[mt][1], o[mt][3]);
    }
    if (g == 0) {  // max -inf and sum 0 when the slot had no tokens
      mml[((size_t)slot * GM + ha) * 2] = m0;
      mml[((size_t)slot * GM + ha) * 2 + 1] = l0;
      mml[((size_t)slot * GM + hb) * 2] = m1;
      mml[((size_t)slot * GM + hb) * 2 + 1] = l1;
    }
  }
  __syncthreads();

  // ---- merge the slots: every thread merges its items (head h, dims d..d+3)
  // itself; the head's max over the slots and each slot's rescale factor come
  // from the slots' (max, sum)
  const int items = (G < GM ? G : GM) * (D / 4);
  const size_t th0 = (size_t)t * a.Hq + h0;
  for (int idx = tid; idx < items; idx += NTHR) {
    const int h = idx / (D / 4), d = 4 * (idx % (D / 4));
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < SL; ++w) M = fmaxf(M, mml[(w * GM + h) * 2]);
    float L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < SL; ++w) {
      const float mw = mml[(w * GM + h) * 2];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);  // -inf: the slot had no tokens
      const float4 v = ga_ld_o4<SH>(mo + ((size_t)w * GM + h) * OS, d);
      L = fmaf(mml[(w * GM + h) * 2 + 1], f, L);
      O.x = fmaf(v.x, f, O.x); O.y = fmaf(v.y, f, O.y); O.z = fmaf(v.z, f, O.z); O.w = fmaf(v.w, f, O.w);
    }
    const size_t th = th0 + h;
    if (S > 1) {  // this chunk's partial, for the combine kernel
      *reinterpret_cast<float4*>(ws_o + (th * S + s) * D + d) = O;
      if (d == 0) {
        ws_ml[(th * S + s) * 2] = M;
        ws_ml[(th * S + s) * 2 + 1] = L;
      }
    } else {
      const float inv = L > 0.f ? vmul / L : 0.f;
      if constexpr (sizeof(OT) == 4) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + th * D + d) =
            make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
      } else {
        __nv_bfloat162 p[2] = {__floats2bfloat162_rn(O.x * inv, O.y * inv),
                               __floats2bfloat162_rn(O.z * inv, O.w * inv)};
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + th * D + d) =
            *reinterpret_cast<const uint2*>(p);
      }
      if (d == 0 && a.lse) a.lse[th] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
  }
}

template <bool FP8, int D, typename QT, typename OT>
cudaError_t launch_ga_typed(const AttnArgs& a, float qk, float vmul, const GatherPlan& p, void* ws,
                            cudaStream_t s) {
  const int G = a.Hq / a.Hkv;
  float* ws_o = p.S > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  float* ws_ml = ws_o ? ws_o + (size_t)a.T * a.Hq * p.S * D : nullptr;
  auto go = [&](auto kern, auto nt_tag) -> cudaError_t {
    constexpr int NT = decltype(nt_tag)::value;
    const size_t smem = (size_t)GaSmem<FP8, D, NT>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(a.T * a.Hkv * p.S), dim3(ga_slots(FP8, NT) * NT * 32), smem, s, 1, a, qk,
                    vmul, p.S, p.C, ws_o, ws_ml);
  };
  return G > 8 ? go(attn_gather_kernel<FP8, D, QT, OT, 2>, std::integral_constant<int, 2>())
               : go(attn_gather_kernel<FP8, D, QT, OT, 1>, std::integral_constant<int, 1>());
}

template <bool FP8, int D>
cudaError_t launch_ga_q(const AttnArgs& a, float qk, float vmul, const GatherPlan& p, void* ws, cudaStream_t s) {
  if (a.q_dt == QSA_BF16) {
    if (a.out_dt == QSA_BF16) return launch_ga_typed<FP8, D, __nv_bfloat16, __nv_bfloat16>(a, qk, vmul, p, ws, s);
    return launch_ga_typed<FP8, D, __nv_bfloat16, float>(a, qk, vmul, p, ws, s);
  }
  if (a.out_dt == QSA_BF16) return launch_ga_typed<FP8, D, float, __nv_bfloat16>(a, qk, vmul, p, ws, s);
  return launch_ga_typed<FP8, D, float, float>(a, qk, vmul, p, ws, s);
}

}  // namespace

GatherPlan attn_gather_plan(int T, int Hq, int Hkv, int D, int W, qsa_dtype_t kv_dt) {
  (void)D;
  GatherPlan p{1, 16};
  const int rows = T * Hkv > 0 ? T * Hkv : 1;
  const int G = Hkv > 0 ? Hq / Hkv : 1;
  const int SL = ga_slots(kv_dt == QSA_FP8_E4M3, G > 8 ? 2 : 1);
  const int tiles = (W + 15) / 16;
  int S = kGaSMs / rows;                               // one wave of one CTA per SM
  const int s_max = (tiles + SL - 1) / SL;             // at least one tile per slot
  if (S > s_max) S = s_max;
  const int s_min = (W + kGaMaxChunk - 1) / kGaMaxChunk;  // the row-index table's capacity
  if (S < s_min) S = s_min;
  if (S < 1) S = 1;
  p.S = S;
  p.C = ((W + S - 1) / S + 15) / 16 * 16;              // <= kGaMaxChunk as S >= s_min; S * C >= W
  return p;
}

bool attn_gather_supported(const AttnArgs& a) {
  // D and dtypes as the other tensor-core kernels, up to 16 query heads per KV head
  return attn_mma_supported(a) && a.Hq / a.Hkv <= 16;
}

cudaError_t launch_sparse_attn_gather(const AttnArgs& a, float qk, float vmul, const GatherPlan& p, void* ws,
                                      cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  if (a.D == 256) return fp8 ? launch_ga_q<true, 256>(a, qk, vmul, p, ws, s) : launch_ga_q<false, 256>(a, qk, vmul, p, ws, s);
  if (a.D == 128) return fp8 ? launch_ga_q<true, 128>(a, qk, vmul, p, ws, s) : launch_ga_q<false, 128>(a, qk, vmul, p, ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace qsa
