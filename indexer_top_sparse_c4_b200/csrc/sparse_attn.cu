// sparse_attn.cu -- stage 4 of QSA: GQA attention over only the selected
// tokens of a paged KV cache ("Qwen3.8-27B QSA - BF16 source weights", "QSA in
// brief": the selection decides which cache entries are read, nothing is
// compressed; Ascend CANN article, "Was der Pull Request tatsächlich
// hinzufügt": empty rows produce exact zeros, the 1/sqrt(D) scale is kept).
//
// General kernel (every dtype, D in {64,128,256}, up to 16 query heads per KV
// head).  CTA = (token split, KV head, query token).  Each warp walks every
// 4th selected token of the split: lane l holds dims [l*D/32, (l+1)*D/32) of
// the gathered K and V rows (one coalesced vector load each), the per-head
// dots are finished with a warp all-reduce, and an online softmax in base 2
// keeps a running max / sum per head with the unnormalised output in shared
// memory.  The four warps are merged at the end; with several splits the
// partial (o, max, sum) go to the workspace and a combine kernel finishes.
#include <math.h>

#include "qsa_internal.cuh"

namespace qsa {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxG = 16;
constexpr float kLn2 = 0.69314718055994530942f;

struct AttnScales {
  float qk;    // softmax scale * log2(e) (* k_scale for FP8): logits in base 2
  float vmul;  // v_scale for FP8, 1 otherwise
};

template <typename OT> __device__ __forceinline__ void store_out(OT* p, size_t i, float v);
template <> __device__ __forceinline__ void store_out<float>(float* p, size_t i, float v) { p[i] = v; }
template <> __device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, size_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

template <int D, typename QT, typename KVT, typename OT>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnArgs a, AttnScales sc, int splits,
                                                             int chunk, float* ws_o, float* ws_ml) {
  constexpr int VPT = D / 32;
  extern __shared__ __align__(16) float smem[];
  const int G = a.Hq / a.Hkv;
  float* q_s = smem;                        // [G][D]       scaled query
  float* o_s = q_s + G * D;                 // [warps][G][D] unnormalised outputs
  float* ml_s = o_s + kWarps * G * D;       // [warps][kMaxG][2] running max / sum
  const int s = blockIdx.x, kvh = blockIdx.y, t = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h0 = kvh * G;

  const QT* qp = reinterpret_cast<const QT*>(a.q) + ((size_t)t * a.Hq + h0) * D;
  for (int i = tid; i < G * D; i += kThreads) q_s[i] = Elem<QT>::get(qp, i) * sc.qk;
  for (int i = tid; i < kWarps * G * D; i += kThreads) o_s[i] = 0.f;
  __syncthreads();

  float m[kMaxG], l[kMaxG];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) { m[h] = -INFINITY; l[h] = 0.f; }

  int r = a.q_req ? a.q_req[t] : t;
  int nt = a.n_tok[t];
  nt = nt < 0 ? 0 : (nt > a.W ? a.W : nt);
  if (r < 0 || r >= a.pt_rows) {  // the whole row is skipped: zero output
    if (tid == 0 && s == 0) flag(a.status, QSA_DEV_BAD_REQUEST);
    r = 0;
    nt = 0;
  }
  const int beg = s * chunk;
  const int end = nt < beg + chunk ? nt : beg + chunk;
  const int32_t* trow = a.tok + (size_t)t * a.W;
  const int32_t* pt = a.page_table + (size_t)r * a.pt_stride;
  const KVT* kc = reinterpret_cast<const KVT*>(a.k_pages);
  const KVT* vc = reinterpret_cast<const KVT*>(a.v_pages);
  float* o_w = o_s + warp * G * D;

  for (int i = beg + warp; i < end; i += kWarps) {
    const int j = __ldg(trow + i);
    if (j == -1) continue;
    if (j < -1 || (j / kPageTokens) >= a.pt_stride) {
      if (lane == 0) flag(a.status, QSA_DEV_BAD_TOKEN);
      continue;
    }
    const int page = __ldg(pt + j / kPageTokens);
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0) flag(a.status, QSA_DEV_BAD_PAGE);
      continue;
    }
    const size_t base = (((size_t)page * kPageTokens + (j % kPageTokens)) * a.Hkv + kvh) * D + lane * VPT;
    float kf[VPT], vf[VPT];
    VecLoad<KVT, VPT>::get(kc, base, kf);
    VecLoad<KVT, VPT>::get(vc, base, vf);
    float dot[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      if (h < G) {
        const float* qh = q_s + h * D + lane * VPT;
        float d = 0.f;
#pragma unroll
        for (int jj = 0; jj < VPT; ++jj) d = fmaf(qh[jj], kf[jj], d);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        dot[h] = d;
      }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      if (h < G) {
        const float mn = fmaxf(m[h], dot[h]);
        const float alpha = exp2f(m[h] - mn);
        const float pr = exp2f(dot[h] - mn);
        l[h] = l[h] * alpha + pr;
        m[h] = mn;
        float* oh = o_w + h * D + lane * VPT;
#pragma unroll
        for (int jj = 0; jj < VPT; ++jj) oh[jj] = fmaf(oh[jj], alpha, pr * vf[jj]);
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      if (h < G) {
        ml_s[(warp * kMaxG + h) * 2] = m[h];
        ml_s[(warp * kMaxG + h) * 2 + 1] = l[h];
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, ml_s[(w * kMaxG + h) * 2]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = ml_s[(w * kMaxG + h) * 2];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - M);
        L = fmaf(ml_s[(w * kMaxG + h) * 2 + 1], f, L);
        O = fmaf(o_s[(w * G + h) * D + d], f, O);
      }
    }
    const size_t th = (size_t)t * a.Hq + h0 + h;
    if (splits == 1) {
      store_out<OT>(reinterpret_cast<OT*>(a.out), th * D + d, L > 0.f ? O / L * sc.vmul : 0.f);
      if (d == 0 && a.lse) a.lse[th] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    } else {
      ws_o[(th * splits + s) * D + d] = O;
      if (d == 0) {
        ws_ml[(th * splits + s) * 2] = M;
        ws_ml[(th * splits + s) * 2 + 1] = L;
      }
    }
  }
}

// Merge the per-split partials of one (query, head): every split's weight
// 2^(max_s - max) is computed once into shared memory, then each thread folds
// one float4 of the output over the splits.
template <typename OT>
__global__ void __launch_bounds__(256) attn_combine_kernel(AttnArgs a, AttnScales sc, int splits,
                                                           const float* ws_o, const float* ws_ml) {
  extern __shared__ __align__(16) float fs[];  // [splits] weights, then the group partials
  __shared__ float red[8];
  pdl_wait();
  const size_t th = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const float* ml = ws_ml + th * splits * 2;
  // thread -> (float4 column, split group); the first kPre partials of the
  // thread's group are loaded now, so their L2 latency overlaps the
  // reductions of the (max, sum) pairs below
  const float* po = ws_o + th * splits * a.D;
  const int ncol = a.D / 4;
  const int ngrp = blockDim.x / ncol;  // >= 1
  const int col = tid % ncol, grp = tid / ncol;
  constexpr int kPre = 4;
  float4 pre[kPre];
#pragma unroll
  for (int u = 0; u < kPre; ++u) {
    const int s = grp + u * ngrp;
    pre[u] = (grp < ngrp && s < splits) ? *reinterpret_cast<const float4*>(po + (size_t)s * a.D + 4 * col)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float M = -INFINITY;
  for (int s = tid; s < splits; s += blockDim.x) M = fmaxf(M, ml[2 * s]);
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
  for (int w = 1; w < nw; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  float L = 0.f;
  for (int s = tid; s < splits; s += blockDim.x) {
    const float ms = ml[2 * s];
    const float f = (M == -INFINITY || ms == -INFINITY) ? 0.f : exp2f(ms - M);
    fs[s] = f;
    L = fmaf(ml[2 * s + 1], f, L);
  }
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) L += __shfl_xor_sync(0xffffffffu, L, d);
  if (lane == 0) red[warp] = L;
  __syncthreads();
  L = 0.f;
  for (int w = 0; w < nw; ++w) L += red[w];
  pdl_launch_dependents();
  __syncthreads();  // fs complete
  const float inv = L > 0.f ? sc.vmul / L : 0.f;
  // the groups' sums meet in shared memory
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
  if (grp < ngrp) {
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
      const int s = grp + u * ngrp;
      const float f = s < splits ? fs[s] : 0.f;
      O.x = fmaf(pre[u].x, f, O.x); O.y = fmaf(pre[u].y, f, O.y);
      O.z = fmaf(pre[u].z, f, O.z); O.w = fmaf(pre[u].w, f, O.w);
    }
    int s = grp + kPre * ngrp;
    for (; s + 3 * ngrp < splits; s += 4 * ngrp) {  // four loads in flight
      float4 v[4];
      float f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        v[u] = *reinterpret_cast<const float4*>(po + (size_t)(s + u * ngrp) * a.D + 4 * col);
        f[u] = fs[s + u * ngrp];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        O.x = fmaf(v[u].x, f[u], O.x); O.y = fmaf(v[u].y, f[u], O.y);
        O.z = fmaf(v[u].z, f[u], O.z); O.w = fmaf(v[u].w, f[u], O.w);
      }
    }
    for (; s < splits; s += ngrp) {
      const float4 v = *reinterpret_cast<const float4*>(po + (size_t)s * a.D + 4 * col);
      const float f = fs[s];
      O.x = fmaf(v.x, f, O.x); O.y = fmaf(v.y, f, O.y); O.z = fmaf(v.z, f, O.z); O.w = fmaf(v.w, f, O.w);
    }
  }
  float4* part = reinterpret_cast<float4*>(fs + ((splits + 3) & ~3));  // [ngrp - 1][ncol]
  if (grp > 0 && grp < ngrp) part[(grp - 1) * ncol + col] = O;
  __syncthreads();
  if (grp == 0) {
    for (int q = 1; q < ngrp; ++q) {
      const float4 v = part[(q - 1) * ncol + col];
      O.x += v.x; O.y += v.y; O.z += v.z; O.w += v.w;
    }
    const size_t o0 = th * a.D + 4 * col;
    store_out<OT>(reinterpret_cast<OT*>(a.out), o0, O.x * inv);
    store_out<OT>(reinterpret_cast<OT*>(a.out), o0 + 1, O.y * inv);
    store_out<OT>(reinterpret_cast<OT*>(a.out), o0 + 2, O.z * inv);
    store_out<OT>(reinterpret_cast<OT*>(a.out), o0 + 3, O.w * inv);
  }
  if (tid == 0 && a.lse) a.lse[th] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

template <int D, typename QT, typename KVT, typename OT>
cudaError_t launch_typed(const AttnArgs& a, const AttnScales& sc, int splits, void* ws,
                         cudaStream_t s) {
  const int G = a.Hq / a.Hkv;
  const size_t smem = ((size_t)(1 + kWarps) * G * D + kWarps * kMaxG * 2) * sizeof(float);
  auto kern = attn_simt_kernel<D, QT, KVT, OT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int chunk = (a.W + splits - 1) / splits;
  float* ws_o = reinterpret_cast<float*>(ws);
  float* ws_ml = ws_o ? ws_o + (size_t)a.T * a.Hq * splits * D : nullptr;
  kern<<<dim3(splits, a.Hkv, a.T), kThreads, smem, s>>>(a, sc, splits, chunk, ws_o, ws_ml);
  return cudaGetLastError();
}

cudaError_t launch_combine(const AttnArgs& a, const AttnScales& sc, int splits, void* ws,
                           cudaStream_t s) {
  const float* ws_o = reinterpret_cast<const float*>(ws);
  const float* ws_ml = ws_o + (size_t)a.T * a.Hq * splits * a.D;
  // D/4 float4 columns x 4 split groups (128 threads at D = 128, 256 at D = 256)
  const int threads = a.D;
  const size_t smem = ((size_t)splits + 4) * sizeof(float) + (size_t)3 * (a.D / 4) * sizeof(float4);
  if (a.out_dt == QSA_F32)
    return launch_k(attn_combine_kernel<float>, dim3(a.T * a.Hq), dim3(threads), smem, s, 1, a, sc,
                    splits, ws_o, ws_ml);
  return launch_k(attn_combine_kernel<__nv_bfloat16>, dim3(a.T * a.Hq), dim3(threads), smem, s, 1,
                  a, sc, splits, ws_o, ws_ml);
}

template <int D, typename QT, typename KVT>
cudaError_t launch_out(const AttnArgs& a, const AttnScales& sc, int splits, void* ws, cudaStream_t s) {
  if (a.out_dt == QSA_F32) return launch_typed<D, QT, KVT, float>(a, sc, splits, ws, s);
  return launch_typed<D, QT, KVT, __nv_bfloat16>(a, sc, splits, ws, s);
}

template <int D, typename QT>
cudaError_t launch_kv(const AttnArgs& a, const AttnScales& sc, int splits, void* ws, cudaStream_t s) {
  switch (a.kv_dt) {
    case QSA_F32: return launch_out<D, QT, float>(a, sc, splits, ws, s);
    case QSA_BF16: return launch_out<D, QT, __nv_bfloat16>(a, sc, splits, ws, s);
    default: return launch_out<D, QT, __nv_fp8_e4m3>(a, sc, splits, ws, s);
  }
}

template <int D>
cudaError_t launch_q(const AttnArgs& a, const AttnScales& sc, int splits, void* ws, cudaStream_t s) {
  if (a.q_dt == QSA_F32) return launch_kv<D, float>(a, sc, splits, ws, s);
  return launch_kv<D, __nv_bfloat16>(a, sc, splits, ws, s);
}

}  // namespace

bool attn_mma_supported(const AttnArgs& a) {
  return (a.kv_dt == QSA_BF16 || a.kv_dt == QSA_FP8_E4M3) && (a.D == 128 || a.D == 256) &&
         a.Hq / a.Hkv <= 16;
}

DecodePlan attn_decode_plan(int T, int Hq, int Hkv, int D, int W, qsa_dtype_t kv_dt) {
  AttnArgs probe{};
  probe.kv_dt = kv_dt;
  probe.D = D;
  probe.Hq = Hq;
  probe.Hkv = Hkv > 0 ? Hkv : 1;
  DecodePlan p;
  if (attn_gather_supported(probe) && T * probe.Hkv < 148) {
    // fewer (query, KV head) rows than SMs: every row spread over CTAs on all
    // SMs, their partials merged by the combine kernel
    p.gather = true;
    p.gp = attn_gather_plan(T, Hq, probe.Hkv, D, W, kv_dt);
    p.s = p.gp.S;
  } else if (attn_mma_supported(probe)) {
    // enough rows to fill the GPU: one warp streams each row
    p.stream = true;
  } else {
    // general kernel: enough splits to spread small batches over the GPU
    const int rows = T * Hkv > 0 ? T * Hkv : 1;
    int s = (4 * 148 + rows - 1) / rows;
    const int max_s = (W + 63) / 64;
    p.s = s < max_s ? s : max_s;
    if (p.s < 1) p.s = 1;
  }
  return p;
}

size_t attn_decode_ws_bytes(int T, int Hq, int D, int splits) {
  if (splits <= 1) return 0;
  return (size_t)T * Hq * splits * (D + 2) * sizeof(float);
}

cudaError_t launch_sparse_attn(const AttnArgs& a, DecodePlan plan, void* ws, cudaStream_t s,
                               bool decode) {
  if (!decode) {
    plan = DecodePlan{};
    plan.stream = true;
  }
  const int splits = plan.s;
  if (a.T == 0) return cudaSuccess;
  const double scale = a.sm_scale > 0.f ? (double)a.sm_scale : 1.0 / sqrt((double)a.D);
  const bool fp8 = a.kv_dt == QSA_FP8_E4M3;
  AttnScales sc;
  sc.qk = (float)(scale * 1.4426950408889634 * (fp8 ? (double)a.k_scale : 1.0));
  sc.vmul = fp8 ? a.v_scale : 1.f;
  cudaError_t e;
  if (plan.gather) {
    e = launch_sparse_attn_gather(a, sc.qk, sc.vmul, plan.gp, ws, s);
  } else if (plan.stream && attn_mma_supported(a)) {
    e = launch_sparse_attn_prefill_rows(a, sc.qk, sc.vmul, s);
  } else {
    switch (a.D) {
      case 64: e = launch_q<64>(a, sc, splits, ws, s); break;
      case 128: e = launch_q<128>(a, sc, splits, ws, s); break;
      case 256: e = launch_q<256>(a, sc, splits, ws, s); break;
      default: return cudaErrorInvalidValue;
    }
  }
  if (e != cudaSuccess || splits == 1) return e;
  return launch_combine(a, sc, splits, ws, s);
}

}  // namespace qsa
