// qsa_internal.cuh -- shared device helpers and the internal launcher
// declarations of libqsa.so.  Not part of the public ABI (include/qsa.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <utility>

#include "../../include/qsa.h"

namespace qsa {

constexpr int kPageTokens = 64;                        // tokens per KV page
constexpr int kGroupTokens = 4;                        // tokens per compressed group (C4)
constexpr int kPageGroups = kPageTokens / kGroupTokens;  // groups per page

// ---- value loads ----------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float get(const float* p, size_t i) { return __ldg(p + i); }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float get(const __nv_bfloat16* p, size_t i) {
    return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short*>(p) + i));
  }
};
template <> struct Elem<__nv_fp8_e4m3> {
  static __device__ __forceinline__ float get(const __nv_fp8_e4m3* p, size_t i) {
    const __nv_fp8_storage_t c = __ldg(reinterpret_cast<const unsigned char*>(p) + i);
    return __half2float(__half(__nv_cvt_fp8_to_halfraw(c, __NV_E4M3)));
  }
};

// Load N consecutive elements starting at element index i (i*sizeof(T) and
// N*sizeof(T) chosen by the callers so the access is a single aligned vector
// load) and widen them to float.
template <typename T, int N> struct VecLoad;
template <int N> struct VecLoad<float, N> {
  static __device__ __forceinline__ void get(const float* p, size_t i, float* out) {
    if constexpr (N == 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(p + i));
      out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    } else if constexpr (N == 2) {
      const float2 v = __ldg(reinterpret_cast<const float2*>(p + i));
      out[0] = v.x; out[1] = v.y;
    } else if constexpr (N == 8) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(p + i));
      const float4 b = __ldg(reinterpret_cast<const float4*>(p + i + 4));
      out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
      out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) out[j] = __ldg(p + i + j);
    }
  }
};
template <int N> struct VecLoad<__nv_bfloat16, N> {
  static __device__ __forceinline__ void get(const __nv_bfloat16* p, size_t i, float* out) {
    const unsigned short* s = reinterpret_cast<const unsigned short*>(p) + i;
    if constexpr (N == 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(s));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        out[2 * j] = __uint_as_float(w[j] << 16);
        out[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    } else if constexpr (N == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(s));
      out[0] = __uint_as_float(v.x << 16); out[1] = __uint_as_float(v.x & 0xffff0000u);
      out[2] = __uint_as_float(v.y << 16); out[3] = __uint_as_float(v.y & 0xffff0000u);
    } else if constexpr (N == 2) {
      const uint32_t v = __ldg(reinterpret_cast<const unsigned int*>(s));
      out[0] = __uint_as_float(v << 16); out[1] = __uint_as_float(v & 0xffff0000u);
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) out[j] = bf16_bits_to_f32(__ldg(s + j));
    }
  }
};
template <int N> struct VecLoad<__nv_fp8_e4m3, N> {
  static __device__ __forceinline__ void get(const __nv_fp8_e4m3* p, size_t i, float* out) {
    const unsigned char* s = reinterpret_cast<const unsigned char*>(p) + i;
    if constexpr (N == 8) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(s));
      const uint32_t w[2] = {v.x, v.y};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] & 0xffffu), __NV_E4M3);
        const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[j] >> 16), __NV_E4M3);
        const float2 a = __half22float2(__half2(lo));
        const float2 b = __half22float2(__half2(hi));
        out[4 * j] = a.x; out[4 * j + 1] = a.y; out[4 * j + 2] = b.x; out[4 * j + 3] = b.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < N; ++j) out[j] = Elem<__nv_fp8_e4m3>::get(p, i + j);
    }
  }
};

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// ---- score order ---------------------------------------------------------------
// float -> uint32 whose unsigned order equals the float order; -0 maps like +0.
// 0 is below every finite or infinite score: the Top-K uses it for "no candidate".
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
// Prefix histogram of a score row: counts of the top kPrefixBits bits of the
// order keys of the row's candidate scores (QSA_PREFIX_HIST_BINS per row).
constexpr int kPrefixBits = 12;
constexpr int kPrefixBins = 1 << kPrefixBits;
constexpr int kPrefixShift = 32 - kPrefixBits;
static_assert(kPrefixBins == QSA_PREFIX_HIST_BINS, "prefix histogram width");

// ---- radix select helper -------------------------------------------------------
// The bin (0..255) holding the need-th largest of the counted keys, scanning
// from the top, and the rank left inside it: warp 0 reads 8 bins per lane,
// finds the lane by a warp scan from the top, then the bin inside the lane.
__device__ __forceinline__ void find_bin_from_top(const int* hist, int need, int* s_bin, int* s_need) {
  const int lane = threadIdx.x & 31;
  if (threadIdx.x >= 32) return;
  // lane l holds bins 255 - 8l .. 248 - 8l (highest first)
  int c[8];
  int sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = hist[255 - 8 * lane - j];
    sum += c[j];
  }
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += y;
  }
  const int excl = incl - sum;
  const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
  const int L = hit ? __ffs(hit) - 1 : 31;
  if (lane == L) {
    int acc = excl, b = 255 - 8 * lane;
    int j = 0;
    for (; j < 7; ++j) {
      if (acc + c[j] >= need) break;
      acc += c[j];
    }
    b -= j;
    *s_bin = b;
    *s_need = need - acc;
  }
}

// ---- programmatic dependent launch (PDL) ----------------------------------------
// Every kernel of the library is launched with programmatic stream
// serialisation, so its CTAs may be scheduled while the previous kernel on the
// stream is still finishing.  pdl_wait() blocks until that kernel has
// completed and its memory is visible; a kernel calls it before its first
// access to global memory (it returns at once when there is no such kernel).
// pdl_launch_dependents() lets the next kernel's CTAs be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kern` on `s` with PDL enabled and, when cluster > 1, a
// (cluster, 1, 1) thread-block cluster.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---- launchers (one per stage; defined in the stage's .cu file) -----------------

struct IndexArgs {
  const void* q_idx; qsa_dtype_t q_dt; const float* w_idx;
  const void* k_idx_pages; qsa_dtype_t k_dt; int num_pages;
  const int32_t* page_table; int pt_rows, pt_stride; const int32_t* q_req; const int32_t* q_pos;
  int T, H_I, D_I; float* scores; int score_stride; uint32_t* status;
  uint32_t* hist = nullptr;  // optional [T][kPrefixBins] prefix histogram (decode scan only)
};
cudaError_t launch_index_scores(const IndexArgs& a, cudaStream_t s);
// Prefill indexer on tcgen05 (BF16 query and keys, H_I = 4, D_I = 128, T >= 32)
bool index_tc_supported(const IndexArgs& a);
cudaError_t launch_index_scores_tc(const IndexArgs& a, cudaStream_t s);

struct TopkArgs {
  const float* scores; int score_stride; const int32_t* q_pos; int T, K;
  int32_t* sel; int32_t* n_sel; uint32_t* status;
  // optional: also expand the kept groups to token ids (no MTP capture);
  // tok == nullptr skips it
  int32_t* tok = nullptr; int32_t* n_tok = nullptr; int W = 0;
  // optional [T][kPrefixBins] prefix histogram from the scan: read in place of
  // the first cluster passes where a row's total matches, then zeroed
  uint32_t* hist = nullptr;
  // guess-verify-refine with self-sampling (no histogram; row and cluster
  // kernels): the guess is a window of key bins read off a strided sample of
  // the row; path (optional) gets 0 dense, 1 the guess verified, 3 the radix passes
  int gvr = 0;
  int32_t* path = nullptr;
};
int topk_cluster_size(int score_stride);       // 0: unsupported
cudaError_t launch_topk_groups(const TopkArgs& a, cudaStream_t s);

struct ExpandArgs {
  const int32_t* sel; const int32_t* n_sel; int K; const int32_t* q_pos;
  const int32_t* capture_pos; int T; int32_t* tok; int32_t* n_tok; int W; uint32_t* status;
};
cudaError_t launch_expand_select(const ExpandArgs& a, cudaStream_t s);
cudaError_t launch_dense_select(const int32_t* q_pos, int T, int threshold, int32_t* tok, int32_t* n_tok, int W,
                                uint32_t* status, cudaStream_t s);

struct AttnArgs {
  const void* q; qsa_dtype_t q_dt; const void* k_pages; const void* v_pages; qsa_dtype_t kv_dt;
  float k_scale, v_scale; int num_pages; const int32_t* page_table; int pt_rows, pt_stride;
  const int32_t* q_req; const int32_t* tok; const int32_t* n_tok; int W, T, Hq, Hkv, D;
  float sm_scale; void* out; qsa_dtype_t out_dt; float* lse; uint32_t* status;
  // selection mode (gather kernel only; tok / n_tok unused): each row's token
  // slots follow from the kept groups as stage 3 would list them -- 4 per
  // kept group of sel [T, K] (n_sel of them), then 4*c(p0) .. p with p0 the
  // capture position (or p) -- cut at W
  const int32_t* sel = nullptr; const int32_t* n_sel = nullptr; int K = 0;
  const int32_t* q_pos = nullptr; const int32_t* capture_pos = nullptr;
};
// Plan of the decode kernel that spreads each (query, KV head) row over S
// CTAs of C token slots each; with S > 1 the combine kernel merges the S
// partials of a row.
struct GatherPlan {
  int S, C;
};
// How a decode call is spread over the GPU.
struct DecodePlan {
  int s = 1;             // partials per row merged by the combine kernel (1: none)
  bool stream = false;   // tensor-core path: one warp streams each (query, KV head) row
  bool gather = false;   // tensor-core path: the gather kernel with plan gp (s = gp.S)
  GatherPlan gp{1, 16};
};
DecodePlan attn_decode_plan(int T, int Hq, int Hkv, int D, int W, qsa_dtype_t kv_dt);
size_t attn_decode_ws_bytes(int T, int Hq, int D, int splits);
// decode == true: the decode plan is used; otherwise (prefill) one warp per
// (query, KV head) row streams all of its tokens.
cudaError_t launch_sparse_attn(const AttnArgs& a, DecodePlan plan, void* ws, cudaStream_t s,
                               bool decode);

// Tensor-core attention kernels (BF16 / FP8 caches, D in {128, 256}, <= 16
// query heads per KV head).
bool attn_mma_supported(const AttnArgs& a);
// Many rows: one warp per (query, KV head) row with all its query heads,
// K/V streamed through a per-warp cp.async ring.
cudaError_t launch_sparse_attn_prefill_rows(const AttnArgs& a, float qk_scale_log2, float vmul, cudaStream_t s);
// Decode kernel for few rows on every SM: rows split into chunks of one CTA
// each (one wave, one CTA per SM), token rows resolved once per chunk, K/V
// streamed through per-slot cp.async rings (sparse_attn_gather.cu).
bool attn_gather_supported(const AttnArgs& a);
GatherPlan attn_gather_plan(int T, int Hq, int Hkv, int D, int W, qsa_dtype_t kv_dt);
cudaError_t launch_sparse_attn_gather(const AttnArgs& a, float qk_scale_log2, float vmul, const GatherPlan& p,
                                      void* ws, cudaStream_t s);

// Indexer projection y[T, N] = x[T, H] . w[N, H]^T (indexer_write.cu): a GEMV
// for few tokens, a tcgen05 GEMM for BF16 prefill chunks.
struct ProjectArgs {
  const void* x; const void* w; int T, H, N; float* y; uint32_t* status;
};
bool project_tc_supported(const ProjectArgs& a, qsa_dtype_t x_dt, qsa_dtype_t w_dt);
cudaError_t launch_indexer_project(const ProjectArgs& a, qsa_dtype_t x_dt, qsa_dtype_t w_dt, cudaStream_t s);
// C4 compressed-key write (indexer_write.cu).
struct CompressArgs {
  const float* k_tok; int tok_stride; int n; const int32_t* g_req; const int32_t* g_id;
  const float* wphi; const float* bias; int D_I; void* k_idx_pages; int num_pages;
  const int32_t* page_table; int pt_rows, pt_stride; uint32_t* status;
};
cudaError_t launch_compress_keys(const CompressArgs& c, qsa_dtype_t k_dt, cudaStream_t s);

// Self-test of the bounded mbarrier wait (selftest.cu).
cudaError_t launch_selftest_wait(uint32_t limit_us, uint32_t* status, uint32_t* report, cudaStream_t s);

// Budgets the guess-verify-refine Top-K serves (topk_groups.cu, TopkArgs::gvr).
bool topk_gvr_budget(int K);

// Sequence-sharded decode (dcp.cu).
cudaError_t launch_dcp_positions(const int32_t* q_pos, int T, int g_lo, int g_hi, int32_t* q_pos_local,
                                 cudaStream_t s);
cudaError_t launch_dcp_candidates(const float* scores, int score_stride, const int32_t* sel, const int32_t* n_sel,
                                  int T, int K, int g_lo, float* cand_score, int32_t* cand_id, uint32_t* status,
                                  cudaStream_t s);
int dcp_merge_max_candidates();
cudaError_t launch_dcp_merge_topk(const float* cand_score, const int32_t* cand_id, int R, int T, int K, int32_t* sel,
                                  int32_t* n_sel, cudaStream_t s);
cudaError_t launch_dcp_expand(const int32_t* sel, const int32_t* n_sel, int K, const int32_t* q_pos, int T, int g_lo,
                              int g_hi, int32_t* tok, int32_t* n_tok, int W, uint32_t* status, cudaStream_t s);
cudaError_t launch_dcp_merge_attn(const float* o_parts, const float* lse_parts, int R, int T, int Hq, int D,
                                  void* out, qsa_dtype_t out_dt, float* lse, cudaStream_t s);

// Sets the message qsa_last_error_string() returns on this thread.
void set_last_error(const char* msg);
// The host-side argument checks of the attention calls (shapes, dtypes,
// pointers, alignment, FP8 scales); QSA_OK or the error, with its message set.
qsa_status_t check_attn_args(const void* q, qsa_dtype_t q_dt, const void* k_pages, const void* v_pages,
                             qsa_dtype_t kv_dt, int num_pages, const int32_t* page_table, int pt_rows,
                             int pt_stride, const int32_t* tok, const int32_t* n_tok, int W, int T,
                             int Hq, int Hkv, int D, void* out, qsa_dtype_t out_dt, float k_scale,
                             float v_scale);

}  // namespace qsa
