// attn_common.cuh -- warp-level MMA fragments, FP8 decoding and token-row
// lookup shared by the tensor-core attention kernels of stage 4 (GQA attention
// over the selected tokens of a paged KV cache; "Qwen3.8-27B QSA - BF16 source
// weights", "QSA in brief": only the selected cache entries are read).
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "qsa_internal.cuh"

namespace qsa {
namespace attn {

constexpr float kLn2 = 0.69314718055994530942f;

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// four FP8-E4M3 codes (byte 0 first) -> two f16x2: codes 0, 1 in `lo`,
// codes 2, 3 in `hi`, exact; the word's halves feed the conversion directly
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t four, uint32_t& lo, uint32_t& hi) {
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n cvt.rn.f16x2.e4m3x2 %0, l;\n cvt.rn.f16x2.e4m3x2 %1, h;\n}\n"
      : "=r"(lo), "=r"(hi)
      : "r"(four));
}

// 2^x (base-2 exponential of the softmax; -inf gives +0)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool FP8> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<true>(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<false>(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds16(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }

// Tile geometry for one KV storage type and head dim.
template <bool FP8, int D>
struct Geo {
  static constexpr int EB = FP8 ? 1 : 2;       // bytes per element
  static constexpr int CH = 16 / EB;           // elements per 16-byte chunk
  static constexpr int NCH = D / CH;           // chunks per row
  static constexpr int KJ = NCH / 4;           // K chunks per thread per row
  static constexpr int KS = CH / 4;            // k-steps per chunk
  static constexpr int NKS = D / 16;           // k-steps per row
  static constexpr int VJ = NCH / 8;           // V chunks per thread per token
  static constexpr int MT = D / 16;            // PV m-tiles (output dims / 16)
  static constexpr int MTJ = CH / 2;           // m-tiles fed by one V chunk
  static constexpr int ROWB = D * EB;          // bytes of one K (or V) row of one KV head
  static_assert(NCH % 8 == 0, "V chunks must split over 8 lanes");
};

// Byte offset of the K/V row (this KV head) of token slot `i` of the list, or
// -1 for padding, a slot past `end`, or an id / page outside the cache.
__device__ __forceinline__ long long row_offset(const AttnArgs& a, const int32_t* trow,
                                                const int32_t* pt, int i, int end, int kvh,
                                                size_t row_bytes, size_t head_bytes) {
  if (i >= end) return -1;
  const int j = __ldg(trow + i);
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
  return (long long)(((size_t)page * kPageTokens + (j % kPageTokens)) * row_bytes + (size_t)kvh * head_bytes);
}

}  // namespace attn
}  // namespace qsa
