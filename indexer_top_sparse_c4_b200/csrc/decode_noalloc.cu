// decode_noalloc.cu -- qsa_sparse_attn_decode_noalloc: the split-K decode
// attention with its scratch held in a fixed buffer inside the library, for
// callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not an option -- inside a
// CUDA-graph capture that must not allocate, under a memory pool that is
// already carved up, from a plugin or driver layer that was handed only the
// input and output buffers -- and so cannot provide the workspace that
// qsa_sparse_attn_decode asks for.
//
// The scratch is a file-scope __device__ array.  Every GPU that loads this
// library holds it until the process exits, so it is kept modest: requests
// whose split-K partials do not fit are refused with QSA_ERR_WORKSPACE.
// Host code may not pass the array's name to a kernel (in host code the name
// is a host-side shadow, not a device address), so the device address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on it.  The cached address belongs to the
// device's primary context (the one the CUDA runtime uses); a process that
// resets the device (cudaDeviceReset) or drives the library from another
// context must not call this entry point again on that device.
#include <stdio.h>

#include <mutex>

#include "qsa_internal.cuh"

namespace {

constexpr size_t kScratchFloats = QSA_DECODE_NOALLOC_SCRATCH_BYTES / sizeof(float);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_decode_scratch[kScratchFloats];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's scratch array (looked up once per device).
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

qsa_status_t qsa_sparse_attn_decode_noalloc(const void* q, qsa_dtype_t q_dt, const void* k_pages,
                                            const void* v_pages, qsa_dtype_t kv_dt, float k_scale,
                                            float v_scale, int num_pages,
                                            const int32_t* page_table, int pt_rows, int pt_stride,
                                            const int32_t* q_req, const int32_t* tok,
                                            const int32_t* n_tok, int W, int T, int Hq, int Hkv,
                                            int D, float sm_scale, void* out, qsa_dtype_t out_dt,
                                            float* lse, uint32_t* dev_status, qsa_stream_t stream) {
  // same checks and kernels as qsa_sparse_attn_decode; only the scratch
  // differs.  The arguments are checked first, so that a bad or unsupported
  // shape is reported as such and not as a scratch shortage.
  const qsa_status_t st = qsa::check_attn_args(q, q_dt, k_pages, v_pages, kv_dt, num_pages, page_table,
                                               pt_rows, pt_stride, tok, n_tok, W, T, Hq, Hkv, D, out,
                                               out_dt, k_scale, v_scale);
  if (st != QSA_OK || T == 0) return st;
  const size_t need = qsa_sparse_attn_decode_workspace_size(T, Hq, Hkv, D, W, kv_dt);
  if (need > kScratchFloats * sizeof(float)) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "qsa_sparse_attn_decode_noalloc: this shape needs %zu bytes of scratch; the built-in "
             "buffer holds %zu (use qsa_sparse_attn_decode with a workspace)",
             need, kScratchFloats * sizeof(float));
    qsa::set_last_error(msg);
    return QSA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof msg, "qsa_sparse_attn_decode_noalloc: scratch lookup failed: %s",
               cudaGetErrorString(e));
      qsa::set_last_error(msg);
      return QSA_ERR_CUDA;
    }
  }
  return qsa_sparse_attn_decode(q, q_dt, k_pages, v_pages, kv_dt, k_scale, v_scale, num_pages,
                                page_table, pt_rows, pt_stride, q_req, tok, n_tok, W, T, Hq, Hkv,
                                D, sm_scale, out, out_dt, lse, scratch,
                                kScratchFloats * sizeof(float), dev_status, stream);
}

}  // extern "C"
