// Decode attention for callers that cannot allocate device memory.
//
// Same computation and kernels as gva_decode_attention; the only difference is
// where the split-KV scratch lives: in a fixed-size array in this library's own
// device memory instead of a caller-provided workspace.
#include <stdio.h>

#include <mutex>

#include "common.cuh"

namespace gva {
void set_error_message(const char* msg);   // defined in api.cu
gva_status_t decode_attention_clearing_status(const gva_shape_t* shape, const float* q_abs,
                                              const void* V_cache, const void* kr_cache,
                                              const int32_t* seq_offset, const int32_t* seq_len,
                                              int64_t max_total_tokens, int64_t num_slots,
                                              void* out, float* lse, void* workspace,
                                              size_t ws_bytes, void* stream);   // api.cu
}

namespace {

// The scratch itself.  Every GPU that loads this library holds it until exit,
// and all calls on a device share it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GVA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch on the current device, looked up once per device
// (the array's host-side name is only a stand-in and must never reach a kernel).
void* scratch_address() {
  static void* addr[64];
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    gva::set_error_message("no current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      char msg[200];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the static scratch failed: %s",
               cudaGetErrorString(e));
      gva::set_error_message(msg);
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" gva_status_t gva_decode_attention_noalloc(const gva_shape_t* shape, const float* q_abs,
                                                     const void* V_cache, const void* kr_cache,
                                                     const int32_t* seq_offset,
                                                     const int32_t* seq_len,
                                                     int64_t max_total_tokens, int64_t num_slots,
                                                     void* out, float* lse, void* stream) {
  const size_t need = gva_decode_workspace_size(shape, max_total_tokens);
  if (need == 0) return GVA_ERR_INVALID_ARG;   // reason already recorded
  if (need > (size_t)GVA_NOALLOC_SCRATCH_BYTES) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "this shape needs %zu bytes of scratch; the static scratch holds %zu "
             "(use gva_decode_attention with a workspace)",
             need, (size_t)GVA_NOALLOC_SCRATCH_BYTES);
    gva::set_error_message(msg);
    return GVA_ERR_WORKSPACE;
  }
  void* ws = scratch_address();
  if (!ws) return GVA_ERR_CUDA;
  // The previous call's device status word must not leak into this one: the
  // decode zeroes it on the stream after all its checks have passed, so a call
  // rejected on the host writes nothing into the shared scratch.
  return gva::decode_attention_clearing_status(shape, q_abs, V_cache, kr_cache, seq_offset, seq_len,
                                               max_total_tokens, num_slots, out, lse, ws,
                                               (size_t)GVA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" gva_status_t gva_noalloc_status(int32_t* status_out, void* stream) {
  if (!status_out) {
    gva::set_error_message("status_out is NULL");
    return GVA_ERR_INVALID_ARG;
  }
  void* ws = scratch_address();
  if (!ws) return GVA_ERR_CUDA;
  // the status word is the first int32 of the scratch (the workspace layout)
  const cudaError_t e = cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDefault,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    char msg[200];
    snprintf(msg, sizeof(msg), "copying the static scratch status word failed: %s",
             cudaGetErrorString(e));
    gva::set_error_message(msg);
    return GVA_ERR_CUDA;
  }
  return GVA_OK;
}
