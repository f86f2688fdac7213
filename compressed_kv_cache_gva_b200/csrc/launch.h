// Internal launchers (host side), one per kernel family.  Called by api.cu after
// argument validation; each returns the launch's cudaError_t.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/gva.h"

#include <utility>

namespace gva {

struct DecodeArgs;

// Function attributes already applied on the current device (launch.cu): a
// launcher sets an attribute only when attr_applied() says the device has not
// yet received that value (or a larger one) for the kernel.
bool attr_applied(const void* kernel, int attr, long long value);
void attr_record(const void* kernel, int attr, long long value);

// Raise a kernel's dynamic shared-memory limit to at least `smem` bytes, once
// per kernel, device and size.
template <typename... KArgs>
cudaError_t ensure_max_smem(void (*k)(KArgs...), size_t smem) {
  const void* key = reinterpret_cast<const void*>(k);
  const int attr = (int)cudaFuncAttributeMaxDynamicSharedMemorySize;
  if (attr_applied(key, attr, (long long)smem)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) attr_record(key, attr, (long long)smem);
  return e;
}

// Launch with programmatic stream serialization allowed (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  // Every kernel asks for the maximum shared-memory carveout (once per device), so
  // consecutive kernels never force the SM to reconfigure its L1/shared split.
  const void* key = reinterpret_cast<const void*>(k);
  const int carve = (int)cudaFuncAttributePreferredSharedMemoryCarveout;
  if (!attr_applied(key, carve, 1) &&
      cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess)
    attr_record(key, carve, 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// early_trigger: let the next kernel launch at once.  The library's own calls pass
// false: the next kernel then launches once this one has exited with its stores
// made visible, since a decode reads the queries and cache rows before its wait.
cudaError_t launch_absorb(const gva_shape_t& sh, const void* q, const void* M, const int* q_pos,
                          float* q_abs, float c, cudaStream_t st, bool early_trigger = false);
size_t absorb_smem_bytes(const gva_shape_t& sh);

cudaError_t launch_append(const gva_shape_t& sh, int N, const void* v_new, const void* kpe_new,
                          const int* slot, const int* pos, long long num_slots, void* V_cache,
                          void* kr_cache, int* err_flag, cudaStream_t st,
                          bool early_trigger = false);

// Append and absorb of the fused decode step in one launch; it lets the next
// kernel launch at once.
cudaError_t launch_prep_step(const gva_shape_t& sh, const void* q, const void* M, const int* q_pos,
                             float* q_abs, float c, int N, const void* v_new, const void* kpe_new,
                             const int* slot, const int* pos, long long num_slots, void* V_cache,
                             void* kr_cache, int* err_flag, cudaStream_t st);

// Same-shape GQA: append (key rotated over d_h, value copied) and the first
// kernel of its decode step (query rotation + append; the next kernel may launch
// at once).
cudaError_t launch_gqa_append(const gva_shape_t& sh, int N, const void* k_new, const void* v_new,
                              const int* slot, const int* pos, long long num_slots, void* K_cache,
                              void* V_cache, int* err_flag, cudaStream_t st);
cudaError_t launch_gqa_prep(const gva_shape_t& sh, const void* q, const int* q_pos, float* q_rot,
                            int N, const void* k_new, const void* v_new, const int* slot,
                            const int* pos, long long num_slots, void* K_cache, void* V_cache,
                            int* err_flag, cudaStream_t st);

// Multi-token attention on tcgen05 (prefill_tc.cu): nq new tokens per sequence,
// causal among them, rows = tokens x heads of a group in blocks of 128.  The
// value tensor map's box is prefill_tile_rows(sh) x 64, the k_rope map's
// prefill_tile_rows(sh) x (16 or 32).  Writes out/lse directly (no workspace).
bool prefill_supported(const gva_shape_t& sh, int nq);
int prefill_tile_rows(const gva_shape_t& sh);
cudaError_t launch_prefill(const gva_shape_t& sh, int nq, const float* q_abs,
                           const int32_t* seq_offset, const int32_t* seq_len, long long num_slots,
                           void* out, float* lse, int* status, const CUtensorMap& tv,
                           const CUtensorMap& tk, cudaStream_t st);

// CUDA-core split kernel (any dtype / shape within limits).  Returns
// cudaErrorNotSupported for shapes it is not built for.
bool simt_supported(const gva_shape_t& sh, bool gqa);
int simt_grid(const gva_shape_t& sh, int num_sms, long long max_total_tokens, bool gqa);
int simt_tile();
cudaError_t launch_decode_simt(const gva_shape_t& sh, bool gqa, DecodeArgs& a, cudaStream_t st);

// Tensor-core split kernel with TMA staging (bf16 caches).
bool mma_supported(const gva_shape_t& sh, bool gqa);
int mma_grid(const gva_shape_t& sh, int num_sms, long long max_total_tokens, bool gqa);
int mma_tile(const gva_shape_t& sh, bool gqa);
cudaError_t launch_decode_mma(const gva_shape_t& sh, bool gqa, DecodeArgs& a,
                              const CUtensorMap& tm_x, const CUtensorMap& tm_v,
                              const CUtensorMap& tm_kr, cudaStream_t st);

// Opt-in tcgen05 split kernel (decode_tc.cu): one-token GVA decode with H/G = 4, bf16
// caches, d_h in {64, 128}, G in {4, 8}, d_r <= 32.  Tiles of 128 / G tokens; the
// value tensor map's box is that many rows x 64 columns, the k_rope map's that
// many rows x (16 or 32) columns.  Same partials and combine as the mma.sync kernel.
bool tc_decode_supported(const gva_shape_t& sh);
int tc_decode_tile(const gva_shape_t& sh);
int tc_decode_grid(const gva_shape_t& sh, int num_sms, long long max_total_tokens);
cudaError_t launch_decode_tc(const gva_shape_t& sh, DecodeArgs& a, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_kr, cudaStream_t st);

// Merge of R normalised states (out, lse) of the same queries (sequence split).
cudaError_t launch_merge_states(const gva_shape_t& sh, int R, const float* outs, const float* lses,
                                void* out, float* lse, cudaStream_t st);

// Log-sum-exp combine of the partials into the output.
cudaError_t launch_combine(const gva_shape_t& sh, const DecodeArgs& a, void* out, float* lse,
                           cudaStream_t st);

}  // namespace gva
