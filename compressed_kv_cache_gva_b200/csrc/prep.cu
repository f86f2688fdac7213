// Query absorption and cache append for GVA decode.
//
// absorb: q~_h = q_h^nope M_h^T and RoPE(q_h^rope, pos), both times
//         softmax_scale*log2(e)  (onedev.kr review of GVA, "How it works": the
//         map is folded into the query once per token and head; "What differs":
//         only the positional slice is rotated).
// append: copy the grouped value, rotate the shared positional key by its own
//         position and store it rounded once to the cache type ("What differs":
//         k_rope = (x_j W_r) R_j^T, cached separately, shared by all heads).
#include "common.cuh"
#include "launch.h"

namespace gva {

// Nearest bf16 of a double, ties to even, without double rounding: truncate to
// float, then force the float's last bit to 1 when the truncation was inexact
// ("round to odd", Boldo & Melquiond 2008); a second rounding of that float to the
// 8-bit bf16 significand then equals the direct rounding of the double.
__device__ __forceinline__ __nv_bfloat16 f64_to_bf16_rne(double x) {
  float r = __double2float_rz(x);
  if ((double)r != x && isfinite(x)) r = __int_as_float(__float_as_int(r) | 1);
  return __float2bfloat16_rn(r);
}

template <typename T>
__device__ __forceinline__ void store_rounded(T* p, double x);
template <>
__device__ __forceinline__ void store_rounded<float>(float* p, double x) {
  *p = __double2float_rn(x);
}
template <>
__device__ __forceinline__ void store_rounded<__nv_bfloat16>(__nv_bfloat16* p, double x) {
  *p = f64_to_bf16_rne(x);
}

// Rotation of pair (i, i + d_r/2) at position pos; angle in float64.
__device__ __forceinline__ void rope_pair(double x1, double x2, double pos, int i, int d_r,
                                          double base, double& y1, double& y2) {
  const double inv_freq = pow(base, -2.0 * (double)i / (double)d_r);
  double s, c;
  sincos(pos * inv_freq, &s, &c);
  y1 = x1 * c - x2 * s;
  y2 = x1 * s + x2 * c;
}

// One CTA per head h: M_h staged in shared memory as float, then every query of
// the batch is multiplied by it.  Thread i < d_h owns output element i.
template <typename TQ>
__global__ void absorb_query_kernel(int B, int H, int d_h, int d_n, int d_r, double base,
                                    float c, const TQ* __restrict__ q, const TQ* __restrict__ M,
                                    const int* __restrict__ q_pos, float* __restrict__ q_abs) {
  extern __shared__ float sm[];
  float* Ms = sm;                       // [d_h][d_n + 1] (padded row)
  float* qs = sm + d_h * (d_n + 1);     // [d_n + d_r]
  const int h = blockIdx.x;
  const int ld = d_n + 1;
  for (int e = threadIdx.x; e < d_h * d_n; e += blockDim.x)
    Ms[(e / d_n) * ld + (e % d_n)] = to_f32(M[(size_t)h * d_h * d_n + e]);
  const int dq = d_n + d_r, dout = d_h + d_r;
  for (int b = 0; b < B; ++b) {
    __syncthreads();
    for (int e = threadIdx.x; e < dq; e += blockDim.x)
      qs[e] = to_f32(q[((size_t)b * H + h) * dq + e]);
    __syncthreads();
    float* o = q_abs + ((size_t)b * H + h) * dout;
    for (int i = threadIdx.x; i < d_h; i += blockDim.x) {
      float acc = 0.f;
      const float* row = Ms + i * ld;
      for (int k = 0; k < d_n; ++k) acc = fmaf(qs[k], row[k], acc);
      o[i] = acc * c;
    }
    const int half = d_r / 2;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
      double y1, y2;
      rope_pair(qs[d_n + i], qs[d_n + half + i], (double)q_pos[b], i, d_r, base, y1, y2);
      o[d_h + i] = (float)(y1 * (double)c);
      o[d_h + half + i] = (float)(y2 * (double)c);
    }
  }
}

// One warp per token: 16-byte copies of the value row, lanes 0..d_r/2-1 rotate
// one pair each of the positional key.
template <typename T>
__global__ void append_cache_kernel(int N, int row_elems, int d_r, double base,
                                    const T* __restrict__ v_new, const T* __restrict__ kpe_new,
                                    const int* __restrict__ slot, const int* __restrict__ pos,
                                    long long num_slots, T* __restrict__ V_cache,
                                    T* __restrict__ kr_cache, int* __restrict__ err_flag) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long long i = (long long)blockIdx.x * warps + (threadIdx.x >> 5); i < N;
       i += (long long)gridDim.x * warps) {
    const long long s = slot[i];
    if (s < 0 || s >= num_slots) {
      if (lane == 0 && err_flag) atomicExch(err_flag, 1);
      continue;
    }
    const int vec = 16 / sizeof(T);
    const uint4* src = reinterpret_cast<const uint4*>(v_new + i * row_elems);
    uint4* dst = reinterpret_cast<uint4*>(V_cache + s * row_elems);
    for (int e = lane; e < row_elems / vec; e += 32) dst[e] = src[e];
    const int half = d_r / 2;
    for (int p = lane; p < half; p += 32) {
      double y1, y2;
      rope_pair((double)to_f32(kpe_new[i * d_r + p]), (double)to_f32(kpe_new[i * d_r + half + p]),
                (double)pos[i], p, d_r, base, y1, y2);
      store_rounded(kr_cache + s * d_r + p, y1);
      store_rounded(kr_cache + s * d_r + half + p, y2);
    }
  }
}

cudaError_t launch_absorb(const gva_shape_t& sh, const void* q, const void* M, const int* q_pos,
                          float* q_abs, float c, cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)sh.d_h * (sh.d_n + 1) + sh.d_n + sh.d_r);
  const int threads = 128;
  if (sh.q_dtype == GVA_BF16) {
    auto k = absorb_query_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<sh.H, threads, smem, st>>>(sh.B, sh.H, sh.d_h, sh.d_n, sh.d_r, sh.rope_base, c,
                                   (const __nv_bfloat16*)q, (const __nv_bfloat16*)M, q_pos, q_abs);
  } else {
    auto k = absorb_query_kernel<float>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<sh.H, threads, smem, st>>>(sh.B, sh.H, sh.d_h, sh.d_n, sh.d_r, sh.rope_base, c,
                                   (const float*)q, (const float*)M, q_pos, q_abs);
  }
  return cudaGetLastError();
}

cudaError_t launch_append(const gva_shape_t& sh, int N, const void* v_new, const void* kpe_new,
                          const int* slot, const int* pos, long long num_slots, void* V_cache,
                          void* kr_cache, int* err_flag, cudaStream_t st) {
  const int threads = 256, warps = threads / 32;
  long long blocks = ((long long)N + warps - 1) / warps;
  int grid = (int)(blocks < 65535 * 8 ? blocks : 65535 * 8);
  const int row = sh.G * sh.d_h;
  if (sh.cache_dtype == GVA_BF16)
    append_cache_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
        N, row, sh.d_r, sh.rope_base, (const __nv_bfloat16*)v_new, (const __nv_bfloat16*)kpe_new,
        slot, pos, num_slots, (__nv_bfloat16*)V_cache, (__nv_bfloat16*)kr_cache, err_flag);
  else
    append_cache_kernel<float><<<grid, threads, 0, st>>>(
        N, row, sh.d_r, sh.rope_base, (const float*)v_new, (const float*)kpe_new, slot, pos,
        num_slots, (float*)V_cache, (float*)kr_cache, err_flag);
  return cudaGetLastError();
}

}  // namespace gva
