// Log-sum-exp combine of split-KV partials (flash-decoding merge).
//
// For sequence b and head h with pieces c = 1..n holding (m_c, l_c, o_c) in base 2:
//   m* = max_c m_c,  L = sum_c 2^(m_c - m*) l_c,  out = sum_c 2^(m_c - m*) o_c / L,
//   lse = (m* + log2 L) * ln 2  (natural log of sum_j exp(s_j)).
// The merge order is fixed by piece index, so results do not depend on which CTA
// finished first.  One CTA per (sequence, block of heads); one thread per output
// element.
#include "common.cuh"
#include "launch.h"

namespace gva {

template <typename TO>
__global__ void __launch_bounds__(128)
    combine_kernel(const DecodeArgs a, TO* __restrict__ out, float* __restrict__ lse) {
  const int b = blockIdx.x;
  const int d_h = a.d_h, H = a.H;
  const int hpb = d_h >= 128 ? 1 : 128 / d_h;
  if (d_h < 128 && (int)threadIdx.x >= hpb * d_h) return;
  const int h = blockIdx.y * hpb + (d_h >= 128 ? 0 : threadIdx.x / d_h);
  if (h >= H) return;
  const int2 meta = a.meta[b];
  const int base = meta.x, n = meta.y;
  float mx = -INFINITY;
  for (int c = 0; c < n; ++c) mx = fmaxf(mx, a.part_ml[(size_t)(base + c) * H + h].x);
  float wsum = 0.f;
  for (int c = 0; c < n; ++c) {
    const float2 ml = a.part_ml[(size_t)(base + c) * H + h];
    wsum += ex2(ml.x - mx) * ml.y;
  }
  const float inv = n > 0 ? 1.f / wsum : 0.f;
  const int dstep = d_h >= 128 ? 128 : d_h;
  for (int d = (d_h >= 128 ? threadIdx.x : threadIdx.x % d_h); d < d_h; d += dstep) {
    float acc = 0.f;
    for (int c = 0; c < n; ++c) {
      const float w = ex2(a.part_ml[(size_t)(base + c) * H + h].x - mx);
      acc = fmaf(w, a.part_o[((size_t)(base + c) * H + h) * d_h + d], acc);
    }
    const float v = acc * inv;
    if constexpr (sizeof(TO) == 2) out[((size_t)b * H + h) * d_h + d] = __float2bfloat16_rn(v);
    else out[((size_t)b * H + h) * d_h + d] = v;
    if (d == 0 && lse) lse[(size_t)b * H + h] = n > 0 ? (mx + log2f(wsum)) * kLn2 : -INFINITY;
  }
}

cudaError_t launch_combine(const gva_shape_t& sh, const DecodeArgs& a, void* out, float* lse,
                           cudaStream_t st) {
  const int hpb = sh.d_h >= 128 ? 1 : 128 / sh.d_h;
  dim3 grid(sh.B, (sh.H + hpb - 1) / hpb);
  if (sh.out_dtype == GVA_BF16)
    combine_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(a, (__nv_bfloat16*)out, lse);
  else
    combine_kernel<float><<<grid, 128, 0, st>>>(a, (float*)out, lse);
  return cudaGetLastError();
}

}  // namespace gva
