// Log-sum-exp combine of split-KV partials (flash-decoding merge).
//
// For sequence b and head h with pieces c = 1..n holding (m_c, l_c, o_c) in base 2:
//   m* = max_c m_c,  L = sum_c 2^(m_c - m*) l_c,  out = sum_c 2^(m_c - m*) o_c / L,
//   lse = (m* + log2 L) * ln 2  (natural log of sum_j exp(s_j)).
// The merge order is fixed by piece index, so results do not depend on which CTA
// finished first.
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace gva {

constexpr int kCombineScanMaxB = 64;   // batches up to this size find their pieces
                                        // from the lengths before waiting
// Target pieces per thread of the combine (loads requested at once); the launcher
// picks the block size from it and the expected pieces per sequence.
#ifndef GVA_COMBINE_PIECES   // measured on B200: 4 beats 8 on every decode workload here
#define GVA_COMBINE_PIECES 4
#endif
constexpr int kCombinePieces = GVA_COMBINE_PIECES;

// grid (B, H, ceil(d_h / 32)); block = 32 output columns x PG piece groups.
// Thread (pg, lane) merges pieces pg, pg+PG, ... of column d = 32*z + lane with
// its own running max; all its loads are requested before the first merge.  The
// PG running states are then merged through shared memory.  For small batches
// the piece range of sequence b is recomputed from the lengths (caller input)
// before waiting on the split kernel, so that after the wait only the partials
// are read.
template <typename TO, int PPT>
__global__ void __launch_bounds__(1024)
    combine_kernel(const DecodeArgs a, TO* __restrict__ out, float* __restrict__ lse) {
  __shared__ float sm_m[32][33], sm_l[32][33], sm_o[32][33];
  __shared__ int4 s_meta;
  const int b = blockIdx.x, h = blockIdx.y, d = blockIdx.z * 32 + (threadIdx.x & 31);
  const int H = a.H, d_h = a.d_h;
  const int tid = threadIdx.x, lane = tid & 31, pg = tid >> 5, npg = blockDim.x >> 5;
  // The next kernel may launch at once: every kernel of this library waits for its
  // predecessor before it reads what that one writes, so in a decode-step loop the
  // next step's first kernel and split kernel start (and the split kernel streams
  // its cache into SMs the finished split CTAs leave) while this combine runs.
  pdl_trigger();
  const bool scan = a.B <= kCombineScanMaxB;
  if (scan && pg == 0) {
    // tokens of the whole batch, tiles of sequences < b, of b and of the batch
    // (one warp), then the CTAs that own the first and last tile of b
    long long total = 0, before = 0, tiles = 0;
    int nb = 0;
    for (int j = lane; j < a.B; j += 32) {
      const int L = max(__ldg(a.seq_len + j), 0);
      const int n = (L + a.tile - 1) / a.tile;
      total += L;
      tiles += n;
      if (j < b) before += n;
      if (j == b) nb = n;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      total += __shfl_xor_sync(0xffffffffu, total, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
      tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
      nb += __shfl_xor_sync(0xffffffffu, nb, o);
    }
    if (lane == 0) {
      int4 m = make_int4(0, 0, 0, 0);
      if (nb > 0 && total < (1ll << 31)) {
        const TileSplit ts = make_split((int)tiles, a.grid, a.pool_per_cta);
        m = ts.slots(b, (int)before, (int)before + nb, a.B);
      }
      s_meta = m;
    }
  }
  pdl_wait();
  // the split kernel has completed: reset its pool counter for the next call
  if (a.pool_ctr && tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    *a.pool_ctr = 0;
#ifdef GVA_TRACE
  const int cid = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  if (a.trace && tid == 0 && cid < 16384) {
    unsigned long long tt;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tt));
    a.trace[4096 * 8 + cid * 2] = tt;
  }
#endif
  int4 meta;
  if (scan) {
    __syncthreads();
    meta = s_meta;
  } else {
    meta = a.meta[b];
  }
  // pieces 0 .. sc-1 are the static slots meta.x + c, pieces sc .. n-1 the pool
  // slots meta.z + c - sc, merged in this fixed order
  const int sc = meta.y, n = meta.y + meta.w;
  const int pool_shift = meta.z - meta.x - sc;
  const bool col = d < d_h;
  const float2* ml = a.part_ml + (size_t)meta.x * H + h;
  const float* po = a.part_o + ((size_t)meta.x * H + h) * d_h + (col ? d : 0);
  const size_t mstride = H, ostride = (size_t)H * d_h;
  float m = -INFINITY, l = 0.f, o = 0.f;
  for (int c0 = pg; c0 < n; c0 += PPT * npg) {
    float2 e[PPT];
    float x[PPT];
#pragma unroll
    for (int u = 0; u < PPT; ++u) {
      const int c = c0 + u * npg;
      if (c < n) {
        const long long sl = c < sc ? c : (long long)c + pool_shift;   // relative to meta.x
        e[u] = ml[sl * (long long)mstride];
        x[u] = po[sl * (long long)ostride];
      }
    }
#pragma unroll
    for (int u = 0; u < PPT; ++u) {
      if (c0 + u * npg >= n) break;
      if (e[u].x == -INFINITY) continue;          // piece past this query's causal limit
      const float mn = fmaxf(m, e[u].x);
      const float f = ex2(m - mn), w = ex2(e[u].x - mn);
      l = l * f + w * e[u].y;
      o = o * f + w * x[u];
      m = mn;
    }
  }
  sm_m[pg][lane] = m;
  sm_l[pg][lane] = l;
  sm_o[pg][lane] = o;
  __syncthreads();
  if (pg != 0) return;
  float M = -INFINITY;
  for (int u = 0; u < npg; ++u) M = fmaxf(M, sm_m[u][lane]);
  float L = 0.f, O = 0.f;
  for (int u = 0; u < npg; ++u) {
    const float mu = sm_m[u][lane];
    if (mu == -INFINITY) continue;                 // a group that saw no piece
    const float f = ex2(mu - M);
    L = fmaf(f, sm_l[u][lane], L);
    O = fmaf(f, sm_o[u][lane], O);
  }
  if (col) {
    const float v = L > 0.f ? O / L : 0.f;
    if constexpr (sizeof(TO) == 2) out[((size_t)b * H + h) * d_h + d] = __float2bfloat16_rn(v);
    else out[((size_t)b * H + h) * d_h + d] = v;
  }
  if (lane == 0 && blockIdx.z == 0 && lse)
    lse[(size_t)b * H + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
#ifdef GVA_TRACE
  if (a.trace && tid == 0 && cid < 16384) {
    unsigned long long tt;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tt));
    a.trace[4096 * 8 + cid * 2 + 1] = tt;
  }
#endif
}

cudaError_t launch_combine(const gva_shape_t& sh, const DecodeArgs& a, void* out, float* lse,
                           cudaStream_t st) {
  const dim3 grid(sh.B, sh.H, (sh.d_h + 31) / 32);
  // a sequence has about grid/B + 1 pieces (ragged batches: more for the long
  // ones); aim at ~kCombinePieces pieces per thread, 1..32 piece groups
  const int per_seq = a.grid * (1 + a.pool_per_cta) / (sh.B > 0 ? sh.B : 1) + 2;
  int npg = (per_seq + kCombinePieces - 1) / kCombinePieces;
  npg = npg < 1 ? 1 : (npg > 32 ? 32 : npg);
  // loads per thread: enough that one round covers the expected pieces when the
  // block is at its 1024-thread limit (a second round costs a full L2 latency)
  const int need = (per_seq + npg - 1) / npg;
  const int ppt = need <= kCombinePieces ? kCombinePieces : 16;   // 32 would spill at 1024 threads
  static_assert(kCombinePieces <= 16, "pieces per thread");
  auto go = [&](auto ppt_c, auto* o) {
    constexpr int K = decltype(ppt_c)::value;
    using TO = std::remove_pointer_t<decltype(o)>;
    return launch_pdl(combine_kernel<TO, K>, grid, dim3(32 * npg), 0, st, a, o, lse);
  };
  using K8 = std::integral_constant<int, kCombinePieces>;
  using K16 = std::integral_constant<int, (kCombinePieces > 16 ? kCombinePieces : 16)>;
  if (sh.out_dtype == GVA_BF16) {
    auto* o = (__nv_bfloat16*)out;
    return ppt <= kCombinePieces ? go(K8{}, o) : go(K16{}, o);
  }
  auto* o = (float*)out;
  return ppt <= kCombinePieces ? go(K8{}, o) : go(K16{}, o);
}

// Merge of R normalised attention states of the same queries over disjoint parts
// of each sequence's cache (one part per GPU when a sequence is split across
// GPUs): lse = log sum_r exp(lse_r), out = sum_r exp(lse_r - lse) out_r.
// One CTA per (sequence, head); threads over d_h.
template <typename TO>
__global__ void __launch_bounds__(128)
    merge_states_kernel(int R, int BH, int d_h, const float* __restrict__ outs,
                        const float* __restrict__ lses, TO* __restrict__ out,
                        float* __restrict__ lse) {
  const int bh = blockIdx.x;
  pdl_trigger();   // as in the combine: successors wait before they read
  pdl_wait();
  float mx = -INFINITY;
  for (int r = 0; r < R; ++r) mx = fmaxf(mx, lses[(size_t)r * BH + bh]);
  float z = 0.f;
  if (mx != -INFINITY)
    for (int r = 0; r < R; ++r) z += ex2((lses[(size_t)r * BH + bh] - mx) * kLog2e);
  for (int d = threadIdx.x; d < d_h; d += blockDim.x) {
    float acc = 0.f;
    if (mx != -INFINITY)
      for (int r = 0; r < R; ++r) {
        const float l = lses[(size_t)r * BH + bh];
        if (l == -INFINITY) continue;              // an empty part contributes nothing
        acc = fmaf(ex2((l - mx) * kLog2e), outs[((size_t)r * BH + bh) * d_h + d], acc);
      }
    const float v = mx != -INFINITY ? acc / z : 0.f;
    if constexpr (sizeof(TO) == 2) out[(size_t)bh * d_h + d] = __float2bfloat16_rn(v);
    else out[(size_t)bh * d_h + d] = v;
  }
  if (threadIdx.x == 0 && lse) lse[bh] = mx != -INFINITY ? mx + log2f(z) * kLn2 : -INFINITY;
}

cudaError_t launch_merge_states(const gva_shape_t& sh, int R, const float* outs, const float* lses,
                                void* out, float* lse, cudaStream_t st) {
  const int BH = sh.B * sh.H;
  const int threads = sh.d_h >= 128 ? 128 : ((sh.d_h + 31) / 32) * 32;
  if (sh.out_dtype == GVA_BF16)
    return launch_pdl(merge_states_kernel<__nv_bfloat16>, dim3(BH), dim3(threads), 0, st, R, BH,
                      sh.d_h, outs, lses, (__nv_bfloat16*)out, lse);
  return launch_pdl(merge_states_kernel<float>, dim3(BH), dim3(threads), 0, st, R, BH, sh.d_h,
                    outs, lses, (float*)out, lse);
}

}  // namespace gva
