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

// Rotation of pair (i, i + d_r/2) at position pos; the angle pos * base^(-2i/d_r)
// is formed in float64 from a float64 frequency table.
__device__ __forceinline__ void rope_pair(double x1, double x2, double pos, double inv_freq,
                                          double& y1, double& y2) {
  double s, c;
  sincos(pos * inv_freq, &s, &c);
  y1 = x1 * c - x2 * s;
  y2 = x1 * s + x2 * c;
}

constexpr int kAbsorbQueries = 4;   // queries per CTA
constexpr int kAbsorbVecs = 16;     // 16-byte vectors of an M_h row held in registers

// 8 bf16 (or 4 float) elements of a 16-byte vector, widened to float.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void widen(const uint4& u, float* out) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void widen(const uint4& u, float* out) {
    out[0] = __uint_as_float(u.x); out[1] = __uint_as_float(u.y);
    out[2] = __uint_as_float(u.z); out[3] = __uint_as_float(u.w);
  }
};

// grid (H, ceil(B / 4), ceil(d_h / 32)), 8 warps.  Warp w < 4 computes 32
// elements of q~ for query b0 + w (lane = one row of M_h, whose 16-byte vectors
// are all requested before the first FMA); warp 4 + w rotates the positional
// slice of the same query (float64 angle; CTAs with z == 0 only).  Everything is
// computed before waiting on the preceding kernel (it reads caller inputs only);
// only the stores of q_abs come after.
template <typename TQ>
__device__ __forceinline__ void absorb_block(int h, int by, int bz, int B, int H, int d_h, int d_n,
                                             int d_r, float c, const TQ* __restrict__ q,
                                             const TQ* __restrict__ M,
                                             const int* __restrict__ q_pos,
                                             float* __restrict__ q_abs, const RopeTable& rt,
                                             float* sm, int early_trigger) {
  const int dq = d_n + d_r, dout = d_h + d_r;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = warp % kAbsorbQueries;
  const int b = by * kAbsorbQueries + qi;
  float* qv = sm + qi * dq;
  const bool active = b < B;
  const TQ* qrow = q + ((size_t)(active ? b : 0) * H + h) * dq;
  float* o = q_abs + ((size_t)(active ? b : 0) * H + h) * dout;
  if (warp < kAbsorbQueries) {
    const int i = bz * 32 + lane;                       // output element of this lane
    const bool row_ok = active && i < d_h;
    const TQ* row = M + ((size_t)h * d_h + (row_ok ? i : 0)) * d_n;
    constexpr int V = Vec16<TQ>::N;
    const bool vec = (d_n % V) == 0 && (reinterpret_cast<uintptr_t>(M) & 15) == 0;
    if (active)
      for (int e = lane; e < d_n; e += 32) qv[e] = to_f32(qrow[e]);
    __syncwarp();
    float acc0 = 0.f, acc1 = 0.f;
    if (vec) {
      for (int k0 = 0; k0 < d_n; k0 += kAbsorbVecs * V) {
        uint4 raw[kAbsorbVecs];
#pragma unroll
        for (int u = 0; u < kAbsorbVecs; ++u)
          if (row_ok && k0 + u * V < d_n) raw[u] = *reinterpret_cast<const uint4*>(row + k0 + u * V);
#pragma unroll
        for (int u = 0; u < kAbsorbVecs; ++u) {
          if (!(row_ok && k0 + u * V < d_n)) continue;
          float x[V];
          Vec16<TQ>::widen(raw[u], x);
#pragma unroll
          for (int j = 0; j < V; j += 2) {
            acc0 = fmaf(qv[k0 + u * V + j], x[j], acc0);
            acc1 = fmaf(qv[k0 + u * V + j + 1], x[j + 1], acc1);
          }
        }
      }
    } else if (row_ok) {
      for (int k = 0; k < d_n; ++k) acc0 = fmaf(qv[k], to_f32(row[k]), acc0);
    }
    pdl_wait();
    if (row_ok) o[i] = (acc0 + acc1) * c;
  } else {
    const int half = d_r / 2;
    const bool rope = active && bz == 0;
    const double pos = rope ? (double)q_pos[b] : 0.0;
    double y1[2] = {0.0, 0.0}, y2[2] = {0.0, 0.0};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int p = lane + 32 * u;
      if (rope && p < half)
        rope_pair(to_f32(qrow[d_n + p]), to_f32(qrow[d_n + half + p]), pos, rt.inv_freq[p], y1[u],
                  y2[u]);
    }
    pdl_wait();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int p = lane + 32 * u;
      if (rope && p < half) {
        o[d_h + p] = (float)(y1[u] * (double)c);
        o[d_h + half + p] = (float)(y2[u] * (double)c);
      }
    }
  }
}

template <typename TQ>
__global__ void __launch_bounds__(2 * kAbsorbQueries * 32)
    absorb_query_kernel(int B, int H, int d_h, int d_n, int d_r, float c, const TQ* __restrict__ q,
                        const TQ* __restrict__ M, const int* __restrict__ q_pos,
                        float* __restrict__ q_abs, const RopeTable rt, int early_trigger) {
  extern __shared__ float sm[];
  // With early_trigger the successor may launch right away: it waits on this
  // kernel before it reads q_abs.  A standalone absorb does not trigger: the
  // next kernel launches once every block has exited, its stores made visible
  // first, since a decode reads its query before its own wait.
  if (early_trigger) pdl_trigger();
  absorb_block<TQ>(blockIdx.x, blockIdx.y, blockIdx.z, B, H, d_h, d_n, d_r, c, q, M, q_pos, q_abs,
                   rt, sm, early_trigger);
  if (!early_trigger) __threadfence();
}

// One warp per token: the value row is loaded (16-byte vectors) and the
// positional pairs rotated before waiting on the preceding kernel; the stores
// into the cache come after.
template <typename T>
__device__ __forceinline__ void append_block(long long bx, int N, int row_elems, int d_r,
                                             const T* __restrict__ v_new,
                                             const T* __restrict__ kpe_new,
                                             const int* __restrict__ slot,
                                             const int* __restrict__ pos, long long num_slots,
                                             T* __restrict__ V_cache, T* __restrict__ kr_cache,
                                             int* __restrict__ err_flag, const RopeTable& rt,
                                             int early_trigger) {
  constexpr int kVecPerLane = 4;   // rows up to 32*4*16 bytes = 2 KB in registers
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long i = bx * warps + (threadIdx.x >> 5);
  const bool active = i < N;
  const long long s = active ? slot[i] : -1;
  const bool ok = active && s >= 0 && s < num_slots;
  const int vec = 16 / sizeof(T);
  const int nvec = row_elems / vec;
  const uint4* src = reinterpret_cast<const uint4*>(v_new + (ok ? i : 0) * row_elems);
  uint4 r[kVecPerLane];
#pragma unroll
  for (int u = 0; u < kVecPerLane; ++u)
    if (ok && lane + 32 * u < nvec) r[u] = src[lane + 32 * u];
  const int half = d_r / 2;
  double y1[2] = {0.0, 0.0}, y2[2] = {0.0, 0.0};   // d_r <= 128: two pairs per lane at most
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int p = lane + 32 * u;
    if (ok && p < half)
      rope_pair((double)to_f32(kpe_new[i * d_r + p]), (double)to_f32(kpe_new[i * d_r + half + p]),
                (double)pos[i], rt.inv_freq[p], y1[u], y2[u]);
  }
  pdl_wait();
  // No trigger here: a decode streams cache rows before its own wait, so the
  // kernel after a standalone append may launch only once the append's rows are
  // stored (at its exit).  In a fused step the kernel triggers at entry and the
  // split kernel leaves the appended rows alone until its wait.
  (void)early_trigger;
  if (active && !ok) {
    if (lane == 0 && err_flag) atomicExch(err_flag, 1);
    return;
  }
  if (!ok) return;
  uint4* dst = reinterpret_cast<uint4*>(V_cache + s * row_elems);
#pragma unroll
  for (int u = 0; u < kVecPerLane; ++u)
    if (lane + 32 * u < nvec) dst[lane + 32 * u] = r[u];
  for (int e = lane + 32 * kVecPerLane; e < nvec; e += 32) dst[e] = src[e];   // wider rows
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int p = lane + 32 * u;
    if (p < half) {
      store_rounded(kr_cache + s * d_r + p, y1[u]);
      store_rounded(kr_cache + s * d_r + half + p, y2[u]);
    }
  }
}

template <typename T>
__global__ void append_cache_kernel(int N, int row_elems, int d_r, const T* __restrict__ v_new,
                                    const T* __restrict__ kpe_new, const int* __restrict__ slot,
                                    const int* __restrict__ pos, long long num_slots,
                                    T* __restrict__ V_cache, T* __restrict__ kr_cache,
                                    int* __restrict__ err_flag, const RopeTable rt,
                                    int early_trigger) {
  // With early_trigger (never used by the standalone append) the successor could
  // launch right away; without it the successor launches once every block has
  // exited, its stores made visible first (a decode streams cache rows before
  // its own wait).
  if (early_trigger) pdl_trigger();
  append_block<T>(blockIdx.x, N, row_elems, d_r, v_new, kpe_new, slot, pos, num_slots, V_cache,
                  kr_cache, err_flag, rt, early_trigger);
  if (!early_trigger) __threadfence();
}

// The first two kernels of the fused decode step in one launch: blocks
// [0, n_absorb) absorb the queries (grid (H, ay, az) flattened), the rest append
// the new tokens (8 per block).  Each block does its loads and arithmetic, waits
// on the preceding kernel, then stores.  The successor (the split kernel) may
// launch at once: it streams only cache rows this kernel does not write before
// its own wait, and it waits on this kernel before it reads q_abs.
template <typename TQ, typename T>
__global__ void __launch_bounds__(256)
    prep_step_kernel(int n_absorb, int ay, int az, int B, int H, int d_h, int d_n, int d_r,
                     float c, const TQ* __restrict__ q, const TQ* __restrict__ M,
                     const int* __restrict__ q_pos, float* __restrict__ q_abs, int N,
                     int row_elems, const T* __restrict__ v_new, const T* __restrict__ kpe_new,
                     const int* __restrict__ slot, const int* __restrict__ pos,
                     long long num_slots, T* __restrict__ V_cache, T* __restrict__ kr_cache,
                     int* __restrict__ err_flag, const RopeTable rt) {
  extern __shared__ float sm[];
  pdl_trigger();
  const int bid = blockIdx.x;
  if (bid < n_absorb) {
    const int per_h = ay * az, r = bid % per_h;
    absorb_block<TQ>(bid / per_h, r / az, r % az, B, H, d_h, d_n, d_r, c, q, M, q_pos, q_abs, rt,
                     sm, 1);
  } else {
    append_block<T>(bid - n_absorb, N, row_elems, d_r, v_new, kpe_new, slot, pos, num_slots,
                    V_cache, kr_cache, err_flag, rt, 1);
  }
}

// ---------------------------------------------------------------------------
// Same-shape GQA: the matched baseline caches a key AND a value per group and
// token (onedev.kr review, "What differs": N_GQA = 2*T*G*d_h).  Its keys carry
// RoPE over the whole head width, pair (i, i + d_h/2) rotated by
// pos * base^(-2i/d_h); the key is stored rounded once to the cache type and the
// value unchanged.  The query of a step is rotated the same way (float32 out,
// unscaled: the decode kernel applies softmax_scale).
// ---------------------------------------------------------------------------

// One warp per new token: the value row and the key pairs are loaded and the
// rotation computed (one float64 sincos per pair index, shared by the groups)
// before waiting on the preceding kernel; the stores come after.
constexpr int kGqaMaxGroups = 8;   // key pairs of up to this many groups held in registers
template <typename T>
__device__ __forceinline__ void gqa_append_block(long long bx, int N, int G, int d_h,
                                                 const T* __restrict__ k_new,
                                                 const T* __restrict__ v_new,
                                                 const int* __restrict__ slot,
                                                 const int* __restrict__ pos, long long num_slots,
                                                 T* __restrict__ K_cache, T* __restrict__ V_cache,
                                                 int* __restrict__ err_flag, const RopeTable& rt,
                                                 int early_trigger) {
  constexpr int kVecPerLane = 4;   // value rows up to 2 KB in registers
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long i = bx * warps + (threadIdx.x >> 5);
  const bool active = i < N;
  const long long s = active ? slot[i] : -1;
  const bool ok = active && s >= 0 && s < num_slots;
  const int row = G * d_h, half = d_h / 2;
  const int nvec = row * (int)sizeof(T) / 16;
  const uint4* vs = reinterpret_cast<const uint4*>(v_new + (ok ? i : 0) * row);
  uint4 r[kVecPerLane];
#pragma unroll
  for (int u = 0; u < kVecPerLane; ++u)
    if (ok && lane + 32 * u < nvec) r[u] = vs[lane + 32 * u];
  const T* krow = k_new + (ok ? i : 0) * row;
  const bool kreg = G <= kGqaMaxGroups;
  float kx[kGqaMaxGroups][2][2];   // [group][pair index u][x1, x2]
#pragma unroll
  for (int g = 0; g < kGqaMaxGroups; ++g)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int k = lane + 32 * u;
      const bool on = ok && kreg && g < G && k < half;
      kx[g][u][0] = on ? to_f32(krow[g * d_h + k]) : 0.f;
      kx[g][u][1] = on ? to_f32(krow[g * d_h + half + k]) : 0.f;
    }
  double cs[2] = {1.0, 1.0}, sn[2] = {0.0, 0.0};   // d_h <= 128: two pair indices per lane
  if (ok) {
    const double p = (double)pos[i];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int k = lane + 32 * u;
      if (k < half) sincos(p * rt.inv_freq[k], &sn[u], &cs[u]);
    }
  }
  pdl_wait();
  // No trigger here: a decode streams cache rows before its own wait, so the
  // kernel after a standalone append may launch only once the append's rows are
  // stored (at its exit).  In a fused step the kernel triggers at entry and the
  // split kernel leaves the appended rows alone until its wait.
  (void)early_trigger;
  if (active && !ok) {
    if (lane == 0 && err_flag) atomicExch(err_flag, 1);
    return;
  }
  if (!ok) return;
  // value: bit-exact copy
  uint4* vd = reinterpret_cast<uint4*>(V_cache + s * row);
#pragma unroll
  for (int u = 0; u < kVecPerLane; ++u)
    if (lane + 32 * u < nvec) vd[lane + 32 * u] = r[u];
  for (int e = lane + 32 * kVecPerLane; e < nvec; e += 32) vd[e] = vs[e];   // wider rows
  // key: every group's pairs rotated, rounded once
  T* kd = K_cache + s * row;
  auto put = [&](int g, int u, double x1, double x2) {
    const int k = lane + 32 * u;
    store_rounded(kd + g * d_h + k, x1 * cs[u] - x2 * sn[u]);
    store_rounded(kd + g * d_h + half + k, x1 * sn[u] + x2 * cs[u]);
  };
  if (kreg) {
#pragma unroll
    for (int g = 0; g < kGqaMaxGroups; ++g)
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (g < G && lane + 32 * u < half) put(g, u, kx[g][u][0], kx[g][u][1]);
  } else {
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int k = lane + 32 * u;
        if (k < half) put(g, u, to_f32(krow[g * d_h + k]), to_f32(krow[g * d_h + half + k]));
      }
  }
}

// One warp per (sequence, head) row of the query: q_rot = RoPE(q, q_pos[b])
// over d_h, float32.
template <typename TQ>
__device__ __forceinline__ void gqa_qrot_block(long long bx, int rows, int H, int d_h,
                                               const TQ* __restrict__ q,
                                               const int* __restrict__ q_pos,
                                               float* __restrict__ q_rot, const RopeTable& rt,
                                               int early_trigger) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long r = bx * warps + (threadIdx.x >> 5);
  const bool active = r < rows;
  const int half = d_h / 2;
  double y1[2] = {0.0, 0.0}, y2[2] = {0.0, 0.0};
  if (active) {
    const double p = (double)q_pos[r / H];
    const TQ* qr = q + r * d_h;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int k = lane + 32 * u;
      if (k < half)
        rope_pair((double)to_f32(qr[k]), (double)to_f32(qr[half + k]), p, rt.inv_freq[k], y1[u],
                  y2[u]);
    }
  }
  pdl_wait();
  if (!early_trigger) pdl_trigger();
  if (!active) return;
  float* o = q_rot + r * d_h;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int k = lane + 32 * u;
    if (k < half) {
      o[k] = (float)y1[u];
      o[half + k] = (float)y2[u];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
    gqa_append_kernel(int N, int G, int d_h, const T* __restrict__ k_new,
                      const T* __restrict__ v_new, const int* __restrict__ slot,
                      const int* __restrict__ pos, long long num_slots, T* __restrict__ K_cache,
                      T* __restrict__ V_cache, int* __restrict__ err_flag, const RopeTable rt) {
  // no trigger: the successor launches once every block has exited, its stores
  // made visible first (a decode streams cache rows before its own wait)
  gqa_append_block<T>(blockIdx.x, N, G, d_h, k_new, v_new, slot, pos, num_slots, K_cache, V_cache,
                      err_flag, rt, 0);
  __threadfence();
}

// The first kernel of the GQA decode step, the counterpart of prep_step_kernel:
// blocks [0, n_qrot) rotate the queries (8 rows per block), the rest append the
// new tokens (8 per block).  The successor may launch at once (see
// prep_step_kernel).
template <typename TQ, typename T>
__global__ void __launch_bounds__(256)
    gqa_prep_kernel(int n_qrot, int rows, int H, int d_h, const TQ* __restrict__ q,
                    const int* __restrict__ q_pos, float* __restrict__ q_rot, int N, int G,
                    const T* __restrict__ k_new, const T* __restrict__ v_new,
                    const int* __restrict__ slot, const int* __restrict__ pos, long long num_slots,
                    T* __restrict__ K_cache, T* __restrict__ V_cache, int* __restrict__ err_flag,
                    const RopeTable rt) {
  pdl_trigger();
  if ((int)blockIdx.x < n_qrot)
    gqa_qrot_block<TQ>(blockIdx.x, rows, H, d_h, q, q_pos, q_rot, rt, 1);
  else
    gqa_append_block<T>(blockIdx.x - n_qrot, N, G, d_h, k_new, v_new, slot, pos, num_slots,
                        K_cache, V_cache, err_flag, rt, 1);
}

static RopeTable rope_table_width(double base, int width) {
  RopeTable t{};
  for (int i = 0; i < width / 2 && i < kMaxRopePairs; ++i)
    t.inv_freq[i] = pow(base, -2.0 * (double)i / (double)width);
  return t;
}

cudaError_t launch_gqa_append(const gva_shape_t& sh, int N, const void* k_new, const void* v_new,
                              const int* slot, const int* pos, long long num_slots, void* K_cache,
                              void* V_cache, int* err_flag, cudaStream_t st) {
  const int grid = (int)(((long long)N + 7) / 8);
  const RopeTable rt = rope_table_width(sh.rope_base, sh.d_h);
  if (sh.cache_dtype == GVA_BF16)
    return launch_pdl(gqa_append_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, N, sh.G,
                      sh.d_h, (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, slot, pos,
                      num_slots, (__nv_bfloat16*)K_cache, (__nv_bfloat16*)V_cache, err_flag, rt);
  return launch_pdl(gqa_append_kernel<float>, dim3(grid), dim3(256), 0, st, N, sh.G, sh.d_h,
                    (const float*)k_new, (const float*)v_new, slot, pos, num_slots,
                    (float*)K_cache, (float*)V_cache, err_flag, rt);
}

template <typename TQ, typename T>
static cudaError_t launch_gqa_prep_t(const gva_shape_t& sh, const void* q, const int* q_pos,
                                     float* q_rot, int N, const void* k_new, const void* v_new,
                                     const int* slot, const int* pos, long long num_slots,
                                     void* K_cache, void* V_cache, int* err_flag,
                                     cudaStream_t st) {
  const long long rows = (long long)sh.B * sh.H;
  const long long n_qrot = (rows + 7) / 8, n_app = ((long long)N + 7) / 8;
  if (n_qrot + n_app > 0x7fffffff) return cudaErrorInvalidConfiguration;
  return launch_pdl(gqa_prep_kernel<TQ, T>, dim3((unsigned)(n_qrot + n_app)), dim3(256), 0, st,
                    (int)n_qrot, (int)rows, sh.H, sh.d_h, (const TQ*)q, q_pos, q_rot, N, sh.G,
                    (const T*)k_new, (const T*)v_new, slot, pos, num_slots, (T*)K_cache,
                    (T*)V_cache, err_flag, rope_table_width(sh.rope_base, sh.d_h));
}

cudaError_t launch_gqa_prep(const gva_shape_t& sh, const void* q, const int* q_pos, float* q_rot,
                            int N, const void* k_new, const void* v_new, const int* slot,
                            const int* pos, long long num_slots, void* K_cache, void* V_cache,
                            int* err_flag, cudaStream_t st) {
  using bf = __nv_bfloat16;
  const bool qb = sh.q_dtype == GVA_BF16, cb = sh.cache_dtype == GVA_BF16;
  if (qb && cb)
    return launch_gqa_prep_t<bf, bf>(sh, q, q_pos, q_rot, N, k_new, v_new, slot, pos, num_slots,
                                     K_cache, V_cache, err_flag, st);
  if (qb)
    return launch_gqa_prep_t<bf, float>(sh, q, q_pos, q_rot, N, k_new, v_new, slot, pos,
                                        num_slots, K_cache, V_cache, err_flag, st);
  if (cb)
    return launch_gqa_prep_t<float, bf>(sh, q, q_pos, q_rot, N, k_new, v_new, slot, pos,
                                        num_slots, K_cache, V_cache, err_flag, st);
  return launch_gqa_prep_t<float, float>(sh, q, q_pos, q_rot, N, k_new, v_new, slot, pos,
                                         num_slots, K_cache, V_cache, err_flag, st);
}

static RopeTable rope_table(const gva_shape_t& sh) {
  RopeTable t{};
  for (int i = 0; i < sh.d_r / 2 && i < kMaxRopePairs; ++i)
    t.inv_freq[i] = pow(sh.rope_base, -2.0 * (double)i / (double)sh.d_r);
  return t;
}

size_t absorb_smem_bytes(const gva_shape_t& sh) {
  return sizeof(float) * (size_t)kAbsorbQueries * (sh.d_n + sh.d_r);
}

cudaError_t launch_absorb(const gva_shape_t& sh, const void* q, const void* M, const int* q_pos,
                          float* q_abs, float c, cudaStream_t st, bool early_trigger) {
  const size_t smem = absorb_smem_bytes(sh);
  const dim3 grid(sh.H, (sh.B + kAbsorbQueries - 1) / kAbsorbQueries, (sh.d_h + 31) / 32);
  const dim3 block(2 * kAbsorbQueries * 32);
  const RopeTable rt = rope_table(sh);
  if (sh.q_dtype == GVA_BF16) {
    auto k = absorb_query_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024) ensure_max_smem(k, smem);
    return launch_pdl(k, grid, block, smem, st, sh.B, sh.H, sh.d_h, sh.d_n, sh.d_r, c,
                      (const __nv_bfloat16*)q, (const __nv_bfloat16*)M, q_pos, q_abs, rt,
                      early_trigger ? 1 : 0);
  }
  auto k = absorb_query_kernel<float>;
  if (smem > 48 * 1024) ensure_max_smem(k, smem);
  return launch_pdl(k, grid, block, smem, st, sh.B, sh.H, sh.d_h, sh.d_n, sh.d_r, c, (const float*)q,
                    (const float*)M, q_pos, q_abs, rt, early_trigger ? 1 : 0);
}

template <typename TQ, typename T>
static cudaError_t launch_prep_t(const gva_shape_t& sh, const void* q, const void* M,
                                 const int* q_pos, float* q_abs, float c, int N, const void* v_new,
                                 const void* kpe_new, const int* slot, const int* pos,
                                 long long num_slots, void* V_cache, void* kr_cache, int* err_flag,
                                 cudaStream_t st) {
  const int ay = (sh.B + kAbsorbQueries - 1) / kAbsorbQueries, az = (sh.d_h + 31) / 32;
  const int n_absorb = sh.B > 0 ? sh.H * ay * az : 0;
  const long long n_append = ((long long)N + 7) / 8;     // 256 threads = 8 tokens per block
  const long long blocks = n_absorb + n_append;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const size_t smem = sh.B > 0 ? absorb_smem_bytes(sh) : 0;
  auto k = prep_step_kernel<TQ, T>;
  if (smem > 48 * 1024) ensure_max_smem(k, smem);
  return launch_pdl(k, dim3((unsigned)blocks), dim3(256), smem, st, n_absorb, ay, az, sh.B, sh.H,
                    sh.d_h, sh.d_n, sh.d_r, c, (const TQ*)q, (const TQ*)M, q_pos, q_abs, N,
                    sh.G * sh.d_h, (const T*)v_new, (const T*)kpe_new, slot, pos, num_slots,
                    (T*)V_cache, (T*)kr_cache, err_flag, rope_table(sh));
}

cudaError_t launch_prep_step(const gva_shape_t& sh, const void* q, const void* M, const int* q_pos,
                             float* q_abs, float c, int N, const void* v_new, const void* kpe_new,
                             const int* slot, const int* pos, long long num_slots, void* V_cache,
                             void* kr_cache, int* err_flag, cudaStream_t st) {
  const bool qb = sh.q_dtype == GVA_BF16, cb = sh.cache_dtype == GVA_BF16;
  using bf = __nv_bfloat16;
  if (qb && cb)
    return launch_prep_t<bf, bf>(sh, q, M, q_pos, q_abs, c, N, v_new, kpe_new, slot, pos,
                                 num_slots, V_cache, kr_cache, err_flag, st);
  if (qb)
    return launch_prep_t<bf, float>(sh, q, M, q_pos, q_abs, c, N, v_new, kpe_new, slot, pos,
                                    num_slots, V_cache, kr_cache, err_flag, st);
  if (cb)
    return launch_prep_t<float, bf>(sh, q, M, q_pos, q_abs, c, N, v_new, kpe_new, slot, pos,
                                    num_slots, V_cache, kr_cache, err_flag, st);
  return launch_prep_t<float, float>(sh, q, M, q_pos, q_abs, c, N, v_new, kpe_new, slot, pos,
                                     num_slots, V_cache, kr_cache, err_flag, st);
}

cudaError_t launch_append(const gva_shape_t& sh, int N, const void* v_new, const void* kpe_new,
                          const int* slot, const int* pos, long long num_slots, void* V_cache,
                          void* kr_cache, int* err_flag, cudaStream_t st, bool early_trigger) {
  const int threads = 256, warps = threads / 32;
  const int grid = (int)(((long long)N + warps - 1) / warps);   // N < 2^31: fits the x grid
  const int row = sh.G * sh.d_h;
  const RopeTable rt = rope_table(sh);
  if (sh.cache_dtype == GVA_BF16)
    return launch_pdl(append_cache_kernel<__nv_bfloat16>, dim3(grid), dim3(threads), 0, st, N, row,
                      sh.d_r, (const __nv_bfloat16*)v_new, (const __nv_bfloat16*)kpe_new, slot, pos,
                      num_slots, (__nv_bfloat16*)V_cache, (__nv_bfloat16*)kr_cache, err_flag, rt,
                      early_trigger ? 1 : 0);
  return launch_pdl(append_cache_kernel<float>, dim3(grid), dim3(threads), 0, st, N, row, sh.d_r,
                    (const float*)v_new, (const float*)kpe_new, slot, pos, num_slots,
                    (float*)V_cache, (float*)kr_cache, err_flag, rt, early_trigger ? 1 : 0);
}

}  // namespace gva
