// Split-KV decode on the CUDA cores (FMA path).
//
// Same work list, partial format and combine as the tensor-core kernel, but the
// products run as fp32 FMAs from shared memory.  It serves float32 caches (where
// the 1e-5 relative accuracy needs fp32 products) and shapes the tensor-core
// kernel is not instantiated for, and it is the CUDA-core baseline that the
// tensor-core path is measured against.
//
// Per tile of TT rows: stage rows as fp32 in shared memory; one thread per
// (token, head) computes the score s = q_abs_h . [v_{g(h)} | k_rope]; one warp per
// head does the online-softmax update; each thread owns up to OPT (head, dim)
// outputs of o_h += sum_t p_t v_{t,g(h)}.
#include "common.cuh"
#include "launch.h"

namespace gva {

constexpr int kSimtTT = 16;
constexpr int kSimtThreads = 256;
constexpr int kSimtOPT = 16;   // outputs per thread: H*d_h <= 4096

struct SimtLayout {
  int row;           // elements per cache row (G*d_h)
  size_t xs, vs, krs, qs, ss, mrun, lrun, alpha, prefix, tp, wtmp, total;
};

static SimtLayout simt_layout(const gva_shape_t& sh, bool gqa) {
  SimtLayout L;
  L.row = sh.G * sh.d_h;
  const int dq = sh.d_h + (gqa ? 0 : sh.d_r);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes, 16); return r; };
  L.xs = take(sizeof(float) * kSimtTT * L.row);
  L.vs = gqa ? take(sizeof(float) * kSimtTT * L.row) : L.xs;
  L.krs = take(sizeof(float) * kSimtTT * (gqa ? 0 : sh.d_r));
  L.qs = take(sizeof(float) * sh.H * dq);
  L.ss = take(sizeof(float) * kSimtTT * sh.H);
  L.mrun = take(sizeof(float) * sh.H);
  L.lrun = take(sizeof(float) * sh.H);
  L.alpha = take(sizeof(float) * sh.H);
  L.prefix = take(sizeof(int) * (sh.B + 1));
  L.tp = take(sizeof(int) * (sh.B + 1));
  L.wtmp = take(sizeof(long long) * 33);
  L.total = o;
  return L;
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
    decode_simt_kernel(const DecodeArgs a, const SimtLayout Ly, const int gqa) {
  extern __shared__ __align__(16) unsigned char sm[];
  float* Xs = reinterpret_cast<float*>(sm + Ly.xs);
  float* Vs = reinterpret_cast<float*>(sm + Ly.vs);
  float* KRs = reinterpret_cast<float*>(sm + Ly.krs);
  float* Qs = reinterpret_cast<float*>(sm + Ly.qs);
  float* Ss = reinterpret_cast<float*>(sm + Ly.ss);
  float* mrun = reinterpret_cast<float*>(sm + Ly.mrun);
  float* lrun = reinterpret_cast<float*>(sm + Ly.lrun);
  float* alpha = reinterpret_cast<float*>(sm + Ly.alpha);
  int* prefix = reinterpret_cast<int*>(sm + Ly.prefix);
  int* tp = reinterpret_cast<int*>(sm + Ly.tp);
  long long* wtmp = reinterpret_cast<long long*>(sm + Ly.wtmp);

  const int H = a.H, d_h = a.d_h, hpg = a.H / a.G, row = Ly.row;
  const int d_r = gqa ? 0 : a.d_r;
  const int dq = d_h + d_r;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const T* X = reinterpret_cast<const T*>(a.X);
  const T* Vv = reinterpret_cast<const T*>(a.Vv);
  const T* KR = reinterpret_cast<const T*>(a.KR);

  pdl_wait();
  pdl_trigger();
  const int len_lane = (a.B <= 32 && tid < a.B) ? __ldg(a.seq_len + tid) : 0;
  if (scan_batch<kSimtTT>(a.seq_len, a.B, len_lane, prefix, tp, wtmp) >= (1ll << 31) && tid == 0)
    atomicOr(a.status, GVA_DEVERR_RANGE);
  const TileSplit ts = make_split(tp[a.B], (int)gridDim.x, 0);
  if (blockIdx.x == 0) write_meta(a, prefix, tp, ts);
  const CtaTiles rng{prefix, tp, a.B, ts.first(blockIdx.x), ts.first(blockIdx.x + 1), kSimtTT};
  if (rng.empty()) return;

  for (int b = rng.first_seq(); rng.reaches(b); ++b) {
    int j0, j1;
    if (!rng.piece(b, j0, j1)) continue;
    const long long row0 = __ldg(a.seq_offset + b);
    // query of sequence b, base-2 scaled
    for (int e = tid; e < H * dq; e += blockDim.x) {
      if (!gqa && a.q_raw == nullptr) {
        Qs[e] = a.q_abs[(size_t)b * H * dq + e];
      } else {
        const size_t i = (size_t)b * H * d_h + e;
        float x = a.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q_raw)[i])
                           : reinterpret_cast<const float*>(a.q_raw)[i];
        Qs[e] = x * a.q_scale;
      }
    }
    for (int h = tid; h < H; h += blockDim.x) {
      mrun[h] = -INFINITY;
      lrun[h] = 0.f;
    }
    float o[kSimtOPT];
#pragma unroll
    for (int i = 0; i < kSimtOPT; ++i) o[i] = 0.f;
    __syncthreads();

    for (int t0 = j0; t0 < j1; t0 += kSimtTT) {
      const int nvalid = min(kSimtTT, j1 - t0);
      // stage rows (zero outside the sequence or the cache)
      for (int e = tid; e < kSimtTT * row; e += blockDim.x) {
        const int r = e / row, c = e - r * row;
        const long long slot = row0 + t0 + r;
        const bool ok = r < nvalid && slot >= 0 && slot < a.num_slots;
        Xs[e] = ok ? to_f32(X[slot * row + c]) : 0.f;
        if (gqa) Vs[e] = ok ? to_f32(Vv[slot * row + c]) : 0.f;
      }
      for (int e = tid; e < kSimtTT * d_r; e += blockDim.x) {
        const int r = e / d_r, c = e - r * d_r;
        const long long slot = row0 + t0 + r;
        const bool ok = r < nvalid && slot >= 0 && slot < a.num_slots;
        KRs[e] = ok ? to_f32(KR[slot * d_r + c]) : 0.f;
      }
      __syncthreads();
      // scores
      for (int e = tid; e < kSimtTT * H; e += blockDim.x) {
        const int r = e / H, h = e - r * H;
        const float* q = Qs + h * dq;
        const float* x = Xs + r * row + (h / hpg) * d_h;
        float s = 0.f;
        for (int i = 0; i < d_h; ++i) s = fmaf(q[i], x[i], s);
        const float* kr = KRs + r * d_r;
        for (int i = 0; i < d_r; ++i) s = fmaf(q[d_h + i], kr[i], s);
        Ss[e] = r < nvalid ? s : -INFINITY;
      }
      __syncthreads();
      // online softmax, one warp per head
      for (int h = warp; h < H; h += nwarps) {
        const float s = lane < kSimtTT ? Ss[lane * H + h] : -INFINITY;
        float mx = s;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float mold = mrun[h];
        const float mnew = fmaxf(mold, mx);
        const float p = ex2(s - mnew);
        float sum = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < kSimtTT) Ss[lane * H + h] = p;
        __syncwarp();
        if (lane == 0) {
          const float al = ex2(mold - mnew);
          alpha[h] = al;
          lrun[h] = lrun[h] * al + sum;
          mrun[h] = mnew;
        }
      }
      __syncthreads();
      // P.V
#pragma unroll
      for (int i = 0; i < kSimtOPT; ++i) {
        const int idx = tid + i * blockDim.x;
        if (idx < H * d_h) {
          const int h = idx / d_h, d = idx - h * d_h;
          const float* v = Vs + (h / hpg) * d_h + d;
          float acc = o[i] * alpha[h];
          for (int r = 0; r < nvalid; ++r) acc = fmaf(Ss[r * H + h], v[r * row], acc);
          o[i] = acc;
        }
      }
      __syncthreads();
    }
    // partial of this piece
    const size_t slot = (size_t)blockIdx.x + b;
#pragma unroll
    for (int i = 0; i < kSimtOPT; ++i) {
      const int idx = tid + i * blockDim.x;
      if (idx < H * d_h) a.part_o[slot * H * d_h + idx] = o[i];
    }
    for (int h = tid; h < H; h += blockDim.x) a.part_ml[slot * H + h] = make_float2(mrun[h], lrun[h]);
    __syncthreads();
  }
}

int simt_tile() { return kSimtTT; }

static bool simt_ok(const gva_shape_t& sh, bool gqa) {
  return (long long)sh.H * sh.d_h <= (long long)kSimtThreads * kSimtOPT &&
         simt_layout(sh, gqa).total <= 200 * 1024;
}

bool simt_supported(const gva_shape_t& sh, bool gqa) { return simt_ok(sh, gqa); }

int simt_grid(const gva_shape_t& sh, int num_sms, long long max_total_tokens, bool gqa) {
  const size_t smem = simt_layout(sh, gqa).total;
  int per_sm = (int)((220 * 1024) / (smem + 1024));
  per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
  if (sh.ctas_per_sm > 0) per_sm = sh.ctas_per_sm;
  long long want = (max_total_tokens + kSimtTT - 1) / kSimtTT;
  long long grid = (long long)num_sms * per_sm;
  if (want < grid) grid = want;
  return grid < 1 ? 1 : (int)grid;
}

cudaError_t launch_decode_simt(const gva_shape_t& sh, bool gqa, DecodeArgs& a, cudaStream_t st) {
  if (!simt_ok(sh, gqa)) return cudaErrorNotSupported;
  const SimtLayout Ly = simt_layout(sh, gqa);
  auto k = sh.cache_dtype == GVA_BF16 ? decode_simt_kernel<__nv_bfloat16> : decode_simt_kernel<float>;
  if (Ly.total > 48 * 1024) {
    cudaError_t e = ensure_max_smem(k, Ly.total);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(k, dim3(a.grid), dim3(kSimtThreads), Ly.total, st, a, Ly, gqa ? 1 : 0);
}

}  // namespace gva
