// Multi-token GVA attention on the fifth-generation tensor cores (sm_100a):
// chunked prefill, and speculative blocks too wide for the decode kernel.
//
// The nq new tokens of a sequence are its last nq cache rows; query token i
// attends rows 0 .. L-nq+i (the causal reading of a one-token decode at each
// point).  In the absorbed form every head h of value group g scores the cache
// with its own row q~_h (onedev.kr review, "How it works") plus the shared
// positional key ("What differs"), so the rows of all nq tokens times the H/G
// heads of a group form one M x d_h operand against the group's value tile:
//
//   S[M x TK] = Q~_hi V^T + Q~_lo V^T + Qr_hi Kr^T + Qr_lo Kr^T   (tcgen05, TMEM)
//   online softmax of S rows in fp32 (base 2)                       (4 warps)
//   O[M x d_h] = alpha O + P V                                       (tcgen05, TMEM)
//
// One CTA = one block of M = 128 rows (row = token * H/G + head) of one group
// of one sequence.  Warp 0 streams 64-token value (and k_rope) tiles with 2-D
// TMA loads into a ring (no multicast), one thread of warp 1 issues every MMA
// and owns the tensor memory, warps 4..7 (one TMEM lane quarter each) run the
// softmax, write P to shared memory (two buffers, so the next tile's softmax
// overlaps this tile's P.V) and rescale O, lazily.  The fp32 query is split into
// bf16 hi + lo parts (two MMAs), so the scores keep ~16 bits; P is bf16.
//
// Tensor memory (256 columns): S double buffer in columns [0, 64) and [64, 128),
// O in [128, 128 + d_h).  Every wait is bounded and reported in the status word;
// the memory is freed on every path.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace gva {

struct PrefillArgs {
  int B, H, G, hpr, nq, d_r, d_h;
  const float* q_abs;        // [B, nq, H, d_h + d_r] fp32, pre-scaled (base 2)
  const int32_t* seq_offset;
  const int32_t* seq_len;
  long long num_slots;
  void* out;                 // [B, nq, H, d_h]
  float* lse;                // [B, nq, H] or null
  int out_bf16;
  int* status;
};

template <int D_H_, int DRP_>
struct PfCfg {
  static constexpr int D_H = D_H_, DRP = DRP_;
  static constexpr int M = 128;              // query rows per CTA
  // Cache tokens per tile, the N of the score MMAs.  Each tcgen05 instruction has a
  // fixed cost well above the arithmetic of a 64-column product, so 128-token tiles
  // halve the score instructions per key.  With d_h = 128 the CTA's shared memory
  // allows one CTA per SM either way, and 128-token tiles are 1.5x faster (16384 +
  // 1024 tokens: 514 vs 776 us on B200).  With d_h = 64, 64-token tiles keep two
  // CTAs per SM, which hide each other's hand-offs and win (184 vs 216 us for
  // 8 x (4096 + 512) tokens).
  static constexpr int TK = D_H == 128 ? 128 : 64;
  static constexpr int CB = D_H / 64;        // 128-byte boxes of a value row
  static constexpr int KS = D_H / 16;        // content k-steps
  static constexpr int RS = DRP / 16;        // positional k-steps
  static constexpr int STAGES = (TK == 128 && D_H == 128) ? 2 : 3;
  static constexpr int QB = M * D_H * 2;     // q~ hi (or lo): CB boxes of M rows x 128 B
  static constexpr int QRB = DRP ? (M * DRP * 2 + 1023) / 1024 * 1024 : 0;
  static constexpr int PB = M * TK * 2;      // one P buffer: TK/64 blocks of M rows x 128 B
  static constexpr int VB = CB * TK * 128;   // value tile of the group
  static constexpr int KRB = DRP ? TK * DRP * 2 : 0;
  static constexpr int STAGE = VB + (KRB + 1023) / 1024 * 1024;
  static constexpr int OFF_Q = 0, OFF_QR = 2 * QB, OFF_P = OFF_QR + 2 * QRB;
  static constexpr int OFF_RING = OFF_P + 2 * PB;
  static constexpr int OFF_BAR = OFF_RING + STAGES * STAGE;
  // full[S], empty[S], s_full[2], s_free[2], p_full[2], pv_done[2], fin
  static constexpr int NBAR = 2 * STAGES + 9;
  static constexpr int SMEM = 1024 + OFF_BAR + NBAR * 8 + 16;
  static constexpr uint32_t TMEM_COLS = TK == 128 ? 512 : 256;
  static constexpr uint32_t S_COL = 0, O_COL = 2 * TK;
  static constexpr uint32_t TX = VB + KRB;
  static constexpr int THREADS = 256;
  static constexpr uint32_t SW_R = DRP == 32 ? tc::kSw64 : tc::kSw32;   // k_rope rows of 64 / 32 B
  static constexpr uint32_t SBO_R = DRP * 2 * 8;                         // 8 rows of k_rope
  static_assert(D_H == 64 || D_H == 128, "d_h");
  static_assert(DRP == 0 || DRP == 16 || DRP == 32, "padded d_r");
  static_assert(TK == 64 || TK == 128, "tile");
  static_assert(O_COL + D_H <= TMEM_COLS && SMEM <= 227 * 1024, "budgets");
  static_assert(D_H <= 128, "O columns");
};

// Byte offset of element k (bf16) of row r in a 128-byte-swizzled K-major tile of
// 128-byte rows (the layout TMA writes with 128-byte swizzle and the tensor core
// reads through a SW128 descriptor): 16-byte chunk c of row r lands at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t sw128_off(int r, int chunk) {
  return (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4));
}
// Same for rows of 32 B (32-byte swizzle) and 64 B (64-byte swizzle).
__device__ __forceinline__ uint32_t sw32_off(int r, int chunk) {
  return (uint32_t)(r * 32 + ((chunk ^ ((r >> 2) & 1)) << 4));
}
__device__ __forceinline__ uint32_t sw64_off(int r, int chunk) {
  return (uint32_t)(r * 64 + ((chunk ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ uint4 split_hi(const float* x, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = x[2 * i], b = x[2 * i + 1];
    const float ah = bf16_round(a), bh = bf16_round(b);
    h[i] = pack_bf16(ah, bh);
    l[i] = pack_bf16(a - ah, b - bh);
  }
  lo = make_uint4(l[0], l[1], l[2], l[3]);
  return make_uint4(h[0], h[1], h[2], h[3]);
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_kr) {
  extern __shared__ unsigned char smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  const uint32_t full = smem_u32(bars), empty = full + 8 * C::STAGES;
  const uint32_t s_full = empty + 8 * C::STAGES, s_free = s_full + 16;
  const uint32_t p_full = s_free + 16, pv_done = p_full + 16, fin = pv_done + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int hpr = a.hpr, nq = a.nq;
  // caller inputs, read before waiting on the preceding kernel
  const int L = max(__ldg(a.seq_len + b), 0);
  const long long off = __ldg(a.seq_offset + b);
  const int row0 = blk * C::M;
  const int rows = min(C::M, nq * hpr - row0);                // valid rows of this block
  const int qi_last = (row0 + rows - 1) / hpr;                 // last query token of the block
  const int kv_end = min(L, L - nq + qi_last + 1);             // keys some row of the block sees
  const int kv_all = min(L, L - nq + row0 / hpr + 1);          // keys every row of the block sees
  const int ntiles = kv_end > 0 ? (kv_end + C::TK - 1) / C::TK : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_full + 8, 1);
    mbar_init(s_free, 4);
    mbar_init(s_free + 8, 4);
    mbar_init(p_full, 4);
    mbar_init(p_full + 8, 4);
    mbar_init(pv_done, 1);
    mbar_init(pv_done + 8, 1);
    mbar_init(fin, 1);
    fence_barrier_init();
    if (blk == 0 && g == 0 && L > 0 && (off < 0 || off + L > a.num_slots))
      atomicOr(a.status, GVA_DEVERR_RANGE);
  }
  if (warp == 1) {
    tc::alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tc::relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_v);
    if (C::DRP) prefetch_tmap(&tm_kr);
  }
  pdl_wait();   // q_abs is written by the preceding kernel
  pdl_trigger();

  // ---- queries -> shared memory: bf16 hi and lo halves, swizzled K-major rows
  const int dq = C::D_H + a.d_r;
  for (int e = threadIdx.x; e < C::M * (C::D_H / 8); e += C::THREADS) {
    const int r = e / (C::D_H / 8), c = e % (C::D_H / 8);
    float x[8];
    if (r < rows) {
      const int R = row0 + r, qi = R / hpr, head = g * hpr + R % hpr;
      const float* src = a.q_abs + (((size_t)b * nq + qi) * a.H + head) * dq + c * 8;
      const float4 u = *reinterpret_cast<const float4*>(src);
      const float4 v = *reinterpret_cast<const float4*>(src + 4);
      x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
      x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.f;
    }
    uint4 lo;
    const uint4 hi = split_hi(x, lo);
    const uint32_t o = C::OFF_Q + (c / 8) * (C::M * 128) + sw128_off(r, c % 8);
    *reinterpret_cast<uint4*>(sm + o) = hi;
    *reinterpret_cast<uint4*>(sm + o + C::QB) = lo;
  }
  if constexpr (C::DRP > 0) {
    for (int e = threadIdx.x; e < C::M * (C::DRP / 8); e += C::THREADS) {
      const int r = e / (C::DRP / 8), c = e % (C::DRP / 8);
      float x[8];
      const int R = row0 + r, qi = R / hpr, head = g * hpr + R % hpr;
      const float* src = a.q_abs + (((size_t)b * nq + qi) * a.H + head) * dq + C::D_H;
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = (r < rows && c * 8 + i < a.d_r) ? src[c * 8 + i] : 0.f;
      uint4 lo;
      const uint4 hi = split_hi(x, lo);
      const uint32_t o = C::OFF_QR + (C::DRP == 32 ? sw64_off(r, c) : sw32_off(r, c));
      *reinterpret_cast<uint4*>(sm + o) = hi;
      *reinterpret_cast<uint4*>(sm + o + C::QRB) = lo;
    }
  }
  fence_proxy_async_smem();   // the queries are read by the tensor core (async proxy)
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int k = 0;
      for (; k < ntiles; ++k) {
        const int s = k % C::STAGES;
        if (k >= C::STAGES && !mbar_wait(empty + 8 * s, ((k / C::STAGES) - 1) & 1, a.status)) break;
        const uint32_t fb = full + 8 * s, st = sb + C::OFF_RING + s * C::STAGE;
        const int y = (int)(off + (long long)k * C::TK);
        mbar_arrive_expect_tx(fb, C::TX);
#pragma unroll
        for (int c = 0; c < C::CB; ++c)
          tma_load_2d(st + c * C::TK * 128, &tm_v, g * C::D_H + c * 64, y, fb);
        if constexpr (C::DRP > 0) tma_load_2d(st + C::VB, &tm_kr, 0, y, fb);
      }
      // do not leave while a copy into shared memory is in flight
      for (int kk = max(0, k - C::STAGES); kk < k; ++kk)
        mbar_wait(full + 8 * (kk % C::STAGES), (kk / C::STAGES) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(C::M, C::TK, 0, 0);   // Q (K-major) x V^T (K-major)
      constexpr uint32_t idO = tc::idesc_bf16(C::M, C::D_H, 0, 1);  // P (K-major) x V (MN-major)
      bool ok = true;
      for (int k = 0; k <= ntiles; ++k) {
        if (k < ntiles) {
          const int s = k % C::STAGES;
          ok = ok && mbar_wait(full + 8 * s, (k / C::STAGES) & 1, a.status);
          if (k >= 2) ok = ok && mbar_wait(s_free + 8 * (k & 1), ((k - 2) >> 1) & 1, a.status);
          tc::fence_after();
          if (ok) {
            const uint32_t d = tmem + C::S_COL + (k & 1) * C::TK;
            const uint32_t vt = sb + C::OFF_RING + s * C::STAGE;
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
              const uint32_t kb = (ks >> 2) * (C::M * 128) + (ks & 3) * 32;
              const uint64_t bq = tc::smem_desc(vt + (ks >> 2) * (C::TK * 128) + (ks & 3) * 32, 16,
                                                1024, tc::kSw128);
              tc::mma_bf16(d, tc::smem_desc(sb + C::OFF_Q + kb, 16, 1024, tc::kSw128), bq, idS,
                           ks > 0);
              tc::mma_bf16(d, tc::smem_desc(sb + C::OFF_Q + C::QB + kb, 16, 1024, tc::kSw128), bq,
                           idS, 1);
            }
#pragma unroll
            for (int rs = 0; rs < C::RS; ++rs) {
              const uint64_t bk = tc::smem_desc(vt + C::VB + rs * 32, 16, C::SBO_R, C::SW_R);
              tc::mma_bf16(d, tc::smem_desc(sb + C::OFF_QR + rs * 32, 16, C::SBO_R, C::SW_R), bk,
                           idS, 1);
              tc::mma_bf16(d, tc::smem_desc(sb + C::OFF_QR + C::QRB + rs * 32, 16, C::SBO_R, C::SW_R),
                           bk, idS, 1);
            }
          }
          tc::commit(s_full + 8 * (k & 1));
        }
        if (k >= 1) {   // P.V of the previous tile, P from buffer kp % 2
          const int kp = k - 1, sp = kp % C::STAGES, pb = kp & 1;
          ok = ok && mbar_wait(p_full + 8 * pb, (kp >> 1) & 1, a.status);
          tc::fence_after();
          if (ok) {
            const uint32_t vt = sb + C::OFF_RING + sp * C::STAGE;
            const uint32_t pt = sb + C::OFF_P + pb * C::PB;
#pragma unroll
            for (int kk = 0; kk < C::TK / 16; ++kk)
              tc::mma_bf16(tmem + C::O_COL,
                           tc::smem_desc(pt + (kk >> 2) * (C::M * 128) + (kk & 3) * 32, 16, 1024,
                                         tc::kSw128),
                           tc::smem_desc(vt + kk * 16 * 128, C::TK * 128, 1024, tc::kSw128), idO,
                           (kp > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit(pv_done + 8 * pb);
          tc::commit(empty + 8 * sp);
        }
      }
      // every MMA has completed before the tensor memory is freed
      tc::commit(fin);
      mbar_wait(fin, 0, a.status);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax, P, O rescale, output
    const int quarter = warp & 3, r = 32 * quarter + lane;
    const bool valid = r < rows;
    const int R = row0 + r, qi = R / hpr, head = g * hpr + R % hpr;
    const int lim = L - nq + qi;                       // last visible cache row of this query
    const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int k = 0; k < ntiles; ++k) {
      ok = ok && mbar_wait(s_full + 8 * (k & 1), (k >> 1) & 1, a.status);
      tc::fence_after();
      float s[C::TK];
#pragma unroll
      for (int q4 = 0; q4 < C::TK / 16; ++q4) tc::ld16(trow + C::S_COL + (k & 1) * C::TK + q4 * 16, s + q4 * 16);
      tc::wait_ld();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + 8 * (k & 1));
      const int t0 = k * C::TK;
      float mx = -INFINITY;
      if (ok && t0 + C::TK <= kv_all) {   // every row sees the whole tile: no mask
#pragma unroll
        for (int j = 0; j < C::TK; ++j) mx = fmaxf(mx, s[j]);
      } else {
#pragma unroll
        for (int j = 0; j < C::TK; ++j) {
          const bool vis = ok && valid && t0 + j <= lim && t0 + j < L;
          s[j] = vis ? s[j] : -INFINITY;
          mx = fmaxf(mx, s[j]);
        }
      }
      // Lazy rescaling: a row keeps the max its exponentials are taken against
      // until a tile's max exceeds it by more than 8 (log2 units), so P <= 2^8 and
      // O is touched only then.  m = -inf (nothing seen yet) always takes the new max.
      const bool grow = mx > m + 8.f;
      const float mn = grow ? mx : m;
      const float ms = mn == -INFINITY ? 0.f : mn;    // no visible key yet: p = 0, alpha = 0
      const float alpha = ex2(m - ms);                 // 1 when the max is kept
      // P buffer k % 2 is free once the P.V of tile k - 2 has completed
      const int pb = k & 1;
      if (k >= 2) {
        ok = ok && mbar_wait(pv_done + 8 * pb, ((k - 2) >> 1) & 1, a.status);
        tc::fence_after();
      }
      // P in bf16, one swizzled 16-byte chunk (8 keys) at a time
      float rsum = 0.f;
      uint8_t* prow = sm + C::OFF_P + pb * C::PB;
#pragma unroll
      for (int c = 0; c < C::TK / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = ex2(s[8 * c + 2 * i] - ms), p1 = ex2(s[8 * c + 2 * i + 1] - ms);
          rsum += p0 + p1;
          w[i] = pack_bf16(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + (c >> 3) * (C::M * 128) + sw128_off(r, c & 7)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      l = l * alpha + rsum;
      m = mn;
      // value rows past the sequence end meet P = 0 but may hold anything (NaN):
      // zero them in the last tile before the P.V product reads them
      if (k == ntiles - 1 && t0 + C::TK > L) {
        uint8_t* vt = sm + C::OFF_RING + (k % C::STAGES) * C::STAGE;
        const int r_lo = L - t0, nz = (C::TK - r_lo) * 8;   // 16-byte chunks per box
        for (int e = r; e < nz * C::CB; e += 128) {
          const int c = e / nz, i = e % nz;
          *reinterpret_cast<uint4*>(vt + c * C::TK * 128 + (r_lo + i / 8) * 128 + (i % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      // O *= alpha before this tile's P.V accumulates onto it, once the previous
      // P.V has completed (only when some row of the warp raised its max)
      if (k >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        ok = ok && mbar_wait(pv_done + 8 * ((k - 1) & 1), ((k - 1) >> 1) & 1, a.status);
        tc::fence_after();
#pragma unroll
        for (int q4 = 0; q4 < C::D_H / 16; ++q4) {
          float o[16];
          tc::ld16(trow + C::O_COL + q4 * 16, o);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= alpha;
          tc::st16(trow + C::O_COL + q4 * 16, o);
        }
        tc::wait_st();
      }
      fence_proxy_async_smem();   // P and the zeroed rows are read by the tensor core
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + 8 * pb);
    }
    if (ntiles > 0) {   // the last P.V (and with it every earlier one) has completed
      ok = ok && mbar_wait(pv_done + 8 * ((ntiles - 1) & 1), ((ntiles - 1) >> 1) & 1, a.status);
      tc::fence_after();
    }
    // ---- output: O / l (zero and lse = -inf for a query that sees no cache row)
    const size_t orow = ((size_t)b * nq + qi) * a.H + head;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int q4 = 0; q4 < C::D_H / 16; ++q4) {
      float o[16];
      if (ntiles > 0) {
        tc::ld16(trow + C::O_COL + q4 * 16, o);
        tc::wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = 0.f;
      }
      if (valid) {
        if (a.out_bf16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.out) + orow * C::D_H + q4 * 16;
#pragma unroll
          for (int i = 0; i < 16; ++i) dst[i] = __float2bfloat16_rn(o[i] * inv);
        } else {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + orow * C::D_H +
                                                  q4 * 16);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv,
                                 o[4 * i + 3] * inv);
        }
      }
    }
    if (valid && a.lse) a.lse[orow] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    (void)ok;
  }

  // ---- every role is done with the tensor memory: free it
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::dealloc(tmem, C::TMEM_COLS);
  }
}

// ----------------------------------------------------------------------------- host

namespace {

template <class C>
cudaError_t run_prefill(const PrefillArgs& a, const CUtensorMap& tv, const CUtensorMap& tk,
                        cudaStream_t st) {
  auto k = prefill_tc_kernel<C>;
  cudaError_t e = ensure_max_smem(k, (size_t)C::SMEM);
  if (e != cudaSuccess) return e;
  const int nblk = (a.nq * a.hpr + C::M - 1) / C::M;
  return launch_pdl(k, dim3(nblk, a.G, a.B), dim3(C::THREADS), C::SMEM, st, a, tv, tk);
}

}  // namespace

bool prefill_supported(const gva_shape_t& sh, int nq) {
  if (sh.cache_dtype != GVA_BF16 || (sh.d_h != 64 && sh.d_h != 128)) return false;
  if (sh.d_r < 0 || sh.d_r > 32 || sh.d_r % 8) return false;
  const int hpr = sh.G > 0 ? sh.H / sh.G : 0;
  if (hpr < 1 || 128 % hpr || nq < 1 || sh.B > 65535 || sh.G > 65535) return false;
  return (long long)nq * hpr <= (1ll << 30);
}

int prefill_tile_rows(const gva_shape_t& sh) { return sh.d_h == 128 ? PfCfg<128, 0>::TK : PfCfg<64, 0>::TK; }

cudaError_t launch_prefill(const gva_shape_t& sh, int nq, const float* q_abs,
                           const int32_t* seq_offset, const int32_t* seq_len, long long num_slots,
                           void* out, float* lse, int* status, const CUtensorMap& tv,
                           const CUtensorMap& tk, cudaStream_t st) {
  PrefillArgs a{};
  a.B = sh.B;
  a.H = sh.H;
  a.G = sh.G;
  a.hpr = sh.H / sh.G;
  a.nq = nq;
  a.d_r = sh.d_r;
  a.d_h = sh.d_h;
  a.q_abs = q_abs;
  a.seq_offset = seq_offset;
  a.seq_len = seq_len;
  a.num_slots = num_slots;
  a.out = out;
  a.lse = lse;
  a.out_bf16 = sh.out_dtype == GVA_BF16;
  a.status = status;
  const int drp = sh.d_r == 0 ? 0 : (sh.d_r <= 16 ? 16 : 32);
  if (sh.d_h == 64) {
    if (drp == 0) return run_prefill<PfCfg<64, 0>>(a, tv, tk, st);
    if (drp == 16) return run_prefill<PfCfg<64, 16>>(a, tv, tk, st);
    return run_prefill<PfCfg<64, 32>>(a, tv, tk, st);
  }
  if (drp == 0) return run_prefill<PfCfg<128, 0>>(a, tv, tk, st);
  if (drp == 16) return run_prefill<PfCfg<128, 16>>(a, tv, tk, st);
  return run_prefill<PfCfg<128, 32>>(a, tv, tk, st);
}

}  // namespace gva
