// Split-KV GVA decode on the fifth-generation tensor cores (sm_100a, tcgen05),
// opt-in through GVA_FLAG_TCGEN05_PATH.
//
// Same work split, partial slots and combine as the default mma.sync split kernel
// (decode_mma.cuh); the per-tile products run as asynchronous tcgen05 MMAs with
// fp32 accumulators in tensor memory.  Measured on B200 it is 1.3-1.6x slower than
// the mma.sync kernel (the first version was 1.5-2.3x slower; ncu: tensor pipe ~4%
// active, warps stalled on barriers and mbarrier waits): a decode tile carries only
// four exponentials per softmax thread, so the hand-offs between TMA, tensor core
// and softmax warps set the pace, while the mma.sync kernel keeps a tile's whole
// dependency chain inside one warp.  It is kept as the measured alternative and as
// the starting point for a version that moves several tiles per hand-off.
//
// A tile holds TT = 128 / G cache rows, so the G value groups of the tile stack
// into one 128-row operand: row r = g * TT + t is group g of token t.  Every value
// row is read from HBM once and serves the H/G = 4 heads of its group; the shared
// positional key of a token is loaded once from HBM and placed next to every
// group's rows (the G copies come from L2).
//
//   S[r, n]   = V_g[t] . Qt[n]  +  k_rope[t] . Qr[n]         (tcgen05, TMEM)
//               column n = 8 g' + j: head 4 g' + (j mod 4), the bf16 hi part of
//               its fp32 absorbed query for j < 4 and the lo part for j >= 4;
//               row r uses the 8 columns of its own group (onedev.kr review,
//               "How it works": s = q~_h . v_j + q_h^rope . k_rope_j)
//   softmax   per row and head in fp32, base 2, lazily rescaled (4 warps)
//   O^T[d, n] += V^T[d, t] P^T[n, t]                        (tcgen05, TMEM)
//               two groups share one P^T operand [16 columns x TT tokens]; with
//               d_h = 64 their values stack into the 128 rows of one MMA.
//
// Warp roles: warp 0 streams tiles with 2-D TMA loads (no multicast) into a ring,
// one thread of warp 1 issues every MMA and owns the tensor memory, polling for
// whichever is ready first, the next tile's scores or the next tile's P.V; warps
// 2-3 write each piece's queries (bf16 hi and lo halves) into shared memory, warps
// 4-7 (one tensor-memory lane quarter each) run the softmax, write P, rescale O
// when a row maximum grows by more than 2^8, and store each piece's partial.
// Every wait is bounded and reported in the status word; the tensor memory is
// freed on every path.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace gva {

template <int D_H_, int G_, int DRP_>
struct TcCfg {
  static constexpr int D_H = D_H_, G = G_, DRP = DRP_;
  static constexpr int HPG = 4;                 // query heads per value group
  static constexpr int C = 2 * HPG;             // score columns of a group: hi | lo
  static constexpr int TT = 128 / G;            // tokens per tile: G * TT = 128 rows
  static constexpr int NS = G * C;              // N of the score MMA
  static constexpr int CB = D_H / 64;           // 64-column chunks of a value row
  static constexpr int KS = D_H / 16;           // content k-steps of the scores
  static constexpr int RS = DRP / 16;           // positional k-steps
  static constexpr int KT = TT / 16;            // token k-steps of P.V
  static constexpr int BOX = TT * 128;          // one [TT x 64] bf16 box
  static constexpr int VB = CB * G * BOX;       // value tile, [chunk][group][token][64]
  static constexpr int KR1 = TT * DRP * 2;      // one positional box [TT x DRP]
  static constexpr int KRB = G * KR1;           // one copy per group: [group][token][DRP]
  static constexpr int STAGE = VB + KRB;
  static constexpr int MINB = D_H == 64 ? 2 : 1;      // CTAs per SM the budgets are sized for
  static constexpr int STAGES = (MINB == 2 && DRP == 32) ? 3 : 4;
  static constexpr uint32_t TX = VB + KRB;      // bytes TMA delivers per stage
  static constexpr int NSET = D_H == 64 ? G / 2 : G;   // P.V MMA chains of a tile
  // Tiles in flight between the roles: the issuer scores up to NSB tiles ahead of
  // the softmax (score buffers in tensor memory), and the softmax runs up to NPB
  // tiles ahead of the P.V products (P buffers in shared memory).
  static constexpr int NPB = 4;
  static constexpr uint32_t TMEM_LIMIT = MINB == 2 ? 256 : 512;
  static constexpr int NSB = (4 * NS + NSET * 16 <= (int)TMEM_LIMIT) ? 4
                           : (3 * NS + NSET * 16 <= (int)TMEM_LIMIT) ? 3 : 2;
  static constexpr int PROW = TT * 2;           // bytes of one P^T row (TT tokens)
  static constexpr int PPAIR = 16 * PROW;       // P^T of one pair of groups
  static constexpr int PBUF = (G / 2) * PPAIR;
  static constexpr int QB = CB * NS * 128;      // queries: [chunk][NS rows][64]
  static constexpr int QRB = DRP ? NS * DRP * 2 : 0;
  static constexpr int QBUF = (QB + QRB + 1023) / 1024 * 1024;
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_Q = OFF_RING + STAGES * STAGE;
  static constexpr int OFF_P = OFF_Q + 2 * QBUF;
  // rescale decisions, by tile parity: tag[2][G] then factors[2][G][4]
  static constexpr int OFF_RESC = OFF_P + NPB * PBUF;
  static constexpr int OFF_BAR = OFF_RESC + (2 * G * 5 * 4 + 15) / 16 * 16;
  // full[STAGES], empty[STAGES], s_full[NSB], s_free[NSB], p_full[NPB], pv_done[NPB],
  // q_full[2], q_free[2], o_free, fin
  static constexpr int NBAR = 2 * STAGES + 2 * NSB + 2 * NPB + 6;
  static constexpr int OFF_SCAN = OFF_BAR + NBAR * 8 + 16;
  static constexpr uint32_t S_COL = 0, O_COL = NSB * NS;
  static constexpr uint32_t TMEM_NEED = NSB * NS + NSET * 16;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                      : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int THREADS = 256;
  static constexpr uint32_t SW_R = DRP == 32 ? tc::kSw64 : tc::kSw32;
  static constexpr uint32_t SBO_R = DRP * 2 * 8;
  static constexpr uint32_t SW_P = TT == 32 ? tc::kSw64 : tc::kSw32;
  static constexpr uint32_t SBO_P = PROW * 8;
  static_assert(G == 4 || G == 8, "groups");
  static_assert(D_H == 64 || D_H == 128, "d_h");
  static_assert(DRP == 0 || DRP == 16 || DRP == 32, "padded d_r");
  static_assert(TMEM_NEED <= TMEM_LIMIT && NSB >= 2, "tensor memory");
  static_assert(NSB + NPB < 16, "issuer ring of tile records");
  static_assert(VB % 1024 == 0 && KR1 % 256 == 0 && PPAIR % 512 == 0, "swizzle atoms");

  static size_t smem_bytes(int B) {
    return 1024 + OFF_SCAN + 3 * sizeof(int) * (B + 1) + 16 + sizeof(long long) * 33;
  }
};

// Byte offset of 16-byte chunk `chunk` of row r in a swizzled K-major tile whose
// rows are 128 / 64 / 32 bytes (the layouts TMA writes with that swizzle and the
// tensor core reads through the matching descriptor).
__device__ __forceinline__ uint32_t swz128(int r, int chunk) {
  return (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t swz64(int r, int chunk) {
  return (uint32_t)(r * 64 + ((chunk ^ ((r >> 1) & 3)) << 4));
}
__device__ __forceinline__ uint32_t swz32(int r, int chunk) {
  return (uint32_t)(r * 32 + ((chunk ^ ((r >> 2) & 1)) << 4));
}

// 32 lanes x 8 consecutive 32-bit tensor-memory columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
      : "memory");
}

// Non-blocking test of an mbarrier phase (the MMA issuer polls several at once).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-tile timeline (-DGVA_TRACE builds only): for the first 8 tiles of each CTA,
// trace[131072 + (cta * 8 + k) * 8 + which] holds %globaltimer at: 0 tile requested,
// 1 scores issued, 2 scores seen by the softmax, 3 P buffer free, 4 after the
// rescale barrier, 5 P handed to the tensor core, 6 P.V issued.
__device__ __forceinline__ void tc_trace(const DecodeArgs& a, int k, int which) {
#ifdef GVA_TRACE
  if (a.trace && k < 8) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    a.trace[131072 + (blockIdx.x * 8 + k) * 8 + which] = t;
  }
#else
  (void)a;
  (void)k;
  (void)which;
#endif
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t*>(&b);
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::MINB)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_kr) {
  extern __shared__ unsigned char smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const uint32_t bar0 = sb + C::OFF_BAR;
  const uint32_t full = bar0, empty = full + 8 * C::STAGES;
  const uint32_t s_full = empty + 8 * C::STAGES, s_free = s_full + 8 * C::NSB;
  const uint32_t p_full = s_free + 8 * C::NSB, pv_done = p_full + 8 * C::NPB;
  const uint32_t q_full = pv_done + 8 * C::NPB, q_free = q_full + 16;
  const uint32_t o_free = q_free + 16, fin = o_free + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + C::NBAR * 8);
  int* resc_tag = reinterpret_cast<int*>(sm + C::OFF_RESC);                    // [2][G]
  float* resc_alpha = reinterpret_cast<float*>(sm + C::OFF_RESC) + 2 * C::G;  // [2][G][4]
  int* prefix = reinterpret_cast<int*>(sm + C::OFF_SCAN);
  int* offs = prefix + a.B + 1;
  int* tp = offs + a.B + 1;
  long long* wtmp = reinterpret_cast<long long*>(
      (reinterpret_cast<uintptr_t>(tp + a.B + 1) + 15) & ~uintptr_t(15));

  // Caller inputs no kernel of this library writes, requested before anything else.
  const bool small_b = a.B <= 32;
  int len_lane = 0, off_lane = 0;
  if (small_b && threadIdx.x < a.B) {
    len_lane = __ldg(a.seq_len + threadIdx.x);
    off_lane = __ldg(a.seq_offset + threadIdx.x);
  }
  const long long slot_lane =
      (a.prefetch && (int)threadIdx.x < a.n_new) ? (long long)__ldg(a.new_slots + threadIdx.x) : -1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    for (int i = 0; i < C::NSB; ++i) {
      mbar_init(s_full + 8 * i, 1);
      mbar_init(s_free + 8 * i, 4);
    }
    for (int i = 0; i < C::NPB; ++i) {
      mbar_init(p_full + 8 * i, 4);
      mbar_init(pv_done + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + 8 * i, 2);
      mbar_init(q_free + 8 * i, 1);
    }
    mbar_init(o_free, 4);
    mbar_init(fin, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 2 * C::G) resc_tag[threadIdx.x] = 0;
  if (warp == 1) {
    tc::alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tc::relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_v);
    if (C::DRP) prefetch_tmap(&tm_kr);
  }
  if (small_b) {
    if (threadIdx.x < a.B) offs[threadIdx.x] = off_lane;
  } else {
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) offs[b] = __ldg(a.seq_offset + b);
  }
  if (scan_batch<C::TT>(a.seq_len, a.B, len_lane, prefix, tp, wtmp) >= (1ll << 31) &&
      threadIdx.x == 0)
    atomicOr(a.status, GVA_DEVERR_RANGE);
  const TileSplit ts = make_split(tp[a.B], (int)gridDim.x, 0);
  const CtaTiles rng{prefix, tp, a.B, ts.first(blockIdx.x), ts.first(blockIdx.x + 1), C::TT};
  const bool has_work = !rng.empty();
  const int b_first = rng.first_seq();

  // ------------------------------------------------------------------ producer
  const bool producer = warp == 0 && lane == 0 && has_work;
  int k_issued = 0;
  TileCursor cur{a.B, 0, 0};
  uint64_t pol = 0;
  auto issue = [&](int k) {
    const int s = k % C::STAGES;
    const uint32_t fb = full + 8 * s;
    tc_trace(a, k, 0);
    mbar_arrive_expect_tx(fb, C::TX);
    const uint32_t st = sb + C::OFF_RING + s * C::STAGE;
    const int y = offs[cur.b] + cur.t0;
#pragma unroll
    for (int c = 0; c < C::CB; ++c)
#pragma unroll
      for (int g = 0; g < C::G; ++g)
        tma_load_2d_hint(st + (c * C::G + g) * C::BOX, &tm_v, g * C::D_H + c * 64, y, fb, pol);
    if constexpr (C::DRP > 0) {
#pragma unroll
      for (int g = 0; g < C::G; ++g) tma_load_2d_hint(st + C::VB + g * C::KR1, &tm_kr, 0, y, fb, pol);
    }
  };
  // Tiles without a row a fused step appends are final before this kernel
  // launches and are requested before the PDL wait.
  __shared__ int first_dirty;
  if (a.prefetch) {
    if (threadIdx.x == 0) first_dirty = 0x7fffffff;
    __syncthreads();
    if (has_work)
      for (int i = threadIdx.x; i < a.n_new; i += blockDim.x) {
        const long long sl = i == (int)threadIdx.x ? slot_lane : (long long)__ldg(a.new_slots + i);
        int kbase = 0;
        for (int b = b_first; rng.reaches(b); ++b) {
          int j0, j1;
          if (!rng.piece(b, j0, j1)) continue;
          const long long r0 = (long long)offs[b] + j0, r1 = (long long)offs[b] + j1;
          if (sl >= r0 && sl < r1) atomicMin(&first_dirty, kbase + (int)((sl - r0) / C::TT));
          kbase += (j1 - j0 + C::TT - 1) / C::TT;
        }
      }
    __syncthreads();
  }
  if (producer) {
    pol = policy_evict_first();
    cur.seek(rng, b_first);
    if (a.prefetch) {
      const int limit = min(C::STAGES, first_dirty);
      for (; cur.b < a.B && k_issued < limit; ++k_issued) {
        issue(k_issued);
        cur.next(rng);
      }
    }
  }
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0) write_meta(a, prefix, tp, ts);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;

  if (!has_work) {
    // nothing to do
  } else if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int k = k_issued;
      for (; cur.b < a.B; ++k) {
        const int s = k % C::STAGES;
        if (k >= C::STAGES &&
            !mbar_wait(empty + 8 * s, ((k / C::STAGES) - 1) & 1, a.status))
          break;
        issue(k);
        cur.next(rng);
      }
      for (int kk = max(0, k - C::STAGES); kk < k; ++kk)
        mbar_wait(full + 8 * (kk % C::STAGES), (kk / C::STAGES) & 1, a.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, C::NS, 0, 0);   // V (K-major) x Qt (K-major)
      constexpr uint32_t idO = tc::idesc_bf16(128, 16, 1, 0);      // V^T (MN-major) x P^T (K-major)
      const uint64_t dsw128 = tc::smem_desc(0, 16, 1024, tc::kSw128);
      const uint64_t dswr = tc::smem_desc(0, 16, C::SBO_R, C::SW_R);
      const uint64_t dv = tc::smem_desc(0, C::D_H == 64 ? C::BOX : C::G * C::BOX, 1024, tc::kSw128);
      const uint64_t dp = tc::smem_desc(0, 16, C::SBO_P, C::SW_P);
      TileCursor t;
      t.seek(rng, b_first);
      bool ok = true, scored_all = false;
      int ks = 0, kp = 0, n = -1;   // next tile to score, next tile to multiply by P
      // records of the tiles scored but not yet multiplied: whether a tile opened
      // a piece, and which piece (at most NSB + NPB tiles apart)
      bool inf_first[16];
      int inf_piece[16];
      uint32_t idle = 0;
      while (ok) {
        bool progress = false;
        if (!scored_all) {
          if (t.b >= a.B) {
            scored_all = true;
          } else {
            int j0, j1;
            rng.piece(t.b, j0, j1);
            const bool first = t.t0 == j0;
            const int nn = first ? n + 1 : n;
            const int s = ks % C::STAGES, sbuf = ks % C::NSB;
            const bool ready = (!first || mbar_test(q_full + 8 * (nn & 1), (nn >> 1) & 1)) &&
                               mbar_test(full + 8 * s, (ks / C::STAGES) & 1) &&
                               (ks < C::NSB || mbar_test(s_free + 8 * sbuf, ((ks / C::NSB) - 1) & 1));
            if (ready) {
              n = nn;
              tc::fence_after();
              const uint32_t d = tmem + C::S_COL + sbuf * C::NS;
              const uint32_t vt = sb + C::OFF_RING + s * C::STAGE;
              const uint32_t qt = sb + C::OFF_Q + (n & 1) * C::QBUF;
#pragma unroll
              for (int kx = 0; kx < C::KS; ++kx)
                tc::mma_bf16(d, dsw128 | ((vt + (kx >> 2) * (C::G * C::BOX) + (kx & 3) * 32) >> 4),
                             dsw128 | ((qt + (kx >> 2) * (C::NS * 128) + (kx & 3) * 32) >> 4), idS,
                             kx > 0);
#pragma unroll
              for (int rs = 0; rs < C::RS; ++rs)
                tc::mma_bf16(d, dswr | ((vt + C::VB + rs * 32) >> 4),
                             dswr | ((qt + C::QB + rs * 32) >> 4), idS, 1);
              tc::commit(s_full + 8 * sbuf);
              tc_trace(a, ks, 1);
              // the queries of this piece are free once its last score MMA completes
              if (t.t0 + C::TT >= j1) tc::commit(q_free + 8 * (n & 1));
              inf_first[ks & 15] = first;
              inf_piece[ks & 15] = n;
              t.next(rng);
              ++ks;
              progress = true;
            }
          }
        }
        if (kp < ks) {
          const bool jf = inf_first[kp & 15];
          const int jn = inf_piece[kp & 15], pb = kp % C::NPB;
          // a new piece overwrites O: the previous piece's partial must have been read
          const bool ready = mbar_test(p_full + 8 * pb, (kp / C::NPB) & 1) &&
                             (!(jf && jn >= 1) || mbar_test(o_free, (jn - 1) & 1));
          if (ready) {
            tc::fence_after();
            const uint32_t vt = sb + C::OFF_RING + (kp % C::STAGES) * C::STAGE;
            const uint32_t pt = sb + C::OFF_P + pb * C::PBUF;
#pragma unroll
            for (int set = 0; set < C::NSET; ++set) {
              // d_h = 64: the values of groups 2 set, 2 set + 1 fill the 128 rows;
              // d_h = 128: the two 64-column chunks of group `set`
              const int pair = C::D_H == 64 ? set : set / 2;
              const uint32_t abase = C::D_H == 64 ? vt + (2 * set) * C::BOX : vt + set * C::BOX;
#pragma unroll
              for (int kk = 0; kk < C::KT; ++kk)
                tc::mma_bf16(tmem + C::O_COL + set * 16, dv | ((abase + kk * 16 * 128) >> 4),
                             dp | ((pt + pair * C::PPAIR + kk * 32) >> 4), idO,
                             (jf && kk == 0) ? 0u : 1u);
            }
            tc::commit(pv_done + 8 * pb);
            tc::commit(empty + 8 * (kp % C::STAGES));
            tc_trace(a, kp, 6);
            ++kp;
            progress = true;
          }
        } else if (scored_all) {
          break;   // every tile scored and multiplied
        }
        if (progress) {
          idle = 0;
        } else if (++idle > 4 * kWaitLimit) {
          atomicOr(a.status, GVA_DEVERR_WAIT);
          ok = false;
        }
      }
      tc::commit(fin);
      mbar_wait(fin, 0, a.status);   // every MMA has completed before the tensor memory is freed
    }
  } else if (warp == 2 || warp == 3) {
    // ---------------------------------------------------------------- queries
    const int tid = threadIdx.x - 64;
    const int dq = C::D_H + a.d_r;
    int n = 0;
    for (int b = b_first; rng.reaches(b); ++b) {
      int j0, j1;
      if (!rng.piece(b, j0, j1)) continue;
      if (n >= 2 && !mbar_wait(q_free + 8 * (n & 1), ((n - 2) >> 1) & 1, a.status)) break;
      uint8_t* qt = sm + C::OFF_Q + (n & 1) * C::QBUF;
      for (int e = tid; e < C::NS * (C::D_H / 8); e += 64) {
        const int r = e / (C::D_H / 8), ch = e % (C::D_H / 8);
        const int g = r / C::C, j = r % C::C, head = g * C::HPG + (j & 3);
        const float* src = a.q_abs + ((size_t)b * a.H + head) * dq + ch * 8;
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const float2 v = *reinterpret_cast<const float2*>(src + i);
          x[i] = v.x;
          x[i + 1] = v.y;
        }
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float h0 = bf16_round(x[2 * i]), h1 = bf16_round(x[2 * i + 1]);
          w[i] = j < 4 ? pack_bf16(h0, h1) : pack_bf16(x[2 * i] - h0, x[2 * i + 1] - h1);
        }
        *reinterpret_cast<uint4*>(qt + (ch >> 3) * (C::NS * 128) + swz128(r, ch & 7)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      if constexpr (C::DRP > 0) {
        for (int e = tid; e < C::NS * (C::DRP / 8); e += 64) {
          const int r = e / (C::DRP / 8), ch = e % (C::DRP / 8);
          const int g = r / C::C, j = r % C::C, head = g * C::HPG + (j & 3);
          const float* src = a.q_abs + ((size_t)b * a.H + head) * dq + C::D_H;
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k0 = ch * 8 + 2 * i;
            const float x0 = k0 < a.d_r ? src[k0] : 0.f, x1 = k0 + 1 < a.d_r ? src[k0 + 1] : 0.f;
            const float h0 = bf16_round(x0), h1 = bf16_round(x1);
            w[i] = j < 4 ? pack_bf16(h0, h1) : pack_bf16(x0 - h0, x1 - h1);
          }
          const uint32_t o = C::DRP == 32 ? swz64(r, ch) : swz32(r, ch);
          *reinterpret_cast<uint4*>(qt + C::QB + o) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();   // read by the tensor core (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full + 8 * (n & 1));
      ++n;
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    const int q = warp & 3, r = 32 * q + lane;
    const int g = r / C::TT, tok = r % C::TT;
    const uint32_t lanebase = tmem + ((uint32_t)(32 * q) << 16);
    // lanes of this row's group within the warp: all 32 (TT = 32) or one half (TT = 16)
    const unsigned gmask = C::TT == 32 ? 0xffffffffu : (lane < 16 ? 0x0000ffffu : 0xffff0000u);
    const int gw = C::TT == 32 ? 32 : 16;
    bool ok = true;
    float m_ref[4], l[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      m_ref[h] = -INFINITY;
      l[h] = 0.f;
    }
    TileCursor t;
    t.seek(rng, b_first);
    int k = 0, j0 = 0, j1 = 0;
    for (; t.b < a.B; t.next(rng), ++k) {
      rng.piece(t.b, j0, j1);
      const bool first = t.t0 == j0, last = t.t0 + C::TT >= j1;
      const int nvalid = min(C::TT, j1 - t.t0);
      const bool valid = tok < nvalid;
      const int sbuf = k % C::NSB, pb = k % C::NPB;
      ok = ok && mbar_wait(s_full + 8 * sbuf, (k / C::NSB) & 1, a.status);
      tc::fence_after();
      if (threadIdx.x == 128) tc_trace(a, k, 2);
      float sv[8];
      if constexpr (C::TT == 32) {
        tmem_ld8(lanebase + C::S_COL + sbuf * C::NS + g * C::C, sv);
      } else {
        float w16[16];
        tc::ld16(lanebase + C::S_COL + sbuf * C::NS + (2 * q) * C::C, w16);
#pragma unroll
        for (int i = 0; i < 8; ++i) sv[i] = lane < 16 ? w16[i] : w16[8 + i];
      }
      tc::wait_ld();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + 8 * sbuf);

      const bool live = ok && valid;
      float s[4];
      bool ex = false;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        s[h] = sv[h] + sv[4 + h];
        ex |= live && s[h] > m_ref[h] + 8.f;
      }
      // The exact maximum over the group's rows is needed on a piece's first tile
      // and when some row exceeds the reference by more than 8 (log2 units): lazy
      // rescaling keeps P <= 2^8 otherwise.  The test is warp-uniform, so the
      // shuffles below always run on the whole warp.
      bool resc = false;
      float alpha[4] = {1.f, 1.f, 1.f, 1.f};
      if (first || __ballot_sync(0xffffffffu, ex) != 0) {
        float tm[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) tm[h] = live ? s[h] : -INFINITY;
#pragma unroll
        for (int o = 1; o < gw; o <<= 1)
#pragma unroll
          for (int h = 0; h < 4; ++h) tm[h] = fmaxf(tm[h], __shfl_xor_sync(0xffffffffu, tm[h], o));
        if (first) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            m_ref[h] = tm[h];
            l[h] = 0.f;
          }
        } else {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            if (tm[h] > m_ref[h] + 8.f) {
              alpha[h] = ex2(m_ref[h] - tm[h]);
              m_ref[h] = tm[h];
              l[h] *= alpha[h];
              resc = true;
            }
          if (resc && tok == 0) {
#pragma unroll
            for (int h = 0; h < 4; ++h) resc_alpha[((k & 1) * C::G + g) * 4 + h] = alpha[h];
            resc_tag[(k & 1) * C::G + g] = k + 1;
          }
        }
      }
      float p[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        p[h] = (live && m_ref[h] != -INFINITY) ? ex2(s[h] - m_ref[h]) : 0.f;
        l[h] += p[h];
      }
      // P buffer k % NPB is free once the P.V of tile k - NPB has completed
      if (k >= C::NPB) {
        ok = ok && mbar_wait(pv_done + 8 * pb, ((k / C::NPB) - 1) & 1, a.status);
        tc::fence_after();
      }
      if (threadIdx.x == 128) tc_trace(a, k, 3);
      {
        const uint32_t pt = sb + C::OFF_P + pb * C::PBUF + (g >> 1) * C::PPAIR;
        const int row0 = (g & 1) * 8;
        const int chunk = (tok * 2) >> 4, within = (tok * 2) & 15;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float hi = bf16_round(p[h]);
          const uint32_t ohi = C::TT == 32 ? swz64(row0 + h, chunk) : swz32(row0 + h, chunk);
          const uint32_t olo = C::TT == 32 ? swz64(row0 + 4 + h, chunk) : swz32(row0 + 4 + h, chunk);
          st_shared_u16(pt + ohi + within, bf16_bits(hi));
          st_shared_u16(pt + olo + within, bf16_bits(p[h] - hi));
        }
      }
      // value rows past the piece end meet P = 0 but may hold anything (NaN):
      // zero this row's values before the P.V product reads them
      if (!valid) {
        uint8_t* vt = sm + C::OFF_RING + (k % C::STAGES) * C::STAGE;
#pragma unroll
        for (int c = 0; c < C::CB; ++c) {
          uint4* row = reinterpret_cast<uint4*>(vt + (c * C::G + g) * C::BOX + tok * 128);
#pragma unroll
          for (int i = 0; i < 8; ++i) row[i] = make_uint4(0, 0, 0, 0);
        }
      }
      // all softmax warps see every group's rescale decision of this tile
      named_bar_sync(1, 128);
      if (threadIdx.x == 128) tc_trace(a, k, 4);
      if (!first) {
        // O lanes this warp owns: d_h = 64: group 2 set + (q >> 1) of every set;
        // d_h = 128: every group (set = group)
        bool waited = false;
#pragma unroll
        for (int set = 0; set < C::NSET; ++set) {
          const int gg = C::D_H == 64 ? 2 * set + (q >> 1) : set;
          if (resc_tag[(k & 1) * C::G + gg] != k + 1) continue;
          if (!waited) {
            // O holds every P.V up to tile k - 1
            ok = ok && mbar_wait(pv_done + 8 * ((k - 1) % C::NPB), ((k - 1) / C::NPB) & 1, a.status);
            tc::fence_after();
            waited = true;
          }
          const uint32_t col = C::O_COL + set * 16 + (gg & 1) * 8;
          float o[8];
          tmem_ld8(lanebase + col, o);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] *= resc_alpha[((k & 1) * C::G + gg) * 4 + (i & 3)];
          tmem_st8(lanebase + col, o);
        }
        if (waited) tc::wait_st();
      }
      fence_proxy_async_smem();   // P and zeroed rows are read by the tensor core
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + 8 * pb);
      if (threadIdx.x == 128) tc_trace(a, k, 5);

      if (last) {
        // ---- piece epilogue: (m, l) per head, and O once its last P.V completed
        ok = ok && mbar_wait(pv_done + 8 * pb, (k / C::NPB) & 1, a.status);
        tc::fence_after();
#pragma unroll
        for (int o = 1; o < gw; o <<= 1)
#pragma unroll
          for (int h = 0; h < 4; ++h) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
        const size_t slot = (size_t)blockIdx.x + t.b;
        if (ok && tok == 0) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            a.part_ml[slot * a.H + g * C::HPG + h] = make_float2(m_ref[h], l[h]);
        }
#pragma unroll
        for (int set = 0; set < C::NSET; ++set) {
          const int gg = C::D_H == 64 ? 2 * set + (q >> 1) : set;
          const int d = C::D_H == 64 ? (q & 1) * 32 + lane : 32 * q + lane;
          float o[8];
          tmem_ld8(lanebase + C::O_COL + set * 16 + (gg & 1) * 8, o);
          tc::wait_ld();
          if (ok) {
            float* po = a.part_o + (slot * a.H + gg * C::HPG) * C::D_H + d;
#pragma unroll
            for (int h = 0; h < 4; ++h) po[h * C::D_H] = o[h] + o[4 + h];
          }
        }
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
      }
    }
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
cudaError_t run_tc(const gva_shape_t& sh, DecodeArgs& a, const CUtensorMap& tv,
                   const CUtensorMap& tk, cudaStream_t st) {
  const size_t smem = C::smem_bytes(sh.B);
  auto k = decode_tc_kernel<C>;
  cudaError_t e = ensure_max_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(a.grid), dim3(C::THREADS), smem, st, a, tv, tk);
}

template <class F>
bool tc_dispatch(const gva_shape_t& sh, F&& f) {
  const int drp = sh.d_r == 0 ? 0 : (sh.d_r <= 16 ? 16 : (sh.d_r <= 32 ? 32 : -1));
#define GVA_TC_CASE(DH, NG, DRP)                                      \
  if (sh.d_h == DH && sh.G == NG && drp == DRP) {                     \
    f(TcCfg<DH, NG, DRP>{});                                          \
    return true;                                                      \
  }
  GVA_TC_CASE(64, 4, 0) GVA_TC_CASE(64, 4, 16) GVA_TC_CASE(64, 4, 32)
  GVA_TC_CASE(64, 8, 0) GVA_TC_CASE(64, 8, 16) GVA_TC_CASE(64, 8, 32)
  GVA_TC_CASE(128, 4, 0) GVA_TC_CASE(128, 4, 16) GVA_TC_CASE(128, 4, 32)
  GVA_TC_CASE(128, 8, 0) GVA_TC_CASE(128, 8, 16) GVA_TC_CASE(128, 8, 32)
#undef GVA_TC_CASE
  return false;
}

}  // namespace

bool tc_decode_supported(const gva_shape_t& sh) {
  if (sh.cache_dtype != GVA_BF16 || sh.G <= 0 || sh.H != 4 * sh.G) return false;
  size_t smem = 0;
  if (!tc_dispatch(sh, [&](auto c) { smem = decltype(c)::smem_bytes(sh.B); })) return false;
  return smem <= 227 * 1024;   // the per-sequence scan arrays grow with B
}

int tc_decode_tile(const gva_shape_t& sh) { return sh.G > 0 ? 128 / sh.G : 0; }

int tc_decode_grid(const gva_shape_t& sh, int num_sms, long long max_total_tokens) {
  int minb = 1, tt = 32;
  size_t smem = 0;
  tc_dispatch(sh, [&](auto c) {
    minb = decltype(c)::MINB;
    tt = decltype(c)::TT;
    smem = decltype(c)::smem_bytes(sh.B);
  });
  int per_sm = (int)((227 * 1024) / (smem + 1024));
  per_sm = per_sm < 1 ? 1 : (per_sm > minb ? minb : per_sm);
  if (sh.ctas_per_sm > 0) per_sm = sh.ctas_per_sm < minb ? sh.ctas_per_sm : minb;
  const long long want = (max_total_tokens + tt - 1) / tt;
  long long grid = (long long)num_sms * per_sm;
  if (want < grid) grid = want;
  return grid < 1 ? 1 : (int)grid;
}

cudaError_t launch_decode_tc(const gva_shape_t& sh, DecodeArgs& a, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_kr, cudaStream_t st) {
  cudaError_t err = cudaErrorNotSupported;
  tc_dispatch(sh, [&](auto c) { err = run_tc<decltype(c)>(sh, a, tm_v, tm_kr, st); });
  return err;
}

}  // namespace gva
