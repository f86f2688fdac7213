// Split-KV decode kernel on the tensor cores, TMA-staged (sm_100a).
//
// One CTA = NG consumer warps (warp g serves value group g and its HPG query
// heads) + 1 producer warp that streams tiles of TT cache rows into a STAGES-deep
// shared-memory ring with 2-D TMA loads (128-byte swizzle, no multicast) and
// mbarrier completion.  Every tile is read from HBM once and serves all heads.
//
// Per tile and group (tokens on the MMA M axis, heads on N):
//   scores  S[tok, n] = V_g[tok, :] . Qb[:, n]  (+ k_rope[tok, :] . Qr[:, n])
//   softmax online in fp32, base 2 (the query is pre-scaled by scale*log2 e)
//   output  O^T[d, n] += V_g^T[d, tok] . P[tok, n]
// With HPG = 4 the 8 MMA columns hold [hi(q) of 4 heads | lo(q) of 4 heads],
// q = hi + lo split into two bf16 numbers, so the fp32 query keeps ~16 bits of
// significand at no extra MMA cost; P is split the same way for the second
// product.  HPG = 8 uses two 8-column tiles (hi, lo).  The score fragment
// (tokens on rows) is turned into the B operand of the second product
// (tokens on K) with movmatrix.trans, so probabilities never touch shared memory.
//
// For GQA (same-shape comparison) the scores operand is the K tile, a separate V
// tile is streamed next to it and there is no positional key.
// Groups with fewer query columns than 4 (H/G = 1, 2, 3 with one query token) run
// the 4-column configuration and groups with 5..7 the 8-column one: the spare
// columns carry a zero query, and their outputs are never stored.
#pragma once

#include "common.cuh"

namespace gva {

#ifndef GVA_ROW_PARTS   // consumer warps per group splitting every tile's rows (d_h = 64, G <= 4)
#define GVA_ROW_PARTS 1
#endif

template <int D_H_, int NG_, int HPG_, int DRP_, bool GQA_, int W_ = 0,
          int P_ = (D_H_ == 64 && NG_ <= 4) ? GVA_ROW_PARTS : 1>
struct MmaCfg {
  static constexpr int D_H = D_H_, NG = NG_, HPG = HPG_, DRP = GQA_ ? 0 : DRP_;
  static constexpr bool GQA = GQA_;
  static constexpr int ROW_BYTES = NG * D_H * 2 * (GQA ? 2 : 1);
#ifndef GVA_TILE_BYTES   // bytes of cache rows per pipeline stage (tuning knob)
#define GVA_TILE_BYTES 16384
#endif
  static constexpr int TT_RAW = (GQA ? 2 * GVA_TILE_BYTES : GVA_TILE_BYTES) / ROW_BYTES;
  static constexpr int TT = TT_RAW >= 64 ? 64 : (TT_RAW >= 32 ? 32 : 16);   // tokens per tile
  // A group's values arrive as boxes of VW columns (64, or 32 for d_h = 32), one
  // VROW-byte row per token, swizzled over VROW bytes by the TMA
  static constexpr int VW = D_H < 64 ? D_H : 64;      // columns per box
  static constexpr int VROW = VW * 2;                 // bytes of a box row (= swizzle span)
  static constexpr int CPR = VROW / 16;               // 16-byte chunks per box row
  static constexpr int CB = D_H / VW;                 // boxes per group
  static constexpr int BOX = TT * VROW;               // bytes of one [TT x VW] bf16 box
  static constexpr int XB = NG * CB * BOX;            // scores operand (V or K)
  static constexpr int VB = GQA ? XB : 0;             // separate value tile (GQA)
  static constexpr int KRB = DRP ? TT * DRP * 2 : 0;  // positional key tile
  static constexpr int STAGE = XB + VB + (KRB + 1023) / 1024 * 1024;
#ifndef GVA_PIPE_BYTES   // shared memory of the stage ring per CTA (tuning knob)
#define GVA_PIPE_BYTES (96 * 1024)
#endif
  // consumer warps per group (round robin over tiles).  Measured on B200: one warp
  // per group is fastest for every workload here (a second warp per group adds the
  // end-of-piece merge and contends for the same SM resources), so 0 means 1.
  static constexpr int W = W_ > 0 ? W_ : 1;
  // P warps per group can instead split every tile's 16-row blocks between them
  // (all P consume each tile; their states merge at the end of a piece), which
  // shortens each tile's dependent MMA/softmax chain.  W and P do not combine.
  static constexpr int P = P_ > 0 ? P_ : 1;
  static constexpr int GW = W * P;                    // consumer warps per group
// Ring budget of the 33 KB tiles of eight 128-wide groups: 3 stages instead of
// the 2 that GVA_PIPE_BYTES holds (measured: 131k-token decode 52.2 -> 50.2 us,
// other shapes unaffected); two CTAs per SM still fit.
#ifndef GVA_PIPE_BYTES_WIDE
#define GVA_PIPE_BYTES_WIDE (108 * 1024)
#endif
  static constexpr int PIPE_BUDGET =
      (!GQA && D_H == 128 && NG == 8) ? GVA_PIPE_BYTES_WIDE : GVA_PIPE_BYTES;
  static constexpr int STAGES_RAW = PIPE_BUDGET / STAGE;
  static constexpr int STAGES_CLAMPED = STAGES_RAW < 2 ? 2 : (STAGES_RAW > 12 ? 12 : STAGES_RAW);
  // A multiple of W: tile k lives in stage k % STAGES and is consumed by warp
  // k % W of each group, so every stage always belongs to the same warp and that
  // warp meets the stage's barrier phases one after another.  (With an odd stage
  // count a warp could wait for phase p+2 while the stage is still in phase p+1,
  // and the parity test would pass on stale data.)
  static constexpr int STAGES = STAGES_CLAMPED / W * W < W ? W : STAGES_CLAMPED / W * W;
// When a CTA's whole range fits in its ring (short batches: every tile is
// requested at once), it first requests RAMP tiles and the rest once the first
// has landed, so its consumers start earlier instead of every tile of the burst
// landing late together.  Longer ranges keep the full ring from the start.
// (Measured: 350M decode 10.85 -> 10.15 us; on the long decodes the ramp lost.)
#ifndef GVA_RAMP_TILES
#define GVA_RAMP_TILES 2
#endif
  static constexpr int RAMP = GVA_RAMP_TILES > 0 && GVA_RAMP_TILES < STAGES ? GVA_RAMP_TILES : 0;
// CTAs with at most this many tiles keep one stage fewer in flight (rings of 4+
// stages): when every CTA requests its whole ring at once, the first tiles queue
// behind ~26 MB of requests.  Measured: d_r = 24 decode 18.27 -> 17.63 us, the
// others (ramped, or longer ranges) unchanged.
#ifndef GVA_SHORT_RANGE_TILES
#define GVA_SHORT_RANGE_TILES 16
#endif
  static constexpr int PIPE = STAGES * STAGE;
  static constexpr uint32_t TX = XB + VB + KRB;       // bytes TMA delivers per stage
  static constexpr int MT = TT / 16;                  // 16-token m-tiles per tile
  static constexpr int MW = MT / P;                   // m-tiles per consumer warp and tile
  static constexpr int NCW = NG * GW;                 // consumer warps
  static constexpr int THREADS = (NCW + 1) * 32;
  static constexpr int NT = HPG == 8 ? 2 : 1;         // 8-column MMA tiles
  static constexpr int KS = D_H / 16;                 // content k-steps (= d m-tiles)
  static constexpr int RS = DRP / 16;                 // positional k-steps
  // end-of-piece merge of the GW warps of a group: (m, l) per warp and lane quad,
  // and the output fragments of warps 1..GW-1
  static constexpr int MERGE_ML = GW * 4 * 4;                   // floats per group
  static constexpr int MERGE_O = (GW - 1) * 32 * KS * 4;       // floats per group
  static constexpr int MERGE = GW > 1 ? NG * (MERGE_ML + MERGE_O) * 4 : 0;  // bytes
  static constexpr int KR_SW = DRP * 2;               // swizzle span of the k_rope box
  // resident CTAs per SM the register budget is sized for.  Two CTAs of 9 warps
  // leave 96 registers a thread; 8 columns of d_h = 128 keep ~100 values live in
  // the consumer (query fragments, O^T accumulators, V^T fragments), so that
  // configuration runs one CTA per SM instead of spilling.
  static constexpr int MINB = (NCW >= 8 && HPG == 8 && D_H == 128) ? 1 : 2;
  static_assert(HPG == 4 || HPG == 8, "heads per group");
  static_assert(STAGES % W == 0, "each stage must belong to one warp of a group");
  static_assert(W == 1 || P == 1, "round robin over tiles or rows split, not both");
  static_assert(MT % P == 0, "row parts must divide the tile's 16-row blocks");
  static_assert(D_H == 32 || D_H % 64 == 0, "d_h");
  static_assert(DRP == 0 || DRP == 16 || DRP == 32, "padded d_r");

  static size_t smem_bytes(int B) {
    return 1024 + PIPE + MERGE + 16 * STAGES + 3 * sizeof(int) * (B + 1) + 16 +
           sizeof(long long) * 33;
  }
};

// Query fragments of sequence b for consumer lane (gq, t) of group g (the B
// operand of the score MMA, column n = gq): the absorbed fp32 query
// (pre-scaled), or the raw query in its storage type, scaled here (GQA, and
// GVA with shared keys and values: M = I, d_r = 0), split into bf16 hi / lo.
// Padding columns (past the group's ncol real ones) get a zero query.
template <class C>
__device__ __forceinline__ void load_query(const DecodeArgs& a, const int b, const int g,
                                           const int hpr, const int ncol, const int gq,
                                           const int t, uint32_t (&qbo)[C::NT][C::KS][2],
                                           uint32_t (&qro)[C::NT][C::RS > 0 ? C::RS : 1][2]) {
  const int H = a.H, dq = C::D_H + a.d_r;
#pragma unroll
  for (int nt = 0; nt < C::NT; ++nt) {
    const int hl = C::HPG == 8 ? gq : (gq & 3);     // column within the group
    const bool lo = C::HPG == 8 ? (nt == 1) : (gq >= 4);
    const int vq = hl / hpr, head = g * hpr + hl % hpr;
    float v[C::KS][4];
    float wv[C::RS > 0 ? C::RS : 1][4];
    if (hl >= ncol) {   // padding column: zero query
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) v[ks][e] = 0.f;
#pragma unroll
      for (int rs = 0; rs < (C::RS > 0 ? C::RS : 1); ++rs)
#pragma unroll
        for (int e = 0; e < 4; ++e) wv[rs][e] = 0.f;
    } else if (!C::GQA && a.q_raw == nullptr) {
      const float* qrow = a.q_abs + (((size_t)b * a.nq + vq) * H + head) * dq;
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        const int k0 = ks * 16 + 2 * t;
        const float2 x01 = *reinterpret_cast<const float2*>(qrow + k0);
        const float2 x89 = *reinterpret_cast<const float2*>(qrow + k0 + 8);
        v[ks][0] = x01.x;
        v[ks][1] = x01.y;
        v[ks][2] = x89.x;
        v[ks][3] = x89.y;
      }
#pragma unroll
      for (int rs = 0; rs < C::RS; ++rs) {
        const int k0 = rs * 16 + 2 * t;
        wv[rs][0] = k0 < a.d_r ? qrow[C::D_H + k0] : 0.f;
        wv[rs][1] = k0 + 1 < a.d_r ? qrow[C::D_H + k0 + 1] : 0.f;
        wv[rs][2] = k0 + 8 < a.d_r ? qrow[C::D_H + k0 + 8] : 0.f;
        wv[rs][3] = k0 + 9 < a.d_r ? qrow[C::D_H + k0 + 9] : 0.f;
      }
    } else {
      const void* rawrow = reinterpret_cast<const char*>(a.q_raw) +
          (((size_t)b * a.nq + vq) * H + head) * C::D_H * (a.q_bf16 ? 2 : 4);
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        const int k0 = ks * 16 + 2 * t;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = k0 + (e & 1) + (e >> 1) * 8;
          const float x = a.q_bf16
              ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(rawrow)[kk])
              : reinterpret_cast<const float*>(rawrow)[kk];
          v[ks][e] = x * a.q_scale;
        }
      }
#pragma unroll
      for (int rs = 0; rs < (C::RS > 0 ? C::RS : 1); ++rs)
#pragma unroll
        for (int e = 0; e < 4; ++e) wv[rs][e] = 0.f;
    }
    auto part = [&](float x) { const float h = bf16_round(x); return lo ? x - h : h; };
#pragma unroll
    for (int ks = 0; ks < C::KS; ++ks) {
      qbo[nt][ks][0] = pack_bf16(part(v[ks][0]), part(v[ks][1]));
      qbo[nt][ks][1] = pack_bf16(part(v[ks][2]), part(v[ks][3]));
    }
#pragma unroll
    for (int rs = 0; rs < C::RS; ++rs) {
      qro[nt][rs][0] = pack_bf16(part(wv[rs][0]), part(wv[rs][1]));
      qro[nt][rs][1] = pack_bf16(part(wv[rs][2]), part(wv[rs][3]));
    }
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::MINB)
    decode_mma_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_kr) {
  extern __shared__ unsigned char smraw[];
  uint8_t* pipe = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
  float* merge = reinterpret_cast<float*>(pipe + C::PIPE);
  uint64_t* full = reinterpret_cast<uint64_t*>(pipe + C::PIPE + C::MERGE);
  uint64_t* empty = full + C::STAGES;
  int* prefix = reinterpret_cast<int*>(empty + C::STAGES);
  int* offs = prefix + a.B + 1;
  int* tp = offs + a.B + 1;            // tile prefix
  long long* wtmp = reinterpret_cast<long long*>(
      (reinterpret_cast<uintptr_t>(tp + a.B + 1) + 15) & ~uintptr_t(15));

  // The lengths and offsets are caller inputs that no kernel of this library
  // writes: they are requested first, so that their latency overlaps the barrier
  // setup, and read before waiting on the preceding kernel.
  const bool small_b = a.B <= 32;
  int len_lane = 0, off_lane = 0;
  if (small_b && threadIdx.x < a.B) {
    len_lane = __ldg(a.seq_len + threadIdx.x);
    off_lane = __ldg(a.seq_offset + threadIdx.x);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) trace_mark(a, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), C::NG * C::P);   // the warps of a group that read a tile
    }
    fence_barrier_init();
  }
  if (warp == C::NCW && lane == 0) {
    prefetch_tmap(&tm_x);
    if (C::GQA) prefetch_tmap(&tm_v);
    if (C::DRP) prefetch_tmap(&tm_kr);
  }
  if (small_b) {
    if (threadIdx.x < a.B) offs[threadIdx.x] = off_lane;
  } else {
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) offs[b] = __ldg(a.seq_offset + b);
  }
  // token and tile prefixes (all zeros, and flagged, past 2^31 - 1 tokens)
  if (scan_batch<C::TT>(a.seq_len, a.B, len_lane, prefix, tp, wtmp) >= (1ll << 31) &&
      threadIdx.x == 0)
    atomicOr(a.status, GVA_DEVERR_RANGE);
  // the tail pool needs one consumer warp per group (W == 1): a pool tile is a
  // piece of its own
  const TileSplit ts = make_split(tp[a.B], (int)gridDim.x,
                                  (kPoolTilesPerCta > 0 && C::W == 1) ? a.pool_per_cta : 0);
  const int n_pool = kPoolTilesPerCta > 0 ? ts.pool() : 0;   // compiled out when disabled
  const CtaTiles rng{prefix, tp, a.B, ts.first(blockIdx.x), ts.first(blockIdx.x + 1), C::TT};
  const bool has_work = !rng.empty() || n_pool > 0;
  const int b_first = rng.first_seq();
  // pool tile held by each stage (-1: the pool is empty, no data in the stage)
  __shared__ int pool_tile[C::STAGES];

  // ------------------------------------------------------------------ producer
  // One thread issues every load of the CTA.  The cache is read once per step:
  // its lines are marked first to evict so the partials, queries and outputs of
  // the step stay in L2.
  const bool producer = warp == C::NCW && lane == 0 && has_work;
  int k_issued = 0;
  bool prod_ok = true;
  TileCursor cur;
  uint64_t pol = 0;
  auto issue = [&](int k) {
    const int s = k % C::STAGES;
    const uint32_t fb = smem_u32(full + s);
#ifdef GVA_TEST_WITHHOLD_TILE
    // Failure-detection test builds only: this tile ordinal of every CTA is never
    // requested (no transaction is armed and no copy is in flight for it), so the
    // consumers' bounded wait on its barrier runs out and reports GVA_DEVERR_WAIT.
    if (k == GVA_TEST_WITHHOLD_TILE) return;
#endif
    if (k == 0) trace_mark(a, 2);
    trace_tile(a, k, 0);
    mbar_arrive_expect_tx(fb, C::TX);
    const uint32_t st = smem_u32(pipe + s * C::STAGE);
    const int y = offs[cur.b] + cur.t0;
#pragma unroll
    for (int g = 0; g < C::NG; ++g)
#pragma unroll
      for (int c = 0; c < C::CB; ++c)
        tma_load_2d_hint(st + (g * C::CB + c) * C::BOX, &tm_x, g * C::D_H + c * C::VW, y, fb, pol);
    if constexpr (C::GQA) {
#pragma unroll
      for (int g = 0; g < C::NG; ++g)
#pragma unroll
        for (int c = 0; c < C::CB; ++c)
          tma_load_2d_hint(st + C::XB + (g * C::CB + c) * C::BOX, &tm_v, g * C::D_H + c * C::VW, y, fb,
                           pol);
    }
    if constexpr (C::DRP > 0) tma_load_2d_hint(st + C::XB, &tm_kr, 0, y, fb, pol);
  };
  // Every cache row is final before this kernel launches (the library's kernels
  // that write cache rows let their successor launch only at their exit), except
  // the rows a fused step's own first kernel appends: the first stages are
  // requested before the PDL wait, up to the first tile of this CTA that uses an
  // appended row.  All threads map the appended slots onto this CTA's tile
  // ordinals in parallel.
  // (Rows a tile reads past its piece's end are never used, so only rows inside
  // the pieces count.)
  __shared__ int first_dirty;
  if (a.prefetch) {
    if (threadIdx.x == 0) first_dirty = 0x7fffffff;
    __syncthreads();
    if (has_work)
      for (int i = threadIdx.x; i < a.n_new; i += blockDim.x) {
        const long long sl = __ldg(a.new_slots + i);
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
  // query fragments (B operand of the score MMA), column n = gq, of sequence q_seq
  uint32_t qb[C::NT][C::KS][2];
  uint32_t qr[C::NT][C::RS > 0 ? C::RS : 1][2];
  int q_seq = -1;
  // A plain decode call's queries are its own inputs (no kernel of the call
  // writes them): the consumers load their first sequence's query before the
  // PDL wait, off the critical path.  In a fused step the first kernel writes
  // them, so they wait.
  if (a.q_early && warp < C::NCW && has_work && rng.reaches(b_first)) {
    const int hpr0 = a.H / a.G;
    load_query<C>(a, b_first, warp / C::GW, hpr0, hpr0 * a.nq, lane >> 2, lane & 3, qb, qr);
    q_seq = b_first;
  }
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) trace_mark(a, 1);
  if (blockIdx.x == 0) write_meta(a, prefix, tp, ts);
  if (!has_work) return;

  if (warp == C::NCW) {
    if (lane != 0) return;
    int k = k_issued;
    const bool ramp = C::RAMP > 0 && rng.T1 - rng.T0 <= C::STAGES;
    // depth in flight: one stage fewer for short ranges (tile k waits for tile
    // k - depth's release; consumers release in order, and that stage is not
    // refilled before tile k, so its barrier is still in that tile's phase).
    // Only with one consumer warp per group: with W > 1 the warps of a group
    // release alternate tiles in no fixed order, so the release of tile
    // k - depth says nothing about tile k - STAGES, whose stage tile k reuses
    // (its copy could still be landing when tile k's is armed on the same
    // barrier); those configurations wait for tile k - STAGES itself.
    const int depth = (C::W == 1 && C::STAGES >= 4 && GVA_SHORT_RANGE_TILES > 0 &&
                       rng.T1 - rng.T0 <= GVA_SHORT_RANGE_TILES) ? C::STAGES - 1 : C::STAGES;
    for (; cur.b < a.B; ++k) {
      const int s = k % C::STAGES;
      const int kd = k - depth;
      if (kd >= 0 && !mbar_wait(smem_u32(empty + kd % C::STAGES), (kd / C::STAGES) & 1, a.status)) {
        prod_ok = false;
        break;
      }
      (void)s;
      // ramp: the rest of the ring is requested once the first tile has landed
      if (ramp && k == C::RAMP) mbar_wait(smem_u32(full), 0, a.status);
      issue(k);
      cur.next(rng);
    }
    // Pool tiles, one per ticket once the static range is issued.  The next
    // ticket is requested as soon as the current one is used, so the atomic's
    // latency overlaps the wait for a free stage.  A stage that carries a pool
    // tile names it in pool_tile[] (written before the arrive that completes the
    // stage); -1 with a plain arrive (no bytes) tells the consumers the pool is
    // empty.
    if (prod_ok && n_pool > 0) {
      int u = atomicAdd(a.pool_ctr, 1);
      for (;; ++k) {
        const int s = k % C::STAGES;
        if (k >= C::STAGES &&
            !mbar_wait(smem_u32(empty + s), ((k / C::STAGES) - 1) & 1, a.status)) {
          prod_ok = false;
          break;
        }
        if (u >= n_pool) {
          pool_tile[s] = -1;
          mbar_arrive(smem_u32(full + s));
          ++k;
          break;
        }
        const int v = ts.NS + u;
        pool_tile[s] = v;
        u = atomicAdd(a.pool_ctr, 1);
        cur.b = seq_at(tp, a.B, v);
        cur.t0 = (v - tp[cur.b]) * C::TT;
        issue(k);
      }
    }
    (void)prod_ok;
    // Drain: do not leave while a copy into this CTA's shared memory is in flight.
    for (int kk = max(0, k - C::STAGES); kk < k; ++kk)
      mbar_wait(smem_u32(full + kk % C::STAGES), (kk / C::STAGES) & 1, a.status);
    return;
  }

  // ------------------------------------------------------------------ consumers
  // warp = g * W + w: group g, tiles w, w+W, w+2W, ... of this CTA (round robin,
  // so W tiles per group are in flight); the W running states are merged at the
  // end of every piece
  // warp = g * GW + wi: group g; with W > 1 warp wi takes tiles wi, wi+W, ...,
  // with P > 1 it takes rows [wi*16*MW, (wi+1)*16*MW) of every tile
  const int g = warp / C::GW, wi = warp % C::GW;
  const int w = C::W > 1 ? wi : 0;
  const int r_lo = C::P > 1 ? wi * C::MW * 16 : 0, r_hi = r_lo + C::MW * 16;   // this warp's rows
  const int t = lane & 3, gq = lane >> 2;
  const int mi = lane >> 3, r8 = lane & 7;
  // ldmatrix row/chunk owned by this lane (see the fragment layouts of m16n8k16)
  const int a_row = (mi & 1) * 8 + r8, a_kc = mi >> 1;   // scores A: rows = tokens
  const int v_tok = (mi >> 1) * 8 + r8, v_dc = mi & 1;   // P.V A (trans): rows = tokens
  const int H = a.H;                  // query heads
  const int hpr = a.H / a.G;          // query heads per group; C::HPG = hpr * nq columns
  const int Hp = a.H * a.nq;          // heads of the partials and the output: [query][head]
  const int dq = C::D_H + a.d_r;
  // columns owned after the hi/lo merge: hcol, hcol+1 of this group.  Column c
  // is query c / hpr of the sequence's nq new tokens and head g*hpr + c % hpr.
  // Fewer real columns than the configuration's (H/G * nq below 4, or 5..7 with
  // 8): the rest carry a zero query and are never stored.
  const int ncol = hpr * a.nq;
  const int hcol = (2 * t) & (C::HPG - 1);
  const bool real0 = hcol < ncol, real1 = hcol + 1 < ncol;
  const int qi0 = hcol / hpr, qi1 = (hcol + 1) / hpr;   // differ only when H/G is odd
  const int phead0 = qi0 * H + g * hpr + hcol % hpr;
  const int phead1 = qi1 * H + g * hpr + (hcol + 1) % hpr;
  const bool lo_half = (C::HPG == 4) && (t >= 2);
  float* mg_ml = merge + g * (C::MERGE_ML + C::MERGE_O);
  float* mg_o = mg_ml + C::MERGE_ML;
  bool ok = true;   // false once a bounded wait gave up: skip work, keep barrier order

  int k = 0;
  // One piece: tokens [j0, j1) of sequence b, tiles k, k+1, ... of the ring;
  // its partial state goes to `slot`.
  auto run_piece = [&](const int b, const int j0, const int j1, const size_t slot) {
    if (b != q_seq) {
      load_query<C>(a, b, g, hpr, ncol, gq, t, qb, qr);
      q_seq = b;
    }

    // O^T fragments: d rows x 8 columns.  With 8 columns per group the hi and lo
    // halves of P (two n-tiles) belong to the same heads and share these
    // accumulators; with 4 the lo half sits in the upper 4 columns (merged at the end)
    float o[C::KS][4];
#pragma unroll
    for (int md = 0; md < C::KS; ++md)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[md][e] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    // causal limits of this thread's two columns: the nq new tokens sit at
    // positions L-nq .. L-1 and query i sees the cache up to its own position
    const int lim0 = (prefix[b + 1] - prefix[b]) - a.nq + qi0;
    const int lim1 = lim0 + (qi1 - qi0);

    for (int t0 = j0; t0 < j1; t0 += C::TT, ++k) {
      if (k % C::W != w) continue;                 // another warp of the group takes it
      const int s = k % C::STAGES;
      if (ok) ok = mbar_wait(smem_u32(full + s), (k / C::STAGES) & 1, a.status);
      if (!ok) continue;
      if (warp == 0 && lane == 0 && k == 0) trace_mark(a, 3);
      if (warp == 0 && lane == 0) trace_tile(a, k, 1);
      const int nvalid = min(C::TT, j1 - t0);
      uint8_t* st = pipe + s * C::STAGE;
      uint8_t* xg = st + g * C::CB * C::BOX;
      uint8_t* vg = C::GQA ? st + C::XB + g * C::CB * C::BOX : xg;
      const bool ragged = nvalid < r_hi;
      if (ragged) {
        // rows past the sequence may hold anything (even NaN): zero this warp's
        // rows so that p = 0 really contributes nothing to P.V
        const int r0 = max(nvalid, r_lo), nz = r_hi - r0;
        for (int e = lane; e < nz * C::CPR * C::CB; e += 32) {
          const int c = e / (nz * C::CPR), rr = r0 + (e / C::CPR) % nz, ch = e % C::CPR;
          *reinterpret_cast<uint4*>(vg + c * C::BOX + rr * C::VROW + ch * 16) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      const uint32_t xg_u = smem_u32(xg), vg_u = smem_u32(vg), kr_u = smem_u32(st + C::XB);

      // ---- scores of this warp's MW*16 tokens (two accumulator chains per m-tile)
      float sc[C::MW][4];
#pragma unroll
      for (int mm = 0; mm < C::MW; ++mm) {
        const int arow = a_row + r_lo + mm * 16;
        float acc[2][C::NT][4];
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[c2][nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
          uint32_t a0, a1, a2, a3;
          // k-step ks covers columns [16 ks, 16 ks + 16): box ks / (CPR/2), chunk pair
          // ks % (CPR/2); the swizzle XORs the chunk with row bits (rows of 128 bytes:
          // row & 7, which is r8 here; of 64 bytes: (row >> 1) & 3)
          const uint32_t xoff = C::VROW == 128
              ? (ks >> 2) * C::BOX + arow * 128 + ((((ks & 3) * 2 + a_kc) ^ r8) << 4)
              : (ks / (C::CPR / 2)) * C::BOX +
                    swz<C::VROW>(arow * C::VROW + ((ks % (C::CPR / 2)) * 2 + a_kc) * 16);
          ldsm_x4(xg_u + xoff, a0,
                  a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt)
            mma_bf16(acc[ks & 1][nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
        }
#pragma unroll
        for (int rs = 0; rs < C::RS; ++rs) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kr_u + swz<C::KR_SW>(arow * C::DRP * 2 + (rs * 2 + a_kc) * 16), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt)
            mma_bf16(acc[(C::KS + rs) & 1][nt], a0, a1, a2, a3, qr[nt][rs][0], qr[nt][rs][1]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x;
          if constexpr (C::HPG == 8) x = (acc[0][0][e] + acc[1][0][e]) + (acc[0][1][e] + acc[1][1][e]);
          else {
            x = acc[0][0][e] + acc[1][0][e];
            x += __shfl_xor_sync(0xffffffffu, x, 2);
          }
          const int r = r_lo + mm * 16 + gq + (e >= 2 ? 8 : 0);
          sc[mm][e] = (r < nvalid && t0 + r <= ((e & 1) ? lim1 : lim0)) ? x : -INFINITY;
        }
      }

      // ---- V^T fragments for the second product, requested before the softmax so
      // their shared-memory latency overlaps it
      uint32_t vf[C::MW][C::KS][4];
#pragma unroll
      for (int mm = 0; mm < C::MW; ++mm)
#pragma unroll
        for (int md = 0; md < C::KS; ++md)
          ldsm_x4_t(vg_u + (C::VROW == 128
                                ? (md >> 2) * C::BOX + (v_tok + r_lo + mm * 16) * 128 +
                                      ((((md & 3) * 2 + v_dc) ^ r8) << 4)
                                : (md / (C::CPR / 2)) * C::BOX +
                                      swz<C::VROW>((v_tok + r_lo + mm * 16) * C::VROW +
                                                   ((md % (C::CPR / 2)) * 2 + v_dc) * 16)),
                    vf[mm][md][0], vf[mm][md][1], vf[mm][md][2], vf[mm][md][3]);

      // ---- online softmax (fp32, base 2); this thread owns heads hcol, hcol+1
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int mm = 0; mm < C::MW; ++mm) {
        mx0 = fmaxf(mx0, fmaxf(sc[mm][0], sc[mm][2]));
        mx1 = fmaxf(mx1, fmaxf(sc[mm][1], sc[mm][3]));
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      // a warp may see no valid token yet (its rows all past the piece end):
      // exponentiate against 0 then, so that p = 0 and alpha = 0, never NaN
      const float ms0 = mn0 == -INFINITY ? 0.f : mn0, ms1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = ex2(m0 - ms0), al1 = ex2(m1 - ms1);
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t bp[C::MW][C::NT][2];
#pragma unroll
      for (int mm = 0; mm < C::MW; ++mm) {
        const float p0 = ex2(sc[mm][0] - ms0), p1 = ex2(sc[mm][1] - ms1);
        const float p2 = ex2(sc[mm][2] - ms0), p3 = ex2(sc[mm][3] - ms1);
        rs0 += p0 + p2;
        rs1 += p1 + p3;
        const float h0 = bf16_round(p0), h1 = bf16_round(p1), h2 = bf16_round(p2), h3 = bf16_round(p3);
        if constexpr (C::HPG == 8) {
          bp[mm][0][0] = movm_t(pack_bf16(h0, h1));
          bp[mm][0][1] = movm_t(pack_bf16(h2, h3));
          bp[mm][1][0] = movm_t(pack_bf16(p0 - h0, p1 - h1));
          bp[mm][1][1] = movm_t(pack_bf16(p2 - h2, p3 - h3));
        } else {
          bp[mm][0][0] = movm_t(lo_half ? pack_bf16(p0 - h0, p1 - h1) : pack_bf16(h0, h1));
          bp[mm][0][1] = movm_t(lo_half ? pack_bf16(p2 - h2, p3 - h3) : pack_bf16(h2, h3));
        }
      }
      l0 = l0 * al0 + rs0;
      l1 = l1 * al1 + rs1;
#pragma unroll
      for (int md = 0; md < C::KS; ++md) {
        o[md][0] *= al0;
        o[md][1] *= al1;
        o[md][2] *= al0;
        o[md][3] *= al1;
      }

      // ---- O^T += V^T P over this warp's tokens (V^T fragments loaded above)
#pragma unroll
      for (int mm = 0; mm < C::MW; ++mm)
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
          for (int md = 0; md < C::KS; ++md)
            mma_bf16(o[md], vf[mm][md][0], vf[mm][md][1], vf[mm][md][2], vf[mm][md][3],
                     bp[mm][nt][0], bp[mm][nt][1]);
      if (ragged) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty + s));
      if (warp == 0 && lane == 0) trace_tile(a, k, 2);
    }

    // ---- piece epilogue
    if (warp == 0 && lane == 0) trace_mark(a, 4);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    if constexpr (C::GW > 1) {
      // merge the GW warps of this group: common max, rescale, sum through smem
      const int bar = 1 + g, nthr = C::GW * 32;
      if (gq == 0) {
        float* e = mg_ml + (wi * 4 + t) * 4;
        e[0] = m0; e[1] = m1; e[2] = l0; e[3] = l1;
      }
      named_bar_sync(bar, nthr);
      float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
      for (int u = 0; u < C::GW; ++u) {
        M0 = fmaxf(M0, mg_ml[(u * 4 + t) * 4 + 0]);
        M1 = fmaxf(M1, mg_ml[(u * 4 + t) * 4 + 1]);
      }
      // a column may have no visible token in this piece (all past its causal
      // limit): keep it at (-inf, 0) instead of forming -inf - -inf
      const float Ms0 = M0 == -INFINITY ? 0.f : M0, Ms1 = M1 == -INFINITY ? 0.f : M1;
      float L0 = 0.f, L1 = 0.f;
#pragma unroll
      for (int u = 0; u < C::GW; ++u) {
        const float* e = mg_ml + (u * 4 + t) * 4;
        L0 += e[2] * ex2(e[0] - Ms0);
        L1 += e[3] * ex2(e[1] - Ms1);
      }
      const float f0 = ex2(m0 - Ms0), f1 = ex2(m1 - Ms1);
#pragma unroll
      for (int md = 0; md < C::KS; ++md) {
        o[md][0] *= f0;
        o[md][1] *= f1;
        o[md][2] *= f0;
        o[md][3] *= f1;
      }
      m0 = M0; m1 = M1; l0 = L0; l1 = L1;
      if (wi > 0) {
        float* dst = mg_o + ((wi - 1) * 32 + lane) * (C::KS * 4);
#pragma unroll
        for (int md = 0; md < C::KS; ++md)
          *reinterpret_cast<float4*>(dst + md * 4) =
              make_float4(o[md][0], o[md][1], o[md][2], o[md][3]);
      }
      named_bar_sync(bar, nthr);
      if (wi == 0) {
#pragma unroll
        for (int u = 1; u < C::GW; ++u) {
          const float* src = mg_o + ((u - 1) * 32 + lane) * (C::KS * 4);
#pragma unroll
          for (int md = 0; md < C::KS; ++md) {
            const float4 x = *reinterpret_cast<const float4*>(src + md * 4);
            o[md][0] += x.x;
            o[md][1] += x.y;
            o[md][2] += x.z;
            o[md][3] += x.w;
          }
        }
      }
      named_bar_sync(bar, nthr);   // scratch free for the next piece
    }
    if (wi != 0) return;
    if constexpr (C::HPG == 4) {
#pragma unroll
      for (int md = 0; md < C::KS; ++md)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[md][e] += __shfl_xor_sync(0xffffffffu, o[md][e], 2);
    }
    if (ok && (C::HPG == 8 || t < 2)) {
      float* po0 = a.part_o + (slot * Hp + phead0) * C::D_H;
      float* po1 = a.part_o + (slot * Hp + phead1) * C::D_H;
#pragma unroll
      for (int md = 0; md < C::KS; ++md) {
        const int d = md * 16 + gq;
        if (real0) {
          po0[d] = o[md][0];
          po0[d + 8] = o[md][2];
        }
        if (real1) {
          po1[d] = o[md][1];
          po1[d + 8] = o[md][3];
        }
      }
      if (gq == 0) {
        if (real0) a.part_ml[slot * Hp + phead0] = make_float2(m0, l0);
        if (real1) a.part_ml[slot * Hp + phead1] = make_float2(m1, l1);
      }
    }
    if (warp == 0 && lane == 0) trace_mark(a, 5);
  };

  // static range: its pieces land in slots cta + b
  for (int b = b_first; rng.reaches(b); ++b) {
    int j0, j1;
    if (rng.piece(b, j0, j1)) run_piece(b, j0, j1, (size_t)blockIdx.x + b);
  }
  // pool tiles handed over by the producer, each a piece of one tile with its
  // own slot, until the empty-pool mark
  while (n_pool > 0 && ok) {
    const int s = k % C::STAGES;
    ok = mbar_wait(smem_u32(full + s), (k / C::STAGES) & 1, a.status);
    if (!ok) break;
    const int v = *static_cast<volatile int*>(pool_tile + s);
    if (v < 0) break;
    const int b = seq_at(tp, a.B, v);
    const int j0 = (v - tp[b]) * C::TT;
    run_piece(b, j0, min(j0 + C::TT, prefix[b + 1] - prefix[b]),
              (size_t)gridDim.x + a.B + (size_t)(v - ts.NS));
  }
}

}  // namespace gva
