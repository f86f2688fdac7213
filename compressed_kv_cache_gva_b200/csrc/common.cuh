// Device helpers shared by the GVA decode kernels (sm_100a).
//
// Holds: the split-KV work list (token-balanced spans over a ragged batch), the
// workspace layout, and thin inline-PTX wrappers for mbarrier, TMA bulk-tensor
// loads, ldmatrix, movmatrix and the bf16 m16n8k16 tensor-core MMA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gva.h"

namespace gva {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxBatch = 4096;          // sequences per call (prefix array lives in smem)
constexpr int kMaxQueryRows = 65535 * 4; // query rows of one absorb call (its grid's y extent)
// A bounded mbarrier wait gives up after GVA_WAIT_LIMIT polls or GVA_WAIT_NS
// nanoseconds of %globaltimer, whichever comes first.  The time bound makes the
// worst case independent of how long one poll blocks; the failure-detection test
// build shortens it.
#ifndef GVA_WAIT_LIMIT
#define GVA_WAIT_LIMIT (1u << 22)
#endif
#ifndef GVA_WAIT_NS
#define GVA_WAIT_NS 2000000000ull
#endif
constexpr uint32_t kWaitLimit = GVA_WAIT_LIMIT;
constexpr unsigned long long kWaitNs = GVA_WAIT_NS;

// ---------------------------------------------------------------------------
// Tail pool of the split (see TileSplit): when a batch has at least
// kPoolMinTilesPerCta tiles per CTA, its last kPoolTilesPerCta * grid tiles are
// not assigned statically; CTAs that finish their static range take them one at
// a time.  0 (the default) disables the pool: measured on B200 it made the long
// decodes slower, because all pool partials belong to the batch's last sequences
// and their combine blocks then merge hundreds of pieces each.
// ---------------------------------------------------------------------------
#ifndef GVA_POOL_TILES_PER_CTA
#define GVA_POOL_TILES_PER_CTA 0
#endif
constexpr int kPoolTilesPerCta = GVA_POOL_TILES_PER_CTA;
constexpr int kPoolMinTilesPerCta = 4;

__host__ __device__ inline int pool_tiles(int NT, int grid, int per_cta) {
  if (per_cta <= 0 || (long long)NT < (long long)kPoolMinTilesPerCta * grid) return 0;
  const long long n = (long long)per_cta * grid;
  return n < NT ? (int)n : NT;
}

// ---------------------------------------------------------------------------
// Workspace: [status word, pool counter | meta[B] | partial (m,l)[P][H] |
// partial o[P][H][d_h]].  P = grid * (1 + pool tiles per CTA) + B partial slots:
// the static piece of sequence b handled by CTA i lands in slot i + b (unique,
// see the work list below), pool tile v in slot grid + B + (v - NS).
// ---------------------------------------------------------------------------
struct WsLayout {
  size_t meta_off, ml_off, o_off, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline WsLayout ws_layout(int B, int H, int d_h, int grid, int pool_per_cta) {
  WsLayout w;
  size_t parts = (size_t)grid * (size_t)(1 + (pool_per_cta > 0 ? pool_per_cta : 0)) + (size_t)B;
  w.meta_off = 256;
  w.ml_off = align_up(w.meta_off + sizeof(int4) * (size_t)B, 256);
  w.o_off = align_up(w.ml_off + sizeof(float2) * parts * (size_t)H, 256);
  w.total = align_up(w.o_off + sizeof(float) * parts * (size_t)H * (size_t)d_h, 256);
  return w;
}

struct DecodeArgs {
  int B, H, G, d_h, d_r;
  const float* q_abs;        // GVA: [B,H,d_h+d_r] float32, pre-scaled to base-2 units
  const void* q_raw;         // GQA: [B,H,d_h] q_dtype
  int q_bf16;                // GQA: q stored as bf16 (else float32)
  float q_scale;             // GQA: softmax_scale*log2(e); GVA: unused
  const void* X;             // rows scored against the query: V (GVA) or K (GQA)
  const void* Vv;            // value rows
  const void* KR;            // GVA rotated positional key rows, or null
  const int* seq_offset;
  const int* seq_len;
  long long num_slots;
  int* status;
  int* pool_ctr;             // tickets of the tail pool taken so far (the combine resets it)
  int pool_per_cta;          // pool tiles per CTA of the split kernel (0: no pool)
  int4* meta;                // per sequence: static slots (first, count), pool slots (first, count)
  float2* part_ml;           // [P][H] (running max, running sum), base-2
  float* part_o;             // [P][H][d_h] un-normalised output
  int nq;                    // query tokens per sequence (causal among them), >= 1
  int grid;                  // CTAs of the split kernel
  int tile;                  // span granularity in tokens
  int q_early;               // read the queries before the PDL wait (no kernel of the call writes them)
  int prefetch;              // stream the cache before the PDL wait, except
  const int* new_slots;      //   tiles holding one of these n_new slots, written by the
  int n_new;                 //   append of the same step
  unsigned long long* trace; // per-CTA timestamps, only with -DGVA_TRACE (else unused)
};

// Optional timeline instrumentation: with -DGVA_TRACE each CTA of the split kernel
// stores %globaltimer (ns) at fixed points of its life into trace[cta * 8 + slot].
__device__ __forceinline__ void trace_mark(const DecodeArgs& a, int slot) {
#ifdef GVA_TRACE
  if (a.trace) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    a.trace[blockIdx.x * 8 + slot] = t;
  }
#else
  (void)a;
  (void)slot;
#endif
}

// Per-tile timeline (same build flag): for the first 16 tiles of each of the
// first 2048 CTAs of the split kernel, trace[65536 + (cta * 16 + k) * 4 + which]
// holds %globaltimer when tile k was requested (which = 0), ready for group 0 (1)
// and released by it (2); trace[200000 + cta] holds the CTA's SM.
__device__ __forceinline__ void trace_tile(const DecodeArgs& a, int k, int which) {
#ifdef GVA_TRACE
  if (a.trace && k < 16 && blockIdx.x < 2048) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    a.trace[65536 + (blockIdx.x * 16 + k) * 4 + which] = t;
    if (k == 0 && which == 0) {
      unsigned sm;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
      a.trace[200000 + blockIdx.x] = sm;
    }
  }
#else
  (void)a;
  (void)k;
  (void)which;
#endif
}

// ---------------------------------------------------------------------------
// Split-KV work list.  Sequence b is cut into nt_b = ceil(L_b / TT) tiles of TT
// tokens (the last one ragged); the tiles of the batch are numbered in batch
// order (tile prefix tp[b]) and CTA i owns tiles [first(i), first(i+1)) with
// first(i) = floor(i * NT / grid).  Cutting at tile boundaries keeps every CTA at
// ceil(NT / grid) tiles or fewer: a token-balanced cut would hand a CTA whose
// range crosses the end of a sequence two ragged tiles.  The tiles CTA i owns in
// sequence b form one "piece"; it is written to partial slot i + b.  Two
// non-empty pieces (b, i) and (b', i') with b + i = b' + i' cannot exist:
// sequences are contiguous in the tile order, so b' > b forces i' >= i.
// The grid is sized on the host from an upper bound of the batch's tokens, so it
// can exceed the batch's tiles.  The split then runs over the first NT CTAs only
// (one tile each): cut over all of them, some CTAs would own no tile although they
// sit inside a sequence's run of slots, and the combine would read slots that no
// CTA wrote.  With NT >= grid, used() == grid and nothing changes.
//
// Tail pool: only the first NS tiles are cut this way; tiles [NS, NT) (the last
// pool_tiles(...) of the batch) go to whichever CTA asks first once its static
// range is issued, one tile per ticket from a counter in the workspace.  A CTA's
// static range ends when its DRAM requests have been served, which varies by a
// few tiles between CTAs; the pool lets the early ones absorb that spread.
// Each pool tile keeps its own partial slot, so the merge order, and the result,
// do not depend on which CTA took it.
// ---------------------------------------------------------------------------
struct TileSplit {
  int NT;     // tiles in the batch
  int grid;   // CTAs launched
  int NS;     // statically assigned tiles; [NS, NT) is the pool
  // CTAs that own static tiles; the rest own none
  __device__ __forceinline__ int used() const { return grid < NS ? grid : (NS > 0 ? NS : 1); }
  __device__ __forceinline__ bool narrow() const { return NS <= 0x7fffffff / used(); }
  __device__ __forceinline__ int first(int i) const {
    const int g = used();
    i = i < g ? i : g;
    return narrow() ? (int)((unsigned)(i * NS) / (unsigned)g)
                    : (int)((long long)i * NS / g);
  }
  // the CTA that owns static tile u (0 <= u < NS): the last i with first(i) <= u
  __device__ __forceinline__ int cta_of(int u) const {
    const int g = used();
    return narrow() ? (int)((unsigned)((u + 1) * g - 1) / (unsigned)NS)
                    : (int)(((long long)(u + 1) * g - 1) / NS);
  }
  __device__ __forceinline__ int pool() const { return NT - NS; }
  // Partial slots of sequence b whose tiles are [t0, t1) in batch order:
  // (first static slot, static count, first pool slot, pool count).
  __device__ __forceinline__ int4 slots(int b, int t0, int t1, int B) const {
    int4 m = make_int4(0, 0, 0, 0);
    const int s1 = t1 < NS ? t1 : NS;
    if (t0 < s1) {
      const int f = cta_of(t0), l = cta_of(s1 - 1);
      m.x = f + b;
      m.y = l - f + 1;
    }
    const int u0 = t0 > NS ? t0 : NS;
    if (u0 < t1) {
      m.z = grid + B + (u0 - NS);
      m.w = t1 - u0;
    }
    return m;
  }
};

__device__ __forceinline__ TileSplit make_split(int NT, int grid, int pool_per_cta) {
  return TileSplit{NT, grid, NT - pool_tiles(NT, grid, pool_per_cta)};
}

// Exclusive prefix sums of val(0..B-1) (each >= 0) into prefix[0..B], for the
// whole block; returns the total.  If the total does not fit in int, every
// entry is 0 (the caller flags it).
template <class F>
__device__ inline long long block_scan(int B, F val, int* prefix, long long* warp_tmp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (B + nt - 1) / nt;
  const int beg = min(tid * per, B), end = min(beg + per, B);
  long long sum = 0;
  for (int b = beg; b < end; ++b) sum += val(b);
  const int lane = tid & 31, w = tid >> 5;
  long long incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tmp[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = (nt + 31) >> 5;
    long long v = lane < nw ? warp_tmp[lane] : 0;
    long long iv = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long u = __shfl_up_sync(0xffffffffu, iv, o);
      if (lane >= o) iv += u;
    }
    if (lane < nw) warp_tmp[lane] = iv - v;
    if (lane == nw - 1) warp_tmp[32] = iv;   // grand total
  }
  __syncthreads();
  long long run = warp_tmp[w] + incl - sum;
  const long long total = warp_tmp[32];
  const bool fits = total < (1ll << 31);
  for (int b = beg; b < end; ++b) {
    prefix[b] = fits ? (int)run : 0;
    run += val(b);
  }
  if (tid == 0) prefix[B] = fits ? (int)total : 0;
  __syncthreads();   // prefix complete; warp_tmp free again
  return total;
}

// Token prefix of the lengths (negative lengths count as 0).
__device__ inline long long block_scan_lengths(const int* __restrict__ seq_len, int B,
                                               int* prefix, long long* warp_tmp) {
  return block_scan(B, [&](int b) { return (long long)max(__ldg(seq_len + b), 0); }, prefix,
                    warp_tmp);
}

// Tile prefix tp[] from the token prefix, tiles of tt tokens.
__device__ inline int block_scan_tiles(const int* prefix, int B, int tt, int* tp,
                                       long long* warp_tmp) {
  return (int)block_scan(
      B, [&](int b) { return (long long)((prefix[b + 1] - prefix[b] + tt - 1) / tt); }, tp,
      warp_tmp);
}

// Token prefix prefix[0..B] and tile prefix tp[0..B] (tiles of TT tokens) of the
// batch for the whole block; returns the token total (every entry is 0 when the
// total exceeds 2^31 - 1, which the caller flags).  For B <= 32 one warp scans
// the lengths its lanes already loaded (len_lane: the lane's length, 0 for lanes
// >= B), with no block-wide scan; larger batches take two block scans.
template <int TT>
__device__ inline long long scan_batch(const int* __restrict__ seq_len, int B, int len_lane,
                                       int* prefix, int* tp, long long* warp_tmp) {
  if (B > 32) {
    const long long total = block_scan_lengths(seq_len, B, prefix, warp_tmp);
    block_scan_tiles(prefix, B, TT, tp, warp_tmp);
    return total;
  }
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int L = max(len_lane, 0);
    const unsigned n = (unsigned)(L + TT - 1) / TT;
    long long x = L;
    unsigned y = n;          // tiles never exceed tokens, so they fit whenever the total does
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, x, o);
      const unsigned v = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) {
        x += u;
        y += v;
      }
    }
    const long long total = __shfl_sync(0xffffffffu, x, 31);
    const unsigned tiles = __shfl_sync(0xffffffffu, y, 31);
    const bool fits = total < (1ll << 31);
    if (lane < B) {
      prefix[lane] = fits ? (int)(x - L) : 0;
      tp[lane] = fits ? (int)(y - n) : 0;
    }
    if (lane == 0) {
      prefix[B] = fits ? (int)total : 0;
      tp[B] = fits ? (int)tiles : 0;
      warp_tmp[32] = total;
    }
  }
  __syncthreads();
  return warp_tmp[32];
}

// First sequence whose range in a prefix array ends after `pos` (skips empty
// sequences).
__device__ inline int seq_at(const int* prefix, int B, int pos) {
  int lo = 0, hi = B;  // answer in [0, B]
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid + 1] > pos) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// The tile range [T0, T1) of one CTA and its pieces.
struct CtaTiles {
  const int* prefix;   // token prefix [B+1]
  const int* tp;       // tile prefix [B+1]
  int B, T0, T1, tt;
  __device__ __forceinline__ bool empty() const { return T1 <= T0; }
  __device__ __forceinline__ int first_seq() const { return empty() ? B : seq_at(tp, B, T0); }
  // does sequence b start before this CTA's range ends?
  __device__ __forceinline__ bool reaches(int b) const { return b < B && tp[b] < T1; }
  // token range [j0, j1) of sequence b inside this CTA's tiles; false if empty
  __device__ __forceinline__ bool piece(int b, int& j0, int& j1) const {
    const int u0 = max(T0, tp[b]) - tp[b], u1 = min(T1, tp[b + 1]) - tp[b];
    j0 = u0 * tt;
    j1 = min(u1 * tt, prefix[b + 1] - prefix[b]);
    return j1 > j0;
  }
};

// Walks the tiles of one CTA: sequence b, tile start t0 (token index in the
// sequence) and the piece end j1.  Empty sequences are skipped; b == B means done.
struct TileCursor {
  int b, t0, j1;
  __device__ void seek(const CtaTiles& r, int from) {
    for (b = from; r.reaches(b); ++b) {
      int j0;
      if (r.piece(b, j0, j1)) {
        t0 = j0;
        return;
      }
    }
    b = r.B;
  }
  __device__ void next(const CtaTiles& r) {
    t0 += r.tt;
    if (t0 >= j1) seek(r, b + 1);
  }
};

// CTA 0 records, for every sequence, where its pieces land and how many there are,
// and flags sequences whose slots leave the cache.
__device__ inline void write_meta(const DecodeArgs& a, const int* prefix, const int* tp,
                                  TileSplit ts) {
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    int L = prefix[b + 1] - prefix[b];
    int4 m = make_int4(0, 0, 0, 0);
    if (L > 0) {
      m = ts.slots(b, tp[b], tp[b + 1], a.B);
      long long off = __ldg(a.seq_offset + b);
      if (off < 0 || off + L > a.num_slots) atomicOr(a.status, GVA_DEVERR_RANGE);
    }
    a.meta[b] = m;
  }
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel here runs a prologue that reads
// nothing the preceding kernel of the stream writes, then waits for that kernel
// (griddepcontrol.wait: it has completed and its writes are visible) before it
// reads or writes anything a predecessor touches.  A kernel whose wait returned
// knows its predecessor completed, and that one waited on its own predecessor,
// so the chain stays ordered transitively.  The split kernels trigger their
// successor after their wait; the first kernel of a fused step and the combine
// trigger at entry, so the next split kernel can launch early: before its own
// wait it only reads caller inputs and cache rows no kernel in flight writes.
// A dependent launches only once every CTA of its predecessor has triggered, so
// a waiting successor never holds the SM resources its predecessors still need.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// RoPE inverse frequencies base^(-2i/d_r), evaluated in float64 on the host.
constexpr int kMaxRopePairs = 64;
struct RopeTable {
  double inv_freq[kMaxRopePairs];
};

// ---------------------------------------------------------------------------
// Small numeric helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {  // 2^x on the SFU (PTX ex2.approx)
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// ---------------------------------------------------------------------------
// PTX wrappers (sm_90+/sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: gives up after kWaitLimit polls or kWaitNs nanoseconds and reports
// it in the status word.  The clock is read only once the first poll has failed,
// and then every 64 polls.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0 && global_ns() - t0 > kWaitNs) break;
  }
  atomicOr(status, GVA_DEVERR_WAIT);
  return false;
}

// 2-D tiled TMA load global -> shared, completion counted on an mbarrier.
// No multicast: every CTA fetches its own tiles.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Same, with an L2 eviction-priority policy (from createpolicy) for data read once.
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Barrier among `count` threads (a multiple of 32) of the CTA, id 1..15.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Register-only operations (movmatrix, mma) are not `volatile`: the compiler may
// schedule them by their data dependencies, overlapping independent chains.
// Shared-memory loads (ldmatrix) stay volatile so that they keep their place
// after the barrier waits and the writes that produce their data.
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset inside a TMA-swizzled tile: the 16-byte chunk index (bits 4..)
// is XORed with bits 7.. of the offset; SW is the swizzle span in bytes.
template <int SW>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
  if constexpr (SW == 128) return off ^ ((off >> 3) & 0x70);
  else if constexpr (SW == 64) return off ^ ((off >> 3) & 0x30);
  else if constexpr (SW == 32) return off ^ ((off >> 3) & 0x10);
  else return off;
}

}  // namespace gva
