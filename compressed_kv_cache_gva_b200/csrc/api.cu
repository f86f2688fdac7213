// C ABI of the GVA decode library: argument validation, kernel selection, TMA
// descriptor encoding and launches.  No allocation, no synchronisation.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace {

thread_local char g_err[320] = "";
#ifdef GVA_TRACE
unsigned long long* g_trace = nullptr;
#endif

gva_status_t fail(gva_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

gva_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(GVA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elt(int dtype) { return dtype == GVA_F32 ? 4 : 2; }

bool dtype_ok(int d) { return d == GVA_F32 || d == GVA_BF16; }

// SM count of the current device (cached per device).
int num_sms() {
  static int cache[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// max_b: the decode keeps per-sequence prefix arrays in shared memory (kMaxBatch);
// the absorb only needs its grid to fit (kMaxQueryRows query rows).
gva_status_t check_shape(const gva_shape_t* sh, bool gqa, int max_b = gva::kMaxBatch) {
  if (!sh) return fail(GVA_ERR_INVALID_ARG, "shape is NULL");
  if (sh->B < 0 || sh->B > max_b)
    return fail(GVA_ERR_INVALID_ARG, "B=%d outside [0, %d]", sh->B, max_b);
  if (sh->H < 1 || sh->G < 1 || sh->H % sh->G)
    return fail(GVA_ERR_INVALID_ARG, "need H >= 1, G >= 1, H %% G == 0 (H=%d G=%d)", sh->H, sh->G);
  if (sh->d_h < 1 || sh->d_h > 512) return fail(GVA_ERR_INVALID_ARG, "d_h=%d outside [1,512]", sh->d_h);
  if (!gqa) {
    if (sh->d_n < 0 || sh->d_n > 1024) return fail(GVA_ERR_INVALID_ARG, "d_n=%d outside [0,1024]", sh->d_n);
    if (sh->d_r < 0 || sh->d_r > 2 * gva::kMaxRopePairs || (sh->d_r & 1))
      return fail(GVA_ERR_INVALID_ARG, "d_r=%d must be even and in [0,%d]", sh->d_r,
                  2 * gva::kMaxRopePairs);
    if (!(sh->rope_base > 0.0) || !isfinite(sh->rope_base))
      return fail(GVA_ERR_INVALID_ARG, "rope_base must be positive and finite");
  }
  if (!dtype_ok(sh->cache_dtype) || !dtype_ok(sh->q_dtype) || !dtype_ok(sh->out_dtype))
    return fail(GVA_ERR_INVALID_ARG, "dtype codes must be GVA_F32 or GVA_BF16");
  if (sh->softmax_scale < 0.f || !isfinite(sh->softmax_scale))
    return fail(GVA_ERR_INVALID_ARG, "softmax_scale must be >= 0 and finite");
  if (sh->ctas_per_sm < 0 || sh->ctas_per_sm > 32)
    return fail(GVA_ERR_INVALID_ARG, "ctas_per_sm=%d outside [0,32]", sh->ctas_per_sm);
  return GVA_OK;
}

float scale_of(const gva_shape_t& sh, bool gqa) {
  if (sh.softmax_scale > 0.f) return sh.softmax_scale;
  const int w = gqa ? sh.d_h : sh.d_n + sh.d_r;
  return w > 0 ? (float)(1.0 / sqrt((double)w)) : 1.f;
}

// ---------------------------------------------------------------- TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 view [rows, cols] with row pitch `pitch_elems`, box [box_rows, box_cols].
gva_status_t encode_2d(CUtensorMap* m, const void* base, long long rows, int cols, int pitch_elems,
                       int box_rows, int box_cols, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(GVA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable from the driver");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)pitch_elems * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(GVA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rows=%lld cols=%d box=%dx%d", (int)r,
                rows, cols, box_rows, box_cols);
  return GVA_OK;
}

struct Plan {
  bool mma;   // tensor-core split kernel (mma.sync or tcgen05)
  bool tc;    // the tcgen05 one
  int grid;
  int pool;   // tail-pool tiles per CTA of the split kernel (0: none)
  gva::WsLayout ws;
};

// allow_tc: a one-token GVA decode with an absorbed query, the only case the
// opt-in tcgen05 kernel covers; multi-token, shared-key and GQA calls always run
// on the mma.sync kernel.
gva_status_t plan_decode(const gva_shape_t& sh, bool gqa, long long max_total, Plan* p,
                         bool allow_tc) {
  const int sms = num_sms();
  if (sms <= 0) return fail(GVA_ERR_CUDA, "no CUDA device");
  p->mma = !(sh.flags & GVA_FLAG_FMA_PATH) && gva::mma_supported(sh, gqa);
  p->tc = p->mma && allow_tc && !gqa && (sh.flags & GVA_FLAG_TCGEN05_PATH) &&
          gva::tc_decode_supported(sh);
  p->grid = p->tc ? gva::tc_decode_grid(sh, sms, max_total)
          : p->mma ? gva::mma_grid(sh, sms, max_total, gqa) : gva::simt_grid(sh, sms, max_total, gqa);
  p->pool = (p->mma && !p->tc) ? gva::kPoolTilesPerCta : 0;   // the mma.sync split kernel only
  p->ws = gva::ws_layout(sh.B, sh.H, sh.d_h, p->grid, p->pool);
  return GVA_OK;
}

// Every check of a decode call (sh already carries the nq * H heads), before
// anything is launched; fills the plan.
gva_status_t decode_check(const gva_shape_t& sh, bool gqa, const void* q, const void* X,
                          const void* Vv, const void* KR, const int32_t* seq_offset,
                          const int32_t* seq_len, int64_t max_total_tokens, int64_t num_slots,
                          const void* out, const float* lse, const void* workspace,
                          size_t ws_bytes, int nq, bool raw_q, Plan* pp) {
  gva_status_t s;
  Plan& p = *pp;
  if (!q || !X || !Vv || !seq_offset || !seq_len || !out || !workspace)
    return fail(GVA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!gqa && sh.d_r > 0 && !KR) return fail(GVA_ERR_INVALID_ARG, "kr_cache is NULL with d_r > 0");
  if (!aligned16(q) || !aligned16(X) || !aligned16(Vv) || (KR && !aligned16(KR)) || !aligned16(out) ||
      !aligned16(workspace) || !aligned16(seq_offset) || !aligned16(seq_len) || (lse && !aligned16(lse)))
    return fail(GVA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (num_slots < 1 || num_slots >= (1ll << 31))
    return fail(GVA_ERR_INVALID_ARG, "num_slots=%lld outside [1, 2^31)", (long long)num_slots);
  if (max_total_tokens < 0 || max_total_tokens >= (1ll << 31))
    return fail(GVA_ERR_INVALID_ARG, "max_total_tokens=%lld outside [0, 2^31)", (long long)max_total_tokens);
  const int e = elt(sh.cache_dtype);
  if ((sh.G * sh.d_h * e) % 16 || (!gqa && (sh.d_r * e) % 16))
    return fail(GVA_ERR_INVALID_ARG, "cache rows must be multiples of 16 bytes (G*d_h*elt=%d, d_r*elt=%d)",
                sh.G * sh.d_h * e, gqa ? 0 : sh.d_r * e);
  if ((s = plan_decode(sh, gqa, max_total_tokens, &p, !gqa && !raw_q && nq == 1)) != GVA_OK)
    return s;
  if (nq > 1 && !p.mma)
    return fail(GVA_ERR_UNSUPPORTED, "several query tokens need the tensor-core kernel "
                "(bf16 cache, (H/G)*n_query <= 8, d_h in {32, 64, 128})");
  if (ws_bytes < p.ws.total)
    return fail(GVA_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, p.ws.total);

  if (!p.mma && !gva::simt_supported(sh, gqa))
    return fail(GVA_ERR_UNSUPPORTED, "no decode kernel for H=%d G=%d d_h=%d d_r=%d", sh.H, sh.G,
                sh.d_h, sh.d_r);
  return GVA_OK;
}

gva_status_t decode_common(const gva_shape_t* shp, bool gqa, const void* q, const void* X,
                           const void* Vv, const void* KR, const int32_t* seq_offset,
                           const int32_t* seq_len, int64_t max_total_tokens, int64_t num_slots,
                           void* out, float* lse, void* workspace, size_t ws_bytes, void* stream,
                           const int32_t* new_slots = nullptr,
                           int n_new = 0, int nq = 1, bool raw_q = false,
                           bool clear_status = false, bool step = false) {
  gva_status_t s = check_shape(shp, gqa);
  if (s != GVA_OK) return s;
  if (nq < 1 || nq > 64) return fail(GVA_ERR_INVALID_ARG, "n_query=%d outside [1,64]", nq);
  // nq query tokens per sequence run as nq * H/G columns per value group: the
  // kernels and the workspace see H * nq heads, the queries see H heads each
  gva_shape_t shv = *shp;
  shv.H = shp->H * nq;
  const gva_shape_t& sh = shv;
  if (sh.B == 0) return GVA_OK;
  Plan p;
  if ((s = decode_check(sh, gqa, q, X, Vv, KR, seq_offset, seq_len, max_total_tokens, num_slots,
                        out, lse, workspace, ws_bytes, nq, raw_q, &p)) != GVA_OK)
    return s;

  gva::DecodeArgs a{};
  a.B = sh.B;
  a.H = shp->H;
  a.nq = nq;
  a.G = sh.G;
  a.d_h = sh.d_h;
  a.d_r = gqa ? 0 : sh.d_r;
  a.q_abs = (gqa || raw_q) ? nullptr : static_cast<const float*>(q);
  a.q_raw = (gqa || raw_q) ? q : nullptr;
  a.q_bf16 = sh.q_dtype == GVA_BF16;
  a.q_scale = scale_of(sh, gqa) * gva::kLog2e;
  a.X = X;
  a.Vv = Vv;
  a.KR = gqa ? nullptr : KR;
  a.seq_offset = seq_offset;
  a.seq_len = seq_len;
  a.num_slots = num_slots;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = reinterpret_cast<int*>(ws);
  a.pool_ctr = reinterpret_cast<int*>(ws) + 1;
  a.pool_per_cta = p.pool;
  a.meta = reinterpret_cast<int4*>(ws + p.ws.meta_off);
  a.part_ml = reinterpret_cast<float2*>(ws + p.ws.ml_off);
  a.part_o = reinterpret_cast<float*>(ws + p.ws.o_off);
  a.grid = p.grid;
  // Every decode requests its first cache tiles before its PDL wait: the cache
  // rows are final by then (a fused step's own new slots excepted, listed in
  // new_slots), since the kernels of this library that write cache rows let
  // their successor launch only at their exit, or, in a fused step, only ahead
  // of a split kernel that avoids those rows.
  a.prefetch = 1;
  // The queries of a plain decode are caller inputs, final before it launches
  // (the library's absorb lets its successor launch only at its exit); in a fused
  // step the first kernel writes them.
  a.q_early = step ? 0 : 1;
  a.new_slots = new_slots;
  a.n_new = new_slots ? n_new : 0;
#ifdef GVA_TRACE
  a.trace = g_trace;
#endif
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // clear_status: zero the workspace's status word and pool counter on the stream
  // right before the split kernel, once every check has passed (a rejected call
  // enqueues nothing)
  auto clear = [&]() -> cudaError_t {
    return clear_status ? cudaMemsetAsync(a.status, 0, 2 * sizeof(int), st) : cudaSuccess;
  };

  cudaError_t err;
  if (p.tc) {
    a.tile = gva::tc_decode_tile(sh);
    const int tt = a.tile;
    const int row = sh.G * sh.d_h;
    CUtensorMap tv{}, tk{};
    if ((s = encode_2d(&tv, Vv, num_slots, row, row, tt, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != GVA_OK)
      return s;
    tk = tv;
    if (sh.d_r > 0) {
      const int drp = sh.d_r <= 16 ? 16 : 32;
      if ((s = encode_2d(&tk, KR, num_slots, sh.d_r, sh.d_r, tt, drp,
                         drp == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B)) != GVA_OK)
        return s;
    }
    if ((err = clear()) != cudaSuccess) return cuda_fail(err, "clearing the status word");
    err = gva::launch_decode_tc(sh, a, tv, tk, st);
  } else if (p.mma) {
    a.tile = gva::mma_tile(sh, gqa);
    const int tt = a.tile;
    const int row = sh.G * sh.d_h;
    // value (and GQA key) boxes: 64 columns with a 128-byte swizzle, or one
    // 32-column group with a 64-byte swizzle for d_h = 32
    const int vw = sh.d_h < 64 ? sh.d_h : 64;
    const CUtensorMapSwizzle vsw = vw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap tx{}, tv{}, tk{};
    if ((s = encode_2d(&tx, X, num_slots, row, row, tt, vw, vsw)) != GVA_OK) return s;
    tv = tx;
    if (gqa && (s = encode_2d(&tv, Vv, num_slots, row, row, tt, vw, vsw)) != GVA_OK)
      return s;
    tk = tx;
    if (!gqa && sh.d_r > 0) {
      const int drp = sh.d_r <= 16 ? 16 : 32;
      if ((s = encode_2d(&tk, KR, num_slots, sh.d_r, sh.d_r, tt, drp,
                         drp == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B)) != GVA_OK)
        return s;
    }
    if ((err = clear()) != cudaSuccess) return cuda_fail(err, "clearing the status word");
    err = gva::launch_decode_mma(sh, gqa, a, tx, tv, tk, st);
  } else {
    a.tile = gva::simt_tile();
    if ((err = clear()) != cudaSuccess) return cuda_fail(err, "clearing the status word");
    err = gva::launch_decode_simt(sh, gqa, a, st);
    if (err == cudaErrorNotSupported)
      return fail(GVA_ERR_UNSUPPORTED, "no decode kernel for H=%d G=%d d_h=%d d_r=%d", sh.H, sh.G,
                  sh.d_h, sh.d_r);
  }
  if (err != cudaSuccess) return cuda_fail(err, "decode split kernel launch");
  a.H = sh.H;   // the combine sees the nq * H heads of the partials
  err = gva::launch_combine(sh, a, out, lse, st);
  if (err != cudaSuccess) return cuda_fail(err, "combine kernel launch");
  return GVA_OK;
}

}  // namespace

namespace gva {
// Lets other translation units of the library record a reason for gva_last_error.
void set_error_message(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

// gva_decode_attention that also zeroes the workspace's status word on the stream,
// after validation and right before the split kernel (used by the entry point
// whose scratch is shared by all calls).
gva_status_t decode_attention_clearing_status(const gva_shape_t* shape, const float* q_abs,
                                              const void* V_cache, const void* kr_cache,
                                              const int32_t* seq_offset, const int32_t* seq_len,
                                              int64_t max_total_tokens, int64_t num_slots,
                                              void* out, float* lse, void* workspace,
                                              size_t ws_bytes, void* stream) {
  return decode_common(shape, false, q_abs, V_cache, V_cache, kr_cache, seq_offset, seq_len,
                       max_total_tokens, num_slots, out, lse, workspace, ws_bytes, stream,
                       nullptr, 0, 1, false, /*clear_status=*/true);
}
}  // namespace gva

extern "C" {

const char* gva_status_string(gva_status_t s) {
  switch (s) {
    case GVA_OK: return "ok";
    case GVA_ERR_INVALID_ARG: return "invalid argument";
    case GVA_ERR_UNSUPPORTED: return "unsupported shape";
    case GVA_ERR_WORKSPACE: return "workspace too small";
    case GVA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* gva_last_error(void) { return g_err; }

#ifdef GVA_TRACE
// Trace builds only: device buffer of grid * 8 uint64 receiving the timeline of
// the next split kernels (NULL turns tracing off).
void gva_trace_set_buffer(void* dev_buf) { g_trace = static_cast<unsigned long long*>(dev_buf); }
#endif

// Argument checks of the absorb (shape already checked; B > 0).
static gva_status_t absorb_check(const gva_shape_t& sh, const void* q, const void* M,
                                 const int32_t* q_pos, const float* q_abs) {
  if (!q || !q_abs || !q_pos || (sh.d_n > 0 && !M))
    return fail(GVA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(q) || (M && !aligned16(M)) || !aligned16(q_pos) || !aligned16(q_abs))
    return fail(GVA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t smem = gva::absorb_smem_bytes(sh);
  if (smem > 200 * 1024) return fail(GVA_ERR_UNSUPPORTED, "M_h too large for one CTA (%zu bytes)", smem);
  return GVA_OK;
}

// Argument checks of the append (shape already checked; N > 0).
static gva_status_t append_check(const gva_shape_t& sh, const void* v_new, const void* kpe_new,
                                 const int32_t* slot, const int32_t* pos, int64_t num_slots,
                                 const void* V_cache, const void* kr_cache) {
  if (!v_new || !slot || !pos || !V_cache || (sh.d_r > 0 && (!kpe_new || !kr_cache)))
    return fail(GVA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(v_new) || !aligned16(V_cache) || (kpe_new && !aligned16(kpe_new)) ||
      (kr_cache && !aligned16(kr_cache)) || !aligned16(slot) || !aligned16(pos))
    return fail(GVA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((sh.G * sh.d_h * elt(sh.cache_dtype)) % 16)
    return fail(GVA_ERR_INVALID_ARG, "value rows must be multiples of 16 bytes");
  if (num_slots < 1) return fail(GVA_ERR_INVALID_ARG, "num_slots=%lld < 1", (long long)num_slots);
  return GVA_OK;
}

static gva_status_t absorb_impl(const gva_shape_t* shp, const void* q, const void* M,
                                const int32_t* q_pos, float* q_abs, void* stream, bool early) {
  gva_status_t s = check_shape(shp, false, gva::kMaxQueryRows);
  if (s != GVA_OK) return s;
  const gva_shape_t& sh = *shp;
  if (sh.B == 0) return GVA_OK;
  if ((s = absorb_check(sh, q, M, q_pos, q_abs)) != GVA_OK) return s;
  const float c = scale_of(sh, false) * gva::kLog2e;
  cudaError_t e =
      gva::launch_absorb(sh, q, M, q_pos, q_abs, c, static_cast<cudaStream_t>(stream), early);
  return e == cudaSuccess ? GVA_OK : cuda_fail(e, "absorb launch");
}

static gva_status_t append_impl(const gva_shape_t* shp, int32_t N, const void* v_new,
                                const void* kpe_new, const int32_t* slot, const int32_t* pos,
                                int64_t num_slots, void* V_cache, void* kr_cache,
                                int32_t* err_flag, void* stream, bool early) {
  gva_status_t s = check_shape(shp, false);
  if (s != GVA_OK) return s;
  const gva_shape_t& sh = *shp;
  if (N < 0) return fail(GVA_ERR_INVALID_ARG, "N=%d < 0", N);
  if (N == 0) return GVA_OK;
  if ((s = append_check(sh, v_new, kpe_new, slot, pos, num_slots, V_cache, kr_cache)) != GVA_OK)
    return s;
  cudaError_t e = gva::launch_append(sh, N, v_new, kpe_new, slot, pos, num_slots, V_cache, kr_cache,
                                     err_flag, static_cast<cudaStream_t>(stream), early);
  return e == cudaSuccess ? GVA_OK : cuda_fail(e, "append launch");
}

gva_status_t gva_absorb_query(const gva_shape_t* shp, const void* q, const void* M,
                              const int32_t* q_pos, float* q_abs, void* stream) {
  return absorb_impl(shp, q, M, q_pos, q_abs, stream, false);
}

gva_status_t gva_append_cache(const gva_shape_t* shp, int32_t N, const void* v_new,
                              const void* kpe_new, const int32_t* slot, const int32_t* pos,
                              int64_t num_slots, void* V_cache, void* kr_cache, int32_t* err_flag,
                              void* stream) {
  return append_impl(shp, N, v_new, kpe_new, slot, pos, num_slots, V_cache, kr_cache, err_flag,
                     stream, false);
}

size_t gva_decode_workspace_size(const gva_shape_t* shp, int64_t max_total_tokens) {
  if (check_shape(shp, false) != GVA_OK && check_shape(shp, true) != GVA_OK) return 0;
  if (max_total_tokens < 0) return 0;
  size_t best = 0;
  for (int gqa = 0; gqa < 2; ++gqa) {
    if (check_shape(shp, gqa) != GVA_OK) continue;
    for (int tc = 0; tc < 2; ++tc) {   // large enough for either split kernel
      Plan p;
      if (plan_decode(*shp, gqa, max_total_tokens, &p, tc == 1) != GVA_OK) return 0;
      if (p.ws.total > best) best = p.ws.total;
    }
  }
  return best;
}

gva_status_t gva_decode_attention(const gva_shape_t* shape, const float* q_abs, const void* V_cache,
                                  const void* kr_cache, const int32_t* seq_offset,
                                  const int32_t* seq_len, int64_t max_total_tokens, int64_t num_slots,
                                  void* out, float* lse, void* workspace, size_t ws_bytes,
                                  void* stream) {
  return decode_common(shape, false, q_abs, V_cache, V_cache, kr_cache, seq_offset, seq_len,
                       max_total_tokens, num_slots, out, lse, workspace, ws_bytes, stream);
}

gva_status_t gva_decode_step(const gva_shape_t* shape, const void* q, const void* M,
                             const int32_t* q_pos, int32_t n_new, const void* v_new,
                             const void* kpe_new, const int32_t* slot, const int32_t* pos,
                             void* V_cache, void* kr_cache, int64_t num_slots,
                             const int32_t* seq_offset, const int32_t* seq_len,
                             int64_t max_total_tokens, float* q_abs, void* out, float* lse,
                             int32_t* err_flag, void* workspace, size_t ws_bytes, void* stream) {
  gva_status_t s = check_shape(shape, false);
  if (s != GVA_OK) return s;
  if (shape->B == 0 && n_new == 0) return GVA_OK;
  // Validate the decode first (it has the strictest requirements), without launching.
  Plan p;
  if (shape->B > 0 &&
      (s = decode_check(*shape, false, q_abs, V_cache, V_cache, kr_cache, seq_offset, seq_len,
                        max_total_tokens, num_slots, out, lse, workspace, ws_bytes, 1, false, &p)) !=
          GVA_OK)
    return s;
  // 1. new tokens into the cache and absorbed queries (one kernel), 2. decode.
  // The first kernel lets the split kernel launch immediately and waits on the
  // preceding kernel before its first store; the split kernel streams every cache
  // tile without a new slot before it waits on the first kernel, so the cache
  // streams while the queries are absorbed.  Two launches instead of three save
  // one grid-completion wait on the step's critical path.
  if (n_new < 0) return fail(GVA_ERR_INVALID_ARG, "n_new=%d < 0", n_new);
  if (shape->B > 0 && (s = absorb_check(*shape, q, M, q_pos, q_abs)) != GVA_OK) return s;
  if (n_new > 0 &&
      (s = append_check(*shape, v_new, kpe_new, slot, pos, num_slots, V_cache, kr_cache)) != GVA_OK)
    return s;
  {
    const float c = scale_of(*shape, false) * gva::kLog2e;
    cudaError_t e = gva::launch_prep_step(*shape, q, M, q_pos, q_abs, c, n_new, v_new, kpe_new,
                                          slot, pos, num_slots, V_cache, kr_cache, err_flag,
                                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "append + absorb launch");
  }
  if (shape->B == 0) return GVA_OK;
  return decode_common(shape, false, q_abs, V_cache, V_cache, kr_cache, seq_offset, seq_len,
                       max_total_tokens, num_slots, out, lse, workspace, ws_bytes, stream, slot,
                       n_new, 1, false, false, /*step=*/true);
}

size_t gva_decode_workspace_size_multi(const gva_shape_t* shape, int32_t n_query,
                                       int64_t max_total_tokens) {
  if (!shape || n_query < 1 || shape->G <= 0) return 0;
  // wide blocks (tcgen05 kernel) write the output directly: only the status word
  if ((shape->H / shape->G) * (long long)n_query > 8 && !(shape->flags & GVA_FLAG_FMA_PATH))
    return check_shape(shape, false) == GVA_OK && gva::prefill_supported(*shape, n_query) ? 256 : 0;
  if (n_query > 64) return 0;
  gva_shape_t shv = *shape;
  shv.H = shape->H * n_query;
  return gva_decode_workspace_size(&shv, max_total_tokens);
}

// Wide multi-token blocks (more than 8 query columns per value group) run on the
// tcgen05 kernel: one CTA per 128 query rows of a group, output written directly.
static gva_status_t prefill_common(const gva_shape_t* shp, int nq, const float* q_abs,
                                   const void* V_cache, const void* kr_cache,
                                   const int32_t* seq_offset, const int32_t* seq_len,
                                   int64_t num_slots, void* out, float* lse, void* workspace,
                                   size_t ws_bytes, void* stream) {
  const gva_shape_t& sh = *shp;
  if (!q_abs || !V_cache || !seq_offset || !seq_len || !out || !workspace)
    return fail(GVA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (sh.d_r > 0 && !kr_cache) return fail(GVA_ERR_INVALID_ARG, "kr_cache is NULL with d_r > 0");
  if (!aligned16(q_abs) || !aligned16(V_cache) || (kr_cache && !aligned16(kr_cache)) ||
      !aligned16(out) || !aligned16(workspace) || !aligned16(seq_offset) || !aligned16(seq_len) ||
      (lse && !aligned16(lse)))
    return fail(GVA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (num_slots < 1 || num_slots >= (1ll << 31))
    return fail(GVA_ERR_INVALID_ARG, "num_slots=%lld outside [1, 2^31)", (long long)num_slots);
  if (ws_bytes < 4) return fail(GVA_ERR_WORKSPACE, "workspace %zu bytes < 4", ws_bytes);
  const int row = sh.G * sh.d_h, tt = gva::prefill_tile_rows(sh);
  CUtensorMap tv{}, tk{};
  gva_status_t s;
  if ((s = encode_2d(&tv, V_cache, num_slots, row, row, tt, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != GVA_OK)
    return s;
  tk = tv;
  if (sh.d_r > 0) {
    const int drp = sh.d_r <= 16 ? 16 : 32;
    if ((s = encode_2d(&tk, kr_cache, num_slots, sh.d_r, sh.d_r, tt, drp,
                       drp == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B)) != GVA_OK)
      return s;
  }
  cudaError_t e = gva::launch_prefill(sh, nq, q_abs, seq_offset, seq_len, num_slots, out, lse,
                                      static_cast<int*>(workspace), tv, tk,
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GVA_OK : cuda_fail(e, "multi-token tcgen05 kernel launch");
}

gva_status_t gva_decode_attention_multi(const gva_shape_t* shape, int32_t n_query,
                                        const float* q_abs, const void* V_cache,
                                        const void* kr_cache, const int32_t* seq_offset,
                                        const int32_t* seq_len, int64_t max_total_tokens,
                                        int64_t num_slots, void* out, float* lse,
                                        void* workspace, size_t ws_bytes, void* stream) {
  gva_status_t s = check_shape(shape, false);
  if (s != GVA_OK) return s;
  if (n_query < 1) return fail(GVA_ERR_INVALID_ARG, "n_query=%d < 1", n_query);
  if (shape->B == 0) return GVA_OK;
  if ((shape->H / shape->G) * (long long)n_query > 8 && !(shape->flags & GVA_FLAG_FMA_PATH)) {
    if (!gva::prefill_supported(*shape, n_query))
      return fail(GVA_ERR_UNSUPPORTED, "no multi-token kernel for H/G=%d, n_query=%d, d_h=%d, "
                  "d_r=%d (tcgen05 path: bf16 cache, d_h in {64, 128}, d_r in {0, 8, ..., 32}, "
                  "H/G dividing 128)", shape->H / shape->G, n_query, shape->d_h, shape->d_r);
    return prefill_common(shape, n_query, q_abs, V_cache, kr_cache, seq_offset, seq_len,
                          num_slots, out, lse, workspace, ws_bytes, stream);
  }
  return decode_common(shape, false, q_abs, V_cache, V_cache, kr_cache, seq_offset, seq_len,
                       max_total_tokens, num_slots, out, lse, workspace, ws_bytes, stream,
                       nullptr, 0, n_query);
}

gva_status_t gva_shared_kv_decode_attention(const gva_shape_t* shape, const void* q,
                                            const void* V_cache, const int32_t* seq_offset,
                                            const int32_t* seq_len, int64_t max_total_tokens,
                                            int64_t num_slots, void* out, float* lse,
                                            void* workspace, size_t ws_bytes, void* stream) {
  if (!shape) return fail(GVA_ERR_INVALID_ARG, "shape is NULL");
  if (shape->d_r != 0 || shape->d_n != shape->d_h)
    return fail(GVA_ERR_INVALID_ARG, "shared keys and values need d_r == 0 and d_n == d_h (got %d, %d)",
                shape->d_r, shape->d_n);
  // keys are the values (M_h = I): the raw query meets the value tile directly
  return decode_common(shape, false, q, V_cache, V_cache, nullptr, seq_offset, seq_len,
                       max_total_tokens, num_slots, out, lse, workspace, ws_bytes, stream,
                       nullptr, 0, 1, /*raw_q=*/true);
}

gva_status_t gva_merge_states(const gva_shape_t* shape, int32_t R, const float* outs,
                              const float* lses, void* out, float* lse, void* stream) {
  gva_status_t s = check_shape(shape, true);
  if (s != GVA_OK) return s;
  if (R < 1 || R > 1024) return fail(GVA_ERR_INVALID_ARG, "R=%d outside [1,1024]", R);
  if (shape->B == 0) return GVA_OK;
  if (!outs || !lses || !out) return fail(GVA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(outs) || !aligned16(lses) || !aligned16(out) || (lse && !aligned16(lse)))
    return fail(GVA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  cudaError_t e = gva::launch_merge_states(*shape, R, outs, lses, out, lse,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GVA_OK : cuda_fail(e, "merge launch");
}

// Argument checks of the GQA append and query rotation (shape checked as GQA).
static gva_status_t gqa_rope_check(const gva_shape_t& sh) {
  if (sh.d_h % 2 || sh.d_h > 2 * gva::kMaxRopePairs)
    return fail(GVA_ERR_UNSUPPORTED, "GQA RoPE needs an even d_h <= %d (d_h=%d)",
                2 * gva::kMaxRopePairs, sh.d_h);
  if (!(sh.rope_base > 0.0) || !isfinite(sh.rope_base))
    return fail(GVA_ERR_INVALID_ARG, "rope_base must be positive and finite");
  if ((sh.G * sh.d_h * elt(sh.cache_dtype)) % 16)
    return fail(GVA_ERR_INVALID_ARG, "cache rows must be multiples of 16 bytes");
  return GVA_OK;
}

static gva_status_t gqa_append_check(const gva_shape_t& sh, const void* k_new, const void* v_new,
                                     const int32_t* slot, const int32_t* pos, int64_t num_slots,
                                     const void* K_cache, const void* V_cache) {
  if (!k_new || !v_new || !slot || !pos || !K_cache || !V_cache)
    return fail(GVA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(slot) || !aligned16(pos) ||
      !aligned16(K_cache) || !aligned16(V_cache))
    return fail(GVA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (num_slots < 1) return fail(GVA_ERR_INVALID_ARG, "num_slots=%lld < 1", (long long)num_slots);
  return GVA_OK;
}

gva_status_t gqa_append_cache(const gva_shape_t* shape, int32_t N, const void* k_new,
                              const void* v_new, const int32_t* slot, const int32_t* pos,
                              int64_t num_slots, void* K_cache, void* V_cache, int32_t* err_flag,
                              void* stream) {
  gva_status_t s = check_shape(shape, true);
  if (s != GVA_OK) return s;
  if ((s = gqa_rope_check(*shape)) != GVA_OK) return s;
  if (N < 0) return fail(GVA_ERR_INVALID_ARG, "N=%d < 0", N);
  if (N == 0) return GVA_OK;
  if ((s = gqa_append_check(*shape, k_new, v_new, slot, pos, num_slots, K_cache, V_cache)) != GVA_OK)
    return s;
  cudaError_t e = gva::launch_gqa_append(*shape, N, k_new, v_new, slot, pos, num_slots, K_cache,
                                         V_cache, err_flag, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GVA_OK : cuda_fail(e, "GQA append launch");
}

gva_status_t gqa_decode_step(const gva_shape_t* shape, const void* q, const int32_t* q_pos,
                             int32_t n_new, const void* k_new, const void* v_new,
                             const int32_t* slot, const int32_t* pos, void* K_cache,
                             void* V_cache, int64_t num_slots, const int32_t* seq_offset,
                             const int32_t* seq_len, int64_t max_total_tokens, float* q_rot,
                             void* out, float* lse, int32_t* err_flag, void* workspace,
                             size_t ws_bytes, void* stream) {
  gva_status_t s = check_shape(shape, true);
  if (s != GVA_OK) return s;
  if ((s = gqa_rope_check(*shape)) != GVA_OK) return s;
  if (n_new < 0) return fail(GVA_ERR_INVALID_ARG, "n_new=%d < 0", n_new);
  if (shape->B == 0 && n_new == 0) return GVA_OK;
  if (!q_rot || !q || !q_pos || !K_cache || !V_cache || !seq_offset || !seq_len || !out ||
      !workspace)
    return fail(GVA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(q) || !aligned16(q_pos) || !aligned16(q_rot))
    return fail(GVA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (n_new > 0 &&
      (s = gqa_append_check(*shape, k_new, v_new, slot, pos, num_slots, K_cache, V_cache)) != GVA_OK)
    return s;
  // the decode reads the rotated float32 query; every check of it happens here,
  // before the first launch
  gva_shape_t shd = *shape;
  shd.q_dtype = GVA_F32;
  Plan p;
  if (shape->B > 0 &&
      (s = decode_check(shd, true, q_rot, K_cache, V_cache, nullptr, seq_offset, seq_len,
                        max_total_tokens, num_slots, out, lse, workspace, ws_bytes, 1, false, &p)) !=
          GVA_OK)
    return s;
  cudaError_t e = gva::launch_gqa_prep(*shape, q, q_pos, q_rot, n_new, k_new, v_new, slot, pos,
                                       num_slots, K_cache, V_cache, err_flag,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "GQA query rotation + append launch");
  if (shape->B == 0) return GVA_OK;
  return decode_common(&shd, true, q_rot, K_cache, V_cache, nullptr, seq_offset, seq_len,
                       max_total_tokens, num_slots, out, lse, workspace, ws_bytes, stream, slot,
                       n_new, 1, false, false, /*step=*/true);
}

gva_status_t gqa_decode_attention(const gva_shape_t* shape, const void* q, const void* K_cache,
                                  const void* V_cache, const int32_t* seq_offset,
                                  const int32_t* seq_len, int64_t max_total_tokens, int64_t num_slots,
                                  void* out, float* lse, void* workspace, size_t ws_bytes,
                                  void* stream) {
  return decode_common(shape, true, q, K_cache, V_cache, nullptr, seq_offset, seq_len,
                       max_total_tokens, num_slots, out, lse, workspace, ws_bytes, stream);
}

}  // extern "C"
