// Instantiations and host launcher of the tensor-core split kernel.
#include "decode_mma.cuh"
#include "launch.h"

namespace gva {

namespace {

template <class C>
cudaError_t run(const gva_shape_t& sh, DecodeArgs& a, const CUtensorMap& tx, const CUtensorMap& tv,
                const CUtensorMap& tk, cudaStream_t st) {
  const size_t smem = C::smem_bytes(sh.B);
  auto k = decode_mma_kernel<C>;
  cudaError_t e = ensure_max_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(a.grid), dim3(C::THREADS), smem, st, a, tx, tv, tk);
}

// Visit the instantiation matching (d_h, G, H/G, padded d_r, gqa); f receives a
// default-constructed config type.  Returns false when none matches.
template <class F>
bool dispatch(const gva_shape_t& sh, bool gqa, F&& f) {
  // columns per group (heads per group x query tokens), padded up to 4 or 8
  const int cols = sh.H / sh.G;
  const int hpg = cols <= 4 ? 4 : (cols <= 8 ? 8 : -1);
  const int drp = gqa ? 0 : (sh.d_r == 0 ? 0 : (sh.d_r <= 16 ? 16 : (sh.d_r <= 32 ? 32 : -1)));
#define GVA_CASE(DH, NG, HPG, DRP, GQ)                                                     \
  if (sh.d_h == DH && sh.G == NG && hpg == HPG && drp == DRP && gqa == GQ) {              \
    f(MmaCfg<DH, NG, HPG, DRP, GQ>{});                                                     \
    return true;                                                                           \
  }
#define GVA_CASES_NG(DH, HPG, DRP, GQ) \
  GVA_CASE(DH, 2, HPG, DRP, GQ) GVA_CASE(DH, 4, HPG, DRP, GQ) GVA_CASE(DH, 8, HPG, DRP, GQ)
#define GVA_CASES_HPG(DH, DRP, GQ) GVA_CASES_NG(DH, 4, DRP, GQ) GVA_CASES_NG(DH, 8, DRP, GQ)
  GVA_CASES_HPG(32, 0, false)
  GVA_CASES_HPG(32, 16, false)
  GVA_CASES_HPG(32, 32, false)
  GVA_CASES_HPG(64, 0, false)
  GVA_CASES_HPG(64, 16, false)
  GVA_CASES_HPG(64, 32, false)
  GVA_CASES_HPG(128, 0, false)
  GVA_CASES_HPG(128, 16, false)
  GVA_CASES_HPG(128, 32, false)
  GVA_CASES_HPG(32, 0, true)
  GVA_CASES_HPG(64, 0, true)
  GVA_CASES_HPG(128, 0, true)
#undef GVA_CASES_HPG
#undef GVA_CASES_NG
#undef GVA_CASE
  return false;
}

}  // namespace

bool mma_supported(const gva_shape_t& sh, bool gqa) {
  if (sh.cache_dtype != GVA_BF16) return false;
  return dispatch(sh, gqa, [](auto) {});
}

int mma_tile(const gva_shape_t& sh, bool gqa) {
  int tt = 0;
  dispatch(sh, gqa, [&](auto c) { tt = decltype(c)::TT; });
  return tt;
}

int mma_grid(const gva_shape_t& sh, int num_sms, long long max_total_tokens, bool gqa) {
  int tt = 16, minb = 2;
  size_t smem = 0;
  dispatch(sh, gqa, [&](auto c) {
    tt = decltype(c)::TT;
    minb = decltype(c)::MINB;
    smem = decltype(c)::smem_bytes(sh.B);
  });
  int per_sm = (int)((227 * 1024) / (smem + 1024));
  per_sm = per_sm < 1 ? 1 : (per_sm > minb ? minb : per_sm);
  if (sh.ctas_per_sm > 0) per_sm = sh.ctas_per_sm;
  long long want = (max_total_tokens + tt - 1) / tt;
  long long grid = (long long)num_sms * per_sm;
  if (want < grid) grid = want;
  return grid < 1 ? 1 : (int)grid;
}

cudaError_t launch_decode_mma(const gva_shape_t& sh, bool gqa, DecodeArgs& a,
                              const CUtensorMap& tm_x, const CUtensorMap& tm_v,
                              const CUtensorMap& tm_kr, cudaStream_t st) {
  cudaError_t err = cudaErrorNotSupported;
  dispatch(sh, gqa, [&](auto c) { err = run<decltype(c)>(sh, a, tm_x, tm_v, tm_kr, st); });
  return err;
}

}  // namespace gva
