// Record of the function attributes already applied, per kernel and CUDA context.
//
// cudaFuncSetAttribute changes per-context state of a kernel; setting it on every
// launch costs host time on the eager path.  The launchers ask here first and
// apply an attribute only when the current context has not yet received an equal
// or larger value for that kernel.  The record is keyed by the context, so after
// cudaDeviceReset (a new primary context) the attributes are applied again.
#include <cuda.h>
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <tuple>

#include "launch.h"

namespace gva {

namespace {
std::mutex g_mu;
std::map<std::tuple<const void*, const void*, int>, long long> g_applied;   // (kernel, ctx, attr)

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The current context (the runtime makes the device's primary context current).
const void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}
}  // namespace

bool attr_applied(const void* kernel, int attr, long long value) {
  const void* ctx = current_context();
  if (!ctx) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  const auto it = g_applied.find(std::make_tuple(kernel, ctx, attr));
  return it != g_applied.end() && it->second >= value;
}

void attr_record(const void* kernel, int attr, long long value) {
  const void* ctx = current_context();
  if (!ctx) return;
  std::lock_guard<std::mutex> lk(g_mu);
  long long& v = g_applied[std::make_tuple(kernel, ctx, attr)];
  if (value > v) v = value;
}

}  // namespace gva
