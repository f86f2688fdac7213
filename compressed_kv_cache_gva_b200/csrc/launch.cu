// Record of the function attributes already applied, per kernel and device.
//
// cudaFuncSetAttribute changes per-context state of a kernel; setting it on every
// launch costs host time on the eager path.  The launchers ask here first and
// apply an attribute only when the current device has not yet received an equal
// or larger value for that kernel.
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <tuple>

#include "launch.h"

namespace gva {

namespace {
std::mutex g_mu;
std::map<std::tuple<const void*, int, int>, long long> g_applied;   // (kernel, device, attr) -> value
}  // namespace

bool attr_applied(const void* kernel, int attr, long long value) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  const auto it = g_applied.find(std::make_tuple(kernel, dev, attr));
  return it != g_applied.end() && it->second >= value;
}

void attr_record(const void* kernel, int attr, long long value) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  std::lock_guard<std::mutex> lk(g_mu);
  long long& v = g_applied[std::make_tuple(kernel, dev, attr)];
  if (value > v) v = value;
}

}  // namespace gva
