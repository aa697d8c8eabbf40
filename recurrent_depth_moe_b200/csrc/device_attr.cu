// Per-device, thread-safe kernel attributes and device properties.
//
// A kernel's dynamic shared-memory limit (cudaFuncAttributeMaxDynamicSharedMemorySize)
// is a property of the kernel on one device: a process that drives several GPUs must
// raise it once on each of them, and host threads may launch concurrently.  The set of
// (kernel, device) pairs already raised is guarded by a mutex, so the attribute call is
// made once per pair and every later launch only takes the lock and looks the pair up.
#include "common.cuh"
#include "kernels.h"

#include <mutex>
#include <set>
#include <utility>

namespace rdt {
namespace {
std::mutex g_attr_mu;
std::set<std::pair<const void*, int>> g_attr_done;
constexpr int kMaxDev = 64;
int g_sm_count[kMaxDev];
}  // namespace

bool ensure_smem_limit(const void* kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  const std::pair<const void*, int> key(kernel, dev);
  if (g_attr_done.count(key)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  g_attr_done.insert(key);
  return true;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  if (g_sm_count[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

}  // namespace rdt
