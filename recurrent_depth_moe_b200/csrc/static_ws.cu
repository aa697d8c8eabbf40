// Decode step for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or any allocator) at the point
// where they run a decode step: a serving loop that must not allocate once it is warm,
// a host runtime that owns no CUDA allocator of its own, or code running inside a
// memory-pool budget that has no room for a per-call workspace.  For them,
// rdt_recurrent_decode_step_static() runs the same decode step as
// rdt_recurrent_decode_step() with its scratch in the file-scope array below instead of
// a caller-provided workspace.  The library allocates nothing on this path.
//
// The array is a module global: every GPU that loads this library holds
// RDT_STATIC_SCRATCH_BYTES of device memory for it until the process exits.
#include "../../include/rdt.h"
#include "common.cuh"

#include <mutex>

// 32 MiB: enough for the 3B-shaped decode (64 sequences, dim 3072, 64 + 1 experts,
// 4224-position caches needs about 14.5 MiB).
static __device__ __align__(256) unsigned char g_rdt_static_scratch[RDT_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
// Device address of the array, per device, resolved on the first call with that device
// current.  A cudaDeviceReset unloads the library's module and makes the cached address
// stale: this path is not usable across a device reset.
void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  In host code the array's
// name is only a host-side stand-in, so the real address comes from
// cudaGetSymbolAddress, resolved once per device with that device current.
rdt_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RDT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RDT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rdt_static_scratch) != cudaSuccess || !p) return RDT_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return RDT_OK;
}
}  // namespace

extern "C" rdt_status rdt_recurrent_decode_step_static(const rdt_config* cfg, const rdt_weights* w,
                                                       const float* h0, const void* e, int batch,
                                                       const int32_t* cache_len, int n_loops, float act_threshold,
                                                       float* h_out, float* halt_weights, int32_t* expert_ids,
                                                       const rdt_kv_cache* cache, void* stream) {
  if (!cache) return RDT_ERR_INVALID_ARG;
  const size_t need = rdt_workspace_size(cfg, batch, 1, cache->t_max);
  if (need == 0) return RDT_ERR_INVALID_ARG;
  if (need > (size_t)RDT_STATIC_SCRATCH_BYTES) return RDT_ERR_WORKSPACE;   // beyond the fixed maximum
  void* ws = nullptr;
  const rdt_status st = scratch_on_current_device(&ws);
  if (st != RDT_OK) return st;
  return rdt_recurrent_decode_step(cfg, w, h0, e, batch, cache_len, n_loops, act_threshold, h_out, halt_weights,
                                   expert_ids, cache, ws, (size_t)RDT_STATIC_SCRATCH_BYTES, stream);
}

// Device status word of the static-scratch decode: the kernels record bounds violations
// and bounded waits that gave up in the first bytes of the scratch (as they do in a
// caller's workspace), and this reads and clears it.  Synchronises `stream`.
extern "C" rdt_status rdt_read_static_status(void* stream) {
  void* ws = nullptr;
  const rdt_status st = scratch_on_current_device(&ws);
  if (st != RDT_OK) return st;
  return rdt_read_device_status(ws, stream);
}
