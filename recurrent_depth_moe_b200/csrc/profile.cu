// Launch counting and per-kernel-class timing with CUDA events recorded on the
// caller's stream around each launch (for benchmarks; off by default).
#include "../../include/rdt.h"
#include "common.cuh"
#include "kernels.h"

#include <atomic>
#include <string.h>
#include <vector>

namespace rdt {

static std::atomic<unsigned long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {
const char* kClassNames[PC_COUNT] = {"loop_prologue", "qkv_gemm_rope", "attention", "o_gemm_residual",
                                     "ffn_rmsnorm",   "router_gemm",   "route_topk_permute", "expert_up_swiglu",
                                     "expert_down_gate", "combine_lora_inject_act", "other", "dense_block", "lm_head", "embed_cast_greedy",
                                     "depth_kv_fill"};
struct Rec {
  int cls;
  cudaEvent_t a, b;
};
struct Prof {
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t next = 0;
  std::vector<Rec> recs;
  int dropped = 0;
};
Prof g_prof;

cudaEvent_t take_event() {
  if (g_prof.next >= g_prof.pool.size()) return nullptr;
  return g_prof.pool[g_prof.next++];
}
}  // namespace

// Only the outermost scope of a host thread records: a whole-block scope then holds the
// block's attention and GEMM launches once, not again under their own classes.
static thread_local int t_scope_depth = 0;

ProfScope::ProfScope(int cls, cudaStream_t s) : cls_(cls), s_(s), a_(nullptr) {
  if (t_scope_depth++ > 0 || !g_prof.on) return;
  a_ = take_event();
  if (a_) cudaEventRecord((cudaEvent_t)a_, s);
}
ProfScope::~ProfScope() {
  --t_scope_depth;
  if (!g_prof.on || !a_) return;
  cudaEvent_t b = take_event();
  if (!b) {
    ++g_prof.dropped;
    return;
  }
  cudaEventRecord(b, s_);
  g_prof.recs.push_back(Rec{cls_, (cudaEvent_t)a_, b});
}

}  // namespace rdt

using namespace rdt;

extern "C" {

unsigned long long rdt_launch_count(void) { return g_launches.load(); }

rdt_status rdt_profile_start(void) {
  const size_t want = 1 << 16;
  while (g_prof.pool.size() < want) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return RDT_ERR_CUDA;
    g_prof.pool.push_back(e);
  }
  g_prof.next = 0;
  g_prof.recs.clear();
  g_prof.dropped = 0;
  g_prof.on = true;
  return RDT_OK;
}

int rdt_profile_stop(rdt_kernel_time* out, int max_entries) {
  g_prof.on = false;
  double ms[PC_COUNT] = {0};
  int n[PC_COUNT] = {0};
  for (const Rec& r : g_prof.recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return -1;
    ms[r.cls] += t;
    n[r.cls] += 1;
  }
  int k = 0;
  for (int c = 0; c < PC_COUNT && k < max_entries; ++c) {
    if (!n[c]) continue;
    memset(&out[k], 0, sizeof(out[k]));
    strncpy(out[k].name, kClassNames[c], sizeof(out[k].name) - 1);
    out[k].launches = n[c];
    out[k].total_ms = ms[c];
    ++k;
  }
  g_prof.recs.clear();
  return k;
}

}  // extern "C"
