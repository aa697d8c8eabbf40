// Causal softmax attention, generic CUDA-core version: one warp per (query row,
// head), lanes over the head dimensions, online (running max / running sum)
// softmax over the visible keys.  Handles GQA (score dim = hd) and MLA (score dim
// = nope + rope, the rope key part shared by all heads), prefill (keys from this
// call's K/V) and decode (keys from the loop cache, per-sequence key counts).
// Key j is visible to query row r iff key_pos0 + j <= q_pos[r]
// ("OpenMythos 분석", Core Structure: causal mask; RoPE & generation cache).
#include "common.cuh"
#include "kernels.h"

namespace rdt {

constexpr int ATT_MAXQ = 6;   // score dims up to 192
constexpr int ATT_MAXV = 4;   // value dims up to 128

template <typename T>
__global__ void __launch_bounds__(256) k_attn_simt(AttnParams p) {
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long total = (long long)p.B * p.T * p.H;
  if (gw >= total) return;
  const int h = (int)(gw % p.H);
  const long long row = gw / p.H;
  const int b = (int)(row / p.T);
  const int g = h / p.G;
  const int dq = p.dn + p.dr;
  const T* qp = (const T*)p.q + row * p.q_row + (long long)h * p.q_head;
  float q[ATT_MAXQ];
#pragma unroll
  for (int u = 0; u < ATT_MAXQ; ++u) {
    int d = lane + 32 * u;
    q[u] = (d < dq) ? to_f(qp[d]) * p.scale : 0.f;
  }
  const int n_keys = p.n_keys_dev ? p.n_keys_dev[b] : p.n_keys;
  int n_vis = p.q_pos[row] - p.key_pos0 + 1;
  if (n_vis > n_keys) n_vis = n_keys;
  const T* k1 = (const T*)p.k1 + (long long)b * p.k1_b + (long long)g * p.k1_g;
  const T* k2 = p.k2 ? (const T*)p.k2 + (long long)b * p.k2_b : nullptr;
  const T* vp = (const T*)p.v + (long long)b * p.v_b + (long long)g * p.v_g;
  float m = -INFINITY, l = 0.f;
  float o[ATT_MAXV];
#pragma unroll
  for (int u = 0; u < ATT_MAXV; ++u) o[u] = 0.f;
  for (int j = 0; j < n_vis; ++j) {
    float part = 0.f;
#pragma unroll
    for (int u = 0; u < ATT_MAXQ; ++u) {
      int d = lane + 32 * u;
      if (d < p.dn) part += q[u] * to_f(k1[(long long)j * p.k1_j + d]);
      else if (d < dq) part += q[u] * to_f(k2[(long long)j * p.k2_j + (d - p.dn)]);
    }
    float s = warp_sum(part);
    float mn = fmaxf(m, s);
    float corr = expf(m - mn);
    float e = expf(s - mn);
    l = l * corr + e;
#pragma unroll
    for (int u = 0; u < ATT_MAXV; ++u) {
      int d = lane + 32 * u;
      float vv = (d < p.dv) ? to_f(vp[(long long)j * p.v_j + d]) : 0.f;
      o[u] = o[u] * corr + e * vv;
    }
    m = mn;
  }
  T* op = (T*)p.o + row * p.o_row + (long long)h * p.o_head;
  float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
  for (int u = 0; u < ATT_MAXV; ++u) {
    int d = lane + 32 * u;
    if (d < p.dv) op[d] = from_f<T>(o[u] * inv);
  }
}

int launch_attention_simt(int dtype, const AttnParams& p, cudaStream_t s) {
  if (p.dn + p.dr > 32 * ATT_MAXQ || p.dv > 32 * ATT_MAXV) return -1;
  long long warps = (long long)p.B * p.T * p.H;
  unsigned blocks = (unsigned)((warps + 7) / 8);
  if (blocks == 0) return 0;
  if (dtype == 0) { k_attn_simt<float><<<blocks, 256, 0, s>>>(p); note_launch(); }
  else { k_attn_simt<bf16><<<blocks, 256, 0, s>>>(p); note_launch(); }
  return 0;
}

}  // namespace rdt
