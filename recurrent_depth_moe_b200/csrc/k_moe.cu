// MoE routing (S5) and token permutation (S6) of the recurrent block
// ("OpenMythos 분석", MoE: scores = softmax(logits); topk(logits + router_bias);
// gates = scores[idx] renormalised).
//
//  k_router_topk   warp per running row: softmax over E logits, biased top-k by
//                  repeated warp arg-max (ties -> lower expert index), renormalised
//                  gates, and the row's rank inside each chosen expert (atomic
//                  histogram).  Reads one [E] logit row per token: HBM-bound.
//  k_route_scan    one CTA: exclusive scan of segment sizes (E routed experts, then
//                  S shared experts holding every running row) and the grouped-GEMM
//                  tile list (tile_m rows per tile, never crossing a segment).
//  k_route_scatter CTA per running row: slot = offset[e] + rank, writes the
//                  slot <-> token maps and copies the router input row into the
//                  expert-sorted buffer with 16-byte vector moves.
#include "common.cuh"
#include "kernels.h"
#include <limits.h>

namespace rdt {

constexpr int ROUTE_MAXE = 8;   // up to 256 experts (8 per lane)

__global__ void __launch_bounds__(256) k_router_topk(RouteParams p) {
  const int lane = threadIdx.x & 31;
  const int ri = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (ri >= *p.n_run) return;
  const int i = p.run_list[ri];
  const float* lg = p.logits + (long long)i * p.E;
  float raw[ROUTE_MAXE], bl[ROUTE_MAXE];
  float mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < ROUTE_MAXE; ++u) {
    int e = lane + 32 * u;
    raw[u] = (e < p.E) ? lg[e] : -INFINITY;
    bl[u] = (e < p.E) ? raw[u] + p.bias[e] : -INFINITY;
    mx = fmaxf(mx, raw[u]);
  }
  mx = warp_max(mx);
  float sum = 0.f;
#pragma unroll
  for (int u = 0; u < ROUTE_MAXE; ++u) {
    int e = lane + 32 * u;
    if (e < p.E) sum += expf(raw[u] - mx);
  }
  sum = warp_sum(sum);
  float sel_score[32];
  int sel_id[32];
  float gsum = 0.f;
  for (int j = 0; j < p.k; ++j) {
    float bv = -INFINITY;
    int be = INT_MAX;
#pragma unroll
    for (int u = 0; u < ROUTE_MAXE; ++u) {
      int e = lane + 32 * u;
      if (e < p.E && (bl[u] > bv || (bl[u] == bv && e < be))) { bv = bl[u]; be = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    if (be == INT_MAX || be < 0 || be >= p.E) {
      if (lane == 0) record_status(p.st, ST_BOUNDS, 401, be);
      be = 0;
    }
    float rsel = -INFINITY;
#pragma unroll
    for (int u = 0; u < ROUTE_MAXE; ++u) {
      int e = lane + 32 * u;
      if (e == be) { rsel = raw[u]; bl[u] = -INFINITY; }
    }
    rsel = warp_max(rsel);
    float sc = expf(rsel - mx) / sum;
    sel_score[j] = sc;
    sel_id[j] = be;
    gsum += sc;
  }
  if (lane == 0) {
    for (int j = 0; j < p.k; ++j) {
      long long o = (long long)i * p.k + j;
      p.ids[o] = sel_id[j];
      p.gates[o] = sel_score[j] / gsum;
      p.rank[o] = atomicAdd(&p.counts[sel_id[j]], 1);
    }
  }
}

__global__ void k_route_scan(RouteParams p) {
  __shared__ int seg_off[1025];
  __shared__ int tile_off[1025];
  const int nseg = p.E + p.S;
  const int n_run = *p.n_run;
  const int s = threadIdx.x;
  int size = 0;
  if (s < p.E) size = p.counts[s];
  else if (s < nseg) size = n_run;
  int nt = (size + p.tile_m - 1) / p.tile_m;
  // inclusive scans in shared memory (Hillis-Steele), nseg <= blockDim.x <= 1024
  seg_off[s] = (s < nseg) ? size : 0;
  tile_off[s] = (s < nseg) ? nt : 0;
  __syncthreads();
  for (int o = 1; o < blockDim.x; o <<= 1) {
    int a = (s >= o) ? seg_off[s - o] : 0;
    int b = (s >= o) ? tile_off[s - o] : 0;
    __syncthreads();
    seg_off[s] += a;
    tile_off[s] += b;
    __syncthreads();
  }
  int seg_start = seg_off[s] - ((s < nseg) ? size : 0);
  int tile_start = tile_off[s] - ((s < nseg) ? nt : 0);
  if (s < nseg) {
    p.offsets[s] = seg_start;
    for (int q = 0; q < nt; ++q) {
      int ti = tile_start + q;
      if (ti >= p.max_tiles) { record_status(p.st, ST_BOUNDS, 402, ti); break; }
      p.tiles[4 * ti + 0] = s;
      p.tiles[4 * ti + 1] = seg_start + q * p.tile_m;
      p.tiles[4 * ti + 2] = min(p.tile_m, size - q * p.tile_m);
      p.tiles[4 * ti + 3] = 0;
    }
  }
  if (s == blockDim.x - 1) {
    p.offsets[nseg] = seg_off[s];
    *p.n_tiles = min(tile_off[s], p.max_tiles);
  }
}

template <typename T>
__global__ void __launch_bounds__(128) k_route_scatter(RouteParams p) {
  const int ri = blockIdx.x;
  if (ri >= *p.n_run) return;
  const int i = p.run_list[ri];
  const int kS = p.k + p.S;
  __shared__ int slots[64];
  if (threadIdx.x < kS) {
    int j = threadIdx.x;
    int slot;
    float gate;
    if (j < p.k) {
      long long o = (long long)i * p.k + j;
      int e = p.ids[o];
      slot = p.offsets[e] + p.rank[o];
      gate = p.gates[o];
    } else {
      slot = p.offsets[p.E + (j - p.k)] + ri;
      gate = 1.f;
    }
    if (slot < 0 || slot >= p.max_slots) {
      record_status(p.st, ST_BOUNDS, 403, slot);
      slot = -1;
    } else {
      p.tok_of[slot] = i;
      p.gate_of[slot] = gate;
    }
    p.slot_of[(long long)i * kS + j] = slot;
    slots[j] = slot;
  }
  __syncthreads();
  const size_t row_bytes = (size_t)p.D * sizeof(T);
  const char* src = (const char*)p.f + (size_t)i * row_bytes;
  if ((row_bytes & 15) == 0) {
    const int nv = (int)(row_bytes / 16);
    for (int j = 0; j < kS; ++j) {
      if (slots[j] < 0) continue;
      char* dst = (char*)p.xg + (size_t)slots[j] * row_bytes;
      for (int v = threadIdx.x; v < nv; v += blockDim.x)
        ((int4*)dst)[v] = ((const int4*)src)[v];
    }
  } else {
    for (int j = 0; j < kS; ++j) {
      if (slots[j] < 0) continue;
      T* dst = (T*)p.xg + (size_t)slots[j] * p.D;
      for (int d = threadIdx.x; d < p.D; d += blockDim.x) dst[d] = ((const T*)src)[d];
    }
  }
}

// Router logits for few rows (decode), logits[m, e] = f[m, :] . Wr[e, :]: CTA per expert,
// so the weights stream through E CTAs at once (the fused tcgen05 router would be one
// CTA).  Warp w takes the 8 rows 8 w .. 8 w + 7 together: each 16-byte weight load
// serves 8 rows, and the 9 loads of a step are in flight at once.
__global__ void __launch_bounds__(256) k_router_small(const bf16* __restrict__ f, const bf16* __restrict__ wr, int M,
                                                     int K, int E, float* __restrict__ logits) {
  constexpr int RW = 8;
  const int e = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bf16* w = wr + (long long)e * K;
  for (int m0 = warp * RW; m0 < M; m0 += 8 * RW) {
    float acc[RW];
#pragma unroll
    for (int i = 0; i < RW; ++i) acc[i] = 0.f;
    for (int k = lane * 8; k < K; k += 256) {
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(w + k));
      uint4 a[RW];
#pragma unroll
      for (int i = 0; i < RW; ++i)
        a[i] = m0 + i < M ? __ldg(reinterpret_cast<const uint4*>(f + (long long)(m0 + i) * K + k)) : make_uint4(0, 0, 0, 0);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 fb = __bfloat1622float2(b2[q]);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          const float2 fa = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(&a[i])[q]);
          acc[i] = fmaf(fa.x, fb.x, acc[i]);
          acc[i] = fmaf(fa.y, fb.y, acc[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      const float t = warp_sum(acc[i]);
      if (lane == 0 && m0 + i < M) logits[(long long)(m0 + i) * E + e] = t;
    }
  }
}

bool launch_router_small(const void* f, const void* wr, int M, int K, int E, float* logits, cudaStream_t s) {
  if (K % 8 || ((uintptr_t)f & 15) || ((uintptr_t)wr & 15) || M <= 0 || E <= 0) return false;
  k_router_small<<<E, 256, 0, s>>>((const bf16*)f, (const bf16*)wr, M, K, E, logits);
  note_launch();
  return true;
}

void launch_router_topk(const RouteParams& p, cudaStream_t s) {
  { k_router_topk<<<(p.N + 7) / 8, 256, 0, s>>>(p); note_launch(); }
}
void launch_route_scan(const RouteParams& p, cudaStream_t s) {
  int nseg = p.E + p.S;
  int threads = 32;
  while (threads < nseg) threads <<= 1;
  { k_route_scan<<<1, threads, 0, s>>>(p); note_launch(); }
}
void launch_route_scatter(int dtype, const RouteParams& p, cudaStream_t s) {
  if (dtype == 0) { k_route_scatter<float><<<p.N, 128, 0, s>>>(p); note_launch(); }
  else { k_route_scatter<bf16><<<p.N, 128, 0, s>>>(p); note_launch(); }
}

}  // namespace rdt
