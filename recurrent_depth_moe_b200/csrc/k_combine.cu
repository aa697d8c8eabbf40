// S9 as a warp-per-row kernel for row widths that are multiples of 128: the fused
// combine + depth-wise LoRA + LTI injection + freeze + ACT step of one loop.
//
// Lane l holds columns 4l + 128j (j < D/128) of its row in registers, so every global
// access is a coalesced 16-byte vector and every input is read exactly once:
//   trans  = x1 + sum_{j < k+S} y[slot_of[i][j]]          (gates already applied)
//   z_q    = (trans . Wd_q) * scale[min(t, mli-1)]_q       (warp reductions, q < r)
//   trans += sum_q z_q B_q                                 ("OpenMythos 분석", Recurrent Block)
//   h_new  = A h + B_inj e + trans                         (LTIInjection, latent reasoning)
//   rows halted before loop t keep h (frozen)
//   ACT:  p = sigmoid(h_new . w_halt + b + off); w = remainder if cum + p >= thr or
//         last loop, else p; cum += p; h_out += w h_new    ("OpenMythos 분석", ACT)
// The LoRA matrices (2 r D elements) are shared by all rows and stay in L1/L2.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace rdt {

template <typename T> struct Vec4;
template <> struct Vec4<float> {
  static __device__ __forceinline__ float4 load(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
};
template <> struct Vec4<bf16> {
  static __device__ __forceinline__ float4 load(const bf16* p) {
    uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x), b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
};

__device__ __forceinline__ float4 f4_add(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
// Packed fp32x2 arithmetic (two independent fp32 operations per instruction).
__device__ __forceinline__ float4 f4_add2(float4 a, float4 b) {
  const float2 lo = __fadd2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
  const float2 hi = __fadd2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
// a + s b, elementwise
__device__ __forceinline__ float4 f4_fma2(float s, float4 b, float4 a) {
  const float2 lo = __ffma2_rn(make_float2(s, s), make_float2(b.x, b.y), make_float2(a.x, a.y));
  const float2 hi = __ffma2_rn(make_float2(s, s), make_float2(b.z, b.w), make_float2(a.z, a.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
// a + b c, elementwise
__device__ __forceinline__ float4 f4_fmav2(float4 b, float4 c, float4 a) {
  const float2 lo = __ffma2_rn(make_float2(b.x, b.y), make_float2(c.x, c.y), make_float2(a.x, a.y));
  const float2 hi = __ffma2_rn(make_float2(b.z, b.w), make_float2(c.z, c.w), make_float2(a.z, a.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
template <typename T> __device__ __forceinline__ void store4(T* p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
template <> __device__ __forceinline__ void store4<bf16>(bf16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ float f4_dot(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

// Plain 4-element load usable on shared or global memory (generic address).
template <typename T> __device__ __forceinline__ float4 ld4(const T* p);
template <> __device__ __forceinline__ float4 ld4<float>(const float* p) { return *reinterpret_cast<const float4*>(p); }
template <> __device__ __forceinline__ float4 ld4<bf16>(const bf16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
  float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// Warp sums of 16 values at once (a transposed butterfly, 16 shuffles instead of 80):
// at each step a lane keeps one half of its values, sends the other half to its partner
// and adds the partner's copy of the half it kept.  Lanes 2q and 2q + 1 end with the sum
// of v[q] over the warp.
__device__ __forceinline__ float warp_sum16(const float (&v)[16], int lane) {
  float a[8], b[4], c[2];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    a[i] = (hi ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, hi ? v[i] : v[i + 8], 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 8;
    b[i] = (hi ? a[i + 4] : a[i]) + __shfl_xor_sync(0xffffffffu, hi ? a[i] : a[i + 4], 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 4;
    c[i] = (hi ? b[i + 2] : b[i]) + __shfl_xor_sync(0xffffffffu, hi ? b[i] : b[i + 2], 4);
  }
  const bool hi = lane & 2;
  float d = (hi ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, hi ? c[0] : c[1], 2);
  return d + __shfl_xor_sync(0xffffffffu, d, 1);
}

// A row is processed by a group of WPR warps; warp wr of the group owns the float4
// columns 4 lane + 128 j for j in [wr VQ, (wr + 1) VQ), VQ = VPL / WPR.  Row-wide sums go
// through shared memory: each warp reduces its part, lane 0 stores it in slot `slot` of
// the group's scratch, one named barrier (id bar, WPR warps) and every lane adds the
// WPR partials.  Slots are never reused within a row, and the next row's first barrier
// orders them against the previous row, so one barrier per reduction phase suffices.
template <int WPR>
struct Group {
  float* red;   // [WPR][32] partial sums of this group
  int wr, bar;
  __device__ __forceinline__ void sync() const {
    if (WPR > 1) asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(WPR * 32) : "memory");
  }
  // Finish `n` warp-reduced partials held (identically) by every lane in v[0..n).
  template <int NMAX>
  __device__ __forceinline__ void reduce(float (&v)[NMAX], int n, int slot0, int lane) const {
    if (WPR == 1) return;
    if (lane == 0)
      for (int q = 0; q < n; ++q) red[wr * 32 + slot0 + q] = v[q];
    sync();
    for (int q = 0; q < n; ++q) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < WPR; ++w) t += red[w * 32 + slot0 + q];
      v[q] = t;
    }
  }
  __device__ __forceinline__ float reduce1(float v, int slot, int lane) const {
    float a[1] = {v};
    reduce<1>(a, 1, slot, lane);
    return a[0];
  }
};

// Prologue of the next loop for the group's row (x = this warp's part of the state):
//   combined = RMSNorm_rec(x + emb + e) * w_rec ; a = RMSNorm_attn(combined) * w_attn
template <typename T, int VQ, int WPR>
__device__ __forceinline__ void next_prologue(const CombineParams& p, float4 (&x)[VQ], long long rowD, int lane,
                                              int j0, const Group<WPR>& g) {
  const T* er = (const T*)p.e + rowD + 4 * lane;
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < VQ; ++j) {
    const int d = 4 * lane + 128 * (j0 + j);
    float4 ev = Vec4<T>::load(er + 128 * (j0 + j));
    x[j] = f4_add(x[j], ev);
    if (d < p.loop_dim) x[j] = f4_add(x[j], __ldg(reinterpret_cast<const float4*>(p.next_emb + d)));
    ss += f4_dot(x[j], x[j]);
  }
  ss = g.reduce1(warp_sum(ss), 17, lane);
  const float inv = rsqrtf(ss / p.D + p.eps);
  float ss2 = 0.f;
#pragma unroll
  for (int j = 0; j < VQ; ++j) {
    const int d = 4 * lane + 128 * (j0 + j);
    const float4 wv = __ldg(reinterpret_cast<const float4*>(p.w_rec + d));
    x[j] = make_float4(x[j].x * inv * wv.x, x[j].y * inv * wv.y, x[j].z * inv * wv.z, x[j].w * inv * wv.w);
    *reinterpret_cast<float4*>(p.combined_out + rowD + d) = x[j];
    ss2 += f4_dot(x[j], x[j]);
  }
  ss2 = g.reduce1(warp_sum(ss2), 18, lane);
  const float inv2 = rsqrtf(ss2 / p.D + p.eps);
#pragma unroll
  for (int j = 0; j < VQ; ++j) {
    const int d = 4 * lane + 128 * (j0 + j);
    const float4 wv = __ldg(reinterpret_cast<const float4*>(p.w_attn + d));
    store4<T>((T*)p.a_out + rowD + d,
              make_float4(x[j].x * inv2 * wv.x, x[j].y * inv2 * wv.y, x[j].z * inv2 * wv.z, x[j].w * inv2 * wv.w));
  }
}

// One row of S9 by a group of WPR warps; Wd / Bl point at the LoRA matrices (shared or global).
template <typename T, int VPL, int WPR>
__device__ __forceinline__ void combine_row(const CombineParams& p, int i, int lane, const Group<WPR>& g,
                                            float* z, const T* Wd, const T* Bl) {
  constexpr int VQ = VPL / WPR;
  const int j0 = g.wr * VQ;
  const int D = p.D;
  const int kS = p.k + p.S;
  const long long rowD = (long long)i * D;
  const bool lead = (g.wr == 0);
  float4 tr[VQ];
  // this row's loop and output row (rows at their own depth), else loop p.t and row i
  const int t = p.t_row ? p.t_row[i] : p.t;
  const long long wo = p.t_row ? (long long)p.out_row[i] * p.n_loops + t : (long long)t * p.N + i;
  const long long outD = p.t_row ? (long long)p.out_row[i] * D : rowD;
  if (!p.block_only && p.halted[i]) {   // frozen row: no update, zero weight, no experts
    if (p.t_row) return;                // an idle slot: nothing to write
    if (lead && lane == 0) p.halt_w_out[wo] = 0.f;
    if (lead && lane < p.k) p.ids_out[wo * p.k + lane] = -1;
    if (p.next_emb) {                   // its keys / values are still recomputed next loop
#pragma unroll
      for (int j = 0; j < VQ; ++j)
        tr[j] = __ldg(reinterpret_cast<const float4*>(p.h + rowD + 4 * lane + 128 * (j0 + j)));
      next_prologue<T, VQ, WPR>(p, tr, rowD, lane, j0, g);
    }
    return;
  }
  if (p.transformer_off) {
#pragma unroll
    for (int j = 0; j < VQ; ++j) tr[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
#pragma unroll
    for (int j = 0; j < VQ; ++j)
      tr[j] = __ldg(reinterpret_cast<const float4*>(p.x1 + rowD + 4 * lane + 128 * (j0 + j)));
    // the row's slot indices in one warp load; lane s holds slot s (invalid ones -> -1)
    int my_slot = -2;
    if (lane < kS) {
      my_slot = __ldg(p.slot_of + (long long)i * kS + lane);
      if (my_slot < 0 || my_slot >= p.max_slots) {
        if (lead) record_status(p.st, ST_BOUNDS, 202, my_slot);
        my_slot = -1;
      }
    }
    // slot rows two at a time, so two rows' loads are in flight per memory round trip
    for (int s = 0; s < kS; s += 2) {
      const int s0 = __shfl_sync(0xffffffffu, my_slot, s);
      const int s1 = (s + 1 < kS) ? __shfl_sync(0xffffffffu, my_slot, s + 1) : -1;
      const T* y0 = (const T*)p.y + (long long)max(s0, 0) * D + 4 * lane;
      const T* y1 = (const T*)p.y + (long long)max(s1, 0) * D + 4 * lane;
#pragma unroll
      for (int j = 0; j < VQ; ++j) {
        const int c = 128 * (j0 + j);
        const float4 a0 = s0 >= 0 ? Vec4<T>::load(y0 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 a1 = s1 >= 0 ? Vec4<T>::load(y1 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        tr[j] = f4_add2(tr[j], f4_add2(a0, a1));
      }
    }
  }
  if (p.block_only) {
#pragma unroll
    for (int j = 0; j < VQ; ++j) *reinterpret_cast<float4*>(p.out + rowD + 4 * lane + 128 * (j0 + j)) = tr[j];
    return;
  }
  if (!p.transformer_off && p.r > 0) {
    const float* sc = p.lora_scale + (long long)min(t, p.max_loop_iters - 1) * p.r;
    // rank in chunks of 16: partial projections of this warp's columns, one transposed warp
    // reduction, then the group sum; lane q of every warp ends with z[q0 + q]
    for (int q0 = 0; q0 < p.r; q0 += 16) {
      const int nq = min(16, p.r - q0);
      // ranks q and q + 1 share one packed FMA per element: (part_q, part_q+1) += t (w_q, w_q+1)
      float2 part2[8];
#pragma unroll
      for (int q = 0; q < 16; q += 2) {
        part2[q / 2] = make_float2(0.f, 0.f);
        if (q < nq) {
          const T* w0 = Wd + (long long)(q0 + q) * D + 4 * lane;
          const T* w1 = w0 + (q + 1 < nq ? D : 0);   // (the odd rank past nq is discarded below)
#pragma unroll
          for (int j = 0; j < VQ; ++j) {
            const float4 a = ld4<T>(w0 + 128 * (j0 + j)), b = ld4<T>(w1 + 128 * (j0 + j)), t = tr[j];
            float2 acc = part2[q / 2];
            acc = __ffma2_rn(make_float2(t.x, t.x), make_float2(a.x, b.x), acc);
            acc = __ffma2_rn(make_float2(t.y, t.y), make_float2(a.y, b.y), acc);
            acc = __ffma2_rn(make_float2(t.z, t.z), make_float2(a.z, b.z), acc);
            acc = __ffma2_rn(make_float2(t.w, t.w), make_float2(a.w, b.w), acc);
            part2[q / 2] = acc;
          }
        }
      }
      float part[16];
#pragma unroll
      for (int q = 0; q < 16; q += 2) {
        part[q] = part2[q / 2].x;
        part[q + 1] = (q + 1 < nq) ? part2[q / 2].y : 0.f;
      }
      const float ws = warp_sum16(part, lane);           // sum of part[lane >> 1]
      if (WPR == 1) {
        if ((lane & 1) == 0 && (lane >> 1) < nq) z[q0 + (lane >> 1)] = ws * sc[q0 + (lane >> 1)];
      } else {
        if ((lane & 1) == 0) g.red[g.wr * 32 + (lane >> 1)] = ws;
        g.sync();
        if (g.wr == 0 && lane < nq) {
          float t = 0.f;
#pragma unroll
          for (int w = 0; w < WPR; ++w) t += g.red[w * 32 + lane];
          z[q0 + lane] = t * sc[q0 + lane];
        }
        g.sync();   // z complete; slots 0..15 free for the next chunk
      }
    }
    __syncwarp();
    // every z_q is complete, so the delta can be added to the row in place
    for (int q = 0; q < p.r; ++q) {
      const T* bq = Bl + (long long)q * D + 4 * lane;
      const float zv = z[q];
#pragma unroll
      for (int j = 0; j < VQ; ++j) tr[j] = f4_fma2(zv, ld4<T>(bq + 128 * (j0 + j)), tr[j]);
    }
    __syncwarp();
  }
  // h_new = A h + B e + trans (in place in tr)
  const T* er = (const T*)p.e + rowD + 4 * lane;
  float zh = 0.f;
#pragma unroll
  for (int j = 0; j < VQ; ++j) {
    const int d = 4 * lane + 128 * (j0 + j);
    float4 hv = __ldg(reinterpret_cast<const float4*>(p.h + rowD + d));
    float4 av = __ldg(reinterpret_cast<const float4*>(p.A + d));
    float4 bv = __ldg(reinterpret_cast<const float4*>(p.inj_B + d));
    float4 ev = Vec4<T>::load(er + 128 * (j0 + j));
    tr[j] = f4_fmav2(bv, ev, f4_fmav2(av, hv, tr[j]));
    if (p.act_on) zh += f4_dot(tr[j], __ldg(reinterpret_cast<const float4*>(p.halt_wv + d)));
  }
  const bool last = (t == p.n_loops - 1);
  float w;
  if (p.act_on) {
    zh = g.reduce1(warp_sum(zh), 16, lane);
    const float zz = zh + p.halt_b[0] + (p.halt_off ? p.halt_off[i] : 0.f);
    const float prob = 1.f / (1.f + expf(-zz));
    const float cum = p.cum[i];
    const bool stop = (cum + prob >= p.thr) || last;
    w = stop ? fmaxf(1.f - cum, 0.f) : prob;
    g.sync();   // every warp has read cum before the lead updates it
    if (lead && lane == 0) {
      p.cum[i] = cum + prob;
      if (stop) p.halted[i] = 1;
      if (p.p_out) p.p_out[i] = prob;
    }
  } else {
    w = last ? 1.f : 0.f;
  }
#pragma unroll
  for (int j = 0; j < VQ; ++j) {
    const int d = 4 * lane + 128 * (j0 + j);
    float4* ho = reinterpret_cast<float4*>(p.h_out + outD + d);
    if (w != 0.f) {
      float4 o = *ho;
      o.x += w * tr[j].x; o.y += w * tr[j].y; o.z += w * tr[j].z; o.w += w * tr[j].w;
      *ho = o;
    }
    *reinterpret_cast<float4*>(p.h_state + rowD + d) = tr[j];
  }
  if (lead && lane == 0) p.halt_w_out[wo] = w;
  if (lead && lane < p.k) p.ids_out[wo * p.k + lane] = p.transformer_off ? -1 : p.ids[(long long)i * p.k + lane];
  if (p.next_emb) next_prologue<T, VQ, WPR>(p, tr, rowD, lane, j0, g);
}

// Persistent: GROUPS row groups of WPR warps per CTA, one CTA per SM, rows strided over
// the grid.  With LSMEM the LoRA matrices (2 r D elements, or the down one alone) are staged in shared memory once
// per CTA, so the rank-r projections read shared memory instead of L2.
template <typename T, int VPL, int WPR, int GROUPS, int LSMEM>
__global__ void __launch_bounds__(GROUPS * WPR * 32, 1) k_combine_warp(CombineParams p) {
  extern __shared__ __align__(16) uint8_t csm[];
  __shared__ float zs[GROUPS][64];
  __shared__ float red[GROUPS][WPR * 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = warp / WPR;
  Group<WPR> g;
  g.red = red[grp];
  g.wr = warp % WPR;
  g.bar = 1 + grp;
  const T* Wd = (const T*)p.lora_down;
  const T* Bl = (const T*)p.lora_B;
  if (LSMEM && p.r > 0 && !p.transformer_off && !p.block_only) {
    // LSMEM 1: both matrices in shared memory; 2: the down projection only (both do not fit)
    const size_t bytes = (size_t)p.r * p.D * sizeof(T);
    const int4* gs0 = reinterpret_cast<const int4*>(p.lora_down);
    const int4* gs1 = reinterpret_cast<const int4*>(p.lora_B);
    int4* d0 = reinterpret_cast<int4*>(csm);
    int4* d1 = reinterpret_cast<int4*>(csm + bytes);
    for (size_t v = threadIdx.x; v < bytes / 16; v += blockDim.x) {
      d0[v] = __ldg(gs0 + v);
      if (LSMEM == 1) d1[v] = __ldg(gs1 + v);
    }
    __syncthreads();
    Wd = reinterpret_cast<const T*>(csm);
    if (LSMEM == 1) Bl = reinterpret_cast<const T*>(csm + bytes);
  }
  for (int i = blockIdx.x * GROUPS + grp; i < p.N; i += gridDim.x * GROUPS)
    combine_row<T, VPL, WPR>(p, i, lane, g, zs[grp], Wd, Bl);
}

// out = RMSNorm(x) * w for fp32 rows of width D = 128 * VPL, one warp per row; with a row
// list, only rows rows[0 .. *n_rows) (the other rows are left as they are).
template <typename T, int VPL>
__global__ void __launch_bounds__(256) k_rmsnorm_warp(const float* __restrict__ x, const float* __restrict__ w,
                                                      T* __restrict__ out, int N, int D, float eps,
                                                      const int* __restrict__ rows, const int* __restrict__ n_rows) {
  const int lane = threadIdx.x & 31;
  int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (rows) {
    if (i >= *n_rows) return;
    i = rows[i];
  }
  if (i >= N) return;
  const long long rowD = (long long)i * D;
  float4 v[VPL];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    v[j] = __ldg(reinterpret_cast<const float4*>(x + rowD + 4 * lane + 128 * j));
    ss += f4_dot(v[j], v[j]);
  }
  const float inv = rsqrtf(warp_sum(ss) / D + eps);
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int d = 4 * lane + 128 * j;
    const float4 wv = __ldg(reinterpret_cast<const float4*>(w + d));
    store4<T>(out + rowD + d, make_float4(v[j].x * inv * wv.x, v[j].y * inv * wv.y, v[j].z * inv * wv.z,
                                          v[j].w * inv * wv.w));
  }
}

// Returns false when the shape needs the CTA-per-row kernel instead.
static inline bool al(const void* q, int b) { return ((uintptr_t)q % b) == 0; }

bool launch_rmsnorm_warp(int dtype, const float* x, const float* w, void* out, int N, int D, float eps,
                         cudaStream_t s, const int* rows, const int* n_rows) {
  if (D % 128 || !al(x, 16) || !al(w, 16) || !al(out, dtype == 0 ? 16 : 8)) return false;
  const unsigned blocks = (unsigned)((N + 7) / 8);
#define RDT_RW(V)                                                                                             \
  case V:                                                                                                     \
    if (dtype == 0) { k_rmsnorm_warp<float, V><<<blocks, 256, 0, s>>>(x, w, (float*)out, N, D, eps, rows, n_rows); note_launch(); } \
    else { k_rmsnorm_warp<bf16, V><<<blocks, 256, 0, s>>>(x, w, (bf16*)out, N, D, eps, rows, n_rows); note_launch(); }    \
    return true;
  switch (D / 128) {
    RDT_RW(1) RDT_RW(2) RDT_RW(4) RDT_RW(8) RDT_RW(12) RDT_RW(16) RDT_RW(24) RDT_RW(32)
    default: return false;
  }
#undef RDT_RW
}

int combine_sm_count() { return device_sm_count(); }

template <typename T, int VPL>
bool launch_combine_vpl(const CombineParams& p, int n_rows, cudaStream_t s) {
  // a row's columns split over warps so that each lane holds at most 4 float4 of a row
  // (16 registers per row array: wider rows spilled at the 64-register limit of 1024
  // threads), and about 32 warps per SM
  constexpr int WPR = (VPL >= 16 && VPL % 4 == 0) ? VPL / 4 : ((VPL % 4 == 0) ? 4 : ((VPL % 2 == 0) ? 2 : 1));
  constexpr int GROUPS = (32 / WPR) < 8 ? (32 / WPR) : 8;
  // LoRA matrices in shared memory: both when they fit in 160 KB, else the down projection
  // alone when it fits in 200 KB (the row group's per-row reads of it then stay on the SM)
  const size_t one = (size_t)p.r * p.D * sizeof(T);
  const bool al_ok = p.r > 0 && (one % 16) == 0 && ((uintptr_t)p.lora_down % 16) == 0 && ((uintptr_t)p.lora_B % 16) == 0;
  const int lsmem = !al_ok ? 0 : (2 * one <= 160 * 1024 ? 1 : (one <= 200 * 1024 ? 2 : 0));
  const size_t lbytes = lsmem == 1 ? 2 * one : one;
  const int sms = combine_sm_count();
  if (n_rows <= 2 * sms) {
    // few rows (decode): one CTA per row with one warp per 128 columns, so the rows spread
    // over the SMs and each warp's chain of dependent loads is one 16-byte vector deep per
    // array; the LoRA matrices are read through L1 / L2 (staging them would cost more than
    // one row uses)
    constexpr int WPR_S = VPL;
    { k_combine_warp<T, VPL, WPR_S, 1, 0><<<std::max(1, n_rows), WPR_S * 32, 0, s>>>(p); note_launch(); }
    return true;
  }
  const int grid = std::max(1, std::min((n_rows + GROUPS - 1) / GROUPS, sms));
  constexpr int THREADS = GROUPS * WPR * 32;
  if (lsmem == 1) {
    if (!ensure_smem_limit((const void*)k_combine_warp<T, VPL, WPR, GROUPS, 1>, 160 * 1024)) return false;
    { k_combine_warp<T, VPL, WPR, GROUPS, 1><<<grid, THREADS, lbytes, s>>>(p); note_launch(); }
  } else if (lsmem == 2) {
    if (!ensure_smem_limit((const void*)k_combine_warp<T, VPL, WPR, GROUPS, 2>, 200 * 1024)) return false;
    { k_combine_warp<T, VPL, WPR, GROUPS, 2><<<grid, THREADS, lbytes, s>>>(p); note_launch(); }
  } else {
    { k_combine_warp<T, VPL, WPR, GROUPS, 0><<<grid, THREADS, 0, s>>>(p); note_launch(); }
  }
  return true;
}

bool launch_combine_warp(int dtype, const CombineParams& p, int n_rows, cudaStream_t s) {
  // one slot index per lane (combine_row): rows with more than 32 slots take the CTA-per-row kernel
  if (p.D % 128 || p.r > 64 || p.k + p.S > 32) return false;
  const int ev = dtype == 0 ? 16 : 8;   // bytes of a 4-element vector in the model dtype
  if (!al(p.x1, 16) || !al(p.y, ev) || !al(p.h, 16) || !al(p.h_state, 16) || !al(p.h_out, 16) || !al(p.A, 16) ||
      !al(p.inj_B, 16) || !al(p.e, ev) || (p.act_on && !al(p.halt_wv, 16)) || (p.out && !al(p.out, 16)) ||
      (p.r > 0 && (!al(p.lora_down, ev) || !al(p.lora_B, ev))))
    return false;
  if (p.next_emb && (p.loop_dim % 4 || !al(p.next_emb, 16) || !al(p.w_rec, 16) || !al(p.w_attn, 16) ||
                     !al(p.combined_out, 16) || !al(p.a_out, ev)))
    return false;
#define RDT_CW(V)                                                                             \
  case V:                                                                                     \
    return dtype == 0 ? launch_combine_vpl<float, V>(p, n_rows, s) : launch_combine_vpl<bf16, V>(p, n_rows, s);
  switch (p.D / 128) {
    RDT_CW(1) RDT_CW(2) RDT_CW(4) RDT_CW(8) RDT_CW(12) RDT_CW(16) RDT_CW(24) RDT_CW(32)
    default: return false;
  }
#undef RDT_CW
}

}  // namespace rdt
