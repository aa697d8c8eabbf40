// KV-cached decode attention (S3 of the decode step), head dim 128, GQA.
//
// One new query row per sequence attends to its loop cache ("OpenMythos 분석", RoPE &
// generation cache: key j visible iff j <= cache_len[b]).  The keys are split into
// n_split ranges.  bf16 runs the tensor-core kernel further below.  The CUDA-core kernel
// (fp32, or unaligned bf16): each warp owns one (sequence, kv head, range) and serves all G query
// heads of the group from one read of every K and V row: lane l holds dims 4l..4l+3
// (8-byte vectors, so a warp reads a 256-byte row in one instruction), 8 keys are
// loaded per step before any of them is used, and an online softmax keeps (m, l, o)
// per head.  k_attn_decode_combine merges the ranges:
//   O = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s.
// The kernel streams the cache once, so it is HBM-bound: 2 * n_keys * 128 * 2 bytes per
// (sequence, kv head).
#include "common.cuh"
#include "kernels.h"

namespace rdt {

namespace {
template <typename T> struct V4;
template <> struct V4<bf16> {
  static __device__ __forceinline__ float4 ld(const bf16* p) {
    uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
};
template <> struct V4<float> {
  static __device__ __forceinline__ float4 ld(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
};
constexpr int KB = 8;   // keys per step
}  // namespace

template <typename T, int G>
__global__ void __launch_bounds__(128) k_attn_decode(AttnParams p, int n_split, int chunk) {
  const int lane = threadIdx.x & 31;
  const long long wid = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int Hkv = p.H / G;
  const long long total = (long long)p.B * Hkv * n_split;
  if (wid >= total) return;
  const int split = (int)(wid % n_split);
  const int bg = (int)(wid / n_split);
  const int b = bg / Hkv, g = bg % Hkv;
  const long long row = b;   // one query row per sequence
  int n_vis = min(p.n_keys, p.q_pos[row] - p.key_pos0 + 1);
  const int j0 = split * chunk;
  const int j1 = min(j0 + chunk, n_vis);
  float4 q[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float4 v = V4<T>::ld((const T*)p.q + row * p.q_row + (long long)(g * G + h) * p.q_head + 4 * lane);
    q[h] = make_float4(v.x * p.scale, v.y * p.scale, v.z * p.scale, v.w * p.scale);
  }
  const long long lp = p.row_loop ? max(p.row_loop[b], 0) : 0;
  const T* kb = (const T*)p.k1 + lp * p.loop_k + (long long)b * p.k1_b + (long long)g * p.k1_g + 4 * lane;
  const T* vb = (const T*)p.v + lp * p.loop_v + (long long)b * p.v_b + (long long)g * p.v_g + 4 * lane;
  float m[G], l[G];
  float4 acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
    acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int j = j0; j < j1; j += KB) {
    const int nk = min(KB, j1 - j);
    float4 kv[KB], vv[KB];
#pragma unroll
    for (int i = 0; i < KB; ++i) {
      if (i < nk) {
        kv[i] = V4<T>::ld(kb + (long long)(j + i) * p.k1_j);
        vv[i] = V4<T>::ld(vb + (long long)(j + i) * p.v_j);
      }
    }
    float s[KB][G];
#pragma unroll
    for (int i = 0; i < KB; ++i)
#pragma unroll
      for (int h = 0; h < G; ++h)
        s[i][h] = (i < nk) ? q[h].x * kv[i].x + q[h].y * kv[i].y + q[h].z * kv[i].z + q[h].w * kv[i].w : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < KB; ++i)
#pragma unroll
        for (int h = 0; h < G; ++h) s[i][h] += __shfl_xor_sync(0xffffffffu, s[i][h], o);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = m[h];
#pragma unroll
      for (int i = 0; i < KB; ++i)
        if (i < nk) mx = fmaxf(mx, s[i][h]);
      const float corr = __expf(m[h] - mx);
      m[h] = mx;
      float4 a = make_float4(acc[h].x * corr, acc[h].y * corr, acc[h].z * corr, acc[h].w * corr);
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < KB; ++i) {
        if (i < nk) {
          const float e = __expf(s[i][h] - mx);
          sum += e;
          a.x += e * vv[i].x; a.y += e * vv[i].y; a.z += e * vv[i].z; a.w += e * vv[i].w;
        }
      }
      l[h] = l[h] * corr + sum;
      acc[h] = a;
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const long long slot = ((long long)b * p.H + g * G + h) * n_split + split;
    *reinterpret_cast<float4*>(p.part_o + slot * 128 + 4 * lane) = acc[h];
    if (lane == 0) {
      p.part_ml[2 * slot] = m[h];
      p.part_ml[2 * slot + 1] = l[h];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128) k_attn_decode_combine(AttnParams p, int n_split) {
  const int bh = blockIdx.x;           // b * H + h
  const int d = threadIdx.x;           // dim
  const int b = bh / p.H, h = bh % p.H;
  const float* ml = p.part_ml + (long long)bh * n_split * 2;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, ml[2 * s]);
  float L = 0.f, o = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < n_split; ++s) {
      const float w = __expf(ml[2 * s] - M);
      L += w * ml[2 * s + 1];
      o += w * p.part_o[((long long)bh * n_split + s) * 128 + d];
    }
  }
  ((T*)p.o)[(long long)b * p.o_row + (long long)h * p.o_head + d] = from_f<T>(L > 0.f ? o / L : 0.f);
}

// ------------------------------------------------------------------------------------------
// bf16 tensor-core version: CTA = (sequence, kv head, key range); the G query heads are
// the first rows of a 16-row MMA tile.  64-key K / V tiles are double-buffered in
// XOR-swizzled shared memory by cp.async; warp w takes keys [16w, 16w + 16) of each
// tile: S = Q K^T and O += P V on m16n8k16 MMAs, online softmax per row in registers.
// The four warps' (m, l, O) are merged in shared memory into one partial per CTA.
// ------------------------------------------------------------------------------------------
namespace dmma {
constexpr int BKV = 64, ROWB = 256, TILEB = BKV * ROWB;       // 16 KB per K or V tile
constexpr int SMEM = 4 * TILEB;                               // K, V x 2 stages
__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ int swz(int r, int c) { return r * ROWB + ((c ^ (r & 7)) << 4); }
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(ok ? 16 : 0) : "memory");
}
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];" : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];" : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pk2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void load_tile(uint8_t* t, const bf16* src, long long ld, int valid) {
  const uint32_t base = su32(t);
  for (int i = threadIdx.x; i < BKV * 16; i += 128) {
    const int r = i >> 4, c = i & 15;
    const bool ok = r < valid;
    cp16(base + swz(r, c), src + (ok ? (long long)r * ld : 0) + c * 8, ok);
  }
}
}  // namespace dmma

template <int G>
__global__ void __launch_bounds__(128) k_attn_decode_mma(AttnParams p, int n_split, int chunk) {
  using namespace dmma;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* Ks = sm;
  uint8_t* Vs = sm + 2 * TILEB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int Hkv = p.H / G;
  const int split = blockIdx.x % n_split;
  const int bg = blockIdx.x / n_split;
  const int b = bg / Hkv, g = bg % Hkv;
  const long long row = b;
  const int n_vis = min(p.n_keys, p.q_pos[row] - p.key_pos0 + 1);
  const int j0 = split * chunk;
  const int j1 = min(j0 + chunk, n_vis);
  const int nt = j1 > j0 ? (j1 - j0 + BKV - 1) / BKV : 0;
  const long long lp = p.row_loop ? max(p.row_loop[b], 0) : 0;
  const bf16* kg = (const bf16*)p.k1 + lp * p.loop_k + (long long)b * p.k1_b + (long long)g * p.k1_g +
                   (long long)j0 * p.k1_j;
  const bf16* vg = (const bf16*)p.v + lp * p.loop_v + (long long)b * p.v_b + (long long)g * p.v_g +
                   (long long)j0 * p.v_j;
  if (nt > 0) {
    load_tile(Ks, kg, p.k1_j, min(BKV, j1 - j0));
    load_tile(Vs, vg, p.v_j, min(BKV, j1 - j0));
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // query fragments: row gid < G is query head g*G + gid; rows >= G are zero
  uint32_t qf[8][4];
  {
    const bf16* qr = (const bf16*)p.q + row * p.q_row + (long long)(g * G + min(gid, G - 1)) * p.q_head;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t lo = *reinterpret_cast<const uint32_t*>(qr + ks * 16 + tig * 2);
      uint32_t hi = *reinterpret_cast<const uint32_t*>(qr + ks * 16 + 8 + tig * 2);
      qf[ks][0] = gid < G ? lo : 0u;
      qf[ks][1] = 0u;
      qf[ks][2] = gid < G ? hi : 0u;
      qf[ks][3] = 0u;
    }
  }
  const float sl2 = p.scale * 1.4426950408889634f;
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m = -INFINITY, l = 0.f;   // for row gid
  for (int t = 0; t < nt; ++t) {
    const int buf = t & 1;
    if (t + 1 < nt) {
      const int k0n = (t + 1) * BKV;
      load_tile(Ks + (buf ^ 1) * TILEB, kg + (long long)k0n * p.k1_j, p.k1_j, min(BKV, j1 - j0 - k0n));
      load_tile(Vs + (buf ^ 1) * TILEB, vg + (long long)k0n * p.v_j, p.v_j, min(BKV, j1 - j0 - k0n));
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const uint32_t kb = su32(Ks + buf * TILEB), vb = su32(Vs + buf * TILEB);
    const int kbase = t * BKV + warp * 16;            // key offset of this warp inside the range
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int key = warp * 16 + (lane & 7) + ((lane >> 4) << 3);
      const int c = ks * 2 + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm4(kb + swz(key, c), b0, b1, b2, b3);
      mma16816(s[0], qf[ks], b0, b1);
      mma16816(s[1], qf[ks], b2, b3);
    }
    float mx = m;
#pragma unroll
    for (int nn = 0; nn < 2; ++nn)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kj = kbase + nn * 8 + tig * 2 + e;
        float v = s[nn][e] * sl2;
        if (j0 + kj >= j1) v = -INFINITY;
        s[nn][e] = v;
        mx = fmaxf(mx, v);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float base = (mx == -INFINITY) ? 0.f : mx;
    const float corr = exp2f(m - base);
    m = mx;
    const float p0 = exp2f(s[0][0] - base), p1 = exp2f(s[0][1] - base);
    const float p2 = exp2f(s[1][0] - base), p3 = exp2f(s[1][1] - base);
    l = l * corr + (p0 + p1 + p2 + p3);
    uint32_t pf[4] = {pk2(p0, p1), 0u, pk2(p2, p3), 0u};
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      o[dt][0] *= corr;
      o[dt][1] *= corr;
    }
#pragma unroll
    for (int dt = 0; dt < 16; dt += 2) {
      const int key = warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
      const int c = dt + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm4t(vb + swz(key, c), b0, b1, b2, b3);
      mma16816(o[dt], pf, b0, b1);
      mma16816(o[dt + 1], pf, b2, b3);
    }
    __syncthreads();
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // quad sums of l, then merge the four warps (rows < G) through shared memory
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  __syncthreads();
  float* mo = reinterpret_cast<float*>(sm);            // [4][G][128] O, then [4][G] m and l
  float* mm = mo + 4 * G * 128;
  float* ll = mm + 4 * G;
  if (gid < G) {
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      mo[(warp * G + gid) * 128 + dt * 8 + tig * 2] = o[dt][0];
      mo[(warp * G + gid) * 128 + dt * 8 + tig * 2 + 1] = o[dt][1];
    }
    if (tig == 0) {
      mm[warp * G + gid] = m;
      ll[warp * G + gid] = l;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * 128; i += 128) {
    const int r = i >> 7, d = i & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, mm[w * G + r]);
    float L = 0.f, acc = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = exp2f(mm[w * G + r] - M);
        L += f * ll[w * G + r];
        acc += f * mo[(w * G + r) * 128 + d];
      }
    }
    const long long slot = ((long long)b * p.H + g * G + r) * n_split + split;
    p.part_o[slot * 128 + d] = acc;
    if (d == 0) {
      // the combine kernel works in natural-log units: M was kept in log2 units
      p.part_ml[2 * slot] = (M == -INFINITY) ? -INFINITY : M * 0.6931471805599453f;
      p.part_ml[2 * slot + 1] = L;
    }
  }
}

int decode_split_count(int t_max) {
  int n = (t_max + 1023) / 1024;   // about 1024 keys (16 tiles of 64) per CTA
  return n < 1 ? 1 : (n > 32 ? 32 : n);
}

int launch_attention_decode(int dtype, const AttnParams& p, cudaStream_t s) {
  const int G = p.G;
  if (p.dn != 128 || p.dr != 0 || p.dv != 128 || !p.part_o || !p.part_ml || p.T != 1) return -1;
  if (G < 1 || G > 8 || p.H % G) return -1;
  const int n_split = p.n_split;
  const int chunk = ((p.n_keys + n_split - 1) / n_split + KB - 1) / KB * KB;
  const long long warps = (long long)p.B * (p.H / G) * n_split;
  const unsigned blocks = (unsigned)((warps + 3) / 4);
#define RDT_DEC(TT, GG)                                                                   \
  case GG: { k_attn_decode<TT, GG><<<blocks, 128, 0, s>>>(p, n_split, chunk); note_launch(); } break;
  if (dtype == 1 && p.k1_j % 8 == 0 && p.v_j % 8 == 0 && p.q_head % 8 == 0 && p.q_row % 2 == 0 &&
      ((uintptr_t)p.k1 & 15) == 0 && ((uintptr_t)p.v & 15) == 0) {
    const int ctas = p.B * (p.H / G) * n_split;
#define RDT_DECM(GG)                                                                              \
  case GG: {                                                                                      \
    if (!ensure_smem_limit((const void*)k_attn_decode_mma<GG>, dmma::SMEM)) return -1;            \
    { k_attn_decode_mma<GG><<<ctas, 128, dmma::SMEM, s>>>(p, n_split, chunk); note_launch(); }   \
  } break;
    switch (G) { RDT_DECM(1) RDT_DECM(2) RDT_DECM(3) RDT_DECM(4) RDT_DECM(6) RDT_DECM(8) default: return -1; }
#undef RDT_DECM
    { k_attn_decode_combine<bf16><<<p.B * p.H, 128, 0, s>>>(p, n_split); note_launch(); }
  } else if (dtype == 1) {
    switch (G) { RDT_DEC(bf16, 1) RDT_DEC(bf16, 2) RDT_DEC(bf16, 3) RDT_DEC(bf16, 4) RDT_DEC(bf16, 6)
      RDT_DEC(bf16, 8) default: return -1; }
    { k_attn_decode_combine<bf16><<<p.B * p.H, 128, 0, s>>>(p, n_split); note_launch(); }
  } else {
    switch (G) { RDT_DEC(float, 1) RDT_DEC(float, 2) RDT_DEC(float, 3) RDT_DEC(float, 4) RDT_DEC(float, 6)
      RDT_DEC(float, 8) default: return -1; }
    { k_attn_decode_combine<float><<<p.B * p.H, 128, 0, s>>>(p, n_split); note_launch(); }
  }
#undef RDT_DEC
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace rdt
