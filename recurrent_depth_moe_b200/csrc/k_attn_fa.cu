// Causal GQA prefill attention for head dim 128, bf16 (S3 of the recurrent block).
//
// Flash-style: one CTA (4 warps) per (sequence, head, 64-query tile); each warp owns
// 16 query rows.  K and V tiles of 64 keys are double-buffered in XOR-swizzled shared
// memory by cp.async; S = Q K^T and O += P V run on bf16 tensor-core MMAs
// (m16n8k16, fp32 accumulation) with the scores, probabilities and output kept in
// registers; the softmax is online (running max and sum per row, exp2 with the
// 1/sqrt(hd) scale folded in).  Query tiles are issued heaviest first (the causal
// diagonal makes late tiles longer).  Key j is visible to query row r iff
// key_pos0 + j <= q_pos[r] ("OpenMythos 분석", Core Structure: causal mask).
#include "common.cuh"
#include "kernels.h"

namespace rdt {
namespace fa {

constexpr int BQ = 64, BKV = 64, HD = 128;
constexpr int ROW_BYTES = HD * 2;                              // 256 B per key / query row
constexpr int TILE_BYTES = BKV * ROW_BYTES;                    // 16 KB
constexpr int SMEM_BYTES = TILE_BYTES /*Q*/ + 4 * TILE_BYTES;  // Q + 2 x (K, V) = 80 KB

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// byte offset of 16-byte chunk c of row r inside a swizzled [rows][256 B] tile
__device__ __forceinline__ int swz(int r, int c) { return r * ROW_BYTES + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Load `rows` rows (row stride `ld` elements) of 128 bf16 into a swizzled tile; rows >= valid_rows zero-filled.
__device__ __forceinline__ void load_tile(uint8_t* tile, const bf16* src, long long ld, int valid_rows) {
  const uint32_t base = smem_u32(tile);
  for (int i = threadIdx.x; i < BKV * 16; i += blockDim.x) {
    int r = i >> 4, c = i & 15;
    bool ok = r < valid_rows;
    const bf16* g = src + (ok ? (long long)r * ld : 0) + c * 8;
    cp_async16(base + swz(r, c), g, ok);
  }
}

__global__ void __launch_bounds__(128) k_attn_fa(AttnParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* Qs = smem;
  uint8_t* Ks = smem + TILE_BYTES;            // 2 buffers
  uint8_t* Vs = smem + 3 * TILE_BYTES;        // 2 buffers
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (p.T + BQ - 1) / BQ;
  const int BH = p.B * p.H;
  const int qt = n_qt - 1 - (int)(blockIdx.x / BH);   // heaviest (last) query tiles first
  const int bh = blockIdx.x % BH;
  const int h = bh % p.H, b = bh / p.H, g = h / p.G;
  const int q0 = qt * BQ;
  const int q_rows = min(BQ, p.T - q0);
  const long long row0 = (long long)b * p.T + q0;

  const bf16* qg = (const bf16*)p.q + row0 * p.q_row + (long long)h * p.q_head;
  const bf16* kg = (const bf16*)p.k1 + (long long)b * p.k1_b + (long long)g * p.k1_g;
  const bf16* vg = (const bf16*)p.v + (long long)b * p.v_b + (long long)g * p.v_g;

  // visible keys of this tile: up to the last query's position
  const int q_last_pos = p.q_pos[row0 + q_rows - 1];
  int n_keys = min(p.n_keys, q_last_pos - p.key_pos0 + 1);
  if (n_keys < 0) n_keys = 0;
  const int n_kv = (n_keys + BKV - 1) / BKV;

  load_tile(Qs, qg, p.q_row, q_rows);
  cp_commit();
  if (n_kv > 0) {
    load_tile(Ks, kg, p.k1_j, min(BKV, n_keys));
    load_tile(Vs, vg, p.v_j, min(BKV, n_keys));
  }
  cp_commit();

  // per-thread rows: r_a = warp*16 + lane/4, r_b = r_a + 8
  const int gid = lane >> 2, tig = lane & 3;
  const int ra = warp * 16 + gid, rb = ra + 8;
  const int pos_a = (ra < q_rows) ? p.q_pos[row0 + ra] : -1;
  const int pos_b = (rb < q_rows) ? p.q_pos[row0 + rb] : -1;
  const int warp_pos_max = p.q_pos[row0 + min(warp * 16 + 15, q_rows - 1)];
  const float sl2 = p.scale * 1.4426950408889634f;

  cp_wait<1>();
  __syncthreads();
  uint32_t qf[8][4];
  {
    const uint32_t qb = smem_u32(Qs);
    const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      int c = ks * 2 + (lane >> 4);
      ldsm_x4(qb + swz(r, c), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
    }
  }

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int j = 0; j < n_kv; ++j) {
    const int buf = j & 1;
    if (j + 1 < n_kv) {
      const int k0n = (j + 1) * BKV;
      load_tile(Ks + (buf ^ 1) * TILE_BYTES, kg + (long long)k0n * p.k1_j, p.k1_j, min(BKV, n_keys - k0n));
      load_tile(Vs + (buf ^ 1) * TILE_BYTES, vg + (long long)k0n * p.v_j, p.v_j, min(BKV, n_keys - k0n));
    }
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const int k0 = j * BKV;
    const int key_pos_first = p.key_pos0 + k0;
    // warps whose rows see none of this tile skip the math (the barrier below still runs)
    if (key_pos_first <= warp_pos_max) {
      const uint32_t kb = smem_u32(Ks + buf * TILE_BYTES), vb = smem_u32(Vs + buf * TILE_BYTES);
      float s[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          // matrices: (keys nt*8.., dims ks*16..), (keys nt*8.., dims ks*16+8..), same for nt+1
          const int key = nt * 8 + (lane & 7) + ((lane >> 4) << 3);
          const int c = ks * 2 + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + swz(key, c), b0, b1, b2, b3);
          mma_bf16(s[nt], qf[ks], b0, b1);
          mma_bf16(s[nt + 1], qf[ks], b2, b3);
        }
      }
      // mask: invisible keys (beyond n_keys or after the query position)
      const bool need_mask = (key_pos_first + BKV - 1 > pos_a) || (key_pos_first + BKV - 1 > pos_b) ||
                             (k0 + BKV > n_keys);
      float mx_a = m_a, mx_b = m_b;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kj = k0 + nt * 8 + tig * 2 + e;
          const int kp = p.key_pos0 + kj;
          float va = s[nt][e] * sl2, vb2 = s[nt][2 + e] * sl2;
          if (need_mask) {
            if (kj >= n_keys || kp > pos_a) va = -INFINITY;
            if (kj >= n_keys || kp > pos_b) vb2 = -INFINITY;
          }
          s[nt][e] = va;
          s[nt][2 + e] = vb2;
          mx_a = fmaxf(mx_a, va);
          mx_b = fmaxf(mx_b, vb2);
        }
      }
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
      const float base_a = (mx_a == -INFINITY) ? 0.f : mx_a;
      const float base_b = (mx_b == -INFINITY) ? 0.f : mx_b;
      const float corr_a = exp2f(m_a - base_a), corr_b = exp2f(m_b - base_b);
      m_a = mx_a;
      m_b = mx_b;
      float sum_a = 0.f, sum_b = 0.f;
      uint32_t pf[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float p0 = exp2f(s[nt][0] - base_a), p1 = exp2f(s[nt][1] - base_a);
        float p2 = exp2f(s[nt][2] - base_b), p3 = exp2f(s[nt][3] - base_b);
        sum_a += p0 + p1;
        sum_b += p2 + p3;
        const int kc = nt >> 1, hi = nt & 1;
        pf[kc][hi * 2 + 0] = pack_bf16(p0, p1);
        pf[kc][hi * 2 + 1] = pack_bf16(p2, p3);
      }
      l_a = l_a * corr_a + sum_a;
      l_b = l_b * corr_b + sum_b;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt) {
        o[dt][0] *= corr_a;
        o[dt][1] *= corr_a;
        o[dt][2] *= corr_b;
        o[dt][3] *= corr_b;
      }
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
#pragma unroll
        for (int dt = 0; dt < 16; dt += 2) {
          // .trans matrices: (keys kc*16.., dims dt*8..), (keys kc*16+8.., dims dt*8..), same for dt+1
          const int key = kc * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int c = dt + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + swz(key, c), b0, b1, b2, b3);
          mma_bf16(o[dt], pf[kc], b0, b1);
          mma_bf16(o[dt + 1], pf[kc], b2, b3);
        }
      }
    }
    __syncthreads();
  }
  cp_wait<0>();

  // finalise: row sums across the quad, normalise, store bf16
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float ia = l_a > 0.f ? 1.f / l_a : 0.f, ib = l_b > 0.f ? 1.f / l_b : 0.f;
  bf16* og = (bf16*)p.o + row0 * p.o_row + (long long)h * p.o_head;
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    const int col = dt * 8 + tig * 2;
    if (ra < q_rows) *reinterpret_cast<uint32_t*>(og + (long long)ra * p.o_row + col) = pack_bf16(o[dt][0] * ia, o[dt][1] * ia);
    if (rb < q_rows) *reinterpret_cast<uint32_t*>(og + (long long)rb * p.o_row + col) = pack_bf16(o[dt][2] * ib, o[dt][3] * ib);
  }
}

}  // namespace fa

bool attention_fa_supports(int dtype, const AttnParams& p) {
  return dtype == 1 && p.dn == 128 && p.dr == 0 && p.dv == 128 && !p.n_keys_dev && p.T >= 1 &&
         p.q_row % 8 == 0 && p.k1_j % 8 == 0 && p.v_j % 8 == 0 && p.q_head % 8 == 0 && p.k1_g % 8 == 0 &&
         p.v_g % 8 == 0 && p.o_row % 2 == 0 && ((uintptr_t)p.q & 15) == 0 && ((uintptr_t)p.k1 & 15) == 0 &&
         ((uintptr_t)p.v & 15) == 0;
}

int launch_attention_fa(const AttnParams& p, cudaStream_t s) {
  if (!ensure_smem_limit((const void*)fa::k_attn_fa, fa::SMEM_BYTES)) return -1;
  const long long blocks = (long long)((p.T + fa::BQ - 1) / fa::BQ) * p.B * p.H;
  if (blocks <= 0) return 0;
  { fa::k_attn_fa<<<(unsigned)blocks, 128, fa::SMEM_BYTES, s>>>(p); note_launch(); }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace rdt
