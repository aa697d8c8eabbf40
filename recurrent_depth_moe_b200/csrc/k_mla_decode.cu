// MLA decode attention on the latent cache, weight-absorbed form (S3 of the decode step
// with attn_type MLA; "OpenMythos 분석", MLA: the cache keeps c_kv and k_rope, and the
// per-head keys / values are linear in RMSNorm(c_kv); DeepSeek-V2's absorbed decode).
//
// For head h with k_nope = W_k,h n_j, v = W_v,h n_j and n_j = r_j (g ⊙ c_j), where
// r_j = 1 / sqrt(mean(c_j^2) + eps) and g the RMSNorm weight:
//   score(h, j) = scale * ( r_j * (qa_h · c_j) + q_rope,h · k_rope,j ),  qa_h = g ⊙ (W_k,h^T q_nope,h)
//   out_h       = W_v,h ( g ⊙ u_h ),  u_h = sum_j softmax_j(score) r_j c_j
// so one read of the cache row (c_j, k_rope,j) serves every head, and nothing per head is
// rebuilt for the cached positions.  Three kernels:
//   k_mla_q_absorb : qa = g ⊙ (W_k,h^T q_nope,h)                          [B][H][kvr] bf16
//   k_mla_attn     : split-KV latent attention on m16n8k16 MMAs; per (sequence, key
//                    range) CTA all H heads are the rows of 16-row tiles; the cache
//                    tiles are double-buffered in XOR-swizzled shared memory by
//                    cp.async.  Writes unnormalised u partials with (m, l) per range.
//   k_mla_out      : merges the ranges and applies g and W_v,h           [B][H * dv]
// The attention kernel streams the cache once: (kvr + dr) * 2 bytes per visible key.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace rdt {

namespace mla {
constexpr int BKV = 64, NW = 8, THREADS = NW * 32;
constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
// Byte offset of 16-byte chunk c of row r in a row-major tile with W chunks per row.
// W >= 8: the chunk's low three bits are XORed with the row; W < 8: the chunk's slot in
// its 128-byte line is XORed with the line.  Either way the 8 rows one ldmatrix phase
// reads at a fixed chunk land in 8 different bank groups.
template <int W>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  if constexpr (W >= 8) {
    return (uint32_t)(r * W * 16 + ((c ^ (r & 7)) << 4));
  } else {
    const int i = r * W + c;
    return (uint32_t)((i ^ ((i >> 3) & 7)) << 4);
  }
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(ok ? 16 : 0) : "memory");
}
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm2(uint32_t a, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(a));
}
__device__ __forceinline__ void ldsm2t(uint32_t a, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(a));
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
__device__ __forceinline__ float sq2(uint32_t u) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
  return f.x * f.x + f.y * f.y;
}

template <int MT, int KVR, int DR>
struct Shape {
  static constexpr int ROWS = 16 * MT;                       // head rows (H <= ROWS)
  static constexpr int WC = KVR / 8, WR = DR / 8;            // 16-byte chunks per row
  static constexpr int C_BYTES = BKV * KVR * 2, R_BYTES = BKV * DR * 2, STAGE = C_BYTES + R_BYTES;
  static constexpr int QA_BYTES = ROWS * KVR * 2, QR_BYTES = ROWS * DR * 2, P_BYTES = ROWS * BKV * 2;
  static constexpr int RED_BYTES = NW * ROWS * 4;
  static constexpr int SMEM = 2 * STAGE + QA_BYTES + QR_BYTES + P_BYTES + RED_BYTES;
  static constexpr int NT = KVR / 8;                         // n-tiles of the value side
  static constexpr int NPW = (NT + NW - 1) / NW;             // ... per warp
};
}  // namespace mla

// qa[b, h, c] = g[c] * sum_i q_nope[b, h, i] * W_kvu[h (dn + dv) + i, c]: per head a
// [B x dn] . [dn x kvr] product.  CTA = (head, 64 columns, 64 sequences): both operands
// are staged in shared memory with 16-byte loads (all in flight together), then each
// thread accumulates a 4 x 4 block of outputs.
constexpr int QA_BC = 64, QA_BB = 64, QA_KC = 64;   // columns, sequences, dn chunk per CTA
__global__ void __launch_bounds__(256) k_mla_q_absorb(MlaDecodeParams p) {
  __shared__ float ws[QA_KC][QA_BC + 4];   // W_k,h[d, c0 + j]
  __shared__ float qs[QA_KC][QA_BB + 4];   // q_nope[b0 + i, h, d], transposed
  const int h = blockIdx.x, c0 = blockIdx.y * QA_BC, b0 = blockIdx.z * QA_BB;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // columns 4 tx.., sequences 4 ty..
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const bf16* wk = (const bf16*)p.w_kvu + (long long)h * (p.dn + p.dv) * p.kvr;
  const bf16* qn = (const bf16*)p.q + (long long)h * p.q_head;
  for (int d0 = 0; d0 < p.dn; d0 += QA_KC) {
    const int kc = min(QA_KC, p.dn - d0);
    __syncthreads();
    // W rows d0 .. d0 + kc, columns c0 .. c0 + 64: 8 columns per 16-byte load
    for (int i = threadIdx.x; i < QA_KC * (QA_BC / 8); i += 256) {
      const int d = i / (QA_BC / 8), j8 = (i % (QA_BC / 8)) * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (d < kc && c0 + j8 < p.kvr) {
        const uint4 raw = *reinterpret_cast<const uint4*>(wk + (long long)(d0 + d) * p.kvr + c0 + j8);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          v[2 * e] = f.x;
          v[2 * e + 1] = f.y;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ws[d][j8 + e] = v[e];
    }
    // q_nope rows b0 .. b0 + 64, dims d0 .. d0 + kc: 8 dims per 16-byte load
    for (int i = threadIdx.x; i < QA_BB * (QA_KC / 8); i += 256) {
      const int bb = i / (QA_KC / 8), d8 = (i % (QA_KC / 8)) * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (b0 + bb < p.B && d8 < kc) {
        const uint4 raw = *reinterpret_cast<const uint4*>(qn + (long long)(b0 + bb) * p.q_row + d0 + d8);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          v[2 * e] = f.x;
          v[2 * e + 1] = f.y;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) qs[d8 + e][bb] = v[e];
    }
    __syncthreads();
    for (int d = 0; d < kc; ++d) {
      const float4 w4 = *reinterpret_cast<const float4*>(&ws[d][4 * tx]);
      const float4 q4 = *reinterpret_cast<const float4*>(&qs[d][4 * ty]);
      const float wv[4] = {w4.x, w4.y, w4.z, w4.w}, qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += qv[i] * wv[j];
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = b0 + 4 * ty + i;
    if (b >= p.B) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + 4 * tx + j;
      if (c < p.kvr) ((bf16*)p.qa)[((long long)b * p.H + h) * p.kvr + c] = from_f<bf16>(acc[i][j] * p.kv_norm_w[c]);
    }
  }
}

template <int MT, int KVR, int DR>
__global__ void __launch_bounds__(mla::THREADS, 1) k_mla_attn(MlaDecodeParams p, int chunk_tiles) {
  using namespace mla;
  using S = Shape<MT, KVR, DR>;
  constexpr int ROWS = S::ROWS, WC = S::WC, WR = S::WR, NT = S::NT, NPW = S::NPW;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* qa_s = sm + 2 * S::STAGE;
  uint8_t* qr_s = qa_s + S::QA_BYTES;
  uint8_t* p_s = qr_s + S::QR_BYTES;
  float* red = reinterpret_cast<float*>(p_s + S::P_BYTES);   // [NW][ROWS]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int split = blockIdx.x % p.n_split, b = blockIdx.x / p.n_split;
  const int n_vis = min(p.q_pos[b] + 1, p.t_max);            // keys 0 .. cache_len[b]
  const int j0 = split * chunk_tiles * BKV;
  const int j1 = min(j0 + chunk_tiles * BKV, n_vis);
  const int nt = j1 > j0 ? (j1 - j0 + BKV - 1) / BKV : 0;
  const bf16* cg = (const bf16*)p.ckv + ((long long)b * p.t_max + j0) * KVR;
  const bf16* rg = (const bf16*)p.krope + ((long long)b * p.t_max + j0) * DR;
  auto load_tile = [&](int t, int buf) {
    const uint32_t cb = su32(sm + buf * S::STAGE), rb = cb + S::C_BYTES;
    const int valid = min(BKV, j1 - j0 - t * BKV);
    const bf16* cs = cg + (long long)t * BKV * KVR;
    const bf16* rs = rg + (long long)t * BKV * DR;
    for (int i = threadIdx.x; i < BKV * WC; i += THREADS) {
      const int r = i / WC, c = i % WC;
      const bool ok = r < valid;
      cp16(cb + swz<WC>(r, c), cs + (ok ? (long long)r * KVR + c * 8 : 0), ok);
    }
    for (int i = threadIdx.x; i < BKV * WR; i += THREADS) {
      const int r = i / WR, c = i % WR;
      const bool ok = r < valid;
      cp16(rb + swz<WR>(r, c), rs + (ok ? (long long)r * DR + c * 8 : 0), ok);
    }
  };
  // query rows h < H: [qa_h | q_rope,h]; padded rows are zero
  {
    const bf16* qa = (const bf16*)p.qa + (long long)b * p.H * KVR;
    for (int i = threadIdx.x; i < ROWS * WC; i += THREADS) {
      const int r = i / WC, c = i % WC;
      const bool ok = r < p.H;
      cp16(su32(qa_s) + swz<WC>(r, c), qa + (ok ? (long long)r * KVR + c * 8 : 0), ok);
    }
    const bf16* qr = (const bf16*)p.q + (long long)b * p.q_row + p.dn;
    for (int i = threadIdx.x; i < ROWS * WR; i += THREADS) {
      const int r = i / WR, c = i % WR;
      const bool ok = r < p.H;
      cp16(su32(qr_s) + swz<WR>(r, c), qr + (ok ? (long long)r * p.q_head + c * 8 : 0), ok);
    }
  }
  if (nt > 0) load_tile(0, 0);
  asm volatile("cp.async.commit_group;" ::: "memory");

  const float lg2s = p.scale * 1.4426950408889634f;   // scores in log2 units
  float o[MT][NPW][4];
  float m[MT][2], lp[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int i = 0; i < NPW; ++i) o[mt][i][0] = o[mt][i][1] = o[mt][i][2] = o[mt][i][3] = 0.f;
    m[mt][0] = m[mt][1] = -INFINITY;
    lp[mt][0] = lp[mt][1] = 0.f;
  }
  const uint32_t qab = su32(qa_s), qrb = su32(qr_s), pb = su32(p_s);
  for (int t = 0; t < nt; ++t) {
    const int buf = t & 1;
    if (t + 1 < nt) load_tile(t + 1, buf ^ 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const uint32_t cb = su32(sm + buf * S::STAGE), rb = cb + S::C_BYTES;
    // scores of keys [8 warp, 8 warp + 8) of the tile; the B fragments also give the
    // per-key sum of squares of c_j (thread: key gid, dims 2 tig, 2 tig + 1 of each 8)
    float sl[MT][4], sr[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) sl[mt][0] = sl[mt][1] = sl[mt][2] = sl[mt][3] = sr[mt][0] = sr[mt][1] = sr[mt][2] = sr[mt][3] = 0.f;
    float sl2[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) sl2[mt][0] = sl2[mt][1] = sl2[mt][2] = sl2[mt][3] = 0.f;
    float ssq = 0.f;
    const int key = warp * 8 + (lane & 7);
#pragma unroll
    for (int ks = 0; ks < KVR / 16; ks += 2) {
      uint32_t bf[4];
      ldsm4(cb + swz<WC>(key, ks * 2 + (lane >> 3)), bf);
      ssq += sq2(bf[0]) + sq2(bf[1]) + sq2(bf[2]) + sq2(bf[3]);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t a[4];
        ldsm4(qab + swz<WC>(mt * 16 + (lane & 15), ks * 2 + (lane >> 4)), a);
        mma16816(sl[mt], a, bf[0], bf[1]);
        ldsm4(qab + swz<WC>(mt * 16 + (lane & 15), ks * 2 + 2 + (lane >> 4)), a);
        mma16816(sl2[mt], a, bf[2], bf[3]);   // second chain: half the dependent depth
      }
    }
#pragma unroll
    for (int ks = 0; ks < DR / 16; ++ks) {
      uint32_t b0, b1;
      ldsm2(rb + swz<WR>(key, ks * 2 + ((lane >> 3) & 1)), b0, b1);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t a[4];
        ldsm4(qrb + swz<WR>(mt * 16 + (lane & 15), ks * 2 + (lane >> 4)), a);
        mma16816(sr[mt], a, b0, b1);
      }
    }
    ssq += __shfl_xor_sync(FULL, ssq, 1);
    ssq += __shfl_xor_sync(FULL, ssq, 2);
    const float rk = rsqrtf(ssq * (1.f / KVR) + p.eps);               // key 8 warp + gid
    const float r0 = __shfl_sync(FULL, rk, (tig * 2) * 4);            // this thread's columns
    const float r1 = __shfl_sync(FULL, rk, (tig * 2 + 1) * 4);
    const int kcol = j0 + t * BKV + warp * 8 + tig * 2;               // absolute key of column 0
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float r = (e & 1) ? r1 : r0;
        float v = ((sl[mt][e] + sl2[mt][e]) * r + sr[mt][e]) * lg2s;
        if (kcol + (e & 1) >= j1) v = -INFINITY;
        sl[mt][e] = v;
      }
      float a0 = fmaxf(sl[mt][0], sl[mt][1]), a1 = fmaxf(sl[mt][2], sl[mt][3]);
      a0 = fmaxf(a0, __shfl_xor_sync(FULL, a0, 1));
      a0 = fmaxf(a0, __shfl_xor_sync(FULL, a0, 2));
      a1 = fmaxf(a1, __shfl_xor_sync(FULL, a1, 1));
      a1 = fmaxf(a1, __shfl_xor_sync(FULL, a1, 2));
      if (tig == 0) {
        red[warp * ROWS + mt * 16 + gid] = a0;
        red[warp * ROWS + mt * 16 + gid + 8] = a1;
      }
    }
    __syncthreads();
    float corr[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = mt * 16 + gid + 8 * hh;
        float mx = m[mt][hh];
#pragma unroll
        for (int w = 0; w < NW; ++w) mx = fmaxf(mx, red[w * ROWS + row]);
        const float base = (mx == -INFINITY) ? 0.f : mx;
        corr[mt][hh] = exp2f(m[mt][hh] - base);
        m[mt][hh] = mx;
        const float pa = exp2f(sl[mt][2 * hh] - base), pbv = exp2f(sl[mt][2 * hh + 1] - base);
        lp[mt][hh] = lp[mt][hh] * corr[mt][hh] + pa + pbv;
        // P' = p r_j: the value side sums p r_j c_j
        *reinterpret_cast<uint32_t*>(p_s + swz<8>(row, warp) + tig * 4) = pk2(pa * r0, pbv * r1);
      }
    }
    __syncthreads();
    // u += P' C over this warp's value columns
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < NPW; ++i) {
        o[mt][i][0] *= corr[mt][0];
        o[mt][i][1] *= corr[mt][0];
        o[mt][i][2] *= corr[mt][1];
        o[mt][i][3] *= corr[mt][1];
      }
#pragma unroll
    for (int ks = 0; ks < BKV / 16; ++ks) {
      uint32_t a[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) ldsm4(pb + swz<8>(mt * 16 + (lane & 15), ks * 2 + (lane >> 4)), a[mt]);
#pragma unroll
      for (int i = 0; i < NPW; ++i) {
        const int n = warp + NW * i;
        if (n < NT) {
          uint32_t b0, b1;
          ldsm2t(cb + swz<WC>(ks * 16 + (lane & 15), n), b0, b1);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) mma16816(o[mt][i], a[mt], b0, b1);
        }
      }
    }
    __syncthreads();
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // row sums: quad, then the eight warps
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      lp[mt][hh] += __shfl_xor_sync(FULL, lp[mt][hh], 1);
      lp[mt][hh] += __shfl_xor_sync(FULL, lp[mt][hh], 2);
    }
  __syncthreads();
  if (tig == 0) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      red[warp * ROWS + mt * 16 + gid] = lp[mt][0];
      red[warp * ROWS + mt * 16 + gid + 8] = lp[mt][1];
    }
  }
  __syncthreads();
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int row = mt * 16 + gid + 8 * hh;
      if (row < p.H) {
        const long long slot = ((long long)b * p.H + row) * p.n_split + split;
        float* po = p.part_o + slot * KVR;
#pragma unroll
        for (int i = 0; i < NPW; ++i) {
          const int n = warp + NW * i;
          if (n < NT) *reinterpret_cast<float2*>(po + n * 8 + tig * 2) = make_float2(o[mt][i][2 * hh], o[mt][i][2 * hh + 1]);
        }
        if (warp == 0 && tig == 0) {
          float L = 0.f;
#pragma unroll
          for (int w = 0; w < NW; ++w) L += red[w * ROWS + row];
          p.part_ml[2 * slot] = m[mt][hh];       // log2 units
          p.part_ml[2 * slot + 1] = L;
        }
      }
    }
}

// Merge the key ranges (u = sum_s 2^{m_s - M} u_s / sum_s 2^{m_s - M} l_s), scale by the
// RMSNorm weight, and apply W_v,h: out[b, h dv + v] = sum_c W_kvu[h (dn + dv) + dn + v, c] g_c u_c.
// CTA = (head, 8 sequences), so each W_v,h row is read once per 8 sequences.
template <int KVR>
__global__ void __launch_bounds__(256) k_mla_out(MlaDecodeParams p) {
  constexpr int BB = 8;
  __shared__ __align__(16) float us[BB][KVR];
  __shared__ float fs[BB][33];   // split weights (n_split <= 32), then 1 / L
  const int h = blockIdx.x, b0 = blockIdx.y * BB, ns = p.n_split;
  if (threadIdx.x < BB) {
    const int bb = threadIdx.x, b = b0 + bb;
    if (b < p.B) {
      const float* ml = p.part_ml + ((long long)b * p.H + h) * ns * 2;
      float M = -INFINITY;
      for (int s = 0; s < ns; ++s) M = fmaxf(M, ml[2 * s]);
      float L = 0.f;
      for (int s = 0; s < ns; ++s) {
        const float f = (M == -INFINITY) ? 0.f : exp2f(ml[2 * s] - M);
        fs[bb][s] = f;
        L += f * ml[2 * s + 1];
      }
      fs[bb][32] = L > 0.f ? 1.f / L : 0.f;
    }
  }
  __syncthreads();
  // merge: float4 of u per thread and step, four key ranges loaded before they are used
  for (int i = threadIdx.x; i < BB * KVR / 4; i += 256) {
    const int bb = i / (KVR / 4), c = (i % (KVR / 4)) * 4, b = b0 + bb;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (b < p.B) {
      const float* po = p.part_o + ((long long)b * p.H + h) * ns * KVR + c;
      int s = 0;
      for (; s + 4 <= ns; s += 4) {
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = *reinterpret_cast<const float4*>(po + (long long)(s + k) * KVR);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float f = fs[bb][s + k];
          u.x += f * v[k].x; u.y += f * v[k].y; u.z += f * v[k].z; u.w += f * v[k].w;
        }
      }
      for (; s < ns; ++s) {
        const float4 v = *reinterpret_cast<const float4*>(po + (long long)s * KVR);
        const float f = fs[bb][s];
        u.x += f * v.x; u.y += f * v.y; u.z += f * v.z; u.w += f * v.w;
      }
      const float il = fs[bb][32];
      u.x *= il * p.kv_norm_w[c]; u.y *= il * p.kv_norm_w[c + 1];
      u.z *= il * p.kv_norm_w[c + 2]; u.w *= il * p.kv_norm_w[c + 3];
    }
    *reinterpret_cast<float4*>(&us[bb][c]) = u;
  }
  __syncthreads();
  // out[b, h dv + v] = W_v,h[v, :] . u_b: warp per row, two rows per pass
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bf16* wv = (const bf16*)p.w_kvu + ((long long)h * (p.dn + p.dv) + p.dn) * KVR;
  for (int v0 = 2 * warp; v0 < p.dv; v0 += 16) {
    float acc[2][BB];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int bb = 0; bb < BB; ++bb) acc[r][bb] = 0.f;
#pragma unroll
    for (int c8 = lane; c8 < KVR / 8; c8 += 32) {
      uint4 raw[2];
#pragma unroll
      for (int r = 0; r < 2; ++r)
        raw[r] = (v0 + r < p.dv) ? *reinterpret_cast<const uint4*>(wv + (long long)(v0 + r) * KVR + c8 * 8)
                                 : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[r]);
        float wf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          wf[2 * e] = f.x;
          wf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int bb = 0; bb < BB; ++bb) {
          const float4 ua = *reinterpret_cast<const float4*>(&us[bb][c8 * 8]);
          const float4 ub = *reinterpret_cast<const float4*>(&us[bb][c8 * 8 + 4]);
          acc[r][bb] += wf[0] * ua.x + wf[1] * ua.y + wf[2] * ua.z + wf[3] * ua.w + wf[4] * ub.x + wf[5] * ub.y +
                        wf[6] * ub.z + wf[7] * ub.w;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int bb = 0; bb < BB; ++bb) acc[r][bb] = warp_sum(acc[r][bb]);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int bb = 0; bb < BB; ++bb)
          if (v0 + r < p.dv && b0 + bb < p.B)
            ((bf16*)p.o)[(long long)(b0 + bb) * p.o_row + (long long)h * p.dv + v0 + r] = from_f<bf16>(acc[r][bb]);
    }
  }
}

namespace {
template <int MT, int KVR, int DR>
int launch_attn_t(const MlaDecodeParams& p, int chunk_tiles, cudaStream_t s) {
  constexpr int SMEM = mla::Shape<MT, KVR, DR>::SMEM;
  if (!ensure_smem_limit((const void*)k_mla_attn<MT, KVR, DR>, SMEM)) return -1;
  k_mla_attn<MT, KVR, DR><<<(unsigned)(p.B * p.n_split), mla::THREADS, SMEM, s>>>(p, chunk_tiles);
  note_launch();
  return 0;
}
}  // namespace

bool mla_decode_supports(int attn_type, int dtype, int H, int kvr, int dr, int dn, int dv) {
  if (attn_type != 1 || dtype != 1 || H < 1 || H > 32) return false;
  const bool shape = (kvr == 32 && dr == 16) || (kvr == 128 && dr == 32) || (kvr == 512 && dr == 64);
  return shape && dn % 8 == 0 && dn >= 8 && dn <= 256 && dv >= 1;
}

int mla_decode_splits(int B, int t_max, int tile_keys) {
  // key ranges per sequence: fewest waves x (tiles per range + the fixed cost of a CTA:
  // its query load and partial write, about 1.5 tiles) over the SMs, one CTA each
  const int sms = tc_sm_count() > 0 ? tc_sm_count() : 148;
  const int tiles = std::max(1, (t_max + tile_keys - 1) / tile_keys);
  int best = 1;
  long long best_cost = -1;
  for (int ns = 1; ns <= std::min(32, tiles); ++ns) {
    const long long waves = ((long long)B * ns + sms - 1) / sms;
    const long long cost = waves * (2 * ((tiles + ns - 1) / ns) + 3);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = ns; }
  }
  return best;
}

int launch_mla_decode(const MlaDecodeParams& p, cudaStream_t s) {
  if (p.B <= 0) return 0;
  if (p.n_split < 1 || p.n_split > 32) return -1;
  const int tiles = (p.t_max + mla::BKV - 1) / mla::BKV;
  const int chunk_tiles = (tiles + p.n_split - 1) / p.n_split;
  {
    dim3 grid((unsigned)p.H, (unsigned)((p.kvr + QA_BC - 1) / QA_BC), (unsigned)((p.B + QA_BB - 1) / QA_BB));
    k_mla_q_absorb<<<grid, 256, 0, s>>>(p);
    note_launch();
  }
  const int MT = p.H <= 16 ? 1 : 2;
  int rc = -1;
  if (p.kvr == 32 && p.dr == 16) rc = MT == 1 ? launch_attn_t<1, 32, 16>(p, chunk_tiles, s) : launch_attn_t<2, 32, 16>(p, chunk_tiles, s);
  else if (p.kvr == 128 && p.dr == 32) rc = MT == 1 ? launch_attn_t<1, 128, 32>(p, chunk_tiles, s) : launch_attn_t<2, 128, 32>(p, chunk_tiles, s);
  else if (p.kvr == 512 && p.dr == 64) rc = MT == 1 ? launch_attn_t<1, 512, 64>(p, chunk_tiles, s) : launch_attn_t<2, 512, 64>(p, chunk_tiles, s);
  if (rc) return rc;
  dim3 grid((unsigned)p.H, (unsigned)((p.B + 7) / 8));
  if (p.kvr == 32) k_mla_out<32><<<grid, 256, 0, s>>>(p);
  else if (p.kvr == 128) k_mla_out<128><<<grid, 256, 0, s>>>(p);
  else k_mla_out<512><<<grid, 256, 0, s>>>(p);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace rdt
