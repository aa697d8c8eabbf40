// MLA decode attention on the latent cache, weight-absorbed form (S3 of the decode step
// with attn_type MLA; "OpenMythos 분석", MLA: the cache keeps c_kv and k_rope, and the
// per-head keys / values are linear in RMSNorm(c_kv); DeepSeek-V2's absorbed decode).
//
// For head h with k_nope = W_k,h n_j, v = W_v,h n_j and n_j = r_j (g ⊙ c_j), where
// r_j = 1 / sqrt(mean(c_j^2) + eps) and g the RMSNorm weight:
//   score(h, j) = scale * ( r_j * (qa_h · c_j) + q_rope,h · k_rope,j ),  qa_h = g ⊙ (W_k,h^T q_nope,h)
//   out_h       = W_v,h ( g ⊙ u_h ),  u_h = sum_j softmax_j(score) r_j c_j
// so one read of the cache row (c_j, k_rope,j) serves every head, and nothing per head is
// rebuilt for the cached positions.  Three kernels, all on m16n8k16 MMAs:
//   k_mla_q_absorb : qa = g ⊙ (W_k,h^T q_nope,h)                          [B][H][kvr] bf16
//   k_mla_attn     : split-KV latent attention.  Per (sequence, key range) CTA the keys are
//                    the MMA rows and the heads the columns (no padding of H to 16); each
//                    warp keeps its quarter of the query in registers for the whole range.
//                    Writes unnormalised u partials with (m, l) per range.
//   k_mla_out      : merges the ranges and applies g and W_v,h           [B][H * dv]
// The attention kernel streams the cache once: (kvr + dr) * 2 bytes per visible key.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>

namespace rdt {

namespace mla {
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
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm2(uint32_t a, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(a));
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

// k_mla_attn's work split.  A tile holds KG groups of 32 keys, and each group has four
// warps (KG = 1: 128 threads, two CTAs per SM; KG = 2: 256 threads, one CTA per SM).
// Scores S^T[key, head] = C Qa^T (latent) + R Qr^T (rope) per tile: warp = (key group kg:
// keys 32 kg .. 32 kg + 31, K quarter kw).  kw = 0 takes
// the KSR rope k-steps and the first L0 latent k-steps, kw = 1..3 equal shares of the rest,
// so each warp holds at most MAXKS k-steps of query fragments.  The four latent quarters
// and the rope part go to shared memory as five partial sums per key group (the rope part
// is added after the latent one is scaled by r_j).  Values U^T[latent, head] += C^T P'^T:
// warp w owns VPW 16-dim latent tiles for every key of the tile.
template <int NTH, int KVR, int DR, int KG>
struct Shape {
  static constexpr int BKV = 32 * KG, NW = 4 * KG, THREADS = 32 * NW;
  static constexpr int KQ = BKV / 8;                           // key octets: softmax threads per head
  static constexpr int NH8 = 8 * NTH;                          // head columns (H <= NH8)
  static constexpr int KSL = KVR / 16, KSR = DR / 16;
  static constexpr int PER = (KSL + KSR + 3) / 4;
  static constexpr int L0 = PER > KSR ? PER - KSR : 0;
  static constexpr int PER1 = (KSL - L0 + 2) / 3;
  static constexpr int MAXKS = (KSR + L0 > PER1) ? KSR + L0 : PER1;
  static constexpr int WC = KVR / 8, WR = DR / 8;              // 16-byte chunks per row
  static constexpr int C_BYTES = BKV * KVR * 2, R_BYTES = BKV * DR * 2, STAGE = C_BYTES + R_BYTES;
  static constexpr int SPP = 36;                               // floats per head row of 32 keys (+4)
  static constexpr int SP_KG = 5 * NH8 * SPP + 4;              // floats per key group (+4: bank shift)
  static constexpr int SP_BYTES = (2 * SP_KG * 4 + 127) / 128 * 128;
  static constexpr int SSQ_BYTES = 4 * BKV * 4;                // [kw][key]
  static constexpr int P_BYTES = NH8 * BKV * 2;                // P' [head][key] bf16, KQ chunks per row
  static constexpr int SMEM = 2 * STAGE + SP_BYTES + SSQ_BYTES + P_BYTES + NH8 * 4;
  static constexpr int VT = KVR / 16, VPW = (VT + NW - 1) / NW;
  static_assert(NH8 * (KVR + DR) * 2 <= STAGE, "the query staging fits one stage");
  static_assert(KSR >= 1 && KSL >= 1, "latent and rope widths are multiples of 16");
};
// The variant for NTH head columns.  Both run at the same rate on the 3B MLA decode (64
// sequences, 24 heads, 4096 keys: 104 us per launch either way), and two 4-warp CTAs per SM
// need twice the key ranges (more partials to merge), so one 8-warp CTA per SM is used.
constexpr int kg_for(int) { return 2; }
}  // namespace mla

// qa[b, h, c] = g[c] * sum_i q_nope[b, h, i] * W_kvu[h (dn + dv) + i, c]: per head a
// [B x dn] . [dn x kvr] product.  CTA = (head, 64 latent columns, 64 sequences), four
// warps of 16 sequences; dn in chunks of 128, both operands staged by cp.async.
namespace qab {
constexpr int BC = 64, BB = 64, KC = 128;
}
__global__ void __launch_bounds__(128) k_mla_q_absorb(MlaDecodeParams p) {
  using namespace mla;
  __shared__ __align__(128) uint8_t ws[qab::KC * qab::BC * 2];   // W rows i x 64 columns
  __shared__ __align__(128) uint8_t qs[qab::BB * qab::KC * 2];   // q_nope rows b x 128 dims
  constexpr int WCW = qab::BC / 8, WCQ = qab::KC / 8;
  const int h = blockIdx.x, c0 = blockIdx.y * qab::BC, b0 = blockIdx.z * qab::BB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int ncols = min(qab::BC, p.kvr - c0);
  float acc[qab::BC / 8][4];
#pragma unroll
  for (int n = 0; n < qab::BC / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const bf16* wk = (const bf16*)p.w_kvu + (long long)h * (p.dn + p.dv) * p.kvr;
  const bf16* qn = (const bf16*)p.q + (long long)h * p.q_head;
  for (int d0 = 0; d0 < p.dn; d0 += qab::KC) {
    const int kc = min(qab::KC, p.dn - d0);
    __syncthreads();
    for (int i = threadIdx.x; i < qab::KC * WCW; i += 128) {
      const int d = i / WCW, c = i % WCW;
      const bool ok = d < kc && c * 8 < ncols;
      cp16(su32(ws) + swz<WCW>(d, c), wk + (ok ? (long long)(d0 + d) * p.kvr + c0 + c * 8 : 0), ok);
    }
    for (int i = threadIdx.x; i < qab::BB * WCQ; i += 128) {
      const int bb = i / WCQ, c = i % WCQ;
      const bool ok = b0 + bb < p.B && c * 8 < kc;
      cp16(su32(qs) + swz<WCQ>(bb, c), qn + (ok ? (long long)(b0 + bb) * p.q_row + d0 + c * 8 : 0), ok);
    }
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    const int nks = (kc + 15) / 16;
    for (int ks = 0; ks < nks; ++ks) {
      uint32_t a[4];
      ldsm4(su32(qs) + swz<WCQ>(warp * 16 + (lane & 15), 2 * ks + (lane >> 4)), a);
#pragma unroll
      for (int n = 0; n < qab::BC / 8; n += 2) {
        // B[k = i][n = c] = W[i][c], columns contiguous: transposed 8x8 loads of rows i
        uint32_t bq[4];
        ldsm4t(su32(ws) + swz<WCW>(16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8, n + (lane >> 4)), bq);
        mma16816(acc[n], a, bq[0], bq[1]);
        mma16816(acc[n + 1], a, bq[2], bq[3]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < qab::BC / 8; ++n) {
    const int c = c0 + 8 * n + 2 * tig;
    if (c - c0 >= ncols) continue;
    const float g0 = p.kv_norm_w[c], g1 = p.kv_norm_w[c + 1];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int b = b0 + warp * 16 + gid + 8 * hh;
      if (b < p.B)
        *reinterpret_cast<uint32_t*>((bf16*)p.qa + ((long long)b * p.H + h) * p.kvr + c) =
            pk2(acc[n][2 * hh] * g0, acc[n][2 * hh + 1] * g1);
    }
  }
}

template <int NTH, int KVR, int DR, int KG>
__global__ void __launch_bounds__(128 * KG, 3 - KG) k_mla_attn(MlaDecodeParams p, int chunk_tiles) {
  using namespace mla;
  using S = Shape<NTH, KVR, DR, KG>;
  constexpr int NH8 = S::NH8, WC = S::WC, WR = S::WR, KSR = S::KSR, KSL = S::KSL, MAXKS = S::MAXKS;
  constexpr int SPP = S::SPP, SP_KG = S::SP_KG, VPW = S::VPW, VT = S::VT;
  constexpr int BKV = S::BKV, THREADS = S::THREADS, KQ = S::KQ;
  extern __shared__ __align__(128) uint8_t sm[];
  float* sp = reinterpret_cast<float*>(sm + 2 * S::STAGE);          // [kg][5][head][key]
  float* ssq_s = reinterpret_cast<float*>(sm + 2 * S::STAGE + S::SP_BYTES);   // [kw][key]
  uint8_t* p_s = sm + 2 * S::STAGE + S::SP_BYTES + S::SSQ_BYTES;     // P' [head][key] bf16
  float* corr_s = reinterpret_cast<float*>(p_s + S::P_BYTES);       // [head]
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

  // this warp's share of the score product
  const int kg = warp >> 2, kw = warp & 3;
  const int lb = kw == 0 ? 0 : S::L0 + (kw - 1) * S::PER1;
  const int le = kw == 0 ? S::L0 : min(KSL, lb + S::PER1);
  // Query fragments (the B operand of the score MMAs), kept in registers for the range:
  // kw = 0: [0, KSR) rope k-steps, then latent k-steps 0 .. L0 - 1; kw > 0: latent lb ..
  uint32_t qf[MAXKS][NTH][2];
  if (nt > 0) load_tile(0, 0);                          // in flight with the query staging
  {
    const uint32_t qab_s = su32(sm + S::STAGE), qrb_s = qab_s + NH8 * KVR * 2;   // stage 1, still free
    const bf16* qa = (const bf16*)p.qa + (long long)b * p.H * KVR;
    for (int i = threadIdx.x; i < NH8 * WC; i += THREADS) {
      const int r = i / WC, c = i % WC;
      const bool ok = r < p.H;
      cp16(qab_s + swz<WC>(r, c), qa + (ok ? (long long)r * KVR + c * 8 : 0), ok);
    }
    const bf16* qr = (const bf16*)p.q + (long long)b * p.q_row + p.dn;
    for (int i = threadIdx.x; i < NH8 * WR; i += THREADS) {
      const int r = i / WR, c = i % WR;
      const bool ok = r < p.H;
      cp16(qrb_s + swz<WR>(r, c), qr + (ok ? (long long)r * p.q_head + c * 8 : 0), ok);
    }
    cp_commit();
    cp_wait<0>();
    __syncthreads();
#pragma unroll
    for (int i = 0; i < MAXKS; ++i) {
      const bool rope = kw == 0 && i < KSR;
      const int ks = kw == 0 ? i - KSR : lb + i;
#pragma unroll
      for (int n = 0; n < NTH; ++n) {
        qf[i][n][0] = qf[i][n][1] = 0u;
        const int row = 8 * n + (lane & 7), half = (lane >> 3) & 1;
        if (rope) ldsm2(qrb_s + swz<WR>(row, 2 * i + half), qf[i][n][0], qf[i][n][1]);
        else if (ks >= 0 && ks < le) ldsm2(qab_s + swz<WC>(row, 2 * ks + half), qf[i][n][0], qf[i][n][1]);
      }
    }
    __syncthreads();   // stage 1 is read; tile 1 may land there
  }

  const float lg2s = p.scale * 1.4426950408889634f;   // scores in log2 units
  const bool smx = threadIdx.x < NH8 * KQ;             // softmax thread: head sh, key octet kq
  const int sh = threadIdx.x / KQ, kq = threadIdx.x % KQ;
  float m_run = -INFINITY, l_run = 0.f;
  float o[VPW][NTH][4];
#pragma unroll
  for (int v = 0; v < VPW; ++v)
#pragma unroll
    for (int n = 0; n < NTH; ++n) o[v][n][0] = o[v][n][1] = o[v][n][2] = o[v][n][3] = 0.f;

  for (int t = 0; t < nt; ++t) {
    const int buf = t & 1;
    if (t + 1 < nt) load_tile(t + 1, buf ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t cb = su32(sm + buf * S::STAGE), rb = cb + S::C_BYTES;
    // ---- partial scores of this warp's keys over its k-steps; per-key sums of squares
    {
      float acc[2][NTH][4];
      // per-key sums of squares of c_j on the tensor pipe: an A fragment of C (16 keys x 16
      // dims) is also the B fragment of C^T for its keys 0..7 (regs 0, 2) and 8..15 (regs 1,
      // 3), so C C^T of the m-tile accumulates in two 16 x 8 blocks whose diagonals are ssq
      float sq[2][2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int u = 0; u < 2; ++u) sq[mt][u][0] = sq[mt][u][1] = sq[mt][u][2] = sq[mt][u][3] = 0.f;
      auto zero = [&]() {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int n = 0; n < NTH; ++n) acc[mt][n][0] = acc[mt][n][1] = acc[mt][n][2] = acc[mt][n][3] = 0.f;
      };
      // rows = keys 16 mt + gid (+ 8), columns = heads 8 n + 2 tig (+ 1)
      auto store = [&](int q) {
        float* dst = sp + kg * SP_KG + q * NH8 * SPP;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int n = 0; n < NTH; ++n) {
            const int hc = 8 * n + 2 * tig, jj = 16 * mt + gid;
            dst[hc * SPP + jj] = acc[mt][n][0];
            dst[(hc + 1) * SPP + jj] = acc[mt][n][1];
            dst[hc * SPP + jj + 8] = acc[mt][n][2];
            dst[(hc + 1) * SPP + jj + 8] = acc[mt][n][3];
          }
      };
      zero();
#pragma unroll
      for (int i = 0; i < MAXKS; ++i) {
        if (i == KSR && KSR < MAXKS && kw == 0) {   // kw 0: rope part done, latent part next
          store(4);
          zero();
        }
        const bool rope = kw == 0 && i < KSR;
        const int ks = kw == 0 ? i - KSR : lb + i;
        if (!rope && !(ks >= 0 && ks < le)) continue;
        uint32_t a[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int key = 32 * kg + 16 * mt + (lane & 15);
          if (rope) {
            ldsm4(rb + swz<WR>(key, 2 * i + (lane >> 4)), a[mt]);
          } else {
            ldsm4(cb + swz<WC>(key, 2 * ks + (lane >> 4)), a[mt]);
          }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
          for (int n = 0; n < NTH; ++n) mma16816(acc[mt][n], a[mt], qf[i][n][0], qf[i][n][1]);
          if (!rope) {
            mma16816(sq[mt][0], a[mt], a[mt][0], a[mt][2]);
            mma16816(sq[mt][1], a[mt], a[mt][1], a[mt][3]);
          }
        }
      }
      if (KSR >= MAXKS && kw == 0) {   // kw 0 held rope k-steps only
        store(4);
        zero();
      }
      store(kw);
      // diagonal (key gid, key gid) of block 0 and (gid + 8, gid + 8) of block 1: lane tig = gid / 2
      if (tig == (gid >> 1)) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int key = 32 * kg + 16 * mt + gid;
          ssq_s[kw * BKV + key] = (gid & 1) ? sq[mt][0][1] : sq[mt][0][0];
          ssq_s[kw * BKV + key + 8] = (gid & 1) ? sq[mt][1][3] : sq[mt][1][2];
        }
      }
    }
    __syncthreads();
    // ---- online softmax: thread = (head sh, keys 8 kq .. 8 kq + 7 of the tile)
    if (smx) {
      const int g2 = kq >> 2, jl = (kq & 3) * 8;
      const float* src = sp + g2 * SP_KG + sh * SPP + jl;
      float lat[8], rp[8], sq[8];
      {
        const float4 x0 = *reinterpret_cast<const float4*>(src), x1 = *reinterpret_cast<const float4*>(src + 4);
        lat[0] = x0.x; lat[1] = x0.y; lat[2] = x0.z; lat[3] = x0.w;
        lat[4] = x1.x; lat[5] = x1.y; lat[6] = x1.z; lat[7] = x1.w;
      }
#pragma unroll
      for (int q = 1; q < 4; ++q) {
        const float* s2 = src + q * NH8 * SPP;
        const float4 x0 = *reinterpret_cast<const float4*>(s2), x1 = *reinterpret_cast<const float4*>(s2 + 4);
        lat[0] += x0.x; lat[1] += x0.y; lat[2] += x0.z; lat[3] += x0.w;
        lat[4] += x1.x; lat[5] += x1.y; lat[6] += x1.z; lat[7] += x1.w;
      }
      {
        const float* s2 = src + 4 * NH8 * SPP;
        const float4 x0 = *reinterpret_cast<const float4*>(s2), x1 = *reinterpret_cast<const float4*>(s2 + 4);
        rp[0] = x0.x; rp[1] = x0.y; rp[2] = x0.z; rp[3] = x0.w;
        rp[4] = x1.x; rp[5] = x1.y; rp[6] = x1.z; rp[7] = x1.w;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) sq[i] = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float* s2 = ssq_s + q * BKV + 8 * kq;
        const float4 x0 = *reinterpret_cast<const float4*>(s2), x1 = *reinterpret_cast<const float4*>(s2 + 4);
        sq[0] += x0.x; sq[1] += x0.y; sq[2] += x0.z; sq[3] += x0.w;
        sq[4] += x1.x; sq[5] += x1.y; sq[6] += x1.z; sq[7] += x1.w;
      }
      const int kabs = j0 + t * BKV + 8 * kq;          // absolute key of i = 0
      float s[8], r[8], mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        r[i] = rsqrtf(sq[i] * (1.f / KVR) + p.eps);
        s[i] = (kabs + i < j1) ? (lat[i] * r[i] + rp[i]) * lg2s : -INFINITY;
        mx = fmaxf(mx, s[i]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
      if (KQ == 8) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
      // lazy running max: it moves only when a score exceeds it by more than 2^8, so most
      // tiles rescale nothing (p <= 256 meanwhile; l and u are fp32)
      float corr = 1.f;
      if (mx > m_run + 8.f) {
        corr = exp2f(m_run - mx);
        m_run = mx;
      }
      const float base = (m_run == -INFINITY) ? 0.f : m_run;
      float ps = 0.f;
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float pa = exp2f(s[2 * i] - base), pb = exp2f(s[2 * i + 1] - base);
        ps += pa + pb;
        pk[i] = pk2(pa * r[2 * i], pb * r[2 * i + 1]);   // P' = p r_j: the value side sums p r_j c_j
      }
      l_run = l_run * corr + ps;
      *reinterpret_cast<uint4*>(p_s + swz<KQ>(sh, kq)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      if (kq == 0) corr_s[sh] = corr;
    }
    __syncthreads();
    // ---- U^T[latent, head] += C^T P'^T over this warp's latent tiles
    {
      uint32_t pf[BKV / 16][NTH][2];
#pragma unroll
      for (int n = 0; n < NTH; ++n)
#pragma unroll
        for (int q = 0; q < BKV / 32; ++q) {
          uint32_t r4[4];
          ldsm4(su32(p_s) + swz<KQ>(8 * n + (lane & 7), (lane >> 3) + 4 * q), r4);
          pf[2 * q][n][0] = r4[0];
          pf[2 * q][n][1] = r4[1];
          pf[2 * q + 1][n][0] = r4[2];
          pf[2 * q + 1][n][1] = r4[3];
        }
      float c0[NTH], c1[NTH];
#pragma unroll
      for (int n = 0; n < NTH; ++n) {
        c0[n] = corr_s[8 * n + 2 * tig];
        c1[n] = corr_s[8 * n + 2 * tig + 1];
      }
      bool rescale = false;
#pragma unroll
      for (int n = 0; n < NTH; ++n) rescale |= (c0[n] != 1.f) || (c1[n] != 1.f);
#pragma unroll
      for (int v = 0; v < VPW; ++v) {
        const int vm = warp * VPW + v;
        if (vm >= VT) continue;
        if (rescale) {
#pragma unroll
          for (int n = 0; n < NTH; ++n) {
            o[v][n][0] *= c0[n];
            o[v][n][1] *= c1[n];
            o[v][n][2] *= c0[n];
            o[v][n][3] *= c1[n];
          }
        }
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          uint32_t a[4];
          ldsm4t(cb + swz<WC>(16 * kk + (lane & 7) + ((lane >> 4) << 3), 2 * vm + ((lane >> 3) & 1)), a);
#pragma unroll
          for (int n = 0; n < NTH; ++n) mma16816(o[v][n], a, pf[kk][n][0], pf[kk][n][1]);
        }
      }
    }
    __syncthreads();   // the next iteration's load overwrites this tile's buffer
  }
  cp_wait<0>();
  if (smx) {
    float l = l_run;
    l += __shfl_xor_sync(FULL, l, 1);
    l += __shfl_xor_sync(FULL, l, 2);
    if (KQ == 8) l += __shfl_xor_sync(FULL, l, 4);
    if (kq == 0 && sh < p.H) {
      const long long slot = ((long long)b * p.H + sh) * p.n_split + split;
      p.part_ml[2 * slot] = m_run;   // log2 units
      p.part_ml[2 * slot + 1] = l;
    }
  }
#pragma unroll
  for (int v = 0; v < VPW; ++v) {
    const int vm = warp * VPW + v;
    if (vm >= VT) continue;
#pragma unroll
    for (int n = 0; n < NTH; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hc = 8 * n + 2 * tig + (e & 1), c = 16 * vm + gid + 8 * (e >> 1);
        if (hc < p.H) p.part_o[(((long long)b * p.H + hc) * p.n_split + split) * KVR + c] = o[v][n][e];
      }
  }
}

// Merge the key ranges (u = sum_s 2^{m_s - M} u_s / sum_s 2^{m_s - M} l_s), scale by the
// RMSNorm weight, and apply W_v,h: out[b, h dv + v] = sum_c W_kvu[h (dn + dv) + dn + v, c] g_c u_c.
// CTA = (head, 64 value rows, 16 sequences); eight warps of 8 value rows.  The merged
// u_b is split into bf16 hi + lo parts (hi + lo = u to about 2^-16 relative) and both go
// through the MMA against the bf16 W_v,h, so the product keeps fp32-level accuracy.
// W_v,h streams through shared memory in 128-column chunks, double-buffered.
namespace mo {
constexpr int BV = 64, BB = 16, KC = 128;
}
template <int KVR>
struct OutShape {
  static constexpr int KCH = KVR < mo::KC ? KVR : mo::KC;
  static constexpr int WCH = KCH / 8, WU = KVR / 8;
  static constexpr int U_BYTES = mo::BB * KVR * 2, W_BYTES = mo::BV * KCH * 2;
  static constexpr int SMEM = 2 * U_BYTES + 2 * W_BYTES;
};
template <int KVR>
__global__ void __launch_bounds__(256) k_mla_out(MlaDecodeParams p) {
  using namespace mla;
  using S = OutShape<KVR>;
  constexpr int KCH = S::KCH, WCH = S::WCH, WU = S::WU, NKC = KVR / KCH;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* uh = sm;
  uint8_t* ul = sm + S::U_BYTES;
  uint8_t* wsm = sm + 2 * S::U_BYTES;
  __shared__ float fs[mo::BB][33];   // split weights (n_split <= 32), then 1 / L
  const int h = blockIdx.x, v0 = blockIdx.y * mo::BV, b0 = blockIdx.z * mo::BB, ns = p.n_split;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const bf16* wv = (const bf16*)p.w_kvu + ((long long)h * (p.dn + p.dv) + p.dn) * KVR;
  auto load_w = [&](int kc, int buf) {
    const uint32_t base = su32(wsm + buf * S::W_BYTES);
    for (int i = threadIdx.x; i < mo::BV * WCH; i += 256) {
      const int v = i / WCH, c = i % WCH;
      const bool ok = v0 + v < p.dv;
      cp16(base + swz<WCH>(v, c), wv + (ok ? (long long)(v0 + v) * KVR + kc * KCH + c * 8 : 0), ok);
    }
  };
  load_w(0, 0);
  cp_commit();
  if (threadIdx.x < mo::BB) {
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
  // merge: four float4 of u per thread and pass, their partial loads issued together
  constexpr int NU = mo::BB * KVR / 4;   // float4 of u in the CTA
  for (int i0 = threadIdx.x; i0 < NU; i0 += 4 * 256) {
    float4 u[4];
    const float* po[4];
    int bb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = i0 + k * 256;
      bb[k] = i / (KVR / 4);
      const int c = (i % (KVR / 4)) * 4, b = b0 + bb[k];
      po[k] = (i < NU && b < p.B) ? p.part_o + ((long long)b * p.H + h) * ns * KVR + c : nullptr;
      u[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int s = 0; s < ns; ++s) {
      float4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[k] = po[k] ? *reinterpret_cast<const float4*>(po[k] + (long long)s * KVR) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (!po[k]) continue;
        const float f = fs[bb[k]][s];
        u[k].x += f * v[k].x; u[k].y += f * v[k].y; u[k].z += f * v[k].z; u[k].w += f * v[k].w;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = i0 + k * 256;
      if (i >= NU) continue;
      const int c = (i % (KVR / 4)) * 4;
      if (po[k]) {
        const float il = fs[bb[k]][32];
        u[k].x *= il * p.kv_norm_w[c]; u[k].y *= il * p.kv_norm_w[c + 1];
        u[k].z *= il * p.kv_norm_w[c + 2]; u[k].w *= il * p.kv_norm_w[c + 3];
      }
      const __nv_bfloat162 h01 = __floats2bfloat162_rn(u[k].x, u[k].y), h23 = __floats2bfloat162_rn(u[k].z, u[k].w);
      const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
      const uint32_t off = swz<WU>(bb[k], c / 8) + (c % 8) * 2;
      *reinterpret_cast<uint2*>(uh + off) = make_uint2(*reinterpret_cast<const uint32_t*>(&h01),
                                                       *reinterpret_cast<const uint32_t*>(&h23));
      *reinterpret_cast<uint2*>(ul + off) =
          make_uint2(pk2(u[k].x - f01.x, u[k].y - f01.y), pk2(u[k].z - f23.x, u[k].w - f23.y));
    }
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int kc = 0; kc < NKC; ++kc) {
    if (kc + 1 < NKC) load_w(kc + 1, (kc + 1) & 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const uint32_t wb = su32(wsm + (kc & 1) * S::W_BYTES);
#pragma unroll
    for (int ks = 0; ks < KCH / 16; ++ks) {
      const int kglob = kc * (KCH / 16) + ks;
      uint32_t ah[4], al[4], b0, b1;
      ldsm4(su32(uh) + swz<WU>(lane & 15, 2 * kglob + (lane >> 4)), ah);
      ldsm4(su32(ul) + swz<WU>(lane & 15, 2 * kglob + (lane >> 4)), al);
      // B[k = c][n = v] = W_v,h[v][c], rows v: plain 8x8 loads
      ldsm2(wb + swz<WCH>(warp * 8 + (lane & 7), 2 * ks + ((lane >> 3) & 1)), b0, b1);
      mma16816(acc, ah, b0, b1);
      mma16816(acc, al, b0, b1);
    }
    __syncthreads();
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int v = v0 + warp * 8 + 2 * tig + (e & 1), b = b0 + gid + 8 * (e >> 1);
    if (v < p.dv && b < p.B)
      ((bf16*)p.o)[(long long)b * p.o_row + (long long)h * p.dv + v] = from_f<bf16>(acc[e]);
  }
}

namespace {
template <int NTH, int KVR, int DR>
int launch_attn_t(const MlaDecodeParams& p, cudaStream_t s) {
  constexpr int KG = mla::kg_for(NTH);
  using S = mla::Shape<NTH, KVR, DR, KG>;
  if (!ensure_smem_limit((const void*)k_mla_attn<NTH, KVR, DR, KG>, S::SMEM)) return -1;
  const int tiles = (p.t_max + S::BKV - 1) / S::BKV;
  const int chunk_tiles = (tiles + p.n_split - 1) / p.n_split;
  k_mla_attn<NTH, KVR, DR, KG><<<(unsigned)(p.B * p.n_split), S::THREADS, S::SMEM, s>>>(p, chunk_tiles);
  note_launch();
  return 0;
}
template <int KVR, int DR>
int launch_attn_h(const MlaDecodeParams& p, cudaStream_t s) {
  switch ((p.H + 7) / 8) {
    case 1: return launch_attn_t<1, KVR, DR>(p, s);
    case 2: return launch_attn_t<2, KVR, DR>(p, s);
    case 3: return launch_attn_t<3, KVR, DR>(p, s);
    case 4: return launch_attn_t<4, KVR, DR>(p, s);
    default: return -1;
  }
}
template <int KVR>
int launch_out_t(const MlaDecodeParams& p, cudaStream_t s) {
  constexpr int SMEM = OutShape<KVR>::SMEM;
  if (!ensure_smem_limit((const void*)k_mla_out<KVR>, SMEM)) return -1;
  dim3 grid((unsigned)p.H, (unsigned)((p.dv + mo::BV - 1) / mo::BV), (unsigned)((p.B + mo::BB - 1) / mo::BB));
  k_mla_out<KVR><<<grid, 256, SMEM, s>>>(p);
  note_launch();
  return 0;
}
}  // namespace

bool mla_decode_supports(int attn_type, int dtype, int H, int kvr, int dr, int dn, int dv) {
  if (attn_type != 1 || dtype != 1 || H < 1 || H > 32) return false;
  const bool shape = (kvr == 32 && dr == 16) || (kvr == 128 && dr == 32) || (kvr == 512 && dr == 64);
  return shape && dn % 8 == 0 && dn >= 8 && dn <= 256 && dv >= 1;
}

int mla_decode_splits(int B, int H, int t_max) {
  // key ranges per sequence: fewest waves x (tiles per range + the fixed cost of a CTA:
  // its query load and partial write, about 1.5 tiles) over the CTA slots of the SMs
  const int kg = mla::kg_for((std::max(H, 1) + 7) / 8);
  const int tile_keys = 32 * kg, per_sm = 3 - kg;
  const int sms = tc_sm_count() > 0 ? tc_sm_count() : 148;
  const int tiles = std::max(1, (t_max + tile_keys - 1) / tile_keys);
  int best = 1;
  long long best_cost = -1;
  for (int ns = 1; ns <= std::min(32, tiles); ++ns) {
    const long long waves = ((long long)B * ns + (long long)sms * per_sm - 1) / ((long long)sms * per_sm);
    const long long cost = waves * (2 * ((tiles + ns - 1) / ns) + 3);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = ns; }
  }
  return best;
}

int launch_mla_decode(const MlaDecodeParams& p, cudaStream_t s) {
  if (p.B <= 0) return 0;
  if (p.n_split < 1 || p.n_split > 32) return -1;
  {
    dim3 grid((unsigned)p.H, (unsigned)((p.kvr + qab::BC - 1) / qab::BC), (unsigned)((p.B + qab::BB - 1) / qab::BB));
    k_mla_q_absorb<<<grid, 128, 0, s>>>(p);
    note_launch();
  }
  int rc = -1;
  if (p.kvr == 32 && p.dr == 16) rc = launch_attn_h<32, 16>(p, s);
  else if (p.kvr == 128 && p.dr == 32) rc = launch_attn_h<128, 32>(p, s);
  else if (p.kvr == 512 && p.dr == 64) rc = launch_attn_h<512, 64>(p, s);
  if (rc) return rc;
  if (p.kvr == 32) rc = launch_out_t<32>(p, s);
  else if (p.kvr == 128) rc = launch_out_t<128>(p, s);
  else rc = launch_out_t<512>(p, s);
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace rdt
