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
#include "tc_common.cuh"

#include <algorithm>
#include <mutex>

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

// ------------------------------------------------------------------------------------------
// k_mla_attn_tc: the latent attention of kv_lora_rank 512 / rope 64 on the tcgen05 tensor
// cores (same partials as k_mla_attn).  Per (sequence, key range) CTA, tiles of 128 keys:
//   S^T[key, head]   = C Qa^T (latent) and R Qr^T (rope)     M = 128 keys, N = 32 heads
//   U^T[dim, head]  += C^T P'^T                               M = 128 dims (x 4), N = 32
// with C the tile's latent rows [128 keys][512], R its rope rows [128][64], Qa / Qr the
// absorbed and rope query rows of the sequence (heads past H are zero) and P' = p r_j.
// Two TMA streams (no multicast), each with its own producer warp and ring, so that the
// cache keeps streaming while a tile waits for its softmax:
//   warp 0: the score chunks (four 128-dim latent chunks and the rope chunk of each tile,
//           32 KB slots) from HBM;
//   warp 2: the value chunks (the same latent rows again, [64 keys][128 dims] per 16 KB
//           slot), L2 hits since the score pass read them a tile earlier.
// Warps 7..10 (thread = key) read each latent score chunk from shared memory as well and
// sum the key's squares, giving r_j = 1 / sqrt(mean(c_j^2) + eps) per tile; a score slot
// is free once the MMAs and these four warps are done with it.  Warp 1 owns TMEM and
// issues the score MMAs, up to three tiles ahead of the softmax (four S buffers in TMEM),
// so the HBM stream never waits for a softmax; warp 11 issues the value product of each
// tile after its softmax.  Warps 3..6 (thread = key = TMEM lane) stage the query, then per tile read
// the scores and the key's r_j, mask, take the per-head
// tile maximum across the 128 keys, keep a lazy running maximum per head (raised only when
// a score exceeds it by more than 2^8; then the l sums and U^T are rescaled), and write P'
// [head][key] (double-buffered) as the B operand of the value product.  At the end they
// write the unnormalised U rows and (m, l) per head.  Every wait is bounded; a wait that
// gives up aborts the CTA after its copies and MMAs have drained.
namespace mtc {
constexpr int BK = 128, NP = 32, KVR = 512, DR = 64;
constexpr int BOX = BK * 128;                 // 16 KB: [128 keys][64 dims] bf16, 128-byte swizzle
constexpr int SSLOT = 2 * BOX, NS = 3;        // score ring: a 128-dim latent chunk or the rope chunk
constexpr int VBOX = 64 * 128;                // 8 KB: [64 keys][64 dims]
constexpr int VSLOT = 2 * VBOX, NV = 4;       // value ring: [64 keys][128 dims]
constexpr int QBOX = NP * 128;                // 4 KB: [32 heads][64 dims] (or [32 heads][64 keys] of P')
constexpr int NQB = (KVR + DR) / 64;          // 8 latent + 1 rope query boxes
constexpr int PBUF = 2 * QBOX;                // P' [32 heads][128 keys]
constexpr int V_OFF = NS * SSLOT, Q_OFF = V_OFF + NV * VSLOT, P_OFF = Q_OFF + NQB * QBOX, BAR_OFF = P_OFF + 2 * PBUF;
constexpr int NSB = 4, NRB = 8;               // S buffers in TMEM; r_j buffers
constexpr int SMEM = BAR_OFF + 2048 + NRB * BK * 4 + 1024;   // barriers, reduction scratch, r_j, alignment slack
constexpr int THREADS = 384;                  // warps: 0 score loads, 1 score MMAs, 2 value loads, 3..6 softmax,
                                              // 7..10 sums of squares, 11 value MMAs
constexpr int SMX0 = 96, SSQ0 = 224;          // first softmax / sum-of-squares thread
constexpr int TMEM_COLS = 512;                // S buffer sb at 64 sb: latent +0, rope +32; U^T at 256 + 32 q
constexpr int T_U = NSB * 64;
constexpr float RESCALE_LOG2 = 8.f;
constexpr unsigned FULL = 0xffffffffu;

// 3-D tile load with an L2 eviction-priority policy (createpolicy): the score pass keeps
// its lines (evict_last) for the value pass, which reads them for the last time (evict_first).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(tc::smem_u32(dst)),
      "l"((uint64_t)map), "r"(tc::smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}
// (d0, d1) += (a0^2, a1^2) as one packed fp32x2 FMA (two independent fma.rn).
__device__ __forceinline__ void sq2(float& d0, float& d1, float a0, float a1) {
  asm("{\n\t.reg .b64 a, c;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 c, {%0, %1};\n\t"
      "fma.rn.f32x2 c, a, a, c;\n\tmov.b64 {%0, %1}, c;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void tmem_ld32_raw(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Barrier `id` over n threads that also ANDs a predicate across them (every thread gets the
// same answer, so all leave a loop together).
__device__ __forceinline__ bool bar_and(bool v, int id, int n) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// Transposed warp reductions of 32 columns (31 shuffles): lane l ends with the reduction of
// column l over the warp's lanes.
template <bool MAX>
__device__ __forceinline__ float warp_reduce32(const float (&v)[32], int lane) {
  auto op = [](float x, float y) { return MAX ? fmaxf(x, y) : x + y; };
  float a[16], b[8], c[4], d[2];
  bool hi = lane & 16;
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = op(hi ? v[i + 16] : v[i], __shfl_xor_sync(FULL, hi ? v[i] : v[i + 16], 16));
  hi = lane & 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = op(hi ? a[i + 8] : a[i], __shfl_xor_sync(FULL, hi ? a[i] : a[i + 8], 8));
  hi = lane & 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = op(hi ? b[i + 4] : b[i], __shfl_xor_sync(FULL, hi ? b[i] : b[i + 4], 4));
  hi = lane & 2;
#pragma unroll
  for (int i = 0; i < 2; ++i) d[i] = op(hi ? c[i + 2] : c[i], __shfl_xor_sync(FULL, hi ? c[i] : c[i + 2], 2));
  hi = lane & 1;
  return op(hi ? d[1] : d[0], __shfl_xor_sync(FULL, hi ? d[0] : d[1], 1));
}
// A ring of n slots fed by one producer thread and drained by the MMA thread (in order).
struct Ring {
  uint64_t* full;
  uint64_t* empty;
  int n, c;
};
}  // namespace mtc

__global__ void __launch_bounds__(mtc::THREADS, 1)
    k_mla_attn_tc(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
                  const __grid_constant__ CUtensorMap tmV, const MlaDecodeParams p, int chunk_tiles) {
  using namespace tc;
  using namespace mtc;
  extern __shared__ uint8_t mtc_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)mtc_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sring = sm;
  uint8_t* vring = sm + V_OFF;
  uint8_t* sQ = sm + Q_OFF;
  uint8_t* sP = sm + P_OFF;
  uint64_t* sfull = (uint64_t*)(sm + BAR_OFF);
  uint64_t* sempty = sfull + NS;
  uint64_t* vfull = sempty + NS;
  uint64_t* vempty = vfull + NV;
  uint64_t* q_ready = vempty + NV;
  uint64_t* s_full = q_ready + 1;    // [NSB] scores of tile t in TMEM buffer t % NSB
  uint64_t* s_free = s_full + NSB;   // [NSB] the softmax has read them
  uint64_t* r_ready = s_free + NSB;  // [NRB] r_j of tile t in buffer t % NRB
  uint64_t* p_full = r_ready + NRB;  // [2] P' of tile t written into buffer t & 1 (one barrier per
                                     // buffer: the softmax runs ahead of the MMA thread's waits)
  uint64_t* pv_done = p_full + 2;    // [2] value product of tile t (P' buffer t & 1) complete
  uint64_t* done = pv_done + 2;       // [2] each MMA issuer's MMAs complete
  uint32_t* tmem_slot = (uint32_t*)(sm + BAR_OFF + 512);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* red = (float*)(sm + BAR_OFF + 1024);   // [2][4][32]
  float* rbuf = (float*)(sm + BAR_OFF + 2048);  // [NRB][128]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % p.n_split, b = blockIdx.x / p.n_split;
  const int n_vis = min(p.q_pos[b] + 1, p.t_max);            // keys 0 .. cache_len[b]
  const int j0 = split * chunk_tiles * BK;
  const int j1 = min(j0 + chunk_tiles * BK, n_vis);
  const int nt = j1 > j0 ? (j1 - j0 + BK - 1) / BK : 0;
  // first key of tile t: a ragged last tile is moved back to end at j1 (keys before its
  // nominal start are masked; before key 0 the copy reads zeros)
  auto tile_start = [&](int t) { const int k = j0 + t * BK; return k + BK <= j1 ? k : j1 - BK; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sempty[i], 1 + 4);   // the MMAs' commit and the four sum-of-squares warps
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    mbar_init(q_ready, 128);
    for (int i = 0; i < NSB; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    for (int i = 0; i < NRB; ++i) mbar_init(&r_ready[i], 128);
    mbar_init(&p_full[0], 128);
    mbar_init(&p_full[1], 128);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(&done[0], 1);
    mbar_init(&done[1], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if ((warp == 0 || warp == 2) && lane == 0 && nt > 0) {
    // ---------------- TMA producers: chunks in the order the MMAs consume them ----------------
    const bool score = warp == 0;
    Ring rg{score ? sfull : vfull, score ? sempty : vempty, score ? NS : NV, 0};
    const uint64_t pol = score ? policy_evict_last() : policy_evict_first();
    int phase[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) phase[i] = -1;
    auto get = [&](uint32_t bytes) -> int {
      const int s = rg.c % rg.n;
      if (!mbar_wait(&rg.empty[s], ((rg.c / rg.n) & 1) ^ 1, abort_flag)) return -1;
      mbar_expect_tx(&rg.full[s], bytes);
      phase[s] = (rg.c / rg.n) & 1;
      ++rg.c;
      return s;
    };
    bool ok = true;
    const int n_load = p.test_no_loads ? 0 : nt;   // test only: idle producers, so the waits run out
    for (int t = 0; t < n_load && ok; ++t) {
      const int ks = tile_start(t);
      if (score) {
        for (int i = 0; i < 4 && ok; ++i) {
          const int s = get(SSLOT);
          if (!(ok = s >= 0)) break;
          tma_load_3d(sring + s * SSLOT, &tmC, &sfull[s], 128 * i, ks, b, pol);
          tma_load_3d(sring + s * SSLOT + BOX, &tmC, &sfull[s], 128 * i + 64, ks, b, pol);
        }
        if (!ok) break;
        const int s = get(BOX);
        if (!(ok = s >= 0)) break;
        tma_load_3d(sring + s * SSLOT, &tmR, &sfull[s], 0, ks, b, pol);
      } else {
        for (int i = 0; i < 4 && ok; ++i)
          for (int kh = 0; kh < 2 && ok; ++kh) {
            const int s = get(VSLOT);
            if (!(ok = s >= 0)) break;
            tma_load_3d(vring + s * VSLOT, &tmV, &vfull[s], 128 * i, ks + 64 * kh, b, pol);
            tma_load_3d(vring + s * VSLOT + VBOX, &tmV, &vfull[s], 128 * i + 64, ks + 64 * kh, b, pol);
          }
      }
    }
    // copies still in flight (an abort) land before the CTA's shared memory is released
    for (int i = 0; i < rg.n; ++i)
      if (phase[i] >= 0) mbar_drain(&rg.full[i], (uint32_t)phase[i]);
  } else if ((warp == 1 || warp == 11) && lane == 0) {
    // ---------------- MMA issuers: warp 1 the scores, warp 11 the value products ----------------
    // (separate threads, so neither stream waits behind the other's memory latency; they
    // write disjoint TMEM columns and each commit tracks its own thread's MMAs)
    const bool score = warp == 1;
    if (nt > 0) {
      constexpr uint32_t ID_S = idesc_bf16(BK, NP);
      constexpr uint32_t ID_U = idesc_bf16_mn(128, NP, true, false);   // A = C^T: MN-major
      Ring r = score ? Ring{sfull, sempty, NS, 0} : Ring{vfull, vempty, NV, 0};
      auto take = [&]() -> int {
        const int s = r.c % r.n;
        if (!mbar_wait(&r.full[s], (r.c / r.n) & 1, abort_flag)) return -1;
        tc_fence_after();
        ++r.c;
        return s;
      };
      bool ok = true;
      if (score) {
        ok = mbar_wait(q_ready, 0, abort_flag);
        tc_fence_after();
        // the scores of tile t into TMEM buffer t % NSB once the softmax has read tile t - NSB
        for (int t = 0; t < nt && ok; ++t) {
          const int sb = t % NSB;
          if (t >= NSB && !(ok = mbar_wait(&s_free[sb], ((t / NSB) - 1) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t tS = tmem + 64 * sb;
          for (int i = 0; i < 4 && ok; ++i) {
            const int s = take();
            if (!(ok = s >= 0)) break;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t a = smem_desc(sring + s * SSLOT + (kk >> 2) * BOX) + 2 * (kk & 3);
              const uint64_t bq = smem_desc(sQ + (2 * i + (kk >> 2)) * QBOX) + 2 * (kk & 3);
              umma_bf16(tS, a, bq, ID_S, (i > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&sempty[s]);
          }
          if (!ok) break;
          const int s = take();
          if (!(ok = s >= 0)) break;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tS + 32, smem_desc(sring + s * SSLOT) + 2 * kk, smem_desc(sQ + 8 * QBOX) + 2 * kk, ID_S,
                      kk > 0 ? 1u : 0u);
          umma_commit(&sempty[s]);
          umma_commit(&s_full[sb]);
        }
      } else {
        // the value product of tile t once its P' is written
        for (int t = 0; t < nt && ok; ++t) {
          if (!(ok = mbar_wait(&p_full[t & 1], (t >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          const uint8_t* pb = sP + (t & 1) * PBUF;
          for (int i = 0; i < 4 && ok; ++i)
            for (int kh = 0; kh < 2; ++kh) {
              const int s = take();
              if (!(ok = s >= 0)) break;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = smem_desc_mn(vring + s * VSLOT + kk * 2048, VBOX);   // 16 keys = 2 KB
                const uint64_t bp = smem_desc(pb + kh * QBOX) + 2 * kk;
                umma_bf16(tmem + T_U + 32 * i, a, bp, ID_U, (t > 0 || kh > 0 || kk > 0) ? 1u : 0u);
              }
              umma_commit(&vempty[s]);
            }
          if (ok) umma_commit(&pv_done[t & 1]);
        }
      }
    }
    // all issued MMAs complete before TMEM is released (also after an abort)
    umma_commit(&done[score ? 0 : 1]);
    mbar_drain(&done[score ? 0 : 1], 0);
  } else if (warp >= 3 && warp <= 6) {
    // ---------------- softmax: thread = key kl of the tile = TMEM lane ----------------
    const int quarter = warp & 3, kl = quarter * 32 + lane, st = threadIdx.x - SMX0;
    const uint32_t lb = (uint32_t)(quarter * 32) << 16;
    if (nt > 0) {
      // query rows [32 heads][576] in the 128-byte-swizzled K-major layout; heads past H zero
      for (int i = st; i < NP * 72; i += 128) {
        const int n = i / 72, u = i % 72;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (n < p.H) {
          if (u < 64) v = *reinterpret_cast<const uint4*>((const bf16*)p.qa + ((long long)b * p.H + n) * KVR + 8 * u);
          else
            v = *reinterpret_cast<const uint4*>((const bf16*)p.q + (long long)b * p.q_row + (long long)n * p.q_head +
                                                p.dn + 8 * (u - 64));
        }
        *reinterpret_cast<uint4*>(sQ + (u >> 3) * QBOX + n * 128 + (((u & 7) ^ (n & 7)) << 4)) = v;
      }
      fence_async_smem();
      mbar_arrive(q_ready);
    }
    const float lg2s = p.scale * 1.4426950408889634f;   // scores in log2 units
    float m_run = -INFINITY;                             // running maximum of head `lane`
    float lp[NP];                                        // this key's share of l, per head
#pragma unroll
    for (int h = 0; h < NP; ++h) lp[h] = 0.f;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int sb = t & 1, tb = t % NSB;
      ok = bar_and(mbar_wait(&s_full[tb], (t / NSB) & 1, abort_flag) &&
                       mbar_wait(&r_ready[t % NRB], (t / NRB) & 1, abort_flag),
                   1, 128);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = tmem + lb + 64 * tb;
      uint32_t rl[32], rr[32];
      tmem_ld32_raw(tS, rl);
      tmem_ld32_raw(tS + 32, rr);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(&s_free[tb]);                  // the scores of tile t + NSB may land there
      const float r = rbuf[(t % NRB) * BK + kl];
      const int kabs = tile_start(t) + kl;
      const bool valid = kabs >= j0 + t * BK && kabs < j1;
      float s[NP];
#pragma unroll
      for (int h = 0; h < NP; ++h)
        s[h] = (valid && h < p.H) ? (__uint_as_float(rl[h]) * r + __uint_as_float(rr[h])) * lg2s : -INFINITY;
      // the tile's maximum per head over its 128 keys (lane h of every warp: head h)
      red[(sb * 4 + quarter) * 32 + lane] = warp_reduce32<true>(s, lane);
      bar_sync(1, 128);
      const float* rs = red + sb * 128;
      const float mt = fmaxf(fmaxf(rs[lane], rs[32 + lane]), fmaxf(rs[64 + lane], rs[96 + lane]));
      float corr = 1.f;
      if (mt > m_run + RESCALE_LOG2) {
        corr = exp2f(m_run - mt);
        m_run = mt;
      }
      const bool resc = t > 0 && __any_sync(FULL, corr != 1.f);   // the same in every warp
      const float base = (m_run == -INFINITY) ? 0.f : m_run;
      float pr[NP];
#pragma unroll
      for (int h = 0; h < NP; ++h) pr[h] = exp2f(s[h] - __shfl_sync(FULL, base, h));
      if (resc) {
#pragma unroll
        for (int h = 0; h < NP; ++h) lp[h] *= __shfl_sync(FULL, corr, h);
      }
#pragma unroll
      for (int h = 0; h < NP; ++h) lp[h] += pr[h];
      // P' buffer t & 1 was read by the value product of tile t - 2; a rescale of U^T waits
      // for that of tile t - 1
      bool w = t < 2 || mbar_wait(&pv_done[sb], ((t >> 1) - 1) & 1, abort_flag);
      if (w && resc) w = mbar_wait(&pv_done[sb ^ 1], ((t - 1) >> 1) & 1, abort_flag);
      ok = bar_and(w, 1, 128);
      if (!ok) break;
      tc_fence_after();
      if (resc) {
        float cf[NP];
#pragma unroll
        for (int h = 0; h < NP; ++h) cf[h] = __shfl_sync(FULL, corr, h);
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float v[32];
          tmem_ld32(tmem + lb + T_U + 32 * q, v);
#pragma unroll
          for (int h = 0; h < NP; ++h) v[h] *= cf[h];
          tmem_st32(tmem + lb + T_U + 32 * q, v);
        }
        tmem_st_wait();
      }
      // P'[head][key] = p r_j (the value side sums p r_j c_j), K-major with 128-byte swizzle
      uint8_t* pcol = sP + sb * PBUF + (kl >> 6) * QBOX + (kl & 7) * 2;
      const int unit = (kl & 63) >> 3;
#pragma unroll
      for (int h = 0; h < NP; ++h)
        *reinterpret_cast<bf16*>(pcol + h * 128 + ((unit ^ (h & 7)) << 4)) = __float2bfloat16_rn(pr[h] * r);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }
    // ---- the range's partials: U rows (unnormalised), m (log2 units) and l per head
    if (ok && nt > 0) ok = bar_and(mbar_wait(&pv_done[(nt - 1) & 1], ((nt - 1) >> 1) & 1, abort_flag), 1, 128);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float v[32];
        if (nt > 0) {
          tmem_ld32(tmem + lb + T_U + 32 * q, v);
        } else {
#pragma unroll
          for (int h = 0; h < NP; ++h) v[h] = 0.f;
        }
        const int c = 128 * q + kl;
#pragma unroll
        for (int h = 0; h < NP; ++h)
          if (h < p.H) p.part_o[(((long long)b * p.H + h) * p.n_split + split) * KVR + c] = v[h];
      }
      const float lw = warp_reduce32<false>(lp, lane);
      bar_sync(1, 128);   // the last tile's reads of red are done
      red[quarter * 32 + lane] = lw;
      bar_sync(1, 128);
      if (quarter == 0 && lane < p.H) {
        const long long slot = ((long long)b * p.H + lane) * p.n_split + split;
        p.part_ml[2 * slot] = m_run;
        p.part_ml[2 * slot + 1] = red[lane] + red[32 + lane] + red[64 + lane] + red[96 + lane];
      }
    }
  } else if (warp >= 7 && warp <= 10) {
    // ---------------- sums of squares: thread = key kl of the tile ----------------
    const int kl = threadIdx.x - SSQ0;
    int c = 0;
    bool ok = true;
    for (int t = 0; t < nt && ok; ++t) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int ch = 0; ch < 5; ++ch) {          // the tile's four latent chunks, then its rope chunk
        const int s = c % NS;
        if (!(ok = mbar_wait(&sfull[s], (c / NS) & 1, abort_flag))) break;
        if (ch < 4) {
          const uint8_t* row = sring + s * SSLOT + kl * 128;
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const uint4 v = *reinterpret_cast<const uint4*>(row + bx * BOX + ((u ^ (kl & 7)) << 4));
              const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                sq2(acc[2 * e], acc[2 * e + 1], __uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[s]);
        ++c;
        if (ch == 3) {
          const float ssq = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          rbuf[(t % NRB) * BK + kl] = rsqrtf(ssq * (1.f / KVR) + p.eps);
          mbar_arrive(&r_ready[t % NRB]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) record_status(p.st, ST_TIMEOUT, 611, blockIdx.x);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
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

// 3-D bf16 map [d2][d1][d0] (row stride s1 bytes, plane stride s2 bytes), box {64, box1, 1},
// 128-byte swizzle; coordinates outside the tensor read zeros.
typedef CUresult (*EncodeTiled3Fn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
bool make_map3(CUtensorMap* m, const void* base, unsigned long long d0, unsigned long long d1, unsigned long long d2,
               unsigned long long s1, unsigned long long s2, unsigned box1) {
  static EncodeTiled3Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiled3Fn)ptr;
  });
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool mla_tc_shape(int H, int kvr, int dr, int t_max) {
  return kvr == mtc::KVR && dr == mtc::DR && H >= 1 && H <= mtc::NP && t_max >= mtc::BK;
}

// 1: not this kernel's shape or layout (the caller takes the mma.sync kernel), 0: launched,
// -1: error.
int launch_attn_tc(const MlaDecodeParams& p, cudaStream_t s) {
  if (!mla_tc_shape(p.H, p.kvr, p.dr, p.t_max)) return 1;
  auto a16 = [](const void* q) { return ((uintptr_t)q & 15) == 0; };
  if (!a16(p.ckv) || !a16(p.krope) || !a16(p.qa) || !a16(p.q) || p.q_row % 8 || p.q_head % 8 || p.dn % 8) return 1;
  CUtensorMap mC, mR;
  const unsigned long long tm = (unsigned long long)p.t_max, B = (unsigned long long)p.B;
  if (!make_map3(&mC, p.ckv, mtc::KVR, tm, B, mtc::KVR * 2ull, tm * mtc::KVR * 2ull, mtc::BK)) return 1;
  if (!make_map3(&mR, p.krope, mtc::DR, tm, B, mtc::DR * 2ull, tm * mtc::DR * 2ull, mtc::BK)) return 1;
  CUtensorMap mV;   // the value chunks: [64 keys][64 dims] boxes of the latent cache
  if (!make_map3(&mV, p.ckv, mtc::KVR, tm, B, mtc::KVR * 2ull, tm * mtc::KVR * 2ull, 64)) return 1;
  if (!ensure_smem_limit((const void*)k_mla_attn_tc, mtc::SMEM)) return -1;
  const int tiles = (p.t_max + mtc::BK - 1) / mtc::BK;
  const int chunk_tiles = (tiles + p.n_split - 1) / p.n_split;
  k_mla_attn_tc<<<(unsigned)(p.B * p.n_split), mtc::THREADS, mtc::SMEM, s>>>(mC, mR, mV, p, chunk_tiles);
  note_launch();
  return 0;
}
}  // namespace

bool mla_decode_supports(int attn_type, int dtype, int H, int kvr, int dr, int dn, int dv) {
  if (attn_type != 1 || dtype != 1 || H < 1 || H > 32) return false;
  const bool shape = (kvr == 32 && dr == 16) || (kvr == 128 && dr == 32) || (kvr == 512 && dr == 64);
  return shape && dn % 8 == 0 && dn >= 8 && dn <= 256 && dv >= 1;
}

int mla_decode_splits(int B, int H, int kvr, int dr, int t_max) {
  const int sms = tc_sm_count() > 0 ? tc_sm_count() : 148;
  if (mla_tc_shape(H, kvr, dr, t_max)) {
    // tensor-core kernel: one CTA per SM, 128-key tiles; fewest waves x (tiles per range +
    // about 2 tiles of fixed cost: the query staging, the first scores, the partial write)
    const int tiles = (t_max + mtc::BK - 1) / mtc::BK;
    int best = 1;
    long long best_cost = -1;
    for (int ns = 1; ns <= std::min(32, tiles); ++ns) {
      const long long waves = ((long long)B * ns + sms - 1) / sms;
      const long long cost = waves * ((tiles + ns - 1) / ns + 2);
      if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = ns; }
    }
    return best;
  }
  // key ranges per sequence: fewest waves x (tiles per range + the fixed cost of a CTA:
  // its query load and partial write, about 1.5 tiles) over the CTA slots of the SMs
  const int kg = mla::kg_for((std::max(H, 1) + 7) / 8);
  const int tile_keys = 32 * kg, per_sm = 3 - kg;
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
  if (p.test_no_loads) return launch_attn_tc(p, s) == 0 ? 0 : -1;   // test only: the attention alone
  {
    dim3 grid((unsigned)p.H, (unsigned)((p.kvr + qab::BC - 1) / qab::BC), (unsigned)((p.B + qab::BB - 1) / qab::BB));
    k_mla_q_absorb<<<grid, 128, 0, s>>>(p);
    note_launch();
  }
  int rc = -1;
  if (p.kvr == 32 && p.dr == 16) rc = launch_attn_h<32, 16>(p, s);
  else if (p.kvr == 128 && p.dr == 32) rc = launch_attn_h<128, 32>(p, s);
  else if (p.kvr == 512 && p.dr == 64) {
    rc = launch_attn_tc(p, s);
    if (rc > 0) rc = launch_attn_h<512, 64>(p, s);
  }
  if (rc) return rc;
  if (p.kvr == 32) rc = launch_out_t<32>(p, s);
  else if (p.kvr == 128) rc = launch_out_t<128>(p, s);
  else rc = launch_out_t<512>(p, s);
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace rdt
