// Causal GQA prefill attention on the sm_100a tensor cores (S3 of the recurrent block),
// head dim 128, bf16 operands, fp32 softmax and accumulation.
//
// One CTA per (sequence, head, 128-query tile), heaviest tiles first.
//   warp 0      TMA: Q once; K and V^T tiles of 128 keys into a 2-stage ring
//   warp 1      TMEM owner; lane 0 issues  S_j = Q K_j^T  (into one of two TMEM S
//               buffers, so QK^T of tile j+1 overlaps the softmax of tile j) and
//               O += P_j V_j  (TMEM O accumulator)
//   warps 2..5  softmax: thread = query row = TMEM lane.  Reads its S row, masks
//               (key j visible iff key_pos0 + j <= q_pos, "OpenMythos 분석", Core
//               Structure causal mask), keeps a running max m and sum l in the log2
//               domain, writes P = exp2(s - m) as bf16 into 128B-swizzled shared
//               memory (the A operand of the PV MMA).  The running max is raised only
//               when it grows by more than 2^8, and only then is the O row rescaled in
//               TMEM, so probabilities stay <= 256 and most tiles skip the rescale.
// V is consumed transposed (V^T[b][g][dim][t], written by the QKV GEMM epilogue) so
// both MMAs read K-major operands.  Every wait is bounded (RDT_ERR_DEVICE_TIMEOUT).
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace rdt {

bool tc_make_map(CUtensorMap* m, const void* base, unsigned long long rows, unsigned long long cols,
                 unsigned long long ld, unsigned box_rows);
int tc_sm_count();

namespace fat {

constexpr int BQ = 128, BKV = 128, HD = 128;
constexpr int TILE = 128 * 128 * 2;   // 32 KB: two 64-column swizzle atoms of 16 KB
constexpr int HALF = TILE / 2;
constexpr int SMEM = TILE /*Q*/ + 2 * TILE /*K*/ + 2 * TILE /*V^T*/ + TILE /*P*/ + 1024 + 256;
constexpr int TMEM_COLS = 512;        // S0 [0,128), S1 [128,256), O [256,384)
constexpr float RESCALE_LOG2 = 8.f;   // lazy rescale threshold (factor 256)

struct Args {
  int B, T, H, G, Hkv;
  const int* q_pos;
  int key_pos0, n_keys;
  float sl2;               // softmax scale * log2(e)
  bf16* o;
  long long o_row;         // output row stride (elements); head h at column h * 128
  int q_col0, k_col0;      // qkv columns of query head 0 and key head 0
  DevStatus* st;
};

using namespace rdt::tc;

__global__ void __launch_bounds__(192, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQK, const __grid_constant__ CUtensorMap tmVt, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TILE;            // 2 stages
  uint8_t* sV = sK + 2 * TILE;        // 2 stages
  uint8_t* sP = sV + 2 * TILE;
  uint64_t* bars = (uint64_t*)(sP + TILE);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;       // [2]
  uint64_t* kv_empty = bars + 3;      // [2]
  uint64_t* s_full = bars + 5;        // [2]
  uint64_t* p_full = bars + 7;
  uint64_t* pv_done = bars + 8;
  uint64_t* done = bars + 9;
  uint32_t* tmem_slot = (uint32_t*)(bars + 10);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int n_qt = (a.T + BQ - 1) / BQ;
  const int BH = a.B * a.H;
  const int qt = n_qt - 1 - (int)(blockIdx.x / BH);
  const int bh = blockIdx.x % BH;
  const int b = bh / a.H, h = bh % a.H, g = h / a.G;
  const int q0 = qt * BQ;
  const int q_rows = min(BQ, a.T - q0);
  const long long row0 = (long long)b * a.T + q0;
  int n_vis = min(a.n_keys, a.q_pos[row0 + q_rows - 1] - a.key_pos0 + 1);
  if (n_vis < 0) n_vis = 0;
  const int nt = (n_vis + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(done, 1);
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

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    mbar_expect_tx(q_full, TILE);
    const int qx = a.q_col0 + h * HD;
    tma_load_2d(sQ, &tmQK, q_full, qx, (int)row0);
    tma_load_2d(sQ + HALF, &tmQK, q_full, qx + 64, (int)row0);
    const int kx = a.k_col0 + g * HD;
    const int vy = (b * a.Hkv + g) * HD;
    for (int j = 0; j < nt; ++j) {
      const int st = j & 1;
      if (!mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1, abort_flag)) break;
      mbar_expect_tx(&kv_full[st], 2 * TILE);
      const int ky = b * a.T + j * BKV;
      tma_load_2d(sK + st * TILE, &tmQK, &kv_full[st], kx, ky);
      tma_load_2d(sK + st * TILE + HALF, &tmQK, &kv_full[st], kx + 64, ky);
      tma_load_2d(sV + st * TILE, &tmVt, &kv_full[st], j * BKV, vy);
      tma_load_2d(sV + st * TILE + HALF, &tmVt, &kv_full[st], j * BKV + 64, vy);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t IDESC = idesc_bf16(128, 128);
    const uint32_t tO = tmem + 256;
    bool ok = mbar_wait(q_full, 0, abort_flag);
    auto issue_pv = [&](int jj) -> bool {
      if (!mbar_wait(p_full, jj & 1, abort_flag)) return false;
      tc_fence_after();
      const int st = jj & 1;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad = smem_desc(sP + (kk >> 2) * HALF) + 2 * (kk & 3);
        const uint64_t bd = smem_desc(sV + st * TILE + (kk >> 2) * HALF) + 2 * (kk & 3);
        umma_bf16(tO, ad, bd, IDESC, (jj > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(pv_done);
      umma_commit(&kv_empty[st]);
      return true;
    };
    for (int j = 0; j < nt && ok; ++j) {
      const int st = j & 1;
      if (!(ok = mbar_wait(&kv_full[st], (j >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t tS = tmem + st * 128;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad = smem_desc(sQ + (kk >> 2) * HALF) + 2 * (kk & 3);
        const uint64_t bd = smem_desc(sK + st * TILE + (kk >> 2) * HALF) + 2 * (kk & 3);
        umma_bf16(tS, ad, bd, IDESC, kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[st]);
      if (j >= 1) ok = issue_pv(j - 1);
    }
    if (ok && nt > 0) issue_pv(nt - 1);
    umma_commit(done);
    mbar_wait(done, 0, abort_flag);
  } else if (warp >= 2) {
    // ---------------- softmax ----------------
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const bool row_valid = rl < q_rows;
    const int my_pos = row_valid ? a.q_pos[row0 + rl] : -1;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    uint8_t* prow0 = sP + rl * 128;           // keys 0..63 of this row
    uint8_t* prow1 = sP + HALF + rl * 128;    // keys 64..127
    for (int j = 0; j < nt; ++j) {
      const int st = j & 1;
      if (!(ok = mbar_wait(&s_full[st], (j >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + st * 128 + c, v);
#pragma unroll
        for (int q = 0; q < 32; ++q) s[c + q] = v[q];
      }
      const int k0 = j * BKV;
      const int kp0 = a.key_pos0 + k0;
      const bool need_mask = (kp0 + BKV - 1 > my_pos) || (k0 + BKV > n_vis);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float x = s[c] * a.sl2;
        if (need_mask && (kp0 + c > my_pos || k0 + c >= n_vis)) x = -INFINITY;
        s[c] = x;
        mx = fmaxf(mx, x);
      }
      float alpha = 1.f;
      if (j == 0) {
        m_used = mx;
      } else if (mx > m_used + RESCALE_LOG2) {
        alpha = exp2f(m_used - mx);
        m_used = mx;
        l *= alpha;
      }
      const float base = (m_used == -INFINITY) ? 0.f : m_used;
      // P_j into registers (packed bf16) before the shared buffer is free again
      uint32_t pk[64];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = exp2f(s[c] - base), p1 = exp2f(s[c + 1] - base);
        sum += p0 + p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[c >> 1] = *reinterpret_cast<uint32_t*>(&h2);
      }
      l += sum;
      if (j >= 1) {
        // PV of tile j-1 done: O is stable and the P buffer is free
        if (!(ok = mbar_wait(pv_done, (j - 1) & 1, abort_flag))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            float v[32];
            tmem_ld32(tmem + lane_base + 256 + c, v);
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= alpha;
            tmem_st32(tmem + lane_base + 256 + c, v);
          }
          tmem_st_wait();
        }
      }
      // 16-byte chunk c (8 keys) of a 128-byte row goes to chunk c ^ (row & 7)
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint8_t* rowp = (c < 8) ? prow0 : prow1;
        const int ch = (c & 7) ^ (rl & 7);
        *reinterpret_cast<uint4*>(rowp + ch * 16) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // final: O / l
    if (ok && nt > 0 && mbar_wait(pv_done, (nt - 1) & 1, abort_flag)) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      bf16* orow = a.o + (row0 + rl) * a.o_row + (long long)h * HD;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        float v[32];
        tmem_ld32(tmem + lane_base + 256 + c, v);
        if (row_valid) {
#pragma unroll
          for (int q = 0; q < 32; q += 8) {
            uint4 u;
            uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h2 = __floats2bfloat162_rn(v[q + 2 * e] * inv, v[q + 2 * e + 1] * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&h2);
            }
            *reinterpret_cast<uint4*>(orow + c + q) = u;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) record_status(a.st, ST_TIMEOUT, 601, blockIdx.x);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace fat

// The prefill attention of a bf16 GQA block with head dim 128 can run here when the
// values were also written transposed (p.vt) and rows are 16-byte aligned.
bool attention_tc_supports(int dtype, const AttnParams& p) {
  return dtype == 1 && p.vt && p.dn == 128 && p.dr == 0 && p.dv == 128 && !p.n_keys_dev && p.T % 8 == 0 &&
         p.vt_ld == p.T && p.q_row % 8 == 0 && p.k1_j == p.q_row && p.k1_b == (long long)p.T * p.q_row &&
         p.o_row % 8 == 0 && ((uintptr_t)p.q & 15) == 0 && ((uintptr_t)p.vt & 15) == 0 &&
         ((uintptr_t)p.o & 15) == 0;
}

int launch_attention_tc(const AttnParams& p, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(fat::k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, fat::SMEM) != cudaSuccess)
      return -1;
    attr = true;
  }
  const int Hkv = p.H / p.G;
  // Q and K live in the qkv rows [B*T, q_row]; k1 points at key head 0 inside those rows
  const long long k_col0 = ((const bf16*)p.k1 - (const bf16*)p.q);
  CUtensorMap mQK, mVt;
  if (!tc_make_map(&mQK, p.q, (unsigned long long)p.B * p.T, (unsigned long long)p.q_row, p.q_row, 128)) return -1;
  if (!tc_make_map(&mVt, p.vt, (unsigned long long)p.B * Hkv * 128, (unsigned long long)p.T, p.vt_ld, 128))
    return -1;
  fat::Args a;
  a.B = p.B; a.T = p.T; a.H = p.H; a.G = p.G; a.Hkv = Hkv;
  a.q_pos = p.q_pos; a.key_pos0 = p.key_pos0; a.n_keys = p.n_keys;
  a.sl2 = p.scale * 1.4426950408889634f;
  a.o = (bf16*)p.o; a.o_row = p.o_row;
  a.q_col0 = 0; a.k_col0 = (int)k_col0;
  a.st = nullptr;
  const long long blocks = (long long)((p.T + fat::BQ - 1) / fat::BQ) * p.B * p.H;
  if (blocks <= 0) return 0;
  { fat::k_attn_tc<<<(unsigned)blocks, 192, fat::SMEM, s>>>(mQK, mVt, a); note_launch(); }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace rdt
