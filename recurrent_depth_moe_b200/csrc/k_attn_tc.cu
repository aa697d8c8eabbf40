// Causal GQA prefill attention on the sm_100a tensor cores (S3 of the recurrent block),
// head dim 128, bf16 operands, fp32 softmax and accumulation.
//
// One CTA per (sequence, head, pair of 128-query tiles), heaviest pairs first.
//   warp 0      TMA: both Q tiles once; K tiles of 128 keys into a 3-stage ring and V^T
//               tiles into a 2-stage ring (K is freed one iteration before V)
//   warp 1      TMEM owner; lane 0 issues, per key tile j and query tile q,
//               O_q += P_q(j-1) V_(j-1) and then S_qj = Q_q K_j^T into the same TMEM
//               columns (one S buffer per query tile; tcgen05 MMAs of one thread run in
//               order, so S_qj starts after the PV that read P from those columns).
//               Every MMA is 128 x 128 x 16: the issuing thread, not the tensor pipe, is
//               the limit for narrower tiles.
//   warps 2..5  softmax of query tile 0; warps 6..9 softmax of query tile 1.
//               Thread = query row = TMEM lane: reads its S row, masks (key j visible
//               iff key_pos0 + j <= q_pos, "OpenMythos 분석", Core Structure causal
//               mask), keeps a running max m and sum l in the log2 domain, and writes
//               P = exp2(s - m) as bf16 back into the first 64 columns of its S buffer
//               (3 in 8 of the exponentials on the FMA pipe, the rest on the SFU): the
//               PV MMA reads its A operand from TMEM.  The running max is raised only
//               when it grows by more than 2^8, and only then is the O row rescaled (S of
//               tile j completing means the PV of tile j-1 has too).
// The two query tiles share every K / V tile and their softmax groups overlap each
// other and the tensor core.  V is consumed transposed (V^T[b][g][dim][t], written by
// the QKV GEMM epilogue) so both MMAs read K-major operands.  Every wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace rdt {

bool tc_make_map(CUtensorMap* m, const void* base, unsigned long long rows, unsigned long long cols,
                 unsigned long long ld, unsigned box_rows);

namespace fat {

constexpr int BQ = 128, BKV = 128, HD = 128;   // query / key tile rows; value (and GQA key) head dim
constexpr int BOX = BQ * 64 * 2;                 // 16 KB: one TMA box [128 rows][64 dims], SW128
constexpr int VTILE = HD * BKV * 2;              // 32 KB: two boxes of values
constexpr int VHALF = VTILE / 2;
constexpr float RESCALE_LOG2 = 8.f;              // lazy rescale threshold (factor 256)

// Kernel variants: HQK = score head dim (query and key), NQ = query tiles per CTA, MLA = keys
// from the per-head k_nope columns plus the head-shared k_rope, values read in place
// (MN-major B operand) instead of a transposed copy.
//   GQA: HQK 128, NQ 2, keys and values^T from the QKV projection (3 K stages, 225.5 KB)
//   MLA: HQK 192 (nope 128 + rope 64), NQ 1, keys [k_nope | k_rope], values from the per-head
//        [k_nope | v] rows (2 K stages, 209.5 KB)
template <int HQK_, int NQ_, bool MLA_>
struct Cfg {
  static constexpr int HQK = HQK_, NQ = NQ_;
  static constexpr bool MLA = MLA_;
  static constexpr int NBOX = HQK / 64;                  // 64-dim boxes per query / key row
  static constexpr int QTILE = BQ * HQK * 2, KTILE = BKV * HQK * 2;
  static constexpr int KSTAGES = MLA ? 2 : 3, VSTAGES = 2;
  static constexpr int SMEM = NQ * QTILE + KSTAGES * KTILE + VSTAGES * VTILE + 1024 + 512;
  static constexpr int TMEM_COLS = NQ == 2 ? 512 : 256;  // S[q] at BKV q (P in its first 64); O[q] at BKV NQ + 128 q
  static constexpr int THREADS = 64 + NQ * 128;
};
using CfgGqa = Cfg<128, 2, false>;
using CfgMla = Cfg<192, 1, true>;

struct Args {
  int B, T, H, G, Hkv;
  const int* q_pos;
  int key_pos0, n_keys;
  float sl2;               // softmax scale * log2(e)
  bf16* o;
  long long o_row;         // output row stride (elements); head h at column h * 128
  int q_col0, k_col0;      // GQA: qkv columns of query head 0 and key head 0
  int q_head, k_head;      // columns between heads: queries; keys / values (MLA: nope + v)
  int v_col0;              // MLA: column of the values inside a head's [k_nope | v] row
  // compact queries (or nullptr): the query / output rows of sequence b are the compact rows
  // seq_off[b] .. seq_off[b + 1]; compact row r sits at position q_pos[run_list[r]]
  const int* seq_off;
  const int* run_list;
  DevStatus* st;           // device status word: a wait that gave up is recorded here
};

// position of query row idx (a batch row, or a compact row in compact mode)
__device__ __forceinline__ int query_pos(const Args& a, long long idx) {
  return a.run_list ? a.q_pos[a.run_list[idx]] : a.q_pos[idx];
}

using namespace rdt::tc;

// 32 TMEM columns of this warp's lanes into registers, no wait: the caller issues
// tcgen05.wait::ld before it reads any of r
__device__ __forceinline__ void tmem_ld32_nw(uint32_t taddr, uint32_t* r) {
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the special-function unit
__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for a pair on the FMA pipe (Cody-Waite style range reduction): x = j + f with j the
// nearest integer (added to a 1.5 * 2^23 shifter, whose low mantissa bits then hold j) and
// f in [-1/2, 1/2]; 2^f by a cubic fitted to minimise the relative error on that interval
// (Lawson's reweighted least squares; max relative error 7.5e-5, well inside the bf16
// rounding that P gets); 2^j added into the exponent field.  x is clamped at -125 so the
// exponent stays normal.  Used for a share of the exponentials so that the SFU and the
// FMA pipe finish together.
constexpr float EXP2_C0 = 0.99992806f, EXP2_C1 = 0.69326097f, EXP2_C2 = 0.24261114f, EXP2_C3 = 0.05517167f;
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 jf = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(jf, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
  p = __ffma2_rn(p, f, make_float2(EXP2_C1, EXP2_C1));
  p = __ffma2_rn(p, f, make_float2(EXP2_C0, EXP2_C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// P = 2^(s * sl2 - base) for one row of BKV scores, written as bf16 pairs into the first
// BKV / 2 TMEM columns at tS; returns the fp32 row sum.  Pairs whose index has
// (pair & 7) < 3 (3 in 8) take the FMA-pipe exponential, the rest the SFU; a masked key
// (s = -inf) gives exactly 0 on either.  The choice depends on the column alone, so a row's
// P does not depend on which other rows share its warp (compact query tiles keep causal
// results bit-identical).
__device__ __forceinline__ float exp_row(const float (&s)[BKV], float sl2, float base, uint32_t tS) {
  const float2 sc = make_float2(sl2, sl2), nb = make_float2(-base, -base);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int hh = 0; hh < BKV / 32; ++hh) {
    uint32_t pf[16];
#pragma unroll
    for (int pi = 0; pi < 16; ++pi) {
      const int k = 32 * hh + 2 * pi;
      const float2 x = __ffma2_rn(make_float2(s[k], s[k + 1]), sc, nb);
      float2 p;
      if ((pi & 7) < 3) {   // pair index within the row: (16 hh + pi) & 7 = pi & 7
        p = ex2_poly2(x);
        if (s[k] == -INFINITY) p.x = 0.f;
        if (s[k + 1] == -INFINITY) p.y = 0.f;
      } else {
        p = make_float2(ex2_sfu(x.x), ex2_sfu(x.y));
      }
      acc[pi & 3] = __fadd2_rn(acc[pi & 3], p);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(p.x, p.y);
      pf[pi] = *reinterpret_cast<uint32_t*>(&h2);
    }
    tmem_st16(tS + 16 * hh, pf);
  }
  acc[0] = __fadd2_rn(acc[0], acc[1]);
  acc[2] = __fadd2_rn(acc[2], acc[3]);
  acc[0] = __fadd2_rn(acc[0], acc[2]);
  return acc[0].x + acc[0].y;
}

__device__ __forceinline__ int visible_tiles(const Args& a, long long row_last, int q_rows) {
  if (q_rows <= 0) return 0;
  int n_vis = min(a.n_keys, query_pos(a, row_last) - a.key_pos0 + 1);
  return n_vis > 0 ? (n_vis + BKV - 1) / BKV : 0;
}

// tmQ: query rows; tmK: key rows (GQA qkv / MLA k_nope); tmKR: MLA k_rope rows (unused for
// GQA); tmV: GQA values transposed [b][g][dim][t], MLA the [k_nope | v] rows.
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmKR, const __grid_constant__ CUtensorMap tmV, const Args a) {
  constexpr int NQ = C::NQ, QTILE = C::QTILE, KTILE = C::KTILE, KSTAGES = C::KSTAGES, VSTAGES = C::VSTAGES;
  constexpr int TMEM_COLS = C::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                          // [NQ] query tiles
  uint8_t* sK = sQ + NQ * QTILE;               // [KSTAGES]
  uint8_t* sV = sK + KSTAGES * KTILE;          // [VSTAGES]
  uint64_t* bars = (uint64_t*)(sV + VSTAGES * VTILE);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                 // [KSTAGES]
  uint64_t* k_empty = k_full + KSTAGES;        // [KSTAGES]
  uint64_t* v_full = k_empty + KSTAGES;        // [VSTAGES]
  uint64_t* v_empty = v_full + VSTAGES;        // [VSTAGES]
  uint64_t* s_full = v_empty + VSTAGES;        // [NQ]
  uint64_t* p_full = s_full + NQ;              // [NQ]
  uint64_t* pv_done = p_full + NQ;             // [NQ]
  uint64_t* done = pv_done + NQ;
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int n_qt = (a.T + BQ - 1) / BQ;
  const int n_pairs = (n_qt + NQ - 1) / NQ;
  const int BH = a.B * a.H;
  const int pair = n_pairs - 1 - (int)(blockIdx.x / BH);    // heaviest pairs first
  const int bh = blockIdx.x % BH;
  const int b = bh / a.H, h = bh % a.H, g = h / a.G;
  // this sequence's query rows: rows b T .. b T + T - 1, or its compact rows
  const long long qbase = a.seq_off ? (long long)a.seq_off[b] : (long long)b * a.T;
  const int n_rows = a.seq_off ? a.seq_off[b + 1] - a.seq_off[b] : a.T;
  int q0[NQ], q_rows[NQ], nt[NQ];
  int nt_max = 0;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    q0[q] = (pair * NQ + q) * BQ;
    q_rows[q] = max(0, min(BQ, n_rows - q0[q]));
    nt[q] = visible_tiles(a, qbase + q0[q] + q_rows[q] - 1, q_rows[q]);
    nt_max = max(nt_max, nt[q]);
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KSTAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VSTAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&s_full[q], 1);
      mbar_init(&p_full[q], 128);
      mbar_init(&pv_done[q], 1);
    }
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
    int qbytes = 0;
#pragma unroll
    for (int q = 0; q < NQ; ++q) qbytes += q_rows[q] > 0 ? QTILE : 0;
    mbar_expect_tx(q_full, qbytes);
    const int qx = a.q_col0 + h * a.q_head;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      if (q_rows[q] <= 0) continue;
      const int qy = (int)(qbase + q0[q]);
#pragma unroll
      for (int kb = 0; kb < C::NBOX; ++kb) tma_load_2d(sQ + q * QTILE + kb * BOX, &tmQ, q_full, qx + 64 * kb, qy);
    }
    const int kx = a.k_col0 + g * a.k_head;
    const int vy = (b * a.Hkv + g) * HD;          // GQA: the head's value rows of V^T
    const int vx = g * a.k_head + a.v_col0;       // MLA: the head's value columns
    int k_phase[KSTAGES], v_phase[VSTAGES];   // phase of the last load issued into each stage (-1: none)
#pragma unroll
    for (int s = 0; s < KSTAGES; ++s) k_phase[s] = -1;
#pragma unroll
    for (int s = 0; s < VSTAGES; ++s) v_phase[s] = -1;
    for (int j = 0; j < nt_max; ++j) {
      const int ks = j % KSTAGES, vs = j % VSTAGES;
      if (!mbar_wait(&k_empty[ks], ((j / KSTAGES) & 1) ^ 1, abort_flag)) break;
      mbar_expect_tx(&k_full[ks], KTILE);
      const int ky = b * a.T + j * BKV;
      if (C::MLA) {                               // [k_nope (2 boxes) | k_rope (1 box, shared by the heads)]
        tma_load_2d(sK + ks * KTILE, &tmK, &k_full[ks], kx, ky);
        tma_load_2d(sK + ks * KTILE + BOX, &tmK, &k_full[ks], kx + 64, ky);
        tma_load_2d(sK + ks * KTILE + 2 * BOX, &tmKR, &k_full[ks], 0, ky);
      } else {
#pragma unroll
        for (int kb = 0; kb < C::NBOX; ++kb) tma_load_2d(sK + ks * KTILE + kb * BOX, &tmK, &k_full[ks], kx + 64 * kb, ky);
      }
      k_phase[ks] = (j / KSTAGES) & 1;
      if (!mbar_wait(&v_empty[vs], ((j / VSTAGES) & 1) ^ 1, abort_flag)) break;
      mbar_expect_tx(&v_full[vs], VTILE);
      if (C::MLA) {                               // [128 keys][64 dims] boxes: an MN-major B operand
        tma_load_2d(sV + vs * VTILE, &tmV, &v_full[vs], vx, ky);
        tma_load_2d(sV + vs * VTILE + VHALF, &tmV, &v_full[vs], vx + 64, ky);
      } else {                                    // [128 dims][64 keys] boxes: K-major
        tma_load_2d(sV + vs * VTILE, &tmV, &v_full[vs], j * BKV, vy);
        tma_load_2d(sV + vs * VTILE + VHALF, &tmV, &v_full[vs], j * BKV + 64, vy);
      }
      v_phase[vs] = (j / VSTAGES) & 1;
    }
    // copies still in flight (an abort) land before the CTA's shared memory is released
    if (qbytes > 0) mbar_drain(q_full, 0);
#pragma unroll
    for (int s = 0; s < KSTAGES; ++s)
      if (k_phase[s] >= 0) mbar_drain(&k_full[s], (uint32_t)k_phase[s]);
#pragma unroll
    for (int s = 0; s < VSTAGES; ++s)
      if (v_phase[s] >= 0) mbar_drain(&v_full[s], (uint32_t)v_phase[s]);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t IDESC_S = idesc_bf16(128, BKV);
    constexpr uint32_t IDESC_O = idesc_bf16_mn(128, HD, false, C::MLA);   // MLA values: B MN-major
    bool ok = mbar_wait(q_full, 0, abort_flag);
    // iteration j: PV of tile j - 1 then S of tile j, per query tile (j = nt_max drains)
    for (int j = 0; j <= nt_max && ok; ++j) {
      const int ks = j % KSTAGES, pvs = (j + VSTAGES - 1) % VSTAGES;   // K of tile j, V of tile j - 1
      const bool load = j < nt_max;
      if (load) {
        if (!(ok = mbar_wait(&k_full[ks], (j / KSTAGES) & 1, abort_flag))) break;
        tc_fence_after();
      }
      if (j >= 1) {
        if (!(ok = mbar_wait(&v_full[pvs], ((j - 1) / VSTAGES) & 1, abort_flag))) break;
        tc_fence_after();
      }
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const uint32_t tS = tmem + q * BKV;   // S of tile j; P of tile j - 1 in its first 64 columns
        if (j >= 1 && j - 1 < nt[q]) {
          if (!(ok = mbar_wait(&p_full[q], (j - 1) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t tO = tmem + NQ * BKV + q * 128;
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            const uint64_t bd = C::MLA ? smem_desc_mn(sV + pvs * VTILE + kk * 2048, VHALF)   // 16 keys = 2 atoms
                                       : smem_desc(sV + pvs * VTILE + (kk >> 2) * VHALF) + 2 * (kk & 3);
            umma_bf16_ts(tO, tS + 8 * kk, bd, IDESC_O, (j > 1 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&pv_done[q]);
        }
        if (load && j < nt[q]) {
#pragma unroll
          for (int kk = 0; kk < C::HQK / 16; ++kk) {
            const uint64_t ad = smem_desc(sQ + q * QTILE + (kk >> 2) * BOX) + 2 * (kk & 3);
            const uint64_t bd = smem_desc(sK + ks * KTILE + (kk >> 2) * BOX) + 2 * (kk & 3);
            umma_bf16(tS, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[q]);
        }
      }
      if (!ok) break;
      if (load) umma_commit(&k_empty[ks]);     // K of tile j is consumed once both S MMAs finish
      if (j >= 1) umma_commit(&v_empty[pvs]);  // V of tile j - 1 once both PV MMAs finish
    }
    // all issued MMAs complete before TMEM is released (also after an abort)
    umma_commit(done);
    mbar_drain(done, 0);
  } else if (warp >= 2) {
    // ---------------- softmax of query tile q ----------------
    const int q = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const long long row0 = qbase + q0[q];
    const bool row_valid = rl < q_rows[q];
    const int my_pos = row_valid ? query_pos(a, row0 + rl) : -1;
    const int n_vis = row_valid ? min(a.n_keys, query_pos(a, row0 + q_rows[q] - 1) - a.key_pos0 + 1) : 0;
    const int ntq = nt[q];
    const uint32_t tO = tmem + lane_base + NQ * BKV + q * 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const uint32_t tS = tmem + lane_base + q * BKV;
    for (int j = 0; j < ntq; ++j) {
      // warp-uniform outcome: the TMEM loads and stores below are .sync.aligned
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&s_full[q], j & 1, abort_flag)))) break;
      tc_fence_after();
      uint32_t sr[BKV];
#pragma unroll
      for (int c = 0; c < BKV; c += 32) tmem_ld32_nw(tS + c, &sr[c]);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV; ++c) s[c] = __uint_as_float(sr[c]);
      const int k0 = j * BKV;
      const int kp0 = a.key_pos0 + k0;
      const bool need_mask = (kp0 + BKV - 1 > my_pos) || (k0 + BKV > n_vis);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BKV; ++c)
          if (kp0 + c > my_pos || k0 + c >= n_vis) s[c] = -INFINITY;
      }
      // row max: 8 independent chains of 3-input max, then a tree (exact in any order)
      float mp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mp[k] = fmaxf(s[k], s[8 + k]);
#pragma unroll
      for (int c = 16; c < BKV; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = fmax3(mp[k], s[c + k], s[c + 8 + k]);
      mp[0] = fmax3(mp[0], mp[1], mp[2]);
      mp[3] = fmax3(mp[3], mp[4], mp[5]);
      mp[6] = fmaxf(mp[6], mp[7]);
      const float mx = fmax3(mp[0], mp[3], mp[6]) * a.sl2;   // the scale is positive: max commutes with it
      float alpha = 1.f;
      if (j == 0) {
        m_used = mx;
      } else if (mx > m_used + RESCALE_LOG2) {
        alpha = exp2f(m_used - mx);
        m_used = mx;
        l *= alpha;
      }
      // P over the first 64 columns of the S buffer (S is in registers already)
      const float base = (m_used == -INFINITY) ? 0.f : m_used;
      l += exp_row(s, a.sl2, base, tS);
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // the max moved: O is rescaled before this tile's PV, after P is written so the S
        // row is no longer live (the PV of tile j - 1 is complete: it was issued before S
        // of tile j, whose completion s_full signalled)
#pragma unroll 1
        for (int c = 0; c < HD; c += 32) {
          float v[32];
          tmem_ld32(tO + c, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= alpha;
          tmem_st32(tO + c, v);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[q]);
    }
    // final: O / l
    if (ok && ntq > 0 && __all_sync(0xffffffffu, mbar_wait(&pv_done[q], (ntq - 1) & 1, abort_flag))) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      // line-wise through shared memory: this query tile's Q block is free now (the last PV
      // completing means every S MMA that read it has completed too)
      uint32_t* stg = reinterpret_cast<uint32_t*>(sQ + q * QTILE) + quarter * 32 * BS_LD;
      bf16* obase = a.o + (row0 + quarter * 32) * a.o_row + (long long)h * HD;
#pragma unroll 1
      for (int c = 0; c < HD; c += 32) {
        float v[32];
        tmem_ld32(tO + c, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= inv;
        store_rows_bf16x32(stg, lane, v, obase + c, a.o_row, q_rows[q] - quarter * 32);
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
  // keys in the QKV rows: the same rows as the queries, or (compact queries) their own rows
  const bool keys = p.seq_off ? (p.run_list && p.k1_j % 8 == 0 && p.k1_b == (long long)p.T * p.k1_j &&
                                 ((uintptr_t)p.k1 & 15) == 0 && p.q_row == (long long)p.H * 128)
                              : (p.k1_j == p.q_row && p.k1_b == (long long)p.T * p.q_row);
  return dtype == 1 && p.vt && p.dn == 128 && p.dr == 0 && p.dv == 128 && !p.n_keys_dev && p.T % 8 == 0 &&
         p.vt_ld == p.T && p.q_row % 8 == 0 && keys && p.o_row % 8 == 0 && ((uintptr_t)p.q & 15) == 0 &&
         ((uintptr_t)p.vt & 15) == 0 && ((uintptr_t)p.o & 15) == 0;
}

// The MLA prefill of a bf16 block with nope 128, rope 64 and value 128 (the DeepSeek-V2
// widths) whose keys are this call's rows: k_nope / v in the per-head [k_nope | v] rows of
// k1 (= v - dn), k_rope in k2, one row per position.
bool attention_tc_mla_supports(int dtype, const AttnParams& p) {
  const long long kvw = p.k1_j;
  return dtype == 1 && p.dn == 128 && p.dr == 64 && p.dv == 128 && p.G == 1 && p.k2 && !p.n_keys_dev &&
         p.n_keys == p.T && p.q_head == 192 && p.q_row == (long long)p.H * 192 && p.k1_g == 256 &&
         kvw == (long long)p.H * 256 && p.k1_b == (long long)p.T * kvw && p.k2_j == 64 &&
         p.k2_b == (long long)p.T * 64 && p.v == (const void*)((const bf16*)p.k1 + 128) && p.v_j == kvw &&
         p.v_g == 256 && p.v_b == p.k1_b && p.o_row % 8 == 0 && ((uintptr_t)p.q & 15) == 0 &&
         ((uintptr_t)p.k1 & 15) == 0 && ((uintptr_t)p.k2 & 15) == 0 && ((uintptr_t)p.o & 15) == 0;
}

template <class C>
static int launch_attn_tc_t(const CUtensorMap& mQ, const CUtensorMap& mK, const CUtensorMap& mKR,
                            const CUtensorMap& mV, const fat::Args& a, cudaStream_t s) {
  if (!ensure_smem_limit((const void*)fat::k_attn_tc<C>, C::SMEM)) return -1;
  const int n_qt = (a.T + fat::BQ - 1) / fat::BQ;
  const long long blocks = (long long)((n_qt + C::NQ - 1) / C::NQ) * a.B * a.H;
  if (blocks <= 0) return 0;
  { fat::k_attn_tc<C><<<(unsigned)blocks, C::THREADS, C::SMEM, s>>>(mQ, mK, mKR, mV, a); note_launch(); }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_attention_tc(const AttnParams& p, cudaStream_t s) {
  const int Hkv = p.H / p.G;
  CUtensorMap mQ, mK, mVt;
  const unsigned long long rows = (unsigned long long)p.B * p.T;
  long long k_col0 = 0;
  if (!tc_make_map(&mQ, p.q, rows, (unsigned long long)p.q_row, p.q_row, fat::BQ)) return -1;
  if (p.seq_off) {
    // compact queries in their own buffer; the keys: Hkv heads from key head 0 of the QKV rows
    if (!tc_make_map(&mK, p.k1, rows, (unsigned long long)Hkv * fat::HD, p.k1_j, fat::BKV)) return -1;
  } else {
    // Q and K live in the qkv rows [B*T, q_row]; k1 points at key head 0 inside those rows
    k_col0 = ((const bf16*)p.k1 - (const bf16*)p.q);
    if (!tc_make_map(&mK, p.q, rows, (unsigned long long)p.q_row, p.q_row, fat::BKV)) return -1;
  }
  if (!tc_make_map(&mVt, p.vt, (unsigned long long)p.B * Hkv * fat::HD, (unsigned long long)p.T, p.vt_ld, fat::HD))
    return -1;
  fat::Args a;
  a.B = p.B; a.T = p.T; a.H = p.H; a.G = p.G; a.Hkv = Hkv;
  a.q_pos = p.q_pos; a.key_pos0 = p.key_pos0; a.n_keys = p.n_keys;
  a.sl2 = p.scale * 1.4426950408889634f;
  a.o = (bf16*)p.o; a.o_row = p.o_row;
  a.q_col0 = 0; a.k_col0 = (int)k_col0; a.q_head = fat::HD; a.k_head = fat::HD; a.v_col0 = 0; a.st = p.st;
  a.seq_off = p.seq_off; a.run_list = p.seq_off ? p.run_list : nullptr;
  return launch_attn_tc_t<fat::CfgGqa>(mQ, mK, mK, mVt, a, s);
}

int launch_attention_tc_mla(const AttnParams& p, cudaStream_t s) {
  CUtensorMap mQ, mK, mKR, mV;
  const unsigned long long rows = (unsigned long long)p.B * p.T;
  const unsigned long long kvw = (unsigned long long)p.k1_j;
  if (!tc_make_map(&mQ, p.q, rows, (unsigned long long)p.q_row, p.q_row, fat::BQ)) return -1;
  if (!tc_make_map(&mK, p.k1, rows, kvw, kvw, fat::BKV)) return -1;     // k_nope and v columns
  if (!tc_make_map(&mKR, p.k2, rows, 64, 64, fat::BKV)) return -1;
  mV = mK;
  fat::Args a;
  a.B = p.B; a.T = p.T; a.H = p.H; a.G = 1; a.Hkv = p.H;
  a.q_pos = p.q_pos; a.key_pos0 = p.key_pos0; a.n_keys = p.n_keys;
  a.sl2 = p.scale * 1.4426950408889634f;
  a.o = (bf16*)p.o; a.o_row = p.o_row;
  a.q_col0 = 0; a.k_col0 = 0; a.q_head = 192; a.k_head = 256; a.v_col0 = 128; a.st = p.st;
  a.seq_off = nullptr; a.run_list = nullptr;
  return launch_attn_tc_t<fat::CfgMla>(mQ, mK, mKR, mV, a, s);
}

}  // namespace rdt
