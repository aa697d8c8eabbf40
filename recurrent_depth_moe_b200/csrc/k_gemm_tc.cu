// Tensor-core GEMM for sm_100a: tcgen05.mma with TMEM accumulators, operands staged
// by TMA (no multicast) into 128-byte-swizzled shared memory, persistent CTAs.
//
//   C[M, N] = A[M, K] . B[N, K]^T, bf16 operands, fp32 accumulation.
//   Tile: 128 rows x BN MMA columns (BN = 64, 128 or 256) x 64-deep K stages.
//   Grouped mode (MoE experts): the m-tiles come from a device tile list
//   {group, row0, rows}; B is the group's weight slab.  SwiGLU: the 256 MMA columns
//   are 128 gate rows (W1) and the matching 128 up rows (W3) of the expert, so the
//   epilogue forms silu(gate) * up for 128 output columns in registers.
//   Router (BN = E): each epilogue thread owns one token's E logits and performs the
//   softmax, the biased top-k (ties -> lower expert index), the gate renormalisation
//   and the per-expert histogram ("OpenMythos 분석", MoE) without a second pass.
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA loads; warp 1 owns TMEM
// (alloc / dealloc) and lane 0 issues the MMAs; warps 2..5 are the epilogue, each
// reading its 32-lane quarter of the accumulator with tcgen05.ld (one row per lane).
// The bf16 and residual epilogues pass each 32 x 32 chunk through shared memory, so
// their global loads and stores cover whole row pieces rather than 16 bytes of 32
// rows.  The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue
// of one tile overlaps the MMAs of the next.  Every mbarrier wait is bounded: on timeout the CTA records
// RDT_ERR_DEVICE_TIMEOUT in the status word and leaves its loops.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

#include <cuda.h>
#include <algorithm>
#include <mutex>

namespace rdt {
namespace tc {

constexpr int BM = 128, BK = 64;
// Decode-sized grouped expert GEMMs (EPI_SWIGLU_T / EPI_GATE_T at BN = 256 over a tile list
// with at most TR_ROWS slot rows per expert on average) run their tiles of at most TR_ROWS rows
// with the tokens on the MMA's N side: the stage holds the same
// boxes (128 token rows, then 256 weight rows), but each MMA takes a 128-row weight box as A and
// the token box as B, D^T[weight row, token] = W . X^T, with N = the tile's rows rounded up to
// 16.  An MMA's time follows N (M = 64 costs as much as M = 128; N = 16 / 64 / 128 take about
// 36 / 48 / 64 cycles against 128 for the full 128 x 256 tile), so an expert segment's last,
// partial tile costs about its own rows, and decode tiles of a few rows free their stages
// sooner (3B decode step 17.24 -> 15.97 ms).  Prefill keeps the tokens on M: there the partial
// tiles in this form measured slower (10B step +1.5%), and full tiles would read the token
// operand twice (two 128-wide MMAs), a third more shared-memory traffic than one 256-wide MMA.
//   SwiGLU: gate box -> D_gate, up box -> D_up (128 output columns, N tokens each); the lane of
//           an output column forms silu(gate) * up for its tokens.
//   gate:   the two 128-row boxes of W2 -> two accumulators (256 output columns).
constexpr int TR_ROWS = 64;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
// Epilogue staging in shared memory, one [32 rows][pitch] block per epilogue warp: fp32 rows
// of the residual epilogue (pitch 36 floats, which keeps the row-per-lane writes and the
// line-per-8-lanes reads free of bank conflicts) or bf16 rows of the stores
// (store_rows_bf16x32, pitch BS_LD words).
constexpr int RS_LD = 36, RS_BYTES = 4 * 32 * RS_LD * 4;

template <int BN> struct Shape {
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // ring depth: 192 KB of stages at every width, so the narrow tiles of the decode-sized GEMMs
  // (one 128-row tile of activations, the weights streaming through) keep as many weight bytes
  // in flight per CTA as the wide ones
  static constexpr int STAGES = BN == 64 ? 8 : (BN == 128 ? 6 : 4);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  // the fp32 residual and the bf16 epilogues add the per-warp staging blocks
  static constexpr int smem_bytes(int epi) {
    return SMEM_BYTES + (epi == EPI_ROUTER || epi == EPI_STORE_F32 ? 0 : RS_BYTES);
  }
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;   // power of two >= 32
  static constexpr int B_BOX = BN > 128 ? 128 : BN;             // rows per TMA box
};

struct TcArgs {
  GemmParams p;
  int n_n;             // n tiles
  int m_tiles;         // dense: m tiles; grouped: read from *p.n_tiles
  int b_rows_group;    // rows of B per group (grouped)
  int n_out_tile;      // output columns per tile
  int k_splits;        // > 1: split-K, tile t covers k-blocks of split t / (m_tiles n_n)
  int kb_split;        // k-blocks per split
  long long split_stride;   // elements between the fp32 partials of two splits
  int group_m;         // row tiles per rasterization group (1: column tile fastest)
  int tr_rows;         // tiles of at most this many rows take the tokens-on-N form (0: none)
};

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + __expf(-z)); }

// RoPE pair index of the first column of a 32-column chunk, or -1 when the chunk is
// not rotated.  Descriptors are 32-column aligned (checked on the host), so a chunk is
// either entirely inside one head's rotated range or entirely outside.
__device__ __forceinline__ int rope_chunk(const GemmParams& p, int c) {
  for (int q = 0; q < p.n_rope; ++q) {
    const RopeDesc& r = p.rope[q];
    int rel = c - r.col0;
    if (rel < 0 || rel >= r.n_heads * r.head_stride) continue;
    int o = rel % r.head_stride - r.off;
    if (o >= 0 && o < r.dim) return o >> 1;
  }
  return -1;
}

struct TileInfo { int group, row0, rows, n0, split; };

// Tiles are walked in groups of group_m row tiles: inside a group the row tile varies
// fastest, then the column tile.  The CTAs in flight at any moment then cover a few column
// tiles of up to group_m row tiles, so each weight tile (B) is read from DRAM once per group
// and the group's activation rows (A) stay in L2 across its column tiles.  With the column
// tile fastest (group_m = 1), an expert holding many row tiles -- a popular expert under a
// skewed router -- has its whole weight slab swept once per wave of CTAs, which only L2 can
// absorb when the slab is small; the host picks group_m from the slab size.
__device__ __forceinline__ TileInfo decode_tile(const TcArgs& a, int t, int m_tiles) {
  TileInfo ti;
  ti.split = 0;
  if (a.k_splits > 1) {
    const int per = m_tiles * a.n_n;
    ti.split = t / per;
    t %= per;
  }
  const int per_group = a.group_m * a.n_n;
  const int gm0 = (t / per_group) * a.group_m, r = t % per_group;
  const int gsz = min(a.group_m, m_tiles - gm0);   // the last group may hold fewer row tiles
  const int m_i = gm0 + r % gsz, n_i = r / gsz;
  if (a.p.tiles) {
    ti.group = a.p.tiles[4 * m_i];
    ti.row0 = a.p.tiles[4 * m_i + 1];
    ti.rows = a.p.tiles[4 * m_i + 2];
  } else {
    ti.group = 0;
    ti.row0 = m_i * BM;
    ti.rows = min(BM, a.p.M - ti.row0);
  }
  ti.n0 = n_i * a.n_out_tile;
  return ti;
}

// Router epilogue for one row held by this thread: E logits in TMEM columns [0, E).
template <int E>
__device__ __forceinline__ void route_row(const GemmParams& p, uint32_t tbase, bool valid, long long r) {
  float lg[E];
#pragma unroll
  for (int c = 0; c < E; c += 32) {
    float v[32];
    tmem_ld32(tbase + c, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) lg[c + j] = v[j];
  }
  if (!valid) return;
  float* lrow = (float*)p.C + r * p.ldc;
#pragma unroll
  for (int c = 0; c < E; c += 4) *reinterpret_cast<float4*>(lrow + c) = make_float4(lg[c], lg[c + 1], lg[c + 2], lg[c + 3]);
  if (p.run_idx && p.run_idx[r] < 0) return;      // halted row: logits only
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < E; ++e) mx = fmaxf(mx, lg[e]);
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) sum += __expf(lg[e] - mx);
  uint32_t taken[E / 32];
#pragma unroll
  for (int w = 0; w < E / 32; ++w) taken[w] = 0u;
  int sel[32];
  float sc[32];
  float gsum = 0.f;
  for (int j = 0; j < p.topk; ++j) {
    float bv = -INFINITY;
    int be = -1;
    float braw = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float b = lg[e] + p.bias[e];
      const bool free = !((taken[e >> 5] >> (e & 31)) & 1u);
      if (free && (be < 0 || b > bv)) { bv = b; be = e; braw = lg[e]; }   // strict >: lower index wins ties
    }
    if (be < 0) { record_status(p.st, ST_BOUNDS, 502, j); be = 0; }
#pragma unroll
    for (int w = 0; w < E / 32; ++w)
      if ((be >> 5) == w) taken[w] |= 1u << (be & 31);
    sel[j] = be;
    sc[j] = __expf(braw - mx) / sum;
    gsum += sc[j];
  }
  for (int j = 0; j < p.topk; ++j) {
    const long long o = r * p.topk + j;
    p.ids[o] = sel[j];
    p.gates[o] = sc[j] / gsum;
    p.rank[o] = atomicAdd(&p.counts[sel[j]], 1);
  }
}

template <int EPI, int BN>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const TcArgs args) {
  using S = Shape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + S::STAGES * S::STAGE_BYTES);
  uint64_t* empty = full + S::STAGES;
  uint64_t* tfull = empty + S::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* epi_stage = (float*)(smem + S::STAGES * S::STAGE_BYTES + 256);   // RS_BYTES, not for the router
  const GemmParams& p = args.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(S::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int m_tiles = p.tiles ? min(*p.n_tiles, p.max_tiles) : args.m_tiles;
  const int total = m_tiles * args.n_n * max(args.k_splits, 1);
  const int nk = p.K / BK;
  // k-block range of a tile (all of K unless split)
  auto k_range = [&](const TileInfo& ti, int& k0, int& k1) {
    if (args.k_splits > 1) {
      k0 = ti.split * args.kb_split;
      k1 = min(nk, k0 + args.kb_split);
    } else {
      k0 = 0;
      k1 = nk;
    }
  };

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int stage = 0;
    uint32_t phase = 0;
    int issued_phase[S::STAGES];   // phase of the last load issued into each stage (-1: none)
#pragma unroll
    for (int s = 0; s < S::STAGES; ++s) issued_phase[s] = -1;
    // test hook: a producer that issues nothing starves every consumer wait
    const int n_prod = p.test_no_loads ? 0 : total;
    for (int t = blockIdx.x; t < n_prod && !*abort_flag; t += gridDim.x) {
      const TileInfo ti = decode_tile(args, t, m_tiles);
      const int gb = ti.group * args.b_rows_group;
      int b0, b1;
      if (EPI == EPI_SWIGLU_T) {
        b0 = gb + ti.n0;
        b1 = gb + p.up_off + ti.n0;
      } else {
        b0 = gb + ti.n0;
        b1 = b0 + S::B_BOX;
      }
      int k0, k1;
      k_range(ti, k0, k1);
      for (int ks = k0; ks < k1; ++ks) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
        uint8_t* sa = smem + stage * S::STAGE_BYTES;
        mbar_expect_tx(&full[stage], S::STAGE_BYTES);
        tma_load_2d(sa, &tmA, &full[stage], ks * BK, ti.row0);
        tma_load_2d(sa + A_BYTES, &tmB, &full[stage], ks * BK, b0);
        if (BN > 128) tma_load_2d(sa + A_BYTES + S::B_BOX * BK * 2, &tmB, &full[stage], ks * BK, b1);
        issued_phase[stage] = (int)phase;
        if (++stage == S::STAGES) { stage = 0; phase ^= 1; }
      }
    }
    // copies still in flight (an abort) land before the CTA's shared memory is released
#pragma unroll
    for (int s = 0; s < S::STAGES; ++s)
      if (issued_phase[s] >= 0) mbar_drain(&full[s], (uint32_t)issued_phase[s]);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t IDESC = idesc_bf16(BM, BN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    constexpr bool TRC = (EPI == EPI_SWIGLU_T || EPI == EPI_GATE_T) && BN == 256;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      if (!(ok = mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * BN;
      const TileInfo ti = decode_tile(args, t, m_tiles);
      // tokens on N for a small tile of a tile list: its rows rounded up to 16 (N = 16..64)
      const bool TR = TRC && ti.rows <= args.tr_rows;
      const uint32_t idesc_tr = idesc_bf16(128, TR ? ((max(ti.rows, 1) + 15) & ~15) : 16);
      int k0, k1;
      k_range(ti, k0, k1);
      for (int ks = k0; ks < k1; ++ks) {
        if (!(ok = mbar_wait(&full[stage], phase, abort_flag))) break;
        tc_fence_after();
        uint8_t* sa = smem + stage * S::STAGE_BYTES;
        const uint64_t ad = smem_desc(sa), bd = smem_desc(sa + A_BYTES);
        if (TR) {
          // A = a 128-row weight box, B = the token box; the two boxes into their own accumulators
          const uint64_t wd1 = smem_desc(sa + A_BYTES + S::B_BOX * BK * 2);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t accum = (ks != k0 || k != 0) ? 1u : 0u;
            umma_bf16(d, bd + 2 * k, ad + 2 * k, idesc_tr, accum);
            umma_bf16(d + 128, wd1 + 2 * k, ad + 2 * k, idesc_tr, accum);
          }
        } else {
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(d, ad + 2 * k, bd + 2 * k, IDESC, (ks != k0 || k != 0) ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        if (++stage == S::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      umma_commit(&tfull[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
    // all issued MMAs complete before TMEM is released (also after an abort)
    umma_commit(done);
    mbar_drain(done, 0);
  } else if (warp >= 2) {
    // ---------------- epilogue ----------------
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const TileInfo ti = decode_tile(args, t, m_tiles);
      const bool valid = rl < ti.rows;
      const long long r = (long long)ti.row0 + rl;
      // fp32 residual epilogue, line-wise: a warp's 32 rows x 32 columns pass through shared
      // memory, so lane l handles row 4i + l / 8, columns 4 (l % 8) .. + 3 of instruction i and
      // every residual load and output store covers whole 128-byte lines.  Output / residual
      // rows go through the row map when the product's rows are compact.  The residual does
      // not depend on the accumulator: its first chunk is in flight while this tile's MMAs
      // finish, and chunk c + 1 while chunk c is stored.
      constexpr bool RES = (EPI == EPI_RESID_F32);
      long long ro_i[RES ? 8 : 1];
      bool ok_i[RES ? 8 : 1];
      float4 rcur[RES ? 8 : 1], rnxt[RES ? 8 : 1];
      const int c4 = 4 * (lane & 7);
      if (RES && args.k_splits <= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rw = quarter * 32 + 4 * i + (lane >> 3);
          ok_i[i] = rw < ti.rows;
          const long long rr = (long long)ti.row0 + rw;
          ro_i[i] = ok_i[i] ? (p.row_map ? (long long)p.row_map[rr] : rr) : 0;
          if (ok_i[i]) rcur[i] = __ldg(reinterpret_cast<const float4*>(p.resid + ro_i[i] * p.ld_resid + ti.n0 + c4));
        }
      }
      // warp-uniform outcome: the TMEM loads below are .sync.aligned, so a wait that gave up
      // in some lanes only must not let the others go on to them
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort_flag))) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      uint32_t* const bstg = reinterpret_cast<uint32_t*>(epi_stage) + (warp - 2) * 32 * BS_LD;
      if (RES && args.k_splits <= 1) {
        float* stg = epi_stage + (warp - 2) * 32 * RS_LD;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          if (c + 32 < BN) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (ok_i[i])
                rnxt[i] = __ldg(reinterpret_cast<const float4*>(p.resid + ro_i[i] * p.ld_resid + ti.n0 + c + 32 + c4));
          }
          float v[32];
          tmem_ld32(tbase + c, v);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(stg + lane * RS_LD + 4 * q) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 a = *reinterpret_cast<const float4*>(stg + (4 * i + (lane >> 3)) * RS_LD + c4);
            if (ok_i[i])
              *reinterpret_cast<float4*>((float*)p.C + ro_i[i] * p.ldc + ti.n0 + c + c4) =
                  make_float4(rcur[i].x + a.x, rcur[i].y + a.y, rcur[i].z + a.z, rcur[i].w + a.w);
            rcur[i] = rnxt[i];
          }
          __syncwarp();
        }
      } else if ((EPI == EPI_SWIGLU_T || EPI == EPI_GATE_T) && BN == 256 && ti.rows <= args.tr_rows) {
        // tokens on N: lane = output column (weight row of the box), TMEM columns = the tile's
        // tokens; for a token the warp's 32 lanes write 32 consecutive columns (64 contiguous bytes)
        const int n_tok = ti.rows;
        const int j = quarter * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < n_tok; c += 32) {
          float g[32];
          tmem_ld32(tbase + c, g);
          if (EPI == EPI_SWIGLU_T) {
            float u[32];
            tmem_ld32(tbase + 128 + c, u);
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * u[i];
            bf16* col = (bf16*)p.C + (long long)(ti.row0 + c) * p.ldc + ti.n0 + j;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c + i < n_tok) col[(long long)i * p.ldc] = __float2bfloat16_rn(g[i]);
          } else {
            float u[32];
            tmem_ld32(tbase + 128 + c, u);
            const float gs = (c + lane < n_tok) ? p.row_scale[ti.row0 + c + lane] : 0.f;   // lane i: token c + i
            bf16* col = (bf16*)p.C + (long long)(ti.row0 + c) * p.ldc + ti.n0 + j;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float s = __shfl_sync(0xffffffffu, gs, i);
              if (c + i < n_tok) {
                col[(long long)i * p.ldc] = __float2bfloat16_rn(g[i] * s);
                col[(long long)i * p.ldc + 128] = __float2bfloat16_rn(u[i] * s);
              }
            }
          }
        }
      } else if (EPI == EPI_ROUTER) {
        if (BN == 64 || BN == 128) route_row<(BN == 128 ? 128 : 64)>(p, tbase, valid, r);
      } else if (EPI == EPI_SWIGLU_T) {
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          float g[32], u[32];
          tmem_ld32(tbase + c, g);
          tmem_ld32(tbase + BN / 2 + c, u);
#pragma unroll
          for (int j = 0; j < 32; ++j) g[j] = silu_f(g[j]) * u[j];
          store_rows_bf16x32(bstg, lane, g, (bf16*)p.C + (long long)(ti.row0 + quarter * 32) * p.ldc + ti.n0 + c,
                             p.ldc, ti.rows - quarter * 32);
        }
      } else {
        const float rs = (EPI == EPI_GATE_T && valid) ? p.row_scale[r] : 0.f;
        const int pos = (EPI == EPI_ROPE_T && valid) ? p.pos[r] : 0;
        bf16* const crow0 = (bf16*)p.C + (long long)(ti.row0 + quarter * 32) * p.ldc;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld32(tbase + c, v);
          const int col = ti.n0 + c;
          if (EPI == EPI_STORE_T) {
            store_rows_bf16x32(bstg, lane, v, crow0 + col, p.ldc, ti.rows - quarter * 32);
          } else if (EPI == EPI_GATE_T) {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= rs;
            store_rows_bf16x32(bstg, lane, v, crow0 + col, p.ldc, ti.rows - quarter * 32);
          } else if (EPI == EPI_ROPE_T) {
            const int m0 = rope_chunk(p, col);
            if (m0 >= 0) {
              const float4* cs4 = reinterpret_cast<const float4*>(p.rope_tab + (long long)pos * p.rope_half + m0);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 cs = cs4[q];   // (cos, sin) of pairs m0 + 2q and m0 + 2q + 1
                float a0 = v[4 * q], a1 = v[4 * q + 1], b0 = v[4 * q + 2], b1 = v[4 * q + 3];
                v[4 * q] = a0 * cs.x - a1 * cs.y;
                v[4 * q + 1] = a0 * cs.y + a1 * cs.x;
                v[4 * q + 2] = b0 * cs.z - b1 * cs.w;
                v[4 * q + 3] = b0 * cs.w + b1 * cs.z;
              }
            }
            store_rows_bf16x32(bstg, lane, v, crow0 + col, p.ldc, ti.rows - quarter * 32);
            if (valid && p.vt && col >= p.vt_col0 && col < p.vt_col0 + p.vt_heads * p.vt_hd) {
              // transposed copy of the values: for each dim, the warp's 32 rows are 32
              // consecutive positions, so every store instruction writes 64 contiguous bytes
              const int vc = col - p.vt_col0, g = vc / p.vt_hd, d0 = vc % p.vt_hd;
              const long long b = r / p.vt_T, tpos = r % p.vt_T;
              bf16* vt = (bf16*)p.vt + ((b * p.vt_heads + g) * p.vt_hd + d0) * p.vt_ld + tpos;
#pragma unroll
              for (int j = 0; j < 32; ++j) vt[(long long)j * p.vt_ld] = __float2bfloat16_rn(v[j]);
            }
          } else if (valid) {
            float* dst = (float*)p.C + ti.split * args.split_stride + r * p.ldc + col;
            if (EPI == EPI_RESID_F32) {
              const float4* rs4 = (const float4*)(p.resid + r * p.ld_resid + col);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                float4 a = rs4[q];
                ((float4*)dst)[q] = make_float4(a.x + v[4 * q], a.y + v[4 * q + 1], a.z + v[4 * q + 2], a.w + v[4 * q + 3]);
              }
            } else {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                ((float4*)dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) record_status(p.st, ST_TIMEOUT, 501, blockIdx.x);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS) : "memory");
  }
}

}  // namespace tc

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  });
  return fn;
}

// 2-D bf16 map over [rows, cols] (row stride ld elements), box = 64 columns x box_rows rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, unsigned long long rows, unsigned long long cols,
              unsigned long long ld, unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() { return device_sm_count(); }

inline bool al16(const void* p) { return ((uintptr_t)p & 15) == 0; }
}  // namespace

bool tc_make_map(CUtensorMap* m, const void* base, unsigned long long rows, unsigned long long cols,
                 unsigned long long ld, unsigned box_rows) {
  return make_map(m, base, rows, cols, ld, box_rows);
}
int tc_sm_count() { return sm_count(); }

namespace {
// MMA tile width for an epilogue and output width N (0 = unsupported).
int pick_bn(const GemmParams& p, int epi) {
  if (epi == EPI_SWIGLU_T) return (p.N % 128 == 0) ? 256 : 0;
  if (epi == EPI_ROUTER) return (p.N == 64 || p.N == 128) ? p.N : 0;
  // rows that fit one 128-row tile (decode): the weights are the traffic, so the narrowest
  // tile spreads them over the most CTAs -- unless N is so wide that every CTA gets many
  // tiles anyway (the vocabulary head): then 128-wide tiles halve the re-reads of the
  // shared activation rows, which cross L2 once per tile
  if (!p.tiles && p.M <= tc::BM && !p.vt && p.N % 64 == 0)
    return (p.N % 128 == 0 && p.N / 64 >= 16 * sm_count()) ? 128 : 64;
  if (p.N % 256 == 0) return 256;
  if (p.N % 128 == 0) return 128;
  if (p.N % 64 == 0) return 64;
  return 0;
}

template <int EPI, int BN>
int launch_tc(const CUtensorMap& mA, const CUtensorMap& mB, const tc::TcArgs& a, int grid, cudaStream_t s) {
  constexpr int smem = tc::Shape<BN>::smem_bytes(EPI);
  if (!ensure_smem_limit((const void*)tc::k_gemm_tc<EPI, BN>, smem)) return -1;
  { tc::k_gemm_tc<EPI, BN><<<grid, 192, smem, s>>>(mA, mB, a); note_launch(); }
  return 0;
}

template <int EPI>
int launch_tc_bn(int bn, const CUtensorMap& mA, const CUtensorMap& mB, const tc::TcArgs& a, int grid, cudaStream_t s) {
  switch (bn) {
    case 64: return launch_tc<EPI, 64>(mA, mB, a, grid, s);
    case 128: return launch_tc<EPI, 128>(mA, mB, a, grid, s);
    case 256: return launch_tc<EPI, 256>(mA, mB, a, grid, s);
  }
  return -1;
}
}  // namespace

bool gemm_tc_supports(const GemmParams& p, int epi) {
  if (epi < EPI_STORE_F32 || epi > EPI_ROUTER) return false;
  if (p.K < tc::BK || p.K % tc::BK) return false;
  if (!pick_bn(p, epi)) return false;
  if (p.lda % 8 || p.ldb % 8 || !al16(p.A) || !al16(p.B) || !al16(p.C)) return false;
  if (epi == EPI_STORE_F32 || epi == EPI_RESID_F32 || epi == EPI_ROUTER) {
    if (p.ldc % 4) return false;
  } else if (p.ldc % 8) {
    return false;
  }
  if (epi == EPI_RESID_F32 && (p.ld_resid % 4 || !al16(p.resid))) return false;
  if (epi == EPI_ROPE_T) {
    if (p.rope_half % 2 || !al16(p.rope_tab)) return false;
    for (int q = 0; q < p.n_rope; ++q) {
      const RopeDesc& r = p.rope[q];
      if (r.col0 % 32 || r.head_stride % 32 || r.off % 32 || r.dim % 32) return false;
    }
  }
  if (epi == EPI_ROUTER && (!p.bias || !p.ids || !p.gates || !p.rank || !p.counts || p.topk < 1 || p.topk > 32))
    return false;
  if (p.tiles && (p.b_group_stride % p.ldb || p.b_rows <= 0)) return false;
  if (p.row_map && (epi != EPI_RESID_F32 || !p.tiles)) return false;   // compact rows: tile list, no split
  return encode_fn() != nullptr;
}

// Split-K epilogue: the sum of the fp32 partials in split order (deterministic), then the
// GEMM's own epilogue; two columns per thread (a RoPE pair is two adjacent columns).
__device__ __forceinline__ int rope_pair_col(const GemmParams& p, int c) {
  for (int q = 0; q < p.n_rope; ++q) {
    const RopeDesc& r = p.rope[q];
    const int rel = c - r.col0;
    if (rel < 0 || rel >= r.n_heads * r.head_stride) continue;
    const int o = rel % r.head_stride - r.off;
    if (o >= 0 && o < r.dim) return o >> 1;
  }
  return -1;
}

template <int EPI>
__global__ void __launch_bounds__(256) k_splitk_epilogue(GemmParams p, const float* __restrict__ part, int splits,
                                                        long long stride) {
  const long long r = blockIdx.y;
  const int c = 2 * (blockIdx.x * 256 + threadIdx.x);
  if (c >= p.N) return;
  const float* src = part + r * p.N + c;
  float v0 = 0.f, v1 = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float2 a = *reinterpret_cast<const float2*>(src + (long long)s * stride);
    v0 += a.x;
    v1 += a.y;
  }
  if (EPI == EPI_STORE_F32) {
    *reinterpret_cast<float2*>((float*)p.C + r * p.ldc + c) = make_float2(v0, v1);
  } else if (EPI == EPI_RESID_F32) {
    const float2 a = *reinterpret_cast<const float2*>(p.resid + r * p.ld_resid + c);
    *reinterpret_cast<float2*>((float*)p.C + r * p.ldc + c) = make_float2(a.x + v0, a.y + v1);
  } else {
    if (EPI == EPI_ROPE_T) {
      const int m = rope_pair_col(p, c);
      if (m >= 0) {
        const float2 cs = p.rope_tab[(long long)p.pos[r] * p.rope_half + m];
        const float a0 = v0 * cs.x - v1 * cs.y, a1 = v0 * cs.y + v1 * cs.x;
        v0 = a0;
        v1 = a1;
      }
    }
    *reinterpret_cast<__nv_bfloat162*>((bf16*)p.C + r * p.ldc + c) = __floats2bfloat162_rn(v0, v1);
  }
}

// Splits for rows that fit one tile: enough to give every SM a tile, at least 3 k-blocks
// each, within the caller's scratch.  1 = no split.
static int splitk_count(const GemmParams& p, int epi, int n_tiles) {
  if (!p.split_ws || p.tiles || p.M > tc::BM || p.vt || p.N % 2 || p.ldc % 2) return 1;
  if (epi != EPI_STORE_F32 && epi != EPI_STORE_T && epi != EPI_RESID_F32 && epi != EPI_ROPE_T) return 1;
  if (epi == EPI_RESID_F32 && p.ld_resid % 2) return 1;
  const int nk = p.K / tc::BK;
  int splits = std::min(sm_count() / std::max(n_tiles, 1), nk / 3);
  splits = std::max(1, std::min(splits, 16));
  while (splits > 1 && (long long)splits * p.M * p.N > p.split_ws_elems) --splits;
  return splits;
}

int launch_gemm_tc(int epi, const GemmParams& p, cudaStream_t s) {
  const int bn = pick_bn(p, epi);
  if (!bn) return -1;
  tc::TcArgs a;
  a.p = p;
  a.k_splits = 1;
  a.kb_split = 0;
  a.split_stride = 0;
  a.n_out_tile = (epi == EPI_SWIGLU_T) ? bn / 2 : bn;
  a.n_n = p.N / a.n_out_tile;
  {
    // decode-sized: at most TR_ROWS slot rows per weight group (expert) on average
    const long long rows_group = (p.tiles && p.ldb > 0) ? p.b_group_stride / p.ldb : 0;
    const long long groups = rows_group > 0 ? p.b_rows / rows_group : 0;
    a.tr_rows = (groups > 0 && p.M <= (long long)tc::TR_ROWS * groups && bn == 256 &&
                 (epi == EPI_SWIGLU_T || epi == EPI_GATE_T))
                    ? tc::TR_ROWS
                    : 0;
  }
  a.m_tiles = p.tiles ? 0 : (p.M + tc::BM - 1) / tc::BM;
  a.b_rows_group = p.tiles ? (int)(p.b_group_stride / p.ldb) : 0;
  // weight bytes one row tile sweeps (SwiGLU: gate and up rows): group the row tiles when
  // that slab would not stay resident in L2 between the waves of CTAs
  {
    const long long slab = (long long)((epi == EPI_SWIGLU_T) ? 2 * p.N : p.N) * p.K * 2;
    a.group_m = slab > (32ll << 20) ? 16 : 1;
  }
  // B map extent: the caller's b_rows (all groups' rows), else N rows (SwiGLU: gate then up rows)
  CUtensorMap mA, mB;
  if (!make_map(&mA, p.A, (unsigned long long)p.M, p.K, p.lda, 128)) return -1;
  unsigned long long brows = p.b_rows > 0 ? (unsigned long long)p.b_rows
                                          : (unsigned long long)((epi == EPI_SWIGLU_T) ? p.up_off + p.N : p.N);
  if (!make_map(&mB, p.B, brows, p.K, p.ldb, bn > 128 ? 128 : bn)) return -1;
  int grid;
  if (p.tiles) {
    grid = sm_count();
  } else {
    long long tiles = (long long)a.m_tiles * a.n_n;
    grid = (int)std::min<long long>(tiles, sm_count());
  }
  if (grid <= 0) return 0;
  const int splits = splitk_count(p, epi, a.m_tiles * a.n_n);
  if (splits > 1) {
    // partial sums of K ranges into the scratch with the fp32 epilogue, then the real one
    const int nk = p.K / tc::BK;
    a.kb_split = (nk + splits - 1) / splits;
    a.k_splits = (nk + a.kb_split - 1) / a.kb_split;
    a.split_stride = (long long)p.M * p.N;
    a.p.C = p.split_ws;
    a.p.ldc = p.N;
    grid = (int)std::min<long long>((long long)a.m_tiles * a.n_n * a.k_splits, sm_count());
    int rc = launch_tc_bn<EPI_STORE_F32>(bn, mA, mB, a, grid, s);
    if (rc) return rc;
    dim3 eg((unsigned)((p.N / 2 + 255) / 256), (unsigned)p.M);
    switch (epi) {
      case EPI_STORE_F32: k_splitk_epilogue<EPI_STORE_F32><<<eg, 256, 0, s>>>(p, p.split_ws, a.k_splits, a.split_stride); break;
      case EPI_STORE_T: k_splitk_epilogue<EPI_STORE_T><<<eg, 256, 0, s>>>(p, p.split_ws, a.k_splits, a.split_stride); break;
      case EPI_RESID_F32: k_splitk_epilogue<EPI_RESID_F32><<<eg, 256, 0, s>>>(p, p.split_ws, a.k_splits, a.split_stride); break;
      default: k_splitk_epilogue<EPI_ROPE_T><<<eg, 256, 0, s>>>(p, p.split_ws, a.k_splits, a.split_stride); break;
    }
    note_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  }
  int rc;
  switch (epi) {
    case EPI_STORE_F32: rc = launch_tc_bn<EPI_STORE_F32>(bn, mA, mB, a, grid, s); break;
    case EPI_STORE_T: rc = launch_tc_bn<EPI_STORE_T>(bn, mA, mB, a, grid, s); break;
    case EPI_RESID_F32: rc = launch_tc_bn<EPI_RESID_F32>(bn, mA, mB, a, grid, s); break;
    case EPI_ROPE_T: rc = launch_tc_bn<EPI_ROPE_T>(bn, mA, mB, a, grid, s); break;
    case EPI_SWIGLU_T: rc = launch_tc<EPI_SWIGLU_T, 256>(mA, mB, a, grid, s); break;
    case EPI_GATE_T: rc = launch_tc_bn<EPI_GATE_T>(bn, mA, mB, a, grid, s); break;
    case EPI_ROUTER: rc = (bn == 64) ? launch_tc<EPI_ROUTER, 64>(mA, mB, a, grid, s)
                                     : launch_tc<EPI_ROUTER, 128>(mA, mB, a, grid, s); break;
    default: return -1;
  }
  if (rc) return rc;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace rdt
