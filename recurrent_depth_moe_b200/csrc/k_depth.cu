// Continuous depth-wise batching of decode steps (GeekNews summary, section 6: tokens leave
// the shared block at their own depth and new tokens take their place; "OpenMythos 분석",
// ACT: a token stops looping once its halting weights reach the threshold).
//
// One slot per sequence.  A tick runs the shared block once over all slots, each slot's
// token at its own loop t_row[slot] (per-row loop embedding, LoRA scale row, loop cache and
// last-loop flag).  After the tick, a token that halted (or ran its last loop) leaves:
//   k_depth_fill_list      the (slot, loop) rows to fill this tick, compacted, and their
//                          128-row GEMM tiles,
//   k_depth_fill_prologue  the attention input of its remaining loops u > t_row, from its
//                          frozen state (the loop embedding changes with u, the state not),
//   fill GEMM (host side)  their keys / values (K/V rows of the QKV weight, RoPE at the
//                          token's position), over the device tile list of the fill rows,
//   k_depth_fill_store     those keys / values into the loop caches u at the position,
// so later tokens of its sequence find it at every loop, exactly as when the token stays
// frozen in a lockstep step; then k_depth_refill puts the sequence's next token in the
// slot at loop 0 (or marks the slot idle when the sequence is done).
#include "common.cuh"
#include "kernels.h"

namespace rdt {

// Slots take token 0 of their sequence; outputs start as "not run" (weight 0, id -1).
template <typename T>
__global__ void k_depth_start(DepthParams p) {
  const int b = blockIdx.x;
  const long long D = p.D;
  if (threadIdx.x == 0) {
    int pos = p.cache_len0[b];
    if (pos < 0 || pos + p.S > p.t_max) {
      record_status(p.st, ST_BOUNDS, 701, pos);
      pos = min(max(pos, 0), p.t_max - p.S);
    }
    p.pos[b] = pos;
    p.tok[b] = 0;
    p.t_row[b] = 0;
    p.out_row[b] = b * p.S;
    p.halted[b] = 0;
    p.cum[b] = 0.f;
    p.off_slot[b] = p.off_seq ? p.off_seq[(long long)b * p.S] : 0.f;
    if (b == 0) *p.pending = p.B * p.S;
  }
  const float* hs = p.h0_seq + (long long)b * p.S * D;
  const T* es = (const T*)p.e_seq + (long long)b * p.S * D;
  for (long long d = threadIdx.x; d < D; d += blockDim.x) {
    p.h[b * D + d] = hs[d];
    ((T*)p.e_slot)[b * D + d] = es[d];
  }
}

__device__ __forceinline__ bool slot_finished(const DepthParams& p, int b) {
  const int t = p.t_row[b];
  return t >= 0 && (p.halted[b] || t == p.L - 1);
}

// The fill rows of this tick, in slot order: for each finished slot b, its loops
// u = t_row[b] + 1 .. L - 1.  One CTA: per-thread slot ranges, a block scan of their row
// counts, then the list, its length and its GEMM row tiles (fill_tile_m rows each).
constexpr int FILL_THREADS = 256;
__global__ void __launch_bounds__(FILL_THREADS) k_depth_fill_list(DepthParams p) {
  __shared__ int sums[FILL_THREADS];
  const int t = threadIdx.x;
  const int per = (p.B + FILL_THREADS - 1) / FILL_THREADS;
  const int b0 = min(p.B, t * per), b1 = min(p.B, b0 + per);
  int n = 0;
  for (int b = b0; b < b1; ++b)
    if (slot_finished(p, b)) n += p.L - 1 - p.t_row[b];
  sums[t] = n;
  __syncthreads();
  for (int off = 1; off < FILL_THREADS; off <<= 1) {   // inclusive scan
    const int v = t >= off ? sums[t - off] : 0;
    __syncthreads();
    sums[t] += v;
    __syncthreads();
  }
  int r = sums[t] - n;
  for (int b = b0; b < b1; ++b) {
    if (!slot_finished(p, b)) continue;
    for (int u = p.t_row[b] + 1; u < p.L; ++u, ++r) {
      p.fill_b[r] = b;
      p.fill_u[r] = u;
    }
  }
  const int total = sums[FILL_THREADS - 1], tm = p.fill_tile_m;
  const int ntiles = (total + tm - 1) / tm;
  if (t == 0) {
    *p.fill_n = total;
    *p.fill_ntiles = ntiles;
  }
  for (int i = t; i < ntiles; i += FILL_THREADS) {
    p.fill_tiles[4 * i] = 0;
    p.fill_tiles[4 * i + 1] = tm * i;
    p.fill_tiles[4 * i + 2] = min(tm, total - tm * i);
    p.fill_tiles[4 * i + 3] = 0;
  }
}

// Fill row r (slot b = fill_b[r], loop u = fill_u[r] > t_row[b]): the attention input of
// loop u for the token that just left slot b, from its frozen state:
//   a = RMSNorm_attn(RMSNorm_rec(h + emb_u + e)).  CTAs past the list's length return.
template <typename T>
__global__ void k_depth_fill_prologue(DepthParams p) {
  extern __shared__ float xs[];
  __shared__ float red[32];
  const int r = blockIdx.x;
  if (r >= *p.fill_n) return;
  const int b = p.fill_b[r], u = p.fill_u[r];
  const long long D = p.D;
  T* a = (T*)p.a_fill + (long long)r * D;
  if (threadIdx.x == 0) p.pos_fill[r] = p.pos[b];
  const float* h = p.h + b * D;
  const T* e = (const T*)p.e_slot + b * D;
  const float* emb = p.emb_tab + (long long)u * p.emb_stride;
  float ss = 0.f;
  for (long long d = threadIdx.x; d < D; d += blockDim.x) {
    float x = h[d] + to_f(e[d]);
    if (d < p.loop_dim) x += emb[d];
    xs[d] = x;
    ss += x * x;
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / D + p.eps);
  float ss2 = 0.f;
  for (long long d = threadIdx.x; d < D; d += blockDim.x) {
    const float c = xs[d] * inv * p.w_rec[d];
    xs[d] = c;
    ss2 += c * c;
  }
  ss2 = block_sum(ss2, red);
  const float inv2 = rsqrtf(ss2 / D + p.eps);
  for (long long d = threadIdx.x; d < D; d += blockDim.x) a[d] = from_f<T>(xs[d] * inv2 * p.w_attn[d]);
}

// The filled keys / values (kv_fill row r: Hkv hd rotated key columns, then Hkv hd value
// columns) into loop cache u = fill_u[r] of sequence b = fill_b[r] at the token's position.
template <typename T>
__global__ void k_depth_fill_store(DepthParams p) {
  const int r = blockIdx.x;
  if (r >= *p.fill_n) return;
  const int b = p.fill_b[r], u = p.fill_u[r];
  const int pos = p.pos[b];
  if (pos < 0 || pos >= p.t_max) {
    if (threadIdx.x == 0) record_status(p.st, ST_BOUNDS, 702, pos);
    return;
  }
  const int W = p.Hkv * p.hd;
  const T* src = (const T*)p.kv_fill + (long long)r * 2 * W;
  T* kc = (T*)p.kc + (long long)u * p.loop_elems;
  T* vc = (T*)p.vc + (long long)u * p.loop_elems;
  for (int i = threadIdx.x; i < W; i += blockDim.x) {
    const int g = i / p.hd, d = i % p.hd;
    const long long dst = (((long long)b * p.Hkv + g) * p.t_max + pos) * p.hd + d;
    kc[dst] = src[i];
    vc[dst] = src[W + i];
  }
}

// After the fill: a finished token's slot takes the sequence's next token at loop 0 (or
// becomes idle: t_row = -1, halted = 1); a running token moves to its next loop.
template <typename T>
__global__ void k_depth_refill(DepthParams p) {
  const int b = blockIdx.x;
  const long long D = p.D;
  __shared__ int state;   // 0: nothing to load, 1: next token loaded
  if (threadIdx.x == 0) {
    state = 0;
    const int t = p.t_row[b];
    if (t >= 0) {
      if (!(p.halted[b] || t == p.L - 1)) {
        p.t_row[b] = t + 1;
      } else {
        atomicSub(p.pending, 1);
        const int n = p.tok[b] + 1;
        p.tok[b] = n;
        if (n < p.S) {
          p.t_row[b] = 0;
          p.halted[b] = 0;
          p.cum[b] = 0.f;
          p.out_row[b] = b * p.S + n;
          p.pos[b] = p.pos[b] + 1;            // tokens of a sequence sit at consecutive positions
          p.off_slot[b] = p.off_seq ? p.off_seq[(long long)b * p.S + n] : 0.f;
          state = 1;
        } else {
          p.t_row[b] = -1;                    // the sequence is done: an idle slot
          p.halted[b] = 1;
        }
      }
    }
  }
  __syncthreads();
  if (!state) return;
  const long long src = ((long long)b * p.S + p.tok[b]) * D;
  for (long long d = threadIdx.x; d < D; d += blockDim.x) {
    p.h[b * D + d] = p.h0_seq[src + d];
    ((T*)p.e_slot)[b * D + d] = ((const T*)p.e_seq)[src + d];
  }
}

static inline int depth_threads(int D) { return D >= 2048 ? 256 : 128; }

void launch_depth_start(int dtype, const DepthParams& p, cudaStream_t s) {
  if (dtype == 0) { k_depth_start<float><<<p.B, depth_threads(p.D), 0, s>>>(p); note_launch(); }
  else { k_depth_start<bf16><<<p.B, depth_threads(p.D), 0, s>>>(p); note_launch(); }
}
void launch_depth_fill_list(const DepthParams& p, cudaStream_t s) {
  k_depth_fill_list<<<1, FILL_THREADS, 0, s>>>(p);
  note_launch();
}
void launch_depth_fill_prologue(int dtype, const DepthParams& p, cudaStream_t s) {
  const size_t smem = (size_t)p.D * sizeof(float);
  const unsigned rows = (unsigned)(p.B * (p.L - 1));
  if (rows == 0) return;
  if (dtype == 0) { k_depth_fill_prologue<float><<<rows, depth_threads(p.D), smem, s>>>(p); note_launch(); }
  else { k_depth_fill_prologue<bf16><<<rows, depth_threads(p.D), smem, s>>>(p); note_launch(); }
}
void launch_depth_fill_store(int dtype, const DepthParams& p, cudaStream_t s) {
  const unsigned rows = (unsigned)(p.B * (p.L - 1));
  if (rows == 0) return;
  if (dtype == 0) { k_depth_fill_store<float><<<rows, 128, 0, s>>>(p); note_launch(); }
  else { k_depth_fill_store<bf16><<<rows, 128, 0, s>>>(p); note_launch(); }
}
void launch_depth_refill(int dtype, const DepthParams& p, cudaStream_t s) {
  if (dtype == 0) { k_depth_refill<float><<<p.B, depth_threads(p.D), 0, s>>>(p); note_launch(); }
  else { k_depth_refill<bf16><<<p.B, depth_threads(p.D), 0, s>>>(p); note_launch(); }
}

}  // namespace rdt
