// Continuous depth-wise batching of decode steps (GeekNews summary, section 6: tokens leave
// the shared block at their own depth and new tokens take their place; "OpenMythos 분석",
// ACT: a token stops looping once its halting weights reach the threshold).
//
// One slot per sequence.  A tick runs the shared block once over all slots, each slot's
// token at its own loop t_row[slot] (per-row loop embedding, LoRA scale row, loop cache and
// last-loop flag).  After the tick, a token that halted (or ran its last loop) leaves:
//   k_depth_fill_prologue  the attention input of its remaining loops u > t_row, from its
//                          frozen state (the loop embedding changes with u, the state not),
//   fill GEMM (host side)  their keys / values (K/V rows of the QKV weight, RoPE at the
//                          token's position),
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

// Row r = b (L - 1) + (u - 1), u = 1 .. L - 1: the attention input of loop u for the token
// that just left slot b at loop t_row[b] < u, from its frozen state:
//   a = RMSNorm_attn(RMSNorm_rec(h + emb_u + e)).  Other rows are zero.
template <typename T>
__global__ void k_depth_fill_prologue(DepthParams p) {
  extern __shared__ float xs[];
  __shared__ float red[32];
  const int r = blockIdx.x;
  const int b = r / (p.L - 1), u = r % (p.L - 1) + 1;
  const long long D = p.D;
  T* a = (T*)p.a_fill + (long long)r * D;
  const bool valid = slot_finished(p, b) && u > p.t_row[b];
  if (threadIdx.x == 0) p.pos_fill[r] = valid ? p.pos[b] : 0;
  if (!valid) {
    for (long long d = threadIdx.x; d < D; d += blockDim.x) a[d] = from_f<T>(0.f);
    return;
  }
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
// columns) into loop cache u of sequence b at the token's position.
template <typename T>
__global__ void k_depth_fill_store(DepthParams p) {
  const int r = blockIdx.x;
  const int b = r / (p.L - 1), u = r % (p.L - 1) + 1;
  if (!(slot_finished(p, b) && u > p.t_row[b])) return;
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
