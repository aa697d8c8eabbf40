// Row-wise kernels of the recurrent block: loop prologue (S1), norms, tables, the
// fused combine + depth-wise LoRA + LTI injection + ACT step (S9), running-row
// compaction, K/V cache writes and the MLA latent preparation.
//
// All are HBM-bound row kernels: one CTA per row, 256 threads, the row staged in
// dynamic shared memory so every input element is read once and every output
// element written once.
#include "common.cuh"
#include "kernels.h"
#include <math.h>

#include <algorithm>

namespace rdt {

// ------------------------------------------------------------------------------------------
// tables (double precision, rounded once to fp32)
// ------------------------------------------------------------------------------------------

// A = exp(-exp(clamp(log_dt + log_A, -20, 20))) ("OpenMythos 분석", latent reasoning).
__global__ void k_lti_A(const float* log_A, const float* log_dt, float* A, int D) {
  int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= D) return;
  double z = (double)log_dt[0] + (double)log_A[d];
  z = fmin(fmax(z, -20.0), 20.0);
  A[d] = (float)exp(-exp(z));
}

// Loop-index embedding of loop t: emb[j] = sin(t w_j), emb[half + j] = cos(t w_j),
// w_j = theta^(-2j / loop_dim) ("OpenMythos 분석", Repeating the parameter ...).
__global__ void k_loop_emb(float* emb, int loop_dim, int t, float theta) {
  int half = loop_dim / 2;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    double w = pow((double)theta, -2.0 * j / loop_dim);
    double ang = (double)t * w;
    emb[j] = (float)sin(ang);
    emb[half + j] = (float)cos(ang);
  }
}

// RoPE phasors: tab[p * half + m] = (cos, sin)(p * theta^(-2m / dim)).
__global__ void k_rope_table(float2* tab, int n_pos, int dim, float theta) {
  int half = dim / 2;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)n_pos * half) return;
  int p = (int)(idx / half), m = (int)(idx % half);
  double ang = (double)p * pow((double)theta, -2.0 * m / dim);
  tab[idx] = make_float2((float)cos(ang), (float)sin(ang));
}

// pos[row] = start_pos + row % seq
__global__ void k_positions(int* pos, int N, int seq, int start_pos) {
  int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < N) pos[r] = start_pos + r % seq;
}

// decode: the new token of sequence b sits at cache_len[b]; out-of-range lengths are
// recorded in the status word and clamped so no table or cache access leaves its buffer.
__global__ void k_positions_decode(int* pos, const int* cache_len, int B, int t_max, DevStatus* st) {
  int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= B) return;
  int p = cache_len[r];
  if (p < 0 || p >= t_max) {
    record_status(st, ST_BOUNDS, 102, p);
    p = p < 0 ? 0 : t_max - 1;
  }
  pos[r] = p;
}

// ------------------------------------------------------------------------------------------
// S1: combined = RMSNorm_rec(h + emb_t + e); a = RMSNorm_attn(combined)
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void k_loop_prologue(const float* __restrict__ h, const T* __restrict__ e,
                                const float* __restrict__ emb, int loop_dim,
                                const float* __restrict__ w_rec, const float* __restrict__ w_attn,
                                float* __restrict__ combined, T* __restrict__ a, int D, float eps,
                                const int* __restrict__ row_loop, int emb_stride) {
  extern __shared__ float xs[];
  __shared__ float red[32];
  const long long row = blockIdx.x;
  if (row_loop) emb += (long long)max(row_loop[row], 0) * emb_stride;   // this row's loop embedding
  const float* hr = h + row * D;
  const T* er = e + row * D;
  float ss = 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float x = hr[d] + to_f(er[d]);
    if (d < loop_dim) x += emb[d];
    xs[d] = x;
    ss += x * x;
  }
  ss = block_sum(ss, red);
  float inv = rsqrtf(ss / D + eps);
  float ss2 = 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float c = xs[d] * inv * w_rec[d];
    xs[d] = c;
    combined[row * D + d] = c;
    ss2 += c * c;
  }
  ss2 = block_sum(ss2, red);
  float inv2 = rsqrtf(ss2 / D + eps);
  for (int d = threadIdx.x; d < D; d += blockDim.x) a[row * D + d] = from_f<T>(xs[d] * inv2 * w_attn[d]);
}

// out = RMSNorm(x) * w over rows of width D (fp32 in, model dtype out).
// in_ld / out_ld are the row strides (elements); x may be a column slice.
template <typename TI, typename TO>
__global__ void k_rmsnorm(const TI* __restrict__ x, long long in_ld, const float* __restrict__ w,
                          TO* __restrict__ out, long long out_ld, int D, float eps) {
  extern __shared__ float xs[];
  __shared__ float red[32];
  const long long row = blockIdx.x;
  float ss = 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float v = to_f(x[row * in_ld + d]);
    xs[d] = v;
    ss += v * v;
  }
  ss = block_sum(ss, red);
  float inv = rsqrtf(ss / D + eps);
  for (int d = threadIdx.x; d < D; d += blockDim.x) out[row * out_ld + d] = from_f<TO>(xs[d] * inv * w[d]);
}

// ------------------------------------------------------------------------------------------
// MLA latent preparation: ckv = RMSNorm_kv(kv_raw[:, :kvr]) (model dtype);
// krope = RoPE(kv_raw[:, kvr:]) (model dtype).
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void k_mla_kv_prep(const float* __restrict__ kv_raw, int kvr, int dr,
                              const float* __restrict__ kv_norm_w, float eps,
                              const int* __restrict__ pos, const float2* __restrict__ rope_tab,
                              T* __restrict__ ckv, T* __restrict__ krope) {
  __shared__ float red[32];
  const long long row = blockIdx.x;
  const float* x = kv_raw + row * (kvr + dr);
  float ss = 0.f;
  for (int d = threadIdx.x; d < kvr; d += blockDim.x) ss += x[d] * x[d];
  ss = block_sum(ss, red);
  float inv = rsqrtf(ss / kvr + eps);
  for (int d = threadIdx.x; d < kvr; d += blockDim.x) ckv[row * kvr + d] = from_f<T>(x[d] * inv * kv_norm_w[d]);
  const int p = pos[row];
  for (int m = threadIdx.x; m < dr / 2; m += blockDim.x) {
    float2 cs = rope_tab[(long long)p * (dr / 2) + m];
    float x0 = x[kvr + 2 * m], x1 = x[kvr + 2 * m + 1];
    krope[row * dr + 2 * m] = from_f<T>(x0 * cs.x - x1 * cs.y);
    krope[row * dr + 2 * m + 1] = from_f<T>(x0 * cs.y + x1 * cs.x);
  }
}

// ------------------------------------------------------------------------------------------
// MLA latent cache of one loop: c_kv [B][t_max][kvr] (raw, before its RMSNorm) and the
// rotated k_rope [B][t_max][dr] shared by all heads ("OpenMythos 분석", MLA: the cache
// holds c_kv and k_rope), written at position pos[row].
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void k_mla_to_cache(const float* __restrict__ kv_raw, const T* __restrict__ krope, int kvr, int dr,
                               const int* __restrict__ pos, int seq, int t_max, T* __restrict__ ckv_c,
                               T* __restrict__ kr_c, DevStatus* st) {
  const long long row = blockIdx.x;
  const int b = (int)(row / seq);
  const int p = pos[row];
  if (p < 0 || p >= t_max) {
    if (threadIdx.x == 0) record_status(st, ST_BOUNDS, 103, p);
    return;
  }
  const long long dst = (long long)b * t_max + p;
  for (int d = threadIdx.x; d < kvr; d += blockDim.x) ckv_c[dst * kvr + d] = from_f<T>(kv_raw[row * (kvr + dr) + d]);
  for (int d = threadIdx.x; d < dr; d += blockDim.x) kr_c[dst * dr + d] = krope[row * dr + d];
}

// ------------------------------------------------------------------------------------------
// GQA K/V rows -> per-loop cache [B][Hkv][t_max][hd] at position pos[row].
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void k_kv_to_cache(const T* __restrict__ qkv, long long ld, int k_col, int v_col,
                              int Hkv, int hd, const int* __restrict__ pos, int seq, int t_max,
                              T* __restrict__ kc, T* __restrict__ vc, const int* __restrict__ row_loop,
                              long long loop_elems, DevStatus* st) {
  const long long row = blockIdx.x;
  const int b = (int)(row / seq);
  const int p = pos[row];
  if (row_loop) {                       // rows at their own loop depth; < 0: an idle row
    const int lp = row_loop[row];
    if (lp < 0) return;
    kc += lp * loop_elems;
    vc += lp * loop_elems;
  }
  if (p < 0 || p >= t_max) {
    if (threadIdx.x == 0) record_status(st, ST_BOUNDS, 101, p);
    return;
  }
  for (int i = threadIdx.x; i < Hkv * hd; i += blockDim.x) {
    int g = i / hd, d = i % hd;
    long long dst = (((long long)b * Hkv + g) * t_max + p) * hd + d;
    kc[dst] = qkv[row * ld + k_col + i];
    vc[dst] = qkv[row * ld + v_col + i];
  }
}

// ------------------------------------------------------------------------------------------
// S9: combine + depth-wise LoRA + LTI injection + freeze + ACT, one CTA per row.
//   trans = x1 + sum_j y[slot_of[i][j]]                (routed, gate already applied; shared)
//   trans += ((trans Wd^T) * scale[min(t, mli-1)]) B_lora
//   h_new = A h + B_inj e + trans;  rows halted before loop t keep h (frozen)
//   ACT: p = sigmoid(h_new . w_halt + b_halt + off); w = remainder if cum + p >= thr or
//   last loop, else p; cum += p; h_out += w h_new.   ACT off: w = [t == L-1].
// block_only: out = trans (one plain block, no LoRA / injection / ACT).
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void k_combine_inject_act(CombineParams p) {
  extern __shared__ float sm[];
  float* tr = sm;                 // [D] trans, then h_new
  float* zq = sm + p.D;           // [r] LoRA projections
  __shared__ float red[32];
  const int i = blockIdx.x;
  const int D = p.D;
  const int kS = p.k + p.S;
  // this row's loop and output row (rows at their own depth), else loop p.t and row i
  const int t = p.t_row ? p.t_row[i] : p.t;
  const long long wo = p.t_row ? (long long)p.out_row[i] * p.n_loops + t : (long long)t * p.N + i;
  const long long orow = p.t_row ? (long long)p.out_row[i] : (long long)i;
  if (!p.block_only && p.halted[i]) {   // frozen row
    if (p.t_row) return;                // an idle slot: nothing to write
    if (threadIdx.x == 0) p.halt_w_out[wo] = 0.f;
    for (int j = threadIdx.x; j < p.k; j += blockDim.x) p.ids_out[wo * p.k + j] = -1;
    return;
  }
  const float* x1 = p.x1 + (long long)i * D;
  if (p.transformer_off) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) tr[d] = 0.f;
  } else {
    for (int d = threadIdx.x; d < D; d += blockDim.x) tr[d] = x1[d];
    for (int j = 0; j < kS; ++j) {
      int slot = p.slot_of[(long long)i * kS + j];
      if (slot < 0 || slot >= p.max_slots) {
        if (threadIdx.x == 0) record_status(p.st, ST_BOUNDS, 201, slot);
        continue;
      }
      const T* yr = (const T*)p.y + (long long)slot * D;
      for (int d = threadIdx.x; d < D; d += blockDim.x) tr[d] += to_f(yr[d]);
    }
  }
  __syncthreads();
  if (p.block_only) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) p.out[(long long)i * D + d] = tr[d];
    return;
  }
  if (!p.transformer_off && p.r > 0) {
    const T* Wd = (const T*)p.lora_down;
    const T* Bl = (const T*)p.lora_B;
    const float* sc = p.lora_scale + (long long)min(t, p.max_loop_iters - 1) * p.r;
    for (int q = 0; q < p.r; ++q) {
      float part = 0.f;
      for (int d = threadIdx.x; d < D; d += blockDim.x) part += tr[d] * to_f(Wd[(long long)q * D + d]);
      part = block_sum(part, red);
      if (threadIdx.x == 0) zq[q] = part * sc[q];
    }
    __syncthreads();
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      float acc = 0.f;
      for (int q = 0; q < p.r; ++q) acc += zq[q] * to_f(Bl[(long long)q * D + d]);
      tr[d] += acc;
    }
  }
  const float* hr = p.h + (long long)i * D;
  const T* er = (const T*)p.e + (long long)i * D;
  float zh = 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float hn = p.A[d] * hr[d] + p.inj_B[d] * to_f(er[d]) + tr[d];
    tr[d] = hn;
    if (p.act_on) zh += hn * p.halt_wv[d];
  }
  float w;
  const bool last = (t == p.n_loops - 1);
  if (p.act_on) {
    zh = block_sum(zh, red);
    float z = zh + p.halt_b[0] + (p.halt_off ? p.halt_off[i] : 0.f);
    float prob = 1.f / (1.f + expf(-z));
    float cum = p.cum[i];
    bool stop = (cum + prob >= p.thr) || last;
    w = stop ? fmaxf(1.f - cum, 0.f) : prob;
    __syncthreads();
    if (threadIdx.x == 0) {
      p.cum[i] = cum + prob;
      if (stop) p.halted[i] = 1;
      if (p.p_out) p.p_out[i] = prob;
    }
  } else {
    w = last ? 1.f : 0.f;
  }
  float* ho = p.h_out + orow * D;
  float* hw = p.h_state + (long long)i * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float hn = tr[d];
    ho[d] += w * hn;
    hw[d] = hn;
  }
  if (threadIdx.x == 0) p.halt_w_out[wo] = w;
  for (int j = threadIdx.x; j < p.k; j += blockDim.x)
    p.ids_out[wo * p.k + j] = p.transformer_off ? -1 : p.ids[(long long)i * p.k + j];
}

// ------------------------------------------------------------------------------------------
// running-row compaction (single CTA, ordered): run_list = rows with halted == 0.
// ------------------------------------------------------------------------------------------
__global__ void k_compact(const int* __restrict__ halted, int N, int* __restrict__ run_list,
                          int* __restrict__ run_idx, int* __restrict__ n_run) {
  __shared__ int warp_tot[32];
  __shared__ int base;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int c0 = 0; c0 < N; c0 += blockDim.x) {
    int i = c0 + threadIdx.x;
    int run = (i < N && !halted[i]) ? 1 : 0;
    unsigned m = __ballot_sync(0xffffffffu, run);
    int pre = __popc(m & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[wid] = __popc(m);
    __syncthreads();
    int off = 0;
    for (int w2 = 0; w2 < wid; ++w2) off += warp_tot[w2];
    int total = 0;
    for (int w2 = 0; w2 < nw; ++w2) total += warp_tot[w2];
    if (i < N) {
      int idx = base + off + pre;
      run_idx[i] = run ? idx : -1;
      if (run) run_list[idx] = i;
    }
    __syncthreads();
    if (threadIdx.x == 0) base += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_run = base;
}

__global__ void k_iota(int* run_list, int* run_idx, int* n_run, int N) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < N) { run_list[i] = i; run_idx[i] = i; }
  if (i == 0) *n_run = N;
}

// embedding gather: out[i] = table[ids[i]] (fp32)
template <typename T>
__global__ void k_embed(const T* __restrict__ table, int vocab, const int* __restrict__ ids, int D,
                        float* __restrict__ out, DevStatus* st) {
  const long long i = blockIdx.x;
  int id = ids[i];
  if (id < 0 || id >= vocab) {
    if (threadIdx.x == 0) record_status(st, ST_BOUNDS, 301, id);
    id = 0;
  }
  for (int d = threadIdx.x; d < D; d += blockDim.x) out[i * D + d] = to_f(table[(long long)id * D + d]);
}

// trace: copy rows [row0, row0 + n) of a [*, W] fp32 or model-dtype matrix (+ optional
// per-column bias) into a fp32 destination.
template <typename T>
__global__ void k_trace_rows(const T* __restrict__ src, int W, int row0, const float* __restrict__ bias,
                             float* __restrict__ dst) {
  const long long r = blockIdx.x;
  for (int c = threadIdx.x; c < W; c += blockDim.x)
    dst[r * W + c] = to_f(src[(row0 + r) * (long long)W + c]) + (bias ? bias[c] : 0.f);
}

// ------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------
static inline int nthreads_for(int D) { return D >= 2048 ? 256 : 128; }

void launch_lti_A(const float* log_A, const float* log_dt, float* A, int D, cudaStream_t s) {
  { k_lti_A<<<(D + 255) / 256, 256, 0, s>>>(log_A, log_dt, A, D); note_launch(); }
}
void launch_loop_emb(float* emb, int loop_dim, int t, float theta, cudaStream_t s) {
  if (loop_dim >= 2) { k_loop_emb<<<1, 128, 0, s>>>(emb, loop_dim, t, theta); note_launch(); }
}
void launch_rope_table(float2* tab, int n_pos, int dim, float theta, cudaStream_t s) {
  long long n = (long long)n_pos * (dim / 2);
  if (n > 0) { k_rope_table<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(tab, n_pos, dim, theta); note_launch(); }
}
void launch_positions(int* pos, int N, int seq, int start_pos, cudaStream_t s) {
  { k_positions<<<(N + 255) / 256, 256, 0, s>>>(pos, N, seq, start_pos); note_launch(); }
}
void launch_positions_decode(int* pos, const int* cache_len, int B, int t_max, DevStatus* st, cudaStream_t s) {
  { k_positions_decode<<<(B + 255) / 256, 256, 0, s>>>(pos, cache_len, B, t_max, st); note_launch(); }
}
void launch_loop_prologue(int dtype, const float* h, const void* e, const float* emb, int loop_dim,
                          const float* w_rec, const float* w_attn, float* combined, void* a,
                          int N, int D, float eps, cudaStream_t s, const int* row_loop, int emb_stride) {
  size_t smem = (size_t)D * sizeof(float);
  if (dtype == 0)
    { k_loop_prologue<float><<<N, nthreads_for(D), smem, s>>>(h, (const float*)e, emb, loop_dim, w_rec, w_attn,
                                                           combined, (float*)a, D, eps, row_loop, emb_stride); note_launch(); }
  else
    { k_loop_prologue<bf16><<<N, nthreads_for(D), smem, s>>>(h, (const bf16*)e, emb, loop_dim, w_rec, w_attn,
                                                          combined, (bf16*)a, D, eps, row_loop, emb_stride); note_launch(); }
}
bool launch_rmsnorm_warp(int dtype, const float* x, const float* w, void* out, int N, int D, float eps,
                         cudaStream_t s, const int* rows = nullptr, const int* n_rows = nullptr);

// RMSNorm of the running rows only (row list run_list[0 .. *n_run)), fp32 input rows of
// width D; false when the shape needs the all-rows kernel
bool launch_rmsnorm_rows(int dtype, const float* x, const float* w, void* out, int N, int D, float eps,
                         const int* run_list, const int* n_run, cudaStream_t s) {
  return launch_rmsnorm_warp(dtype, x, w, out, N, D, eps, s, run_list, n_run);
}

void launch_rmsnorm(int in_f32, int dtype, const void* x, long long in_ld, const float* w, void* out,
                    long long out_ld, int rows, int D, float eps, cudaStream_t s) {
  if (in_f32 && in_ld == D && out_ld == D && launch_rmsnorm_warp(dtype, (const float*)x, w, out, rows, D, eps, s))
    return;
  size_t smem = (size_t)D * sizeof(float);
  int nt = nthreads_for(D);
  if (in_f32) {
    if (dtype == 0) { k_rmsnorm<float, float><<<rows, nt, smem, s>>>((const float*)x, in_ld, w, (float*)out, out_ld, D, eps); note_launch(); }
    else { k_rmsnorm<float, bf16><<<rows, nt, smem, s>>>((const float*)x, in_ld, w, (bf16*)out, out_ld, D, eps); note_launch(); }
  } else {
    if (dtype == 0) { k_rmsnorm<float, float><<<rows, nt, smem, s>>>((const float*)x, in_ld, w, (float*)out, out_ld, D, eps); note_launch(); }
    else { k_rmsnorm<bf16, bf16><<<rows, nt, smem, s>>>((const bf16*)x, in_ld, w, (bf16*)out, out_ld, D, eps); note_launch(); }
  }
}
void launch_mla_kv_prep(int dtype, const float* kv_raw, int kvr, int dr, const float* kv_norm_w, float eps,
                        const int* pos, const float2* rope_tab, void* ckv, void* krope, int N, cudaStream_t s) {
  if (dtype == 0)
    { k_mla_kv_prep<float><<<N, 64, 0, s>>>(kv_raw, kvr, dr, kv_norm_w, eps, pos, rope_tab, (float*)ckv, (float*)krope); note_launch(); }
  else
    { k_mla_kv_prep<bf16><<<N, 64, 0, s>>>(kv_raw, kvr, dr, kv_norm_w, eps, pos, rope_tab, (bf16*)ckv, (bf16*)krope); note_launch(); }
}
void launch_kv_to_cache(int dtype, const void* qkv, long long ld, int k_col, int v_col, int Hkv, int hd,
                        const int* pos, int N, int seq, int t_max, void* kc, void* vc, DevStatus* st,
                        cudaStream_t s, const int* row_loop, long long loop_elems) {
  if (dtype == 0)
    { k_kv_to_cache<float><<<N, 128, 0, s>>>((const float*)qkv, ld, k_col, v_col, Hkv, hd, pos, seq, t_max,
                                           (float*)kc, (float*)vc, row_loop, loop_elems, st); note_launch(); }
  else
    { k_kv_to_cache<bf16><<<N, 128, 0, s>>>((const bf16*)qkv, ld, k_col, v_col, Hkv, hd, pos, seq, t_max,
                                          (bf16*)kc, (bf16*)vc, row_loop, loop_elems, st); note_launch(); }
}
bool launch_combine_warp(int dtype, const CombineParams& p, int n_rows, cudaStream_t s);

void launch_mla_to_cache(int dtype, const float* kv_raw, const void* krope, int kvr, int dr, const int* pos, int N,
                         int seq, int t_max, void* ckv_c, void* kr_c, DevStatus* st, cudaStream_t s) {
  if (dtype == 0) { k_mla_to_cache<float><<<N, 64, 0, s>>>(kv_raw, (const float*)krope, kvr, dr, pos, seq, t_max, (float*)ckv_c, (float*)kr_c, st); note_launch(); }
  else { k_mla_to_cache<bf16><<<N, 64, 0, s>>>(kv_raw, (const bf16*)krope, kvr, dr, pos, seq, t_max, (bf16*)ckv_c, (bf16*)kr_c, st); note_launch(); }
}

bool launch_combine(int dtype, const CombineParams& p, int n_rows, cudaStream_t s) {
  if (launch_combine_warp(dtype, p, n_rows, s)) return p.next_emb != nullptr;
  size_t smem = (size_t)(p.D + 64) * sizeof(float);
  int nt = nthreads_for(p.D);
  if (dtype == 0) { k_combine_inject_act<float><<<n_rows, nt, smem, s>>>(p); note_launch(); }
  else { k_combine_inject_act<bf16><<<n_rows, nt, smem, s>>>(p); note_launch(); }
  return false;
}
// Running-row list in two passes over CTAs of 1024 rows: each CTA counts its running rows,
// then each CTA adds the counts of the CTAs before it (in order: the list is the same as a
// sequential scan) and scatters its rows.  No CTA waits for another.
__global__ void __launch_bounds__(1024) k_compact_count(const int* __restrict__ halted, int N, int* __restrict__ cta_count) {
  __shared__ int warp_tot[32];
  const int i = blockIdx.x * 1024 + threadIdx.x, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, i < N && !halted[i]);
  if (lane == 0) warp_tot[wid] = __popc(m);
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < 32; ++w) tot += warp_tot[w];
    cta_count[blockIdx.x] = tot;
  }
}
__global__ void __launch_bounds__(1024) k_compact_scatter(const int* __restrict__ halted, int N,
                                                          const int* __restrict__ cta_count, int* __restrict__ run_list,
                                                          int* __restrict__ run_idx, int* __restrict__ n_run) {
  __shared__ int warp_tot[32];
  __shared__ int base;
  const int i = blockIdx.x * 1024 + threadIdx.x, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x < 32) {
    int b = 0;
    for (int c = threadIdx.x; c < (int)blockIdx.x; c += 32) b += cta_count[c];
    b = warp_sum_int(b);
    if (threadIdx.x == 0) base = b;
  }
  const bool run = i < N && !halted[i];
  const unsigned m = __ballot_sync(0xffffffffu, run);
  if (lane == 0) warp_tot[wid] = __popc(m);
  __syncthreads();
  int off = base;
  for (int w = 0; w < wid; ++w) off += warp_tot[w];
  if (i < N) {
    const int idx = off + __popc(m & ((1u << lane) - 1u));
    run_idx[i] = run ? idx : -1;
    if (run) run_list[idx] = i;
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 1023) {
    int tot = off;
    for (int w = wid; w < 32; ++w) tot += warp_tot[w];
    *n_run = tot;
  }
}

void launch_compact(const int* halted, int N, int* run_list, int* run_idx, int* n_run, int* cta_count,
                    cudaStream_t s) {
  const int ctas = (N + 1023) / 1024;
  if (ctas <= 0) return;
  if (!cta_count || ctas > 4096) { k_compact<<<1, 1024, 0, s>>>(halted, N, run_list, run_idx, n_run); note_launch(); return; }
  if (ctas == 1) {   // one CTA of ceil(N / 32) warps does it in a single launch
    k_compact<<<1, (N + 31) / 32 * 32, 0, s>>>(halted, N, run_list, run_idx, n_run);
    note_launch();
    return;
  }
  k_compact_count<<<ctas, 1024, 0, s>>>(halted, N, cta_count);
  note_launch();
  k_compact_scatter<<<ctas, 1024, 0, s>>>(halted, N, cta_count, run_list, run_idx, n_run);
  note_launch();
}
// seq_off[b] = number of running rows before sequence b (run_list is in row order, so a
// lower bound of b T), and the 128-row tiles of the compact rows.
__global__ void k_compact_meta(const int* __restrict__ run_list, const int* __restrict__ n_run_p, int B, int T,
                               int* __restrict__ seq_off, int* __restrict__ tiles, int* __restrict__ n_tiles) {
  const int n_run = *n_run_p;
  for (int b = threadIdx.x; b <= B; b += blockDim.x) {
    const long long key = (long long)b * T;
    int lo = 0, hi = n_run;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if ((long long)run_list[mid] < key) lo = mid + 1;
      else hi = mid;
    }
    seq_off[b] = lo;
  }
  const int nt = (n_run + 127) / 128;
  if (threadIdx.x == 0) *n_tiles = nt;
  for (int i = threadIdx.x; i < nt; i += blockDim.x) {
    tiles[4 * i] = 0;
    tiles[4 * i + 1] = 128 * i;
    tiles[4 * i + 2] = min(128, n_run - 128 * i);
    tiles[4 * i + 3] = 0;
  }
}
void launch_compact_meta(const int* run_list, const int* n_run, int B, int T, int* seq_off, int* tiles,
                         int* n_tiles, cudaStream_t s) {
  k_compact_meta<<<1, 1024, 0, s>>>(run_list, n_run, B, T, seq_off, tiles, n_tiles);
  note_launch();
}

// dst[r] = src[run_list[r]] for the compact rows r < n_run: a warp per row (rows strided over
// the grid's warps), 16-byte vectors, four loads in flight per lane; with pos_c, also the
// compact rows' positions pos_c[r] = pos[run_list[r]]
__global__ void __launch_bounds__(256) k_gather_rows(const uint8_t* __restrict__ src, long long src_ld,
                                                     uint8_t* __restrict__ dst, long long dst_ld, int nv,
                                                     const int* __restrict__ run_list, const int* __restrict__ n_run,
                                                     const int* __restrict__ pos, int* __restrict__ pos_c) {
  const int lane = threadIdx.x & 31;
  const int n = *n_run;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps) {
    const int i = run_list[r];
    if (pos_c && lane == 0) pos_c[r] = pos[i];
    const int4* s4 = reinterpret_cast<const int4*>(src + (long long)i * src_ld);
    int4* d4 = reinterpret_cast<int4*>(dst + (long long)r * dst_ld);
    for (int v0 = lane; v0 < nv; v0 += 128) {
      int4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (v0 + 32 * u < nv) v[u] = __ldg(s4 + v0 + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (v0 + 32 * u < nv) d4[v0 + 32 * u] = v[u];
    }
  }
}
void launch_gather_rows(const void* src, long long src_ld, void* dst, long long dst_ld, long long bytes,
                        const int* run_list, const int* n_run, int N, cudaStream_t s, const int* pos, int* pos_c) {
  if (N <= 0) return;
  const int grid = (int)std::min<long long>((N + 7) / 8, 8LL * device_sm_count());
  k_gather_rows<<<std::max(grid, 1), 256, 0, s>>>((const uint8_t*)src, src_ld, (uint8_t*)dst, dst_ld,
                                                  (int)(bytes / 16), run_list, n_run, pos, pos_c);
  note_launch();
}

void launch_iota(int* run_list, int* run_idx, int* n_run, int N, cudaStream_t s) {
  { k_iota<<<(N + 255) / 256, 256, 0, s>>>(run_list, run_idx, n_run, N); note_launch(); }
}
// Greedy choice of the next token: CTA per row, argmax over the vocabulary with ties to
// the lowest index; NaN compares below every number (a row of NaN gives 0).
constexpr int GREEDY_THREADS = 512;
__global__ void __launch_bounds__(GREEDY_THREADS) k_greedy(const float* __restrict__ logits, int vocab,
                                                          int* __restrict__ tokens, int out_ld) {
  __shared__ float bv_s[GREEDY_THREADS / 32];
  __shared__ int bi_s[GREEDY_THREADS / 32];
  const float* row = logits + (long long)blockIdx.x * vocab;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  auto take = [&](float x, int v) {
    if (x == x && (x > bv || (x == bv && v < bi))) { bv = x; bi = v; }
  };
  int v0 = 0;
  if ((vocab & 3) == 0 && ((uintptr_t)row & 15) == 0) {   // 16-byte vectors, four in flight per thread
    const float4* r4 = reinterpret_cast<const float4*>(row);
    const int n4 = vocab >> 2;
    for (int q = threadIdx.x; q < n4; q += 4 * GREEDY_THREADS) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) f[u] = q + u * GREEDY_THREADS < n4 ? __ldg(r4 + q + u * GREEDY_THREADS)
                                                                   : make_float4(NAN, NAN, NAN, NAN);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = 4 * (q + u * GREEDY_THREADS);
        take(f[u].x, v); take(f[u].y, v + 1); take(f[u].z, v + 2); take(f[u].w, v + 3);
      }
    }
    v0 = vocab;
  }
  for (int v = v0 + threadIdx.x; v < vocab; v += GREEDY_THREADS) take(row[v], v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { bv_s[w] = bv; bi_s[w] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < GREEDY_THREADS / 32; ++k)
      if (bv_s[k] > bv_s[0] || (bv_s[k] == bv_s[0] && bi_s[k] < bi_s[0])) { bv_s[0] = bv_s[k]; bi_s[0] = bi_s[k]; }
    tokens[(long long)blockIdx.x * out_ld] = bi_s[0] == 0x7fffffff ? 0 : bi_s[0];
  }
}

__global__ void k_to_model_dtype(const float* __restrict__ x, bf16* __restrict__ out, long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(x[i]);
}

void launch_greedy(const float* logits, int n, int vocab, int* tokens, int out_ld, cudaStream_t s) {
  k_greedy<<<n, GREEDY_THREADS, 0, s>>>(logits, vocab, tokens, out_ld);
  note_launch();
}
void launch_to_model_dtype(const float* x, void* out, long long n, cudaStream_t s) {
  const long long blocks = std::min<long long>((n + 255) / 256, 148LL * 16);
  k_to_model_dtype<<<(unsigned)blocks, 256, 0, s>>>(x, (bf16*)out, n);
  note_launch();
}

void launch_embed(int dtype, const void* table, int vocab, const int* ids, int n, int D, float* out,
                  DevStatus* st, cudaStream_t s) {
  if (dtype == 0) { k_embed<float><<<n, 128, 0, s>>>((const float*)table, vocab, ids, D, out, st); note_launch(); }
  else { k_embed<bf16><<<n, 128, 0, s>>>((const bf16*)table, vocab, ids, D, out, st); note_launch(); }
}
void launch_trace_rows(int src_is_model_dtype, int dtype, const void* src, int W, int row0, int n,
                       const float* bias, float* dst, cudaStream_t s) {
  if (n <= 0) return;
  if (!src_is_model_dtype || dtype == 0)
    { k_trace_rows<float><<<n, 128, 0, s>>>((const float*)src, W, row0, bias, dst); note_launch(); }
  else
    { k_trace_rows<bf16><<<n, 128, 0, s>>>((const bf16*)src, W, row0, bias, dst); note_launch(); }
}

}  // namespace rdt
