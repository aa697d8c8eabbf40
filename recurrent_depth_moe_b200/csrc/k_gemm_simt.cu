// CUDA-core GEMM with the recurrent block's epilogues.  Used for the fp32 mode
// (the 1e-4 parity mode: no TF32, plain FFMA) and for shapes the tcgen05 kernel
// does not take (widths that are not multiples of its tile, e.g. the dense
// prelude/coda hidden width 4*dim/3).
//   C[M, N] = A[M, K] . B[N, K]^T, 64 x 64 output tile per CTA, 16-deep K slices
//   staged through shared memory, 4 x 4 outputs per thread.
#include "common.cuh"
#include "kernels.h"

namespace rdt {

namespace {
constexpr int BM = 64, BN = 64, BK = 16;

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// Is column c the first of a rotated pair?  Returns the pair index m (>= 0) or -1.
__device__ __forceinline__ int rope_pair(const GemmParams& p, int c) {
  for (int q = 0; q < p.n_rope; ++q) {
    const RopeDesc& r = p.rope[q];
    int rel = c - r.col0;
    if (rel < 0 || rel >= r.n_heads * r.head_stride) continue;
    int o = rel % r.head_stride - r.off;
    if (o >= 0 && o < r.dim) return o >> 1;
  }
  return -1;
}
}  // namespace

template <typename TA, typename TC, int EPI>
__global__ void __launch_bounds__(256) k_gemm_simt(GemmParams p) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Bu[EPI == EPI_SWIGLU_T ? BK : 1][BN + 4];
  int group = 0, row0, rows;
  if (p.tiles) {
    if ((int)blockIdx.x >= *p.n_tiles) return;
    group = p.tiles[4 * blockIdx.x];
    row0 = p.tiles[4 * blockIdx.x + 1];
    rows = p.tiles[4 * blockIdx.x + 2];
  } else {
    row0 = blockIdx.x * BM;
    rows = min(BM, p.M - row0);
  }
  const int col0 = blockIdx.y * BN;
  const TA* A = (const TA*)p.A;
  const TA* B = (const TA*)p.B + (long long)group * p.b_group_stride;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4], acu[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = acu[i][j] = 0.f;

  for (int k0 = 0; k0 < p.K; k0 += BK) {
    for (int idx = threadIdx.x; idx < BM * BK; idx += 256) {
      int r = idx / BK, kk = idx % BK;
      int k = k0 + kk;
      As[kk][r] = (r < rows && k < p.K) ? to_f(A[(long long)(row0 + r) * p.lda + k]) : 0.f;
      int c = col0 + r;
      Bs[kk][r] = (c < p.N && k < p.K) ? to_f(B[(long long)c * p.ldb + k]) : 0.f;
      if (EPI == EPI_SWIGLU_T)
        Bu[kk][r] = (c < p.N && k < p.K) ? to_f(B[(long long)(p.up_off + c) * p.ldb + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4], u[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b[j] = Bs[kk][tx * 4 + j];
        if (EPI == EPI_SWIGLU_T) u[j] = Bu[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (EPI == EPI_SWIGLU_T) acu[i][j] = fmaf(a[i], u[j], acu[i][j]);
        }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int rl = ty * 4 + i;
    if (rl >= rows) continue;
    long long r = row0 + rl;
    if (EPI == EPI_ROPE_T) {
      int pos = p.pos[r];
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        int c = col0 + tx * 4 + j;
        if (c >= p.N) continue;
        float v0 = acc[i][j], v1 = acc[i][j + 1];
        int m = rope_pair(p, c);
        if (m >= 0) {
          float2 cs = p.rope_tab[(long long)pos * p.rope_half + m];
          float r0 = v0 * cs.x - v1 * cs.y, r1 = v0 * cs.y + v1 * cs.x;
          v0 = r0; v1 = r1;
        }
        ((TC*)p.C)[r * p.ldc + c] = from_f<TC>(v0);
        if (c + 1 < p.N) ((TC*)p.C)[r * p.ldc + c + 1] = from_f<TC>(v1);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int c = col0 + tx * 4 + j;
        if (c >= p.N) continue;
        float v = acc[i][j];
        if (EPI == EPI_STORE_F32 || EPI == EPI_STORE_T) {
          ((TC*)p.C)[r * p.ldc + c] = from_f<TC>(v);
        } else if (EPI == EPI_RESID_F32) {
          ((float*)p.C)[r * p.ldc + c] = p.resid[r * p.ld_resid + c] + v;
        } else if (EPI == EPI_SWIGLU_T) {
          ((TC*)p.C)[r * p.ldc + c] = from_f<TC>(silu_f(v) * acu[i][j]);
        } else if (EPI == EPI_GATE_T) {
          ((TC*)p.C)[r * p.ldc + c] = from_f<TC>(p.row_scale[r] * v);
        }
      }
    }
  }
}

int launch_gemm_simt(int dtype, int epi, const GemmParams& p, cudaStream_t s) {
  dim3 grid(p.tiles ? p.max_tiles : (p.M + BM - 1) / BM, (p.N + BN - 1) / BN);
  if (grid.x == 0 || grid.y == 0) return 0;
#define RDT_SIMT_CASE(TA, TO)                                                              \
  switch (epi) {                                                                           \
    case EPI_STORE_F32: { k_gemm_simt<TA, float, EPI_STORE_F32><<<grid, 256, 0, s>>>(p); note_launch(); } break; \
    case EPI_STORE_T: { k_gemm_simt<TA, TO, EPI_STORE_T><<<grid, 256, 0, s>>>(p); note_launch(); } break;        \
    case EPI_RESID_F32: { k_gemm_simt<TA, float, EPI_RESID_F32><<<grid, 256, 0, s>>>(p); note_launch(); } break; \
    case EPI_ROPE_T: { k_gemm_simt<TA, TO, EPI_ROPE_T><<<grid, 256, 0, s>>>(p); note_launch(); } break;          \
    case EPI_SWIGLU_T: { k_gemm_simt<TA, TO, EPI_SWIGLU_T><<<grid, 256, 0, s>>>(p); note_launch(); } break;      \
    case EPI_GATE_T: { k_gemm_simt<TA, TO, EPI_GATE_T><<<grid, 256, 0, s>>>(p); note_launch(); } break;   \
    default: return -1;                                                                    \
  }
  if (dtype == 0) { RDT_SIMT_CASE(float, float) } else { RDT_SIMT_CASE(bf16, bf16) }
#undef RDT_SIMT_CASE
  return 0;
}

}  // namespace rdt
