// Internal launcher declarations of librdt (host side).  Not part of the ABI.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace rdt {

struct DevStatus;

// Raise `kernel`'s dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device); thread-safe.  Returns false if the CUDA call fails.
bool ensure_smem_limit(const void* kernel, int bytes);
// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Kernel classes for event timing (ProfScope records a CUDA event pair around the
// launches in its scope on the given stream when profiling is on).
enum ProfClass {
  PC_PROLOGUE = 0, PC_QKV, PC_ATTN, PC_OPROJ, PC_FFN_NORM, PC_ROUTER_GEMM, PC_ROUTE, PC_EXPERT_UP,
  PC_EXPERT_DOWN, PC_COMBINE, PC_OTHER, PC_BLOCK, PC_HEAD, PC_TOKENS, PC_DEPTH_FILL, PC_COUNT
};
struct ProfScope {
  ProfScope(int cls, cudaStream_t s);
  ~ProfScope();
  int cls_;
  cudaStream_t s_;
  void* a_;
};

// ------------------------------------------------------------------------------------------
// GEMM: C[M, N] = A[M, K] . B[N, K]^T with A, B K-contiguous (nn.Linear layout for B).
// Grouped mode: tiles[4 * i] = {group, row0, rows, 0}; B advanced by group * b_group_stride.
// ------------------------------------------------------------------------------------------
enum Epi {
  EPI_STORE_F32 = 0,   // C fp32 = acc
  EPI_STORE_T = 1,     // C model dtype = acc
  EPI_RESID_F32 = 2,   // C fp32 = resid + acc
  EPI_ROPE_T = 3,      // C model dtype = RoPE(acc) on the described column ranges
  EPI_SWIGLU_T = 4,    // C model dtype = silu(acc(B rows c)) * acc(B rows up_off + c)
  EPI_GATE_T = 5,      // C model dtype = row_scale[row] * acc
  EPI_ROUTER = 6       // C fp32 = logits; plus softmax / biased top-k / gates / expert histogram
};

struct RopeDesc {        // columns col0 + h * head_stride + off + [0, dim), h < n_heads
  int col0, n_heads, head_stride, off, dim;
};

struct GemmParams {
  const void* A; long long lda;
  const void* B; long long ldb; long long b_group_stride;
  int M, N, K;
  const int* tiles; const int* n_tiles; int max_tiles;  // grouped mode when tiles != nullptr
  int up_off;                                            // SWIGLU: W3 row offset in a group
  void* C; long long ldc;
  const float* resid; long long ld_resid;
  const float* row_scale;
  const int* pos; const float2* rope_tab; int rope_half; int n_rope; RopeDesc rope[2];
  long long b_rows;                                      // rows of the B tensor (0: derive from N)
  int impl;                                              // -1 auto, else a GemmImpl
  // EPI_ROUTER: route the running rows (run_idx >= 0) from their logits row
  const float* bias; const int* run_idx; int topk;
  int* ids; float* gates; int* rank; int* counts;
  // EPI_ROPE_T (optional): also store the value columns [vt_col0, vt_col0 + vt_heads * vt_hd)
  // transposed: vt[((b * vt_heads + g) * vt_hd + d) * vt_ld + t] for row = b * vt_T + t
  void* vt; int vt_col0, vt_heads, vt_hd, vt_T; long long vt_ld;
  // split-K scratch for rows that fit one tile (decode): fp32 partials [splits][M][N];
  // nullptr = no split
  float* split_ws; long long split_ws_elems;
  // test only: the tensor-core producer issues no loads, so the kernel's bounded waits run
  // out and it records a timeout (nothing is ever in flight); 0 in production
  int test_no_loads;
  // EPI_RESID_F32 (optional): row r of the product is written to, and takes its residual
  // from, row row_map[r] of C / resid
  const int* row_map;
  DevStatus* st;
};

// Which implementation handles a GEMM (decided on the host from shape and dtype).
enum GemmImpl { GEMM_SIMT = 0, GEMM_TC = 1 };
int gemm_tile_m(GemmImpl impl);
GemmImpl gemm_pick(int dtype, const GemmParams& p, int epi);
int launch_gemm(int dtype, int epi, const GemmParams& p, cudaStream_t s);   // returns 0 on success

// ------------------------------------------------------------------------------------------
// attention
// ------------------------------------------------------------------------------------------
struct AttnParams {
  const void* q; long long q_row; int q_head;           // q[row, h, 0 : dn + dr]
  const void* k1; long long k1_b, k1_j, k1_g;           // per-kv-head key part, dim dn
  const void* k2; long long k2_b, k2_j;                 // head-shared key part, dim dr (MLA)
  const void* v; long long v_b, v_j, v_g;               // dim dv
  void* o; long long o_row; int o_head;
  int B, T, H, G;                                       // G = H / Hkv
  int dn, dr, dv;
  const int* q_pos;                                     // [B * T] absolute positions
  int key_pos0;                                         // absolute position of key index 0
  const int* n_keys_dev;                                // per sequence (decode) or nullptr
  int n_keys;                                           // keys per sequence (prefill)
  float scale;
  // split-KV decode scratch
  float* part_o; float* part_ml; int n_split;
  // tensor-core prefill: values transposed, vt[((b * Hkv + g) * dv + d) * vt_ld + j]
  const void* vt; long long vt_ld;
  // decode with rows at different loop depths: sequence b reads the loop cache
  // max(row_loop[b], 0), i.e. k1 / v advanced by that many loop_k / loop_v elements
  const int* row_loop; long long loop_k, loop_v;
  // compact queries (tensor-core prefill): q holds only the running rows, in row order, and
  // o receives them in the same order; sequence b's rows are q[seq_off[b] .. seq_off[b + 1])
  // and compact row r is row run_list[r] of the batch (its position q_pos[run_list[r]])
  const int* seq_off; const int* run_list;
  DevStatus* st;                                        // device status word (timeouts); may be null
};
int launch_attention(int dtype, const AttnParams& p, cudaStream_t s);
int launch_attention_decode(int dtype, const AttnParams& p, cudaStream_t s);
bool attention_tc_supports(int dtype, const AttnParams& p);   // the tensor-core prefill kernel takes p

// MLA decode on the latent cache, weight-absorbed (bf16): q absorption, split-KV latent
// attention over all heads of a sequence, range merge + value absorption into o.
struct MlaDecodeParams {
  int B, H, dn, dr, dv, kvr;
  const void* q; long long q_row; int q_head;   // [B][H][dn + dr]: q_nope, rotated q_rope
  const void* w_kvu; const float* kv_norm_w;    // [H (dn + dv)][kvr], [kvr]
  float eps, scale;
  const void* ckv; const void* krope; int t_max;  // this loop's cache: [B][t_max][kvr], [B][t_max][dr]
  const int* q_pos;                             // [B] new-token position = cache_len[b]
  void* qa;                                     // scratch [B][H][kvr]
  float* part_o; float* part_ml; int n_split;   // [B][H][n_split][kvr], [B][H][n_split][2]
  void* o; long long o_row;                     // attention output [B][H dv]
  DevStatus* st;
  int test_no_loads;                            // test only: the tensor-core attention alone, producers idle
};
bool mla_decode_supports(int attn_type, int dtype, int H, int kvr, int dr, int dn, int dv);
int mla_decode_splits(int B, int H, int kvr, int dr, int t_max);   // key ranges per sequence (part_o slots)
int launch_mla_decode(const MlaDecodeParams& p, cudaStream_t s);
int tc_sm_count();

// ------------------------------------------------------------------------------------------
// MoE routing and permutation
// ------------------------------------------------------------------------------------------
struct RouteParams {
  const float* logits; const float* bias;       // [N, E], [E]
  int N, E, k, S;
  const int* run_list; const int* n_run;
  int* ids; float* gates; int* rank; int* counts;   // [N, k], [N, k], [N, k], [E]
  int* offsets;                                  // [E + S + 1]
  int* tiles; int* n_tiles; int max_tiles; int tile_m;
  int* slot_of; int* tok_of; float* gate_of;     // [N, k + S], [M], [M]
  const void* f; void* xg; int D;                // gather source rows / destination
  int max_slots;
  DevStatus* st;
};
void launch_router_topk(const RouteParams& p, cudaStream_t s);
bool launch_router_small(const void* f, const void* wr, int M, int K, int E, float* logits, cudaStream_t s);
void launch_route_scan(const RouteParams& p, cudaStream_t s);
void launch_route_scatter(int dtype, const RouteParams& p, cudaStream_t s);

// ------------------------------------------------------------------------------------------
// row kernels
// ------------------------------------------------------------------------------------------
struct CombineParams {
  int N, D, k, S, r, t, n_loops, max_loop_iters, max_slots;
  int act_on, transformer_off, block_only;
  float thr;
  const float* x1; const void* y; const int* slot_of; const int* ids;   // y in the model dtype
  const void* lora_down; const void* lora_B; const float* lora_scale;
  const float* A; const float* inj_B; const void* e;
  const float* h; float* h_state; float* h_out;
  const float* halt_wv; const float* halt_b; const float* halt_off;
  float* cum; int* halted;
  float* halt_w_out; int* ids_out; float* p_out;
  float* out;   // block_only
  // rows at their own loop depth (continuous depth-wise batching; nullptr: every row at loop
  // t): row i runs loop t_row[i] and its outputs go to output row out_row[i] of h_out
  // [rows][D], halt_w_out [rows][n_loops] and ids_out [rows][n_loops][k]; halted rows are
  // idle slots and write nothing
  const int* t_row; const int* out_row;
  // fused prologue of loop t + 1 (warp-per-row kernel only; next_emb == nullptr: off):
  // combined = RMSNorm_rec(h_new + emb + e), a = RMSNorm_attn(combined)
  const float* next_emb; int loop_dim; const float* w_rec; const float* w_attn; float eps;
  float* combined_out; void* a_out;
  DevStatus* st;
};

// ------------------------------------------------------------------------------------------
// continuous depth-wise batching of decode steps: one slot per sequence, each slot's token at
// its own loop; finished tokens fill their remaining loops' keys / values and the slot takes
// the sequence's next token
// ------------------------------------------------------------------------------------------
struct DepthParams {
  int B, S, L, D, loop_dim, emb_stride, Hkv, hd, t_max;
  const float* h0_seq; const void* e_seq; const float* off_seq;   // [B][S][D], [B][S][D], [B][S] or null
  const int* cache_len0;                                           // [B] position of token 0
  float* h; void* e_slot; float* off_slot; int* pos;               // slot state [B][D], [B][D], [B], [B]
  int* t_row; int* tok; int* out_row; float* cum; int* halted; int* pending;
  const float* emb_tab; const float* w_rec; const float* w_attn; float eps;   // emb_tab [L][emb_stride]
  void* a_fill; int* pos_fill; const void* kv_fill;                // [B (L-1)][D], [B (L-1)], [B (L-1)][2 Hkv hd]
  int* fill_b; int* fill_u; int* fill_n;                           // fill row r = (slot fill_b[r], loop fill_u[r]), r < *fill_n
  int* fill_tiles; int* fill_ntiles; int fill_tile_m;              // GEMM row tiles of the fill rows {0, row0, rows, 0}
  void* kc; void* vc; long long loop_elems;                        // GQA loop caches, elements per loop
  DevStatus* st;
};
void launch_depth_start(int dtype, const DepthParams& p, cudaStream_t s);
void launch_depth_fill_list(const DepthParams& p, cudaStream_t s);
void launch_depth_fill_prologue(int dtype, const DepthParams& p, cudaStream_t s);
void launch_depth_fill_store(int dtype, const DepthParams& p, cudaStream_t s);
void launch_depth_refill(int dtype, const DepthParams& p, cudaStream_t s);

void launch_lti_A(const float* log_A, const float* log_dt, float* A, int D, cudaStream_t s);
void launch_loop_emb(float* emb, int loop_dim, int t, float theta, cudaStream_t s);
void launch_rope_table(float2* tab, int n_pos, int dim, float theta, cudaStream_t s);
void launch_positions(int* pos, int N, int seq, int start_pos, cudaStream_t s);
void launch_positions_decode(int* pos, const int* cache_len, int B, int t_max, DevStatus* st, cudaStream_t s);
// row_loop (optional): row r adds the loop embedding emb + max(row_loop[r], 0) * emb_stride
void launch_loop_prologue(int dtype, const float* h, const void* e, const float* emb, int loop_dim,
                          const float* w_rec, const float* w_attn, float* combined, void* a,
                          int N, int D, float eps, cudaStream_t s, const int* row_loop = nullptr,
                          int emb_stride = 0);
bool launch_rmsnorm_rows(int dtype, const float* x, const float* w, void* out, int N, int D, float eps,
                         const int* run_list, const int* n_run, cudaStream_t s);   // running rows only
void launch_rmsnorm(int in_f32, int dtype, const void* x, long long in_ld, const float* w, void* out,
                    long long out_ld, int rows, int D, float eps, cudaStream_t s);
void launch_mla_kv_prep(int dtype, const float* kv_raw, int kvr, int dr, const float* kv_norm_w, float eps,
                        const int* pos, const float2* rope_tab, void* ckv, void* krope, int N, cudaStream_t s);
// row_loop (optional): row r writes into the loop cache row_loop[r] (loop_elems elements per
// loop), rows with row_loop[r] < 0 write nothing
void launch_kv_to_cache(int dtype, const void* qkv, long long ld, int k_col, int v_col, int Hkv, int hd,
                        const int* pos, int N, int seq, int t_max, void* kc, void* vc, DevStatus* st,
                        cudaStream_t s, const int* row_loop = nullptr, long long loop_elems = 0);
// returns true when the fused next-loop prologue ran (p.next_emb set and supported)
bool launch_combine(int dtype, const CombineParams& p, int n_rows, cudaStream_t s);
void launch_compact(const int* halted, int N, int* run_list, int* run_idx, int* n_run, int* cta_count,
                    cudaStream_t s);
void launch_greedy(const float* logits, int n, int vocab, int* tokens, int out_ld, cudaStream_t s);
void launch_to_model_dtype(const float* x, void* out, long long n, cudaStream_t s);
void launch_mla_to_cache(int dtype, const float* kv_raw, const void* krope, int kvr, int dr, const int* pos, int N,
                         int seq, int t_max, void* ckv_c, void* kr_c, DevStatus* st, cudaStream_t s);
void launch_iota(int* run_list, int* run_idx, int* n_run, int N, cudaStream_t s);
// Compact running rows: per-sequence offsets of run_list (seq_off[b] = first compact index
// of sequence b's rows, [B + 1]) and the 128-row tiles of the n_run compact rows.
void launch_compact_meta(const int* run_list, const int* n_run, int B, int T, int* seq_off, int* tiles,
                         int* n_tiles, cudaStream_t s);
// dst[r] = src[run_list[r]] for r < n_run: `bytes` per row (a multiple of 16), row strides in
// bytes; with pos_c also pos_c[r] = pos[run_list[r]]
void launch_gather_rows(const void* src, long long src_ld, void* dst, long long dst_ld, long long bytes,
                        const int* run_list, const int* n_run, int N, cudaStream_t s, const int* pos = nullptr,
                        int* pos_c = nullptr);
void launch_embed(int dtype, const void* table, int vocab, const int* ids, int n, int D, float* out,
                  DevStatus* st, cudaStream_t s);
void launch_trace_rows(int src_is_model_dtype, int dtype, const void* src, int W, int row0, int n,
                       const float* bias, float* dst, cudaStream_t s);

}  // namespace rdt
