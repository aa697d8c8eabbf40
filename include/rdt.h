/*
 * rdt.h — C ABI of librdt: the looped Recurrent Block of the OpenMythos
 * Recurrent-Depth Transformer on one B200 (sm_100a).
 *
 * Conventions (all entry points):
 *  - Every pointer argument named as "device" is a device pointer owned by the
 *    caller.  The library allocates nothing on these paths; scratch memory is the
 *    caller's workspace `ws` of at least rdt_workspace_size() bytes, 256-byte aligned.
 *  - Matrices are row-major.  Weight matrices use the nn.Linear layout
 *    [out_features, in_features] and are stored in the model dtype
 *    (cfg->dtype: 0 = fp32, 1 = bf16).  Vectors marked "fp32" are always fp32.
 *  - Activations are sequence-major rows: row = b * seq + i for sequence b,
 *    position i.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All calls only
 *    enqueue work on it and return, except rdt_read_device_status (synchronises).
 *  - Arguments are validated on the host before anything is launched; a bad
 *    argument returns RDT_ERR_INVALID_ARG (or RDT_ERR_UNSUPPORTED for a valid but
 *    unimplemented shape) with nothing enqueued.  No C++ exception crosses the ABI.
 *  - Kernels that detect an inconsistency on the device (an index out of range)
 *    record it in a status word inside the workspace instead of trapping; read it
 *    with rdt_read_device_status.
 *
 * Page references (titles and sections of the extracted web pages):
 *  "OpenMythos 분석" (zero.shotlearni.ng): Core Structure, Recurrent Block, latent
 *  reasoning, Repeating the parameter reduces expressiveness, MoE, MLA, RoPE &
 *  generation cache, ACT.  "OpenMythos" README mirror (runchr.com): 사용법,
 *  모델 변형, Attention 구현, 동적 시스템 관점, 해결책.
 */
#ifndef RDT_H_
#define RDT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RDT_API __attribute__((visibility("default")))
#else
#define RDT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RDT_OK = 0,
  RDT_ERR_INVALID_ARG = 1,     /* null pointer, bad size, inconsistent config       */
  RDT_ERR_UNSUPPORTED = 2,     /* valid but not implemented                          */
  RDT_ERR_WORKSPACE = 3,       /* ws too small or misaligned                          */
  RDT_ERR_CUDA = 4,            /* a CUDA runtime call failed                          */
  RDT_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait gave up                  */
  RDT_ERR_DEVICE_BOUNDS = 6    /* a device-side index check failed                   */
} rdt_status;

/* Mirror of MythosConfig (README mirror, 사용법) narrowed to the recurrent block,
 * plus the constants the pages leave open. */
typedef struct {
  int dim;                 /* D                                                    */
  int n_heads;             /* H; GQA head_dim = D / H                              */
  int n_kv_heads;          /* Hkv (GQA); H divisible by Hkv                       */
  int attn_type;           /* 0 = GQA, 1 = MLA                                     */
  int kv_lora_rank;        /* MLA latent width                                     */
  int q_lora_rank;         /* MLA query latent width                               */
  int qk_rope_head_dim;    /* MLA rotary part of the score dim                     */
  int qk_nope_head_dim;    /* MLA non-rotary part of the score dim                 */
  int v_head_dim;          /* MLA value head dim                                   */
  int n_experts;           /* E routed experts (0: dense FFN block)                */
  int n_shared_experts;    /* S always-on experts                                  */
  int top_k;               /* experts per token (n_experts_per_tok)                */
  int expert_dim;          /* F hidden width of routed and shared experts          */
  int lora_rank;           /* r of the depth-wise LoRA                             */
  int max_loop_iters;      /* rows of the LoRA scale table                          */
  int loop_dim;            /* channels carrying the loop-index embedding (even)    */
  float rope_theta;        /* RoPE base (10000)                                    */
  float loop_theta;        /* loop-embedding base (10000)                          */
  float norm_eps;          /* RMSNorm epsilon (1e-6)                                */
  int dtype;               /* 0 = fp32, 1 = bf16 (storage of matrices, e, GEMM inputs) */
} rdt_config;

/* Recurrent-block (or dense prelude/coda block) weights: device pointers.
 * Model-dtype matrices unless marked fp32.  Unused fields may be NULL
 * (e.g. the MLA fields for GQA, routing fields for a dense block). */
typedef struct {
  const float* rec_norm_w;   /* [D] fp32  RecurrentBlock.norm on h_loop + e         */
  const float* attn_norm_w;  /* [D] fp32  pre-attention RMSNorm                      */
  const float* ffn_norm_w;   /* [D] fp32  pre-FFN RMSNorm                            */
  /* GQA */
  const void* w_qkv;         /* [(H + 2 Hkv) hd, D]: q heads, then k heads, then v    */
  const void* w_o;           /* [D, H hd] (GQA) or [D, H v_head_dim] (MLA)            */
  /* MLA (DeepSeek-V2 layout) */
  const void* w_q_down;      /* [q_lora_rank, D]                                      */
  const float* q_norm_w;     /* [q_lora_rank] fp32                                    */
  const void* w_q_up;        /* [H (nope + rope), q_lora_rank], per head [nope|rope]  */
  const void* w_kv_down;     /* [kv_lora_rank + rope, D]: c_kv then k_rope            */
  const float* kv_norm_w;    /* [kv_lora_rank] fp32                                   */
  const void* w_kv_up;       /* [H (nope + v), kv_lora_rank], per head [k_nope|v]     */
  /* MoE ("OpenMythos 분석", MoE) */
  const void* w_router;      /* [E, D]                                                */
  const float* router_bias;  /* [E] fp32, used for selection only                     */
  const void* w13;           /* [E + S][2F][D]: rows [0,F) = W1 (gate), [F,2F) = W3    */
  const void* w2;            /* [E + S][D][F]; experts 0..E-1 routed, E.. shared      */
  /* depth-wise LoRA ("Repeating the parameter ...") */
  const void* lora_down;     /* [r, D]                                                */
  const void* lora_B;        /* [r, D]                                                */
  const float* lora_scale;   /* [max_loop_iters, r] fp32                              */
  /* LTI injection ("latent reasoning") and ACT halting head ("ACT") */
  const float* log_A;        /* [D] fp32                                              */
  const float* log_dt;       /* [1] fp32                                              */
  const float* inj_B;        /* [D] fp32                                              */
  const float* halt_w;       /* [D] fp32                                              */
  const float* halt_b;       /* [1] fp32                                              */
} rdt_weights;

/* One K/V cache per recurrent loop iteration (cache key recurrent_loop_t,
 * "OpenMythos 분석", Recurrent Block / RoPE & generation cache), model dtype,
 * caller-owned device memory; a sequence's positions beyond its length are never read.
 * GQA: k, v [n_loops][batch][Hkv][t_max][hd], post-RoPE keys and values.
 * MLA ("OpenMythos 분석", MLA: the cache keeps the latent, not per-head K/V):
 *      k = c_kv   [n_loops][batch][t_max][kv_lora_rank], before its RMSNorm;
 *      v = k_rope [n_loops][batch][t_max][qk_rope_head_dim], rotated, one for all heads.
 *      Each call rebuilds [k_nope | v] of the cached positions from c_kv. */
typedef struct {
  void* k;
  void* v;
  int n_loops;   /* loop caches held (>= the n_loops of a call that uses it) */
  int batch;     /* sequences held                                          */
  int t_max;     /* positions per sequence                                  */
} rdt_kv_cache;

/* Optional per-loop trace of a row range (tests; NULL in production).
 * Each non-NULL buffer is device memory sized [n_loops][n_rows][...]. */
typedef struct {
  int row0, n_rows;
  float* h_in;           /* [L][n_rows][D]  state entering loop t                    */
  float* f;              /* [L][n_rows][D]  router input RMSNorm_ffn(x1), as stored   */
  float* biased_logits;  /* [L][n_rows][E]  router logits + router_bias              */
  float* p;              /* [L][n_rows]     halting probability (ACT on)             */
} rdt_trace;

enum {
  RDT_FLAG_TRANSFORMER_OFF = 1,  /* debug: Transformer(h, e) term = 0 (pure LTI)      */
  /* test only (no counterpart on the pages): the call runs one tensor-core GEMM (the
   * first attention projection of loop 0) whose TMA producer issues no loads, then
   * returns without launching anything else; outputs are not written.  The GEMM's bounded
   * waits run out (about 2 s), it frees its TMEM with nothing in flight, and the device
   * status word reads RDT_ERR_DEVICE_TIMEOUT.  Needs bf16 and a tensor-core shape, else
   * RDT_ERR_UNSUPPORTED.  Exercises the timeout path without faulting the context. */
  RDT_FLAG_TEST_GEMM_TIMEOUT = 2,
  /* test only (no counterpart on the pages): a one-token call on an MLA latent cache runs
   * loop 0 up to its absorbed latent attention, launches that attention on the tensor
   * cores with its TMA producers idle, and returns without launching anything else;
   * outputs are not written.  The attention's bounded waits run out (about 2 s), every
   * warp role leaves with nothing in flight, TMEM is freed, and the device status word
   * reads RDT_ERR_DEVICE_TIMEOUT.  Needs bf16, kv_lora_rank 512, rope 64, H <= 32 and a
   * cache of at least 128 positions (the tensor-core kernel), else RDT_ERR_UNSUPPORTED. */
  RDT_FLAG_TEST_MLA_ATTN_TIMEOUT = 4
};

/* Bytes of workspace needed by rdt_recurrent_forward / rdt_recurrent_decode_step /
 * rdt_block_forward / rdt_head for `batch` x `seq` rows attending to at most
 * `max_keys` keys per sequence (prefill: start_pos + seq; decode: cache t_max).
 * Returns 0 for an invalid config. */
RDT_API size_t rdt_workspace_size(const rdt_config* cfg, int batch, int seq, int max_keys);

/* RecurrentBlock.forward ("OpenMythos 분석", Recurrent Block; update rule
 * h_{t+1} = A h_t + B e + Transformer(h_t, e), README mirror 동적 시스템 관점).
 *  h0 [N, D] fp32, e [N, D] model dtype, N = batch * seq; positions start_pos + i.
 *  act_threshold <= 0 turns ACT off (h_out = state after the last loop).
 *  halt_logit_offset: NULL or [N] fp32 added to the halting logit (workload hook).
 *  Outputs: h_out [N, D] fp32 (ACT-weighted state), halt_weights [n_loops, N] fp32,
 *  expert_ids [n_loops, N, top_k] int32 (-1 for halted rows).
 *  cache: NULL, or per-loop caches that receive this call's K/V at positions
 *  start_pos..start_pos+seq-1 (and supply earlier keys when start_pos > 0).
 *  trace: NULL or a row-range trace.  flags: RDT_FLAG_*.
 *  Weights of a MoE block are required (n_experts >= 1, top_k >= 1). */
RDT_API rdt_status rdt_recurrent_forward(const rdt_config* cfg, const rdt_weights* w,
                                 const float* h0, const void* e,
                                 int batch, int seq, int start_pos, int n_loops,
                                 float act_threshold, const float* halt_logit_offset,
                                 float* h_out, float* halt_weights, int32_t* expert_ids,
                                 const rdt_kv_cache* cache, const rdt_trace* trace, int flags,
                                 void* ws, size_t ws_bytes, void* stream);

/* One KV-cached decode step of the recurrent block ("OpenMythos 분석", RoPE &
 * generation cache): one new token per sequence b at position cache_len[b]
 * (device int32 [batch]); loop t reads and extends loop cache t (GQA or MLA).
 * The new K/V are written at cache_len[b]; the caller advances cache_len.
 * Outputs as rdt_recurrent_forward with N = batch.
 * CUDA graphs: the call only enqueues kernels and asynchronous copies on `stream`
 * (no host synchronisation, no allocation), and every kernel argument is a function
 * of this call's arguments, never of device data.  A stream capture of it therefore
 * replays correctly while the arguments (pointers, sizes, n_loops, act_threshold)
 * stay the same and the caller updates the pointed-to inputs and cache_len in place.
 * The first call on a device sets kernel attributes once: make it before capturing. */
RDT_API rdt_status rdt_recurrent_decode_step(const rdt_config* cfg, const rdt_weights* w,
                                     const float* h0, const void* e, int batch,
                                     const int32_t* cache_len, int n_loops, float act_threshold,
                                     float* h_out, float* halt_weights, int32_t* expert_ids,
                                     const rdt_kv_cache* cache,
                                     void* ws, size_t ws_bytes, void* stream);

/* rdt_recurrent_decode_step with the optional arguments of rdt_recurrent_forward:
 * halt_logit_offset (NULL or [batch] fp32 added to the halting logit) and a per-loop trace
 * of a row range (tests: the router input f and biased logits per loop, for teacher-forced
 * checks of the decode step's routes).  Both NULL: rdt_recurrent_decode_step. */
RDT_API rdt_status rdt_recurrent_decode_step_ex(const rdt_config* cfg, const rdt_weights* w,
                                        const float* h0, const void* e, int batch,
                                        const int32_t* cache_len, int n_loops, float act_threshold,
                                        const float* halt_logit_offset,
                                        float* h_out, float* halt_weights, int32_t* expert_ids,
                                        const rdt_kv_cache* cache, const rdt_trace* trace,
                                        void* ws, size_t ws_bytes, void* stream);

/* Decode step without a caller workspace, for callers that cannot allocate device
 * memory (a warm serving loop that must not allocate, a host runtime without a CUDA
 * allocator of its own, a memory-pool budget with no room for a per-call workspace).
 * The paper has no counterpart: this is a library convenience around
 * rdt_recurrent_decode_step, which it runs unchanged.
 *  - Scratch: a static device array of RDT_STATIC_SCRATCH_BYTES inside librdt, held
 *    by every GPU that loads the library until the process exits.  Nothing is
 *    allocated by this call (no cudaMalloc / cudaFree / allocating library routine).
 *  - Arguments, layouts and outputs are those of rdt_recurrent_decode_step; the
 *    caller still provides inputs, outputs, weights and the caches.
 *  - Sizes whose workspace (rdt_workspace_size(cfg, batch, 1, cache->t_max)) exceeds
 *    RDT_STATIC_SCRATCH_BYTES are rejected with RDT_ERR_WORKSPACE, nothing enqueued.
 *  - The first call on each device resolves the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call before
 *    any stream capture.
 *  - All calls share the one array: calls that overlap on the GPU (different streams,
 *    or other host threads) race and corrupt each other.  Each call initialises every
 *    part of the array it reads, so leftover contents of earlier calls do not matter.
 *  - The device status word lives in the array: read it with rdt_read_static_status.
 *  - The array's address is cached per device: not usable across a cudaDeviceReset. */
#define RDT_STATIC_SCRATCH_BYTES (32u << 20)
RDT_API rdt_status rdt_recurrent_decode_step_static(const rdt_config* cfg, const rdt_weights* w,
                                                    const float* h0, const void* e, int batch,
                                                    const int32_t* cache_len, int n_loops, float act_threshold,
                                                    float* h_out, float* halt_weights, int32_t* expert_ids,
                                                    const rdt_kv_cache* cache, void* stream);

/* Synchronise `stream`, then read and clear the device status word of the static
 * scratch used by rdt_recurrent_decode_step_static on the current device (as
 * rdt_read_device_status does for a caller workspace).  Allocates nothing. */
RDT_API rdt_status rdt_read_static_status(void* stream);

/* ---- continuous depth-wise batching of decode steps --------------------------------------
 * GeekNews summary, section 6: with ACT ("OpenMythos 분석", ACT) a token may leave the shared
 * block after fewer loops; continuous depth-wise batching lets it leave its batch slot there
 * and puts new work in its place.  Here the work is decode: `batch` sequences each decode
 * `n_tokens` tokens in order.  One slot per sequence; a tick runs the shared block once
 * over all slots, each slot's token at its own loop (its own loop embedding, LoRA scale row,
 * loop cache and last-loop flag).  A token that halts, or has run n_loops loops, leaves its
 * slot: the keys / values of its remaining loops are computed from its frozen state and
 * written into those loop caches (later tokens of the sequence attend to it there, as in a
 * lockstep decode step), and the slot takes the sequence's next token at loop 0.  The results
 * equal n_tokens successive rdt_recurrent_decode_step calls on each sequence (token n at
 * position cache_len[b] + n); the work per tick stays a full batch while tokens halt early.
 * GQA caches only (RDT_ERR_UNSUPPORTED for MLA).  All pointers are caller-owned device memory. */
typedef struct {
  const rdt_config* cfg;           /* host */
  const rdt_weights* w;            /* host struct of device pointers                         */
  const float* h0;                 /* [batch][n_tokens][D] fp32: token n of sequence b         */
  const void* e;                   /* [batch][n_tokens][D] model dtype                         */
  const float* halt_logit_offset;  /* NULL or [batch][n_tokens] fp32, added to the halting logit */
  const int32_t* cache_len;        /* [batch] int32: position of token 0 of sequence b; the   */
                                   /* tokens of b sit at cache_len[b] .. cache_len[b]+n_tokens-1 */
  int batch, n_tokens, n_loops;
  float act_threshold;             /* <= 0: ACT off (every token runs n_loops loops)           */
  float* h_out;                    /* [batch][n_tokens][D] fp32                                */
  float* halt_weights;             /* [batch][n_tokens][n_loops] fp32 (0 after a token halts)  */
  int32_t* expert_ids;             /* [batch][n_tokens][n_loops][top_k] (-1 after it halts)    */
  const rdt_kv_cache* cache;       /* host struct: GQA loop caches, n_loops >= n_loops, batch */
                                   /* >= batch, t_max >= every cache_len[b] + n_tokens         */
  void* ws; size_t ws_bytes;       /* >= rdt_depth_batch_workspace_size, 256-byte aligned;     */
                                   /* holds the slots' state between calls                     */
} rdt_depth_batch;

/* Workspace bytes of a depth-batched decode of `batch` sequences (0 for an invalid config). */
RDT_API size_t rdt_depth_batch_workspace_size(const rdt_config* cfg, int batch, int n_loops, int t_max);
/* Clear the outputs and the device status word, put token 0 of every sequence in its slot. */
RDT_API rdt_status rdt_depth_batch_begin(const rdt_depth_batch* db, void* stream);
/* Enqueue n_ticks ticks (asynchronous; every kernel argument is a function of *db, so a
 * stream capture of a tick replays correctly while *db stays the same).  Ticks after every
 * token finished do no work on the outputs. */
RDT_API rdt_status rdt_depth_batch_tick(const rdt_depth_batch* db, int n_ticks, void* stream);
/* Synchronise `stream` and return the number of tokens not yet finished (-1: CUDA error). */
RDT_API long long rdt_depth_batch_pending(const rdt_depth_batch* db, void* stream);
/* begin, then ticks in chunks of check_every (reading the pending count after each chunk,
 * which synchronises `stream`) until every token finished.  Device errors are recorded in
 * the status word of ws (rdt_read_device_status). */
RDT_API rdt_status rdt_depth_batch_run(const rdt_depth_batch* db, int check_every, void* stream);

/* One pre-norm TransformerBlock: x_out = x1 + FFN(RMSNorm(x1)), x1 = x_in + Attn(RMSNorm(x_in)).
 * FFN is the MoE when cfg->n_experts > 0, else the dense SwiGLU in w13/w2 expert 0
 * with hidden cfg->expert_dim (prelude/coda: Expert(dim, dim*4//3), "OpenMythos 분석", MoE).
 * x_in, x_out [N, D] fp32 (may not alias). */
RDT_API rdt_status rdt_block_forward(const rdt_config* cfg, const rdt_weights* w,
                             const float* x_in, float* x_out, int batch, int seq, int start_pos,
                             void* ws, size_t ws_bytes, void* stream);

/* rdt_block_forward with a KV cache for the block (a prelude or coda layer of the
 * generation loop, "OpenMythos 분석", RoPE & generation cache: one cache per layer).
 *  cache: NULL (same as rdt_block_forward), or the block's cache in the layout of
 *         rdt_kv_cache with n_loops >= 1 (slot 0 is used).
 *  cache_len: NULL for a prefill at positions start_pos..start_pos+seq-1 (written to
 *         the cache; earlier positions are read from it when start_pos > 0), or device
 *         int32 [batch] for a decode step (seq = 1): the new token of sequence b is at
 *         position cache_len[b], written there, and attends to positions 0..cache_len[b].
 *  Workspace: rdt_workspace_size(cfg, batch, seq, max(start_pos + seq, cache->t_max)).
 *  Invalid: decode without a cache or with seq != 1; a prefill past cache->t_max. */
RDT_API rdt_status rdt_block_forward_cached(const rdt_config* cfg, const rdt_weights* w,
                                            const float* x_in, float* x_out, int batch, int seq, int start_pos,
                                            const int32_t* cache_len, const rdt_kv_cache* cache,
                                            void* ws, size_t ws_bytes, void* stream);

/* Token embedding gather ("OpenMythos 분석", Core Structure: self.embed(input_ids)):
 * out[i] = table[ids[i]] widened to fp32.  table [vocab, D] model dtype; ids int32 [n]. */
RDT_API rdt_status rdt_embed(const rdt_config* cfg, const void* table, int vocab, const int32_t* ids, int n,
                     float* out, void* stream);

/* LM head: logits = RMSNorm(x) W_head^T ("OpenMythos 분석", Core Structure:
 * self.head(self.norm(x))).  x [n, D] fp32, norm_w [D] fp32, head [vocab, D] model dtype,
 * logits [n, vocab] fp32. */
RDT_API rdt_status rdt_head(const rdt_config* cfg, const float* x, int n, const float* norm_w,
                    const void* head, int vocab, float* logits,
                    void* ws, size_t ws_bytes, void* stream);

/* rdt_head on n rows of x spaced x_ld floats apart (x_ld >= dim), e.g. the last
 * position of each sequence of a prefill (x_ld = seq * dim).  logits [n, vocab]. */
RDT_API rdt_status rdt_head_rows(const rdt_config* cfg, const float* x, long long x_ld, int n,
                                 const float* norm_w, const void* head, int vocab, float* logits,
                                 void* ws, size_t ws_bytes, void* stream);

/* Greedy next token of generation (the pages print the generation loop but not its
 * sampling rule; the plainest reading is the most likely token): for each row b < n,
 * tokens[b * out_ld] = argmax_v logits[b * vocab + v], ties to the lowest index; NaN
 * is never chosen (a row of NaN gives 0).  logits fp32 and tokens int32, device. */
RDT_API rdt_status rdt_greedy_tokens(const float* logits, int n, int vocab, int32_t* tokens, int out_ld,
                                     void* stream);

/* out[i] = x[i] in the model dtype (fp32 copy, or bf16 round-to-nearest-even), i < n:
 * the recurrent block's injected input e is the prelude output in the model dtype
 * ("OpenMythos 분석", Core Structure: e = x after the prelude).  Device pointers. */
RDT_API rdt_status rdt_to_model_dtype(const rdt_config* cfg, const float* x, void* out, long long n,
                                      void* stream);

/* Synchronise `stream`, read and clear the device status word in `ws`. */
RDT_API rdt_status rdt_read_device_status(void* ws, void* stream);

/* Static description of a status code. */
RDT_API const char* rdt_status_string(rdt_status s);

/* Library build identifier (kernel set and target), static string. */
RDT_API const char* rdt_version(void);

/* ---- measurement support (benchmarks; no effect on results) ---------------- */

/* Number of kernels this library has enqueued since it was loaded (host counter). */
RDT_API unsigned long long rdt_launch_count(void);

/* Per-kernel-class device time: while profiling is on, every library call records a
 * CUDA event pair on its stream around each kernel class it launches. */
typedef struct {
  char name[32];      /* kernel class, e.g. "expert_up_swiglu"          */
  int launches;       /* timed launches of that class                    */
  double total_ms;    /* summed event-to-event device time               */
} rdt_kernel_time;

/* Start (or restart) collection.  Creates the event pool on first use. */
RDT_API rdt_status rdt_profile_start(void);

/* Stop collection, wait for the recorded events and write up to max_entries
 * per-class totals to out.  Returns the number written, or -1 on a CUDA error. */
RDT_API int rdt_profile_stop(rdt_kernel_time* out, int max_entries);

#ifdef __cplusplus
}
#endif
#endif /* RDT_H_ */
