// librdt C ABI: host validation, workspace carving and per-loop orchestration of
// the recurrent block.  Host code only enqueues kernels on the caller's stream;
// nothing here allocates device memory or synchronises (except
// rdt_read_device_status).
#include "../../include/rdt.h"
#include "common.cuh"
#include "kernels.h"

#include <string.h>
#include <algorithm>

using namespace rdt;

namespace rdt {
int decode_split_count(int t_max);
}

namespace {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Layout {
  // byte offsets into the workspace
  size_t status, h, combined, a, qkv, cq_raw, cq, q, kv_raw, ckv, krope, kvu, attn, x1, f, logits;
  size_t ids, gates, rank, counts, offsets, tiles, ntiles, slot_of, tok_of, gate_of, xg, u, y;
  size_t cta_count;                  // per-CTA running-row counts of the compaction
  size_t run_list, run_idx, nrun, cum, halted, Avec, emb, rope, pos, p_buf, part_o, part_ml, xn, vt;
  size_t mla_ckv_all, mla_kvu_all;   // MLA with earlier cached keys: rebuilt per-head keys / values
  size_t mla_qa;                     // MLA absorbed decode: absorbed queries (0 = path not used)
  size_t splitk; long long splitk_elems;   // split-K partials of single-tile GEMMs (decode)
  size_t qc, seq_off, pos_c, otiles, ontiles;   // compact queries of the running rows (GQA prefill; 0 = unused)
  int part_dim;                      // split-KV partial width (head dim, or kv_lora_rank)
  size_t total;
  int max_tiles, max_slots, rope_dim, rope_pos, n_split;
};

int esize(const rdt_config* c) { return c->dtype == 0 ? 4 : 2; }

rdt_status check_config(const rdt_config* c) {
  if (!c) return RDT_ERR_INVALID_ARG;
  if (c->dim <= 0 || c->n_heads <= 0 || (c->dtype != 0 && c->dtype != 1)) return RDT_ERR_INVALID_ARG;
  if (c->attn_type == 0) {
    if (c->n_kv_heads <= 0 || c->dim % c->n_heads || c->n_heads % c->n_kv_heads) return RDT_ERR_INVALID_ARG;
    int hd = c->dim / c->n_heads;
    if (hd % 2 || hd > 192) return RDT_ERR_UNSUPPORTED;
  } else if (c->attn_type == 1) {
    if (c->kv_lora_rank <= 0 || c->q_lora_rank <= 0 || c->qk_rope_head_dim <= 0 || c->qk_nope_head_dim < 0 ||
        c->v_head_dim <= 0 || c->qk_rope_head_dim % 2)
      return RDT_ERR_INVALID_ARG;
    if (c->qk_rope_head_dim + c->qk_nope_head_dim > 192 || c->v_head_dim > 128) return RDT_ERR_UNSUPPORTED;
  } else {
    return RDT_ERR_INVALID_ARG;
  }
  if (c->n_experts < 0 || c->n_shared_experts < 0 || c->top_k < 0 || c->top_k > c->n_experts) return RDT_ERR_INVALID_ARG;
  if (c->n_experts > 256 || c->top_k > 32 || c->n_experts + c->n_shared_experts > 1024 ||
      c->top_k + c->n_shared_experts > 64)
    return RDT_ERR_UNSUPPORTED;
  if (c->n_experts + c->n_shared_experts < 1 || c->expert_dim <= 0) return RDT_ERR_INVALID_ARG;
  if (c->lora_rank < 0 || c->lora_rank > 64 || c->max_loop_iters < 1) return RDT_ERR_INVALID_ARG;
  if (c->loop_dim < 0 || c->loop_dim % 2 || c->loop_dim > c->dim) return RDT_ERR_INVALID_ARG;
  if (!(c->norm_eps >= 0.f) || !(c->rope_theta > 0.f) || !(c->loop_theta > 0.f)) return RDT_ERR_INVALID_ARG;
  return RDT_OK;
}

void make_layout(const rdt_config* c, int B, int T, int max_keys, Layout* L) {
  const size_t N = (size_t)B * T, D = c->dim, es = esize(c);
  const int k = c->top_k, S = c->n_shared_experts, E = c->n_experts, F = c->expert_dim;
  const size_t M = N * (size_t)(k + S);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
  memset(L, 0, sizeof(*L));
  L->status = take(sizeof(DevStatus));
  L->h = take(N * D * 4);
  L->combined = take(N * D * 4);
  L->a = take(N * D * es);
  int H = c->n_heads, dv = 0;
  if (c->attn_type == 0) {
    int hd = c->dim / H;
    L->qkv = take(N * (size_t)(H + 2 * c->n_kv_heads) * hd * es);
    L->vt = take(N * (size_t)c->n_kv_heads * hd * es);   // values transposed per sequence
    dv = hd;
    L->rope_dim = hd;
    if (T > 1 && c->dtype == 1) {   // prefill: the running rows' queries, gathered, and their tiles
      L->qc = take(N * (size_t)H * hd * es);
      L->seq_off = take((size_t)(B + 1) * 4);
      L->pos_c = take(N * 4);
      L->otiles = take(((N + 127) / 128) * 16);
      L->ontiles = take(16);
    }
  } else {
    int dn = c->qk_nope_head_dim, dr = c->qk_rope_head_dim;
    dv = c->v_head_dim;
    L->cq_raw = take(N * c->q_lora_rank * 4);
    L->cq = take(N * c->q_lora_rank * es);
    L->q = take(N * (size_t)H * (dn + dr) * es);
    L->kv_raw = take(N * (size_t)(c->kv_lora_rank + dr) * 4);
    L->ckv = take(N * c->kv_lora_rank * es);
    L->krope = take(N * dr * es);
    L->kvu = take(N * (size_t)H * (dn + dv) * es);
    L->rope_dim = dr;
    if (T == 1 && mla_decode_supports(1, c->dtype, H, c->kv_lora_rank, dr, dn, dv)) {
      // decode on the latent cache in the absorbed form: nothing per head is rebuilt
      L->mla_qa = take((size_t)B * H * c->kv_lora_rank * es);
    } else if (max_keys > T) {   // earlier positions come from the latent cache
      L->mla_ckv_all = take((size_t)B * max_keys * c->kv_lora_rank * es);
      L->mla_kvu_all = take((size_t)B * max_keys * H * (dn + dv) * es);
    }
  }
  L->attn = take(N * (size_t)H * dv * es);
  L->x1 = take(N * D * 4);
  L->f = take(N * D * es);
  L->xn = take(N * D * es);
  L->logits = take(N * (size_t)std::max(E, 1) * 4);
  L->ids = take(N * std::max(k, 1) * 4);
  L->gates = take(N * std::max(k, 1) * 4);
  L->rank = take(N * std::max(k, 1) * 4);
  L->counts = take((size_t)std::max(E, 1) * 4);
  L->offsets = take((size_t)(E + S + 1) * 4);
  L->max_tiles = (int)((M + 63) / 64) + E + S + 1;
  L->tiles = take((size_t)L->max_tiles * 16);
  L->ntiles = take(16);
  L->max_slots = (int)M;
  L->slot_of = take(N * (k + S) * 4);
  L->tok_of = take(M * 4);
  L->gate_of = take(M * 4);
  L->xg = take(M * D * es);
  L->u = take(M * (size_t)F * es);
  L->y = take(M * D * es);   // gate-scaled expert outputs, model dtype
  L->run_list = take(N * 4);
  L->run_idx = take(N * 4);
  L->nrun = take(16);
  L->cta_count = take((size_t)std::max<size_t>((N + 1023) / 1024, 1) * 4);
  L->cum = take(N * 4);
  L->halted = take(N * 4);
  L->p_buf = take(N * 4);
  L->Avec = take(D * 4);
  L->emb = take((size_t)2 * std::max(c->loop_dim, 2) * 4);   // loop embeddings of loops t and t + 1
  L->rope_pos = std::max(max_keys, T);
  L->rope = take((size_t)L->rope_pos * (L->rope_dim / 2) * 8);
  L->pos = take(N * 4);
  // decode layouts (one row per sequence) hold the split-KV attention partials
  L->n_split = (T == 1) ? decode_split_count(std::max(max_keys, 1)) : 0;
  L->part_dim = 128;
  if (L->mla_qa) {
    L->n_split = mla_decode_splits(B, H, c->kv_lora_rank, c->qk_rope_head_dim, std::max(max_keys, 1));
    L->part_dim = c->kv_lora_rank;
  }
  L->part_o = take(L->n_split ? (size_t)B * H * L->n_split * L->part_dim * 4 : 16);
  if (N <= 128) {   // rows that fit one GEMM tile: the weights stream through split-K CTAs
    L->splitk_elems = (long long)N * 16384;
    L->splitk = take((size_t)L->splitk_elems * 4);
  }
  L->part_ml = take(L->n_split ? (size_t)B * H * L->n_split * 2 * 4 : 16);
  L->total = off;
}

template <typename P> P at(void* ws, size_t off) { return (P)((char*)ws + off); }

struct Ctx {
  const rdt_config* c;
  const rdt_weights* w;
  Layout L;
  void* ws;
  cudaStream_t s;
  DevStatus* st;
  int dtype;
  const int* row_loop = nullptr;   // decode rows at their own loop depth (continuous depth-wise batching)
  bool compact_q = false;          // prefill with ACT: attention queries and O projection on the running rows
  bool test_mla_timeout = false;   // test only: RDT_FLAG_TEST_MLA_ATTN_TIMEOUT
  bool test_mla_done = false;      // ... and its attention was launched
};

#define RDT_TRY(x)                          \
  do {                                      \
    if ((x) != 0) return RDT_ERR_CUDA;      \
  } while (0)

GemmParams gemm_base(const Ctx& x) {
  GemmParams g;
  memset(&g, 0, sizeof(g));
  g.st = x.st;
  g.impl = -1;
  if (x.L.splitk) {
    g.split_ws = at<float*>(x.ws, x.L.splitk);
    g.split_ws_elems = x.L.splitk_elems;
  }
  return g;
}

// Attention sub-block (S2 + S3 + S4): x1 = combined + Attn(a).  rows = N (all rows:
// halted rows keep contributing keys/values).
rdt_status attention_block(Ctx& x, int B, int T, const float* combined, const void* a, float* x1,
                           const rdt_kv_cache* cache, int loop_t, int start_pos, bool decode) {
  const rdt_config* c = x.c;
  const rdt_weights* w = x.w;
  const int N = B * T, D = c->dim, H = c->n_heads, es = esize(c);
  const int* pos = at<const int*>(x.ws, x.L.pos);
  const float2* tab = at<const float2*>(x.ws, x.L.rope);
  void* attn = at<void*>(x.ws, x.L.attn);
  AttnParams ap;
  memset(&ap, 0, sizeof(ap));
  ap.B = B; ap.T = T; ap.H = H; ap.q_pos = pos; ap.st = x.st;
  int dv;
  bool absorbed = false;   // MLA decode ran in the absorbed form (attention output written)
  if (c->attn_type == 0) {
    const int Hkv = c->n_kv_heads, hd = D / H, W = (H + 2 * Hkv) * hd;
    void* qkv = at<void*>(x.ws, x.L.qkv);
    GemmParams g = gemm_base(x);
    g.A = a; g.lda = D; g.B = w->w_qkv; g.ldb = D; g.M = N; g.N = W; g.K = D;
    g.C = qkv; g.ldc = W; g.pos = pos; g.rope_tab = tab; g.rope_half = hd / 2; g.n_rope = 2;
    g.rope[0] = RopeDesc{0, H, hd, 0, hd};
    g.rope[1] = RopeDesc{H * hd, Hkv, hd, 0, hd};
    // the tensor-core attention reads V transposed; the QKV epilogue writes that copy
    const bool kv_from_qkv = !(cache && cache->k && (decode || start_pos > 0));
    bool want_vt = x.dtype == 1 && hd == 128 && T % 8 == 0 && kv_from_qkv && !decode;
    if (want_vt) {
      g.vt = at<void*>(x.ws, x.L.vt); g.vt_col0 = (H + Hkv) * hd; g.vt_heads = Hkv; g.vt_hd = hd; g.vt_T = T; g.vt_ld = T;
      if (gemm_pick(x.dtype, g, EPI_ROPE_T) != GEMM_TC) { g.vt = nullptr; want_vt = false; }
    }
    ap.vt = want_vt ? g.vt : nullptr; ap.vt_ld = T;
    // Compact queries (prefill with ACT on the tensor-core attention): keys / values for every
    // row, queries only for the running rows, gathered in row order (their `a` rows into the
    // f buffer, free until the MoE) and projected into their own buffer with RoPE at their
    // positions.
    bool compact = false;
    GemmParams gq, gkv;
    if (x.compact_q && loop_t > 0 && want_vt && x.L.qc) {   // loop 0 runs every row
      gkv = g;
      gkv.B = (const char*)w->w_qkv + (size_t)H * hd * D * es; gkv.N = 2 * Hkv * hd;
      gkv.C = (char*)qkv + (size_t)H * hd * es; gkv.n_rope = 1; gkv.rope[0] = RopeDesc{0, Hkv, hd, 0, hd};
      gkv.vt_col0 = Hkv * hd;
      gq = gemm_base(x);
      gq.A = at<void*>(x.ws, x.L.f); gq.lda = D; gq.B = w->w_qkv; gq.ldb = D; gq.M = N; gq.N = H * hd; gq.K = D;
      gq.tiles = at<const int*>(x.ws, x.L.otiles); gq.n_tiles = at<const int*>(x.ws, x.L.ontiles);
      gq.max_tiles = (N + 127) / 128; gq.b_group_stride = 0; gq.b_rows = (long long)H * hd;
      gq.C = at<void*>(x.ws, x.L.qc); gq.ldc = (long long)H * hd; gq.pos = at<const int*>(x.ws, x.L.pos_c);
      gq.rope_tab = tab; gq.rope_half = hd / 2; gq.n_rope = 1; gq.rope[0] = RopeDesc{0, H, hd, 0, hd};
      compact = gemm_pick(x.dtype, gkv, EPI_ROPE_T) == GEMM_TC && gemm_pick(x.dtype, gq, EPI_ROPE_T) == GEMM_TC;
    }
    if (compact) {
      const int* run_list = at<const int*>(x.ws, x.L.run_list);
      const int* nrun = at<const int*>(x.ws, x.L.nrun);
      {
        ProfScope ps(PC_OTHER, x.s);
        launch_compact_meta(run_list, nrun, B, T, at<int*>(x.ws, x.L.seq_off), at<int*>(x.ws, x.L.otiles),
                            at<int*>(x.ws, x.L.ontiles), x.s);
        launch_gather_rows(a, (long long)D * es, at<void*>(x.ws, x.L.f), (long long)D * es, (long long)D * es,
                           run_list, nrun, N, x.s, pos, at<int*>(x.ws, x.L.pos_c));
      }
      ProfScope ps(PC_QKV, x.s);
      RDT_TRY(launch_gemm(x.dtype, EPI_ROPE_T, gkv, x.s));
      RDT_TRY(launch_gemm(x.dtype, EPI_ROPE_T, gq, x.s));
      ap.q = at<void*>(x.ws, x.L.qc); ap.q_row = (long long)H * hd;
      ap.seq_off = at<const int*>(x.ws, x.L.seq_off); ap.run_list = run_list;
    } else {
      { ProfScope ps(PC_QKV, x.s); RDT_TRY(launch_gemm(x.dtype, EPI_ROPE_T, g, x.s)); }
      ap.q = qkv; ap.q_row = W;
    }
    ap.q_head = hd; ap.dn = hd; ap.dr = 0; ap.dv = hd; ap.G = H / Hkv;
    ap.scale = 1.f / sqrtf((float)hd);
    const bool use_cache = cache && cache->k;
    if (use_cache) {
      const long long loop_elems = (long long)cache->batch * Hkv * cache->t_max * hd;
      size_t per_loop = (size_t)loop_elems * es;
      char* kc = (char*)cache->k + per_loop * loop_t;
      char* vc = (char*)cache->v + per_loop * loop_t;
      {
        ProfScope ps(PC_OTHER, x.s);
        launch_kv_to_cache(x.dtype, qkv, W, H * hd, (H + Hkv) * hd, Hkv, hd, pos, N, T, cache->t_max, kc, vc, x.st,
                           x.s, x.row_loop, loop_elems);
      }
      if (x.row_loop) { ap.row_loop = x.row_loop; ap.loop_k = ap.loop_v = loop_elems; }
      if (decode || start_pos > 0) {
        long long sj = hd, sg = (long long)cache->t_max * hd, sb = (long long)Hkv * sg;
        ap.k1 = kc; ap.k1_b = sb; ap.k1_j = sj; ap.k1_g = sg;
        ap.v = vc; ap.v_b = sb; ap.v_j = sj; ap.v_g = sg;
        ap.key_pos0 = 0;
        ap.n_keys = decode ? cache->t_max : start_pos + T;
        if (decode && x.L.n_split) {
          ap.part_o = at<float*>(x.ws, x.L.part_o); ap.part_ml = at<float*>(x.ws, x.L.part_ml); ap.n_split = x.L.n_split;
        }
      }
    }
    if (!ap.k1) {
      ap.k1 = (const char*)qkv + (size_t)H * hd * es; ap.k1_b = (long long)T * W; ap.k1_j = W; ap.k1_g = hd;
      ap.v = (const char*)qkv + (size_t)(H + Hkv) * hd * es; ap.v_b = (long long)T * W; ap.v_j = W; ap.v_g = hd;
      ap.key_pos0 = start_pos; ap.n_keys = T;
    }
    dv = hd;
  } else {
    const int dn = c->qk_nope_head_dim, dr = c->qk_rope_head_dim, kvr = c->kv_lora_rank, ql = c->q_lora_rank;
    dv = c->v_head_dim;
    float* cq_raw = at<float*>(x.ws, x.L.cq_raw);
    void* cq = at<void*>(x.ws, x.L.cq);
    void* q = at<void*>(x.ws, x.L.q);
    float* kv_raw = at<float*>(x.ws, x.L.kv_raw);
    void* ckv = at<void*>(x.ws, x.L.ckv);
    void* krope = at<void*>(x.ws, x.L.krope);
    void* kvu = at<void*>(x.ws, x.L.kvu);
    {
      ProfScope ps_proj(PC_QKV, x.s);   // the projections, up to the attention proper
      GemmParams g = gemm_base(x);
      g.A = a; g.lda = D; g.B = w->w_q_down; g.ldb = D; g.M = N; g.N = ql; g.K = D; g.C = cq_raw; g.ldc = ql;
      RDT_TRY(launch_gemm(x.dtype, EPI_STORE_F32, g, x.s));
      launch_rmsnorm(1, x.dtype, cq_raw, ql, w->q_norm_w, cq, ql, N, ql, c->norm_eps, x.s);
      g = gemm_base(x);
      g.A = cq; g.lda = ql; g.B = w->w_q_up; g.ldb = ql; g.M = N; g.N = H * (dn + dr); g.K = ql;
      g.C = q; g.ldc = H * (dn + dr); g.pos = pos; g.rope_tab = tab; g.rope_half = dr / 2; g.n_rope = 1;
      g.rope[0] = RopeDesc{0, H, dn + dr, dn, dr};
      RDT_TRY(launch_gemm(x.dtype, EPI_ROPE_T, g, x.s));
      g = gemm_base(x);
      g.A = a; g.lda = D; g.B = w->w_kv_down; g.ldb = D; g.M = N; g.N = kvr + dr; g.K = D; g.C = kv_raw; g.ldc = kvr + dr;
      RDT_TRY(launch_gemm(x.dtype, EPI_STORE_F32, g, x.s));
      launch_mla_kv_prep(x.dtype, kv_raw, kvr, dr, w->kv_norm_w, c->norm_eps, pos, tab, ckv, krope, N, x.s);
      absorbed = T == 1 && cache && cache->k && x.L.mla_qa;   // one row per sequence, keys from the cache
      if (!absorbed) {   // per-head [k_nope | v] of this call's rows
        g = gemm_base(x);
        g.A = ckv; g.lda = kvr; g.B = w->w_kv_up; g.ldb = kvr; g.M = N; g.N = H * (dn + dv); g.K = kvr;
        g.C = kvu; g.ldc = H * (dn + dv);
        RDT_TRY(launch_gemm(x.dtype, EPI_STORE_T, g, x.s));
      }
    }
    const long long kvw = (long long)H * (dn + dv);
    ap.q = q; ap.q_row = H * (dn + dr); ap.q_head = dn + dr; ap.dn = dn; ap.dr = dr; ap.dv = dv; ap.G = 1;
    ap.k1 = kvu; ap.k1_b = (long long)T * kvw; ap.k1_j = kvw; ap.k1_g = dn + dv;
    ap.k2 = krope; ap.k2_b = (long long)T * dr; ap.k2_j = dr;
    ap.v = (const char*)kvu + (size_t)dn * es; ap.v_b = (long long)T * kvw; ap.v_j = kvw; ap.v_g = dn + dv;
    ap.key_pos0 = start_pos; ap.n_keys = T;
    if (cache && cache->k) {
      // latent cache of loop t: c_kv [B][t_max][kvr] (raw) and k_rope [B][t_max][dr]
      const int tm = cache->t_max;
      char* ckv_c = (char*)cache->k + (size_t)loop_t * cache->batch * tm * kvr * es;
      char* kr_c = (char*)cache->v + (size_t)loop_t * cache->batch * tm * dr * es;
      { ProfScope ps(PC_OTHER, x.s); launch_mla_to_cache(x.dtype, kv_raw, krope, kvr, dr, pos, N, T, tm, ckv_c, kr_c, x.st, x.s); }
      if (absorbed) {
        MlaDecodeParams mp;
        memset(&mp, 0, sizeof(mp));
        mp.B = B; mp.H = H; mp.dn = dn; mp.dr = dr; mp.dv = dv; mp.kvr = kvr;
        mp.q = q; mp.q_row = (long long)H * (dn + dr); mp.q_head = dn + dr;
        mp.w_kvu = w->w_kv_up; mp.kv_norm_w = w->kv_norm_w; mp.eps = c->norm_eps;
        mp.scale = 1.f / sqrtf((float)(dn + dr));
        mp.ckv = ckv_c; mp.krope = kr_c; mp.t_max = tm; mp.q_pos = pos;
        mp.qa = at<void*>(x.ws, x.L.mla_qa);
        mp.part_o = at<float*>(x.ws, x.L.part_o); mp.part_ml = at<float*>(x.ws, x.L.part_ml); mp.n_split = x.L.n_split;
        mp.o = attn; mp.o_row = (long long)H * dv; mp.st = x.st;
        if (x.test_mla_timeout) {   // the tensor-core attention alone, its producers idle
          mp.test_no_loads = 1;
          x.test_mla_done = launch_mla_decode(mp, x.s) == 0;
          return x.test_mla_done ? RDT_OK : RDT_ERR_UNSUPPORTED;
        }
        ProfScope ps(PC_ATTN, x.s);
        if (launch_mla_decode(mp, x.s) != 0) return RDT_ERR_CUDA;
      } else if (decode || start_pos > 0) {
        // keys / values of every cached position: [k_nope | v] = RMSNorm(c_kv) W_kvu^T
        if (!x.L.mla_kvu_all) return RDT_ERR_WORKSPACE;
        void* ckv_all = at<void*>(x.ws, x.L.mla_ckv_all);
        void* kvu_all = at<void*>(x.ws, x.L.mla_kvu_all);
        const int rows = B * tm;
        ProfScope ps(PC_OTHER, x.s);
        launch_rmsnorm(0, x.dtype, ckv_c, kvr, w->kv_norm_w, ckv_all, kvr, rows, kvr, c->norm_eps, x.s);
        GemmParams g2 = gemm_base(x);
        g2.A = ckv_all; g2.lda = kvr; g2.B = w->w_kv_up; g2.ldb = kvr; g2.M = rows; g2.N = H * (dn + dv); g2.K = kvr;
        g2.C = kvu_all; g2.ldc = kvw;
        RDT_TRY(launch_gemm(x.dtype, EPI_STORE_T, g2, x.s));
        ap.k1 = kvu_all; ap.k1_b = (long long)tm * kvw; ap.k1_j = kvw; ap.k1_g = dn + dv;
        ap.k2 = kr_c; ap.k2_b = (long long)tm * dr; ap.k2_j = dr;
        ap.v = (const char*)kvu_all + (size_t)dn * es; ap.v_b = (long long)tm * kvw; ap.v_j = kvw; ap.v_g = dn + dv;
        ap.key_pos0 = 0;
        ap.n_keys = decode ? tm : start_pos + T;
      }
    }
    ap.scale = 1.f / sqrtf((float)(dn + dr));
  }
  ap.o = attn; ap.o_row = (long long)H * dv; ap.o_head = dv;
  GemmParams g = gemm_base(x);
  g.A = attn; g.lda = (long long)H * dv; g.B = w->w_o; g.ldb = (long long)H * dv; g.M = N; g.N = D; g.K = H * dv;
  g.C = x1; g.ldc = D; g.resid = combined; g.ld_resid = D;
  // Compact queries: only the running rows get an attention output and x1 (a halted row keeps
  // its state); the O projection runs over their tiles and writes x1 through the row map.
  if (ap.seq_off) {
    GemmParams gc = g;
    gc.tiles = at<const int*>(x.ws, x.L.otiles); gc.n_tiles = at<const int*>(x.ws, x.L.ontiles);
    gc.max_tiles = (N + 127) / 128; gc.b_group_stride = 0; gc.b_rows = D;
    gc.row_map = ap.run_list;
    if (!attention_tc_supports(x.dtype, ap) || gemm_pick(x.dtype, gc, EPI_RESID_F32) != GEMM_TC)
      return RDT_ERR_UNSUPPORTED;   // the shapes were checked before the queries were made compact
    { ProfScope ps(PC_ATTN, x.s); RDT_TRY(launch_attention(x.dtype, ap, x.s)); }
    { ProfScope ps(PC_OPROJ, x.s); RDT_TRY(launch_gemm(x.dtype, EPI_RESID_F32, gc, x.s)); }
    return RDT_OK;
  }
  if (!absorbed) { ProfScope ps(PC_ATTN, x.s); RDT_TRY(launch_attention(x.dtype, ap, x.s)); }
  { ProfScope ps(PC_OPROJ, x.s); RDT_TRY(launch_gemm(x.dtype, EPI_RESID_F32, g, x.s)); }
  return RDT_OK;
}

// MoE FFN (S5 .. S8) on the running rows: y[slot] = gate * Expert_e(f[token]).
rdt_status moe_block(Ctx& x, int N, const float* x1) {
  const rdt_config* c = x.c;
  const rdt_weights* w = x.w;
  const int D = c->dim, E = c->n_experts, k = c->top_k, S = c->n_shared_experts, F = c->expert_dim;
  void* f = at<void*>(x.ws, x.L.f);
  {
    // the router and the experts read f of the running rows only
    ProfScope ps(PC_FFN_NORM, x.s);
    if (!launch_rmsnorm_rows(x.dtype, x1, w->ffn_norm_w, f, N, D, c->norm_eps, at<const int*>(x.ws, x.L.run_list),
                             at<const int*>(x.ws, x.L.nrun), x.s))
      launch_rmsnorm(1, x.dtype, x1, D, w->ffn_norm_w, f, D, N, D, c->norm_eps, x.s);
  }
  float* logits = at<float*>(x.ws, x.L.logits);
  RouteParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.logits = logits; rp.bias = w->router_bias; rp.N = N; rp.E = E; rp.k = k; rp.S = S;
  rp.run_list = at<int*>(x.ws, x.L.run_list); rp.n_run = at<int*>(x.ws, x.L.nrun);
  rp.ids = at<int*>(x.ws, x.L.ids); rp.gates = at<float*>(x.ws, x.L.gates); rp.rank = at<int*>(x.ws, x.L.rank);
  rp.counts = at<int*>(x.ws, x.L.counts); rp.offsets = at<int*>(x.ws, x.L.offsets);
  rp.tiles = at<int*>(x.ws, x.L.tiles); rp.n_tiles = at<int*>(x.ws, x.L.ntiles); rp.max_tiles = x.L.max_tiles;
  rp.slot_of = at<int*>(x.ws, x.L.slot_of); rp.tok_of = at<int*>(x.ws, x.L.tok_of);
  rp.gate_of = at<float*>(x.ws, x.L.gate_of); rp.f = f; rp.xg = at<void*>(x.ws, x.L.xg); rp.D = D;
  rp.max_slots = x.L.max_slots; rp.st = x.st;
  // expert GEMMs pick their tile height from the implementation that will run them
  GemmParams up = gemm_base(x);
  up.A = rp.xg; up.lda = D; up.B = w->w13; up.ldb = D; up.b_group_stride = (long long)2 * F * D;
  up.M = x.L.max_slots; up.N = F; up.K = D; up.up_off = F; up.b_rows = (long long)(E + S) * 2 * F;
  up.tiles = rp.tiles; up.n_tiles = rp.n_tiles; up.max_tiles = x.L.max_tiles;
  up.C = at<void*>(x.ws, x.L.u); up.ldc = F;
  GemmParams dn = gemm_base(x);
  dn.A = up.C; dn.lda = F; dn.B = w->w2; dn.ldb = F; dn.b_group_stride = (long long)D * F;
  dn.M = x.L.max_slots; dn.N = D; dn.K = F; dn.b_rows = (long long)(E + S) * D; dn.tiles = rp.tiles; dn.n_tiles = rp.n_tiles; dn.max_tiles = x.L.max_tiles;
  dn.C = at<void*>(x.ws, x.L.y); dn.ldc = D; dn.row_scale = rp.gate_of;
  // both expert GEMMs consume the same tile list, so they must share one tile height
  GemmImpl iu = gemm_pick(x.dtype, up, EPI_SWIGLU_T), id = gemm_pick(x.dtype, dn, EPI_GATE_T);
  if (iu != id) iu = id = GEMM_SIMT;
  up.impl = dn.impl = (int)iu;
  rp.tile_m = gemm_tile_m(iu);
  if (cudaMemsetAsync(rp.counts, 0, sizeof(int) * std::max(E, 1), x.s) != cudaSuccess) return RDT_ERR_CUDA;
  // router logits; on the tensor-core path the GEMM epilogue also routes the running rows
  GemmParams g = gemm_base(x);
  g.A = f; g.lda = D; g.B = w->w_router; g.ldb = D; g.M = N; g.N = E; g.K = D; g.C = logits; g.ldc = E;
  g.bias = w->router_bias; g.run_idx = at<int*>(x.ws, x.L.run_idx); g.topk = k;
  g.ids = rp.ids; g.gates = rp.gates; g.rank = rp.rank; g.counts = rp.counts;
  // few rows (decode): the logits come from a CTA per expert and top-k runs on its own
  // kernel; otherwise the tcgen05 router GEMM routes in its epilogue
  const bool small_router = x.dtype == 1 && N <= 128;
  const bool fused_route = !small_router && gemm_pick(x.dtype, g, EPI_ROUTER) == GEMM_TC;
  {
    ProfScope ps(PC_ROUTER_GEMM, x.s);
    if (!(small_router && launch_router_small(f, w->w_router, N, D, E, logits, x.s)))
      RDT_TRY(launch_gemm(x.dtype, fused_route ? EPI_ROUTER : EPI_STORE_F32, g, x.s));
  }
  {
    ProfScope ps(PC_ROUTE, x.s);
    if (!fused_route) launch_router_topk(rp, x.s);
    launch_route_scan(rp, x.s);
    launch_route_scatter(x.dtype, rp, x.s);
  }
  { ProfScope ps(PC_EXPERT_UP, x.s); RDT_TRY(launch_gemm(x.dtype, EPI_SWIGLU_T, up, x.s)); }
  { ProfScope ps(PC_EXPERT_DOWN, x.s); RDT_TRY(launch_gemm(x.dtype, EPI_GATE_T, dn, x.s)); }
  return RDT_OK;
}

CombineParams combine_base(Ctx& x, int N) {
  const rdt_config* c = x.c;
  const rdt_weights* w = x.w;
  CombineParams cp;
  memset(&cp, 0, sizeof(cp));
  cp.N = N; cp.D = c->dim; cp.k = c->top_k; cp.S = c->n_shared_experts; cp.r = c->lora_rank;
  cp.max_loop_iters = c->max_loop_iters; cp.max_slots = x.L.max_slots;
  cp.x1 = at<float*>(x.ws, x.L.x1); cp.y = at<void*>(x.ws, x.L.y); cp.slot_of = at<int*>(x.ws, x.L.slot_of);
  cp.ids = at<int*>(x.ws, x.L.ids);
  cp.lora_down = w->lora_down; cp.lora_B = w->lora_B; cp.lora_scale = w->lora_scale;
  cp.A = at<float*>(x.ws, x.L.Avec); cp.inj_B = w->inj_B;
  cp.h = at<float*>(x.ws, x.L.h); cp.h_state = at<float*>(x.ws, x.L.h);
  cp.halt_wv = w->halt_w; cp.halt_b = w->halt_b;
  cp.cum = at<float*>(x.ws, x.L.cum); cp.halted = at<int*>(x.ws, x.L.halted);
  cp.p_out = at<float*>(x.ws, x.L.p_buf);
  cp.st = x.st;
  return cp;
}

rdt_status check_block_weights(const rdt_config* c, const rdt_weights* w, bool moe) {
  if (!w || !w->attn_norm_w || !w->ffn_norm_w || !w->w_o || !w->w13 || !w->w2) return RDT_ERR_INVALID_ARG;
  if (c->attn_type == 0 && !w->w_qkv) return RDT_ERR_INVALID_ARG;
  if (c->attn_type == 1 && (!w->w_q_down || !w->q_norm_w || !w->w_q_up || !w->w_kv_down || !w->kv_norm_w || !w->w_kv_up))
    return RDT_ERR_INVALID_ARG;
  if (moe && (!w->w_router || !w->router_bias || c->n_experts < 1 || c->top_k < 1)) return RDT_ERR_INVALID_ARG;
  return RDT_OK;
}

rdt_status check_ws(void* ws, size_t ws_bytes, const Layout& L) {
  if (!ws || ((uintptr_t)ws & 255)) return RDT_ERR_WORKSPACE;
  if (ws_bytes < L.total) return RDT_ERR_WORKSPACE;
  return RDT_OK;
}

// Shared loop driver of prefill (decode = false) and decode (decode = true).
rdt_status run_recurrent(const rdt_config* c, const rdt_weights* w, const float* h0, const void* e, int B, int T,
                         int start_pos, const int32_t* cache_len, int n_loops, float thr, const float* halt_off,
                         float* h_out, float* halt_weights, int32_t* expert_ids, const rdt_kv_cache* cache,
                         const rdt_trace* trace, int flags, void* ws, size_t ws_bytes, cudaStream_t s, bool decode) {
  rdt_status st = check_config(c);
  if (st != RDT_OK) return st;
  if ((st = check_block_weights(c, w, true)) != RDT_OK) return st;
  if (!w->rec_norm_w || !w->log_A || !w->log_dt || !w->inj_B) return RDT_ERR_INVALID_ARG;
  if (c->lora_rank > 0 && (!w->lora_down || !w->lora_B || !w->lora_scale)) return RDT_ERR_INVALID_ARG;
  if (!h0 || !e || !h_out || !halt_weights || !expert_ids) return RDT_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0 || n_loops <= 0 || start_pos < 0) return RDT_ERR_INVALID_ARG;
  if (thr != thr) return RDT_ERR_INVALID_ARG;   // NaN threshold
  const bool act_on = thr > 0.f;
  if (act_on && (!w->halt_w || !w->halt_b)) return RDT_ERR_INVALID_ARG;
  if ((long long)B * T > (1LL << 30)) return RDT_ERR_UNSUPPORTED;
  int max_keys = start_pos + T;
  if (cache) {
    if (!cache->k || !cache->v || cache->t_max <= 0 || cache->batch < B || cache->n_loops < n_loops)
      return RDT_ERR_INVALID_ARG;
    if (!decode && start_pos + T > cache->t_max) return RDT_ERR_INVALID_ARG;
    max_keys = std::max(max_keys, cache->t_max);
  }
  if (decode && (!cache || !cache_len)) return RDT_ERR_INVALID_ARG;
  if (trace && (trace->row0 < 0 || trace->n_rows < 0 || trace->row0 + trace->n_rows > B * T)) return RDT_ERR_INVALID_ARG;
  Ctx x;
  x.c = c; x.w = w; x.ws = ws; x.s = s; x.dtype = c->dtype;
  make_layout(c, B, T, max_keys, &x.L);
  if ((st = check_ws(ws, ws_bytes, x.L)) != RDT_OK) return st;
  // halted rows drop out of the attention queries and the O projection (prefill with ACT,
  // keys from this call's rows)
  x.compact_q = act_on && !decode && !(cache && cache->k && start_pos > 0);
  x.st = at<DevStatus*>(ws, x.L.status);
  const int N = B * T, D = c->dim, E = c->n_experts;
  const bool transformer_off = (flags & RDT_FLAG_TRANSFORMER_OFF) != 0;
  float* h = at<float*>(ws, x.L.h);
  float* combined = at<float*>(ws, x.L.combined);
  void* a = at<void*>(ws, x.L.a);
  float* x1 = at<float*>(ws, x.L.x1);
  float* emb = at<float*>(ws, x.L.emb);
  int* pos = at<int*>(ws, x.L.pos);
  // per-call set-up
  if (cudaMemsetAsync(x.st, 0, sizeof(DevStatus), s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemcpyAsync(h, h0, (size_t)N * D * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemsetAsync(h_out, 0, (size_t)N * D * 4, s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemsetAsync(at<void*>(ws, x.L.cum), 0, (size_t)N * 4, s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemsetAsync(at<void*>(ws, x.L.halted), 0, (size_t)N * 4, s) != cudaSuccess) return RDT_ERR_CUDA;
  launch_lti_A(w->log_A, w->log_dt, at<float*>(ws, x.L.Avec), D, s);
  launch_rope_table(at<float2*>(ws, x.L.rope), x.L.rope_pos, x.L.rope_dim, c->rope_theta, s);
  if (decode) launch_positions_decode(pos, cache_len, B, cache->t_max, x.st, s);
  else launch_positions(pos, N, T, start_pos, s);
  launch_iota(at<int*>(ws, x.L.run_list), at<int*>(ws, x.L.run_idx), at<int*>(ws, x.L.nrun), N, s);
  CombineParams cp = combine_base(x, N);
  cp.n_loops = n_loops; cp.act_on = act_on; cp.thr = thr; cp.e = e; cp.h_out = h_out;
  cp.halt_off = halt_off; cp.halt_w_out = halt_weights; cp.ids_out = expert_ids;
  cp.transformer_off = transformer_off;
  cp.loop_dim = c->loop_dim; cp.w_rec = w->rec_norm_w; cp.w_attn = w->attn_norm_w; cp.eps = c->norm_eps;
  cp.combined_out = combined; cp.a_out = a;
  x.test_mla_timeout = (flags & RDT_FLAG_TEST_MLA_ATTN_TIMEOUT) != 0;
  if (flags & RDT_FLAG_TEST_GEMM_TIMEOUT) {
    // the first projection of loop 0 with an idle producer; nothing reads its output
    GemmParams g = gemm_base(x);
    g.A = a; g.lda = D; g.M = N; g.K = D; g.test_no_loads = 1;
    if (c->attn_type == 0) {
      const int W = (c->n_heads + 2 * c->n_kv_heads) * (D / c->n_heads);
      g.B = w->w_qkv; g.ldb = D; g.N = W; g.C = at<void*>(ws, x.L.qkv); g.ldc = W;
    } else {
      g.B = w->w_q_down; g.ldb = D; g.N = c->q_lora_rank; g.C = at<void*>(ws, x.L.cq); g.ldc = c->q_lora_rank;
    }
    if (gemm_pick(x.dtype, g, EPI_STORE_T) != GEMM_TC) return RDT_ERR_UNSUPPORTED;
    RDT_TRY(launch_gemm(x.dtype, EPI_STORE_T, g, s));
    return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
  }
  const int emb_stride = std::max(c->loop_dim, 2);
  bool prologue_done = false;   // set when the previous loop's combine kernel computed this loop's prologue
  for (int t = 0; t < n_loops; ++t) {
    float* emb_t = emb + (size_t)(t & 1) * emb_stride;
    if (trace && trace->h_in)
      launch_trace_rows(0, x.dtype, h, D, trace->row0, trace->n_rows, nullptr,
                        trace->h_in + (size_t)t * trace->n_rows * D, s);
    if (!prologue_done) {
      ProfScope ps(PC_PROLOGUE, s);
      launch_loop_emb(emb_t, c->loop_dim, t, c->loop_theta, s);
      launch_loop_prologue(x.dtype, h, e, emb_t, c->loop_dim, w->rec_norm_w, w->attn_norm_w, combined, a, N, D,
                           c->norm_eps, s);
    }
    if (!transformer_off) {
      if ((st = attention_block(x, B, T, combined, a, x1, cache, t, start_pos, decode)) != RDT_OK) return st;
      if (x.test_mla_timeout) {
        if (!x.test_mla_done) return RDT_ERR_UNSUPPORTED;
        return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
      }
      if ((st = moe_block(x, N, x1)) != RDT_OK) return st;
      if (trace && trace->f)
        launch_trace_rows(1, x.dtype, at<void*>(ws, x.L.f), D, trace->row0, trace->n_rows, nullptr,
                          trace->f + (size_t)t * trace->n_rows * D, s);
      if (trace && trace->biased_logits)
        launch_trace_rows(0, x.dtype, at<float*>(ws, x.L.logits), E, trace->row0, trace->n_rows, w->router_bias,
                          trace->biased_logits + (size_t)t * trace->n_rows * E, s);
    }
    cp.t = t;
    cp.next_emb = nullptr;
    if (t + 1 < n_loops && c->loop_dim >= 0) {
      // the combine kernel of loop t also produces combined / a of loop t + 1
      float* emb_n = emb + (size_t)((t + 1) & 1) * emb_stride;
      launch_loop_emb(emb_n, c->loop_dim, t + 1, c->loop_theta, s);
      cp.next_emb = emb_n;
    }
    { ProfScope ps(PC_COMBINE, s); prologue_done = launch_combine(x.dtype, cp, N, s); }
    if (trace && trace->p && act_on)
      launch_trace_rows(0, x.dtype, at<float*>(ws, x.L.p_buf), 1, trace->row0, trace->n_rows, nullptr,
                        trace->p + (size_t)t * trace->n_rows, s);
    if (act_on && t + 1 < n_loops) {
      ProfScope ps(PC_OTHER, s);
      launch_compact(at<int*>(ws, x.L.halted), N, at<int*>(ws, x.L.run_list), at<int*>(ws, x.L.run_idx),
                     at<int*>(ws, x.L.nrun), at<int*>(ws, x.L.cta_count), s);
    }
  }
  if (cudaGetLastError() != cudaSuccess) return RDT_ERR_CUDA;
  return RDT_OK;
}

// ------------------------------------------------------------------------------------------
// continuous depth-wise batching of decode steps
// ------------------------------------------------------------------------------------------
struct DepthLayout {
  size_t t_row, tok, out_row, pending, e_slot, off_slot, emb_tab, a_fill, kv_fill, pos_fill;
  size_t fill_b, fill_u, fill_n, fill_tiles, fill_ntiles, total;
  int emb_stride, fill_max_tiles;
};

// The decode layout of `batch` rows (one slot per sequence) followed by the slot state and
// the fill buffers of the remaining loops of finished tokens.
void make_depth_layout(const rdt_config* c, int B, int L, int t_max, Layout* Lo, DepthLayout* DL) {
  make_layout(c, B, 1, t_max, Lo);
  size_t off = Lo->total;
  auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
  const size_t D = c->dim, es = esize(c), nf = (size_t)B * std::max(L - 1, 1);
  const int hd = c->dim / c->n_heads;
  DL->emb_stride = std::max(c->loop_dim, 2);
  DL->t_row = take((size_t)B * 4);
  DL->tok = take((size_t)B * 4);
  DL->out_row = take((size_t)B * 4);
  DL->pending = take(16);
  DL->e_slot = take((size_t)B * D * es);
  DL->off_slot = take((size_t)B * 4);
  DL->emb_tab = take((size_t)L * DL->emb_stride * 4);
  DL->a_fill = take(nf * D * es);
  DL->kv_fill = take(nf * 2 * (size_t)c->n_kv_heads * hd * es);
  DL->pos_fill = take(nf * 4);
  DL->fill_b = take(nf * 4);
  DL->fill_u = take(nf * 4);
  DL->fill_n = take(16);
  DL->fill_max_tiles = (int)((nf + 63) / 64);   // the smaller of the two GEMM row tiles
  DL->fill_tiles = take((size_t)DL->fill_max_tiles * 16);
  DL->fill_ntiles = take(16);
  DL->total = off;
}

struct DepthCall {
  Ctx x;
  DepthLayout DL;
  DepthParams dp;
  CombineParams cp;
};

rdt_status depth_setup(const rdt_depth_batch* db, cudaStream_t s, DepthCall* dc) {
  if (!db) return RDT_ERR_INVALID_ARG;
  const rdt_config* c = db->cfg;
  const rdt_weights* w = db->w;
  rdt_status st = check_config(c);
  if (st != RDT_OK) return st;
  if ((st = check_block_weights(c, w, true)) != RDT_OK) return st;
  if (c->attn_type != 0) return RDT_ERR_UNSUPPORTED;    // GQA loop caches only
  if (!w->rec_norm_w || !w->log_A || !w->log_dt || !w->inj_B) return RDT_ERR_INVALID_ARG;
  if (c->lora_rank > 0 && (!w->lora_down || !w->lora_B || !w->lora_scale)) return RDT_ERR_INVALID_ARG;
  const int B = db->batch, S = db->n_tokens, L = db->n_loops;
  if (!db->h0 || !db->e || !db->cache_len || !db->h_out || !db->halt_weights || !db->expert_ids || !db->cache)
    return RDT_ERR_INVALID_ARG;
  if (B <= 0 || S <= 0 || L <= 0 || db->act_threshold != db->act_threshold) return RDT_ERR_INVALID_ARG;
  if ((long long)B * S > (1LL << 30) || (long long)B * L > (1LL << 24)) return RDT_ERR_UNSUPPORTED;
  const bool act_on = db->act_threshold > 0.f;
  if (act_on && (!w->halt_w || !w->halt_b)) return RDT_ERR_INVALID_ARG;
  const rdt_kv_cache* cache = db->cache;
  if (!cache->k || !cache->v || cache->t_max <= 0 || cache->batch < B || cache->n_loops < L || S > cache->t_max)
    return RDT_ERR_INVALID_ARG;
  Ctx& x = dc->x;
  x.c = c; x.w = w; x.ws = db->ws; x.s = s; x.dtype = c->dtype;
  make_depth_layout(c, B, L, cache->t_max, &x.L, &dc->DL);
  if (!db->ws || ((uintptr_t)db->ws & 255) || db->ws_bytes < dc->DL.total) return RDT_ERR_WORKSPACE;
  x.st = at<DevStatus*>(db->ws, x.L.status);
  const DepthLayout& DL = dc->DL;
  void* ws = db->ws;
  x.row_loop = at<int*>(ws, DL.t_row);
  const int D = c->dim, hd = D / c->n_heads;
  DepthParams& dp = dc->dp;
  memset(&dp, 0, sizeof(dp));
  dp.B = B; dp.S = S; dp.L = L; dp.D = D; dp.loop_dim = c->loop_dim; dp.emb_stride = DL.emb_stride;
  dp.Hkv = c->n_kv_heads; dp.hd = hd; dp.t_max = cache->t_max;
  dp.h0_seq = db->h0; dp.e_seq = db->e; dp.off_seq = db->halt_logit_offset; dp.cache_len0 = db->cache_len;
  dp.h = at<float*>(ws, x.L.h); dp.e_slot = at<void*>(ws, DL.e_slot); dp.off_slot = at<float*>(ws, DL.off_slot);
  dp.pos = at<int*>(ws, x.L.pos);
  dp.t_row = at<int*>(ws, DL.t_row); dp.tok = at<int*>(ws, DL.tok); dp.out_row = at<int*>(ws, DL.out_row);
  dp.cum = at<float*>(ws, x.L.cum); dp.halted = at<int*>(ws, x.L.halted); dp.pending = at<int*>(ws, DL.pending);
  dp.emb_tab = at<float*>(ws, DL.emb_tab); dp.w_rec = w->rec_norm_w; dp.w_attn = w->attn_norm_w; dp.eps = c->norm_eps;
  dp.a_fill = at<void*>(ws, DL.a_fill); dp.pos_fill = at<int*>(ws, DL.pos_fill); dp.kv_fill = at<void*>(ws, DL.kv_fill);
  dp.fill_b = at<int*>(ws, DL.fill_b); dp.fill_u = at<int*>(ws, DL.fill_u); dp.fill_n = at<int*>(ws, DL.fill_n);
  dp.fill_tiles = at<int*>(ws, DL.fill_tiles); dp.fill_ntiles = at<int*>(ws, DL.fill_ntiles);
  dp.kc = cache->k; dp.vc = cache->v;
  dp.loop_elems = (long long)cache->batch * c->n_kv_heads * cache->t_max * hd;
  dp.st = x.st;
  CombineParams& cp = dc->cp;
  cp = combine_base(x, B);
  cp.n_loops = L; cp.act_on = act_on; cp.thr = db->act_threshold; cp.e = dp.e_slot; cp.h_out = db->h_out;
  cp.halt_off = dp.off_slot; cp.halt_w_out = db->halt_weights; cp.ids_out = db->expert_ids;
  cp.loop_dim = c->loop_dim; cp.w_rec = w->rec_norm_w; cp.w_attn = w->attn_norm_w; cp.eps = c->norm_eps;
  cp.next_emb = nullptr; cp.t_row = dp.t_row; cp.out_row = dp.out_row;
  return RDT_OK;
}

// One tick: every slot's token runs one loop at its own depth; finished tokens fill their
// remaining loops' keys / values and their slots take the next tokens.
rdt_status depth_tick(const rdt_depth_batch* db, DepthCall& dc) {
  Ctx& x = dc.x;
  const rdt_config* c = x.c;
  const rdt_weights* w = x.w;
  const DepthParams& dp = dc.dp;
  const int B = dp.B, L = dp.L, D = c->dim, hd = dp.hd, Hkv = dp.Hkv, H = c->n_heads;
  cudaStream_t s = x.s;
  void* ws = x.ws;
  float* combined = at<float*>(ws, x.L.combined);
  void* a = at<void*>(ws, x.L.a);
  float* x1 = at<float*>(ws, x.L.x1);
  rdt_status st;
  {
    ProfScope ps(PC_PROLOGUE, s);
    launch_loop_prologue(x.dtype, dp.h, dp.e_slot, dp.emb_tab, c->loop_dim, w->rec_norm_w, w->attn_norm_w,
                         combined, a, B, D, c->norm_eps, s, dp.t_row, dp.emb_stride);
  }
  if ((st = attention_block(x, B, 1, combined, a, x1, db->cache, 0, 0, true)) != RDT_OK) return st;
  if ((st = moe_block(x, B, x1)) != RDT_OK) return st;
  { ProfScope ps(PC_COMBINE, s); launch_combine(x.dtype, dc.cp, B, s); }
  if (L > 1) {
    ProfScope ps(PC_DEPTH_FILL, s);
    // the fill rows are compacted on the device; the GEMM runs over their row tiles only
    GemmParams g;
    memset(&g, 0, sizeof(g));
    g.impl = -1; g.st = x.st;
    g.A = dp.a_fill; g.lda = D;
    g.B = (const char*)w->w_qkv + (size_t)H * hd * D * esize(c); g.ldb = D;   // the K and V rows of w_qkv
    g.M = B * (L - 1); g.N = 2 * Hkv * hd; g.K = D;
    g.tiles = dp.fill_tiles; g.n_tiles = dp.fill_ntiles; g.b_group_stride = 0; g.b_rows = g.N;
    g.C = const_cast<void*>(dp.kv_fill); g.ldc = 2 * Hkv * hd;
    g.pos = dp.pos_fill; g.rope_tab = at<const float2*>(ws, x.L.rope); g.rope_half = hd / 2; g.n_rope = 1;
    g.rope[0] = RopeDesc{0, Hkv, hd, 0, hd};
    DepthParams fp = dp;
    fp.fill_tile_m = gemm_tile_m(gemm_pick(x.dtype, g, EPI_ROPE_T));
    g.max_tiles = (g.M + fp.fill_tile_m - 1) / fp.fill_tile_m;
    launch_depth_fill_list(fp, s);
    launch_depth_fill_prologue(x.dtype, fp, s);
    RDT_TRY(launch_gemm(x.dtype, EPI_ROPE_T, g, s));
    launch_depth_fill_store(x.dtype, fp, s);
  }
  {
    ProfScope ps(PC_OTHER, s);
    launch_depth_refill(x.dtype, dp, s);
    launch_compact(dp.halted, B, at<int*>(ws, x.L.run_list), at<int*>(ws, x.L.run_idx), at<int*>(ws, x.L.nrun),
                   at<int*>(ws, x.L.cta_count), s);
  }
  return RDT_OK;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// GEMM dispatch
// ------------------------------------------------------------------------------------------
namespace rdt {
int launch_gemm_simt(int dtype, int epi, const GemmParams& p, cudaStream_t s);
int launch_gemm_tc(int epi, const GemmParams& p, cudaStream_t s);
bool gemm_tc_supports(const GemmParams& p, int epi);
int launch_attention_simt(int dtype, const AttnParams& p, cudaStream_t s);
bool attention_fa_supports(int dtype, const AttnParams& p);
int launch_attention_fa(const AttnParams& p, cudaStream_t s);
bool attention_tc_supports(int dtype, const AttnParams& p);
int launch_attention_tc(const AttnParams& p, cudaStream_t s);
bool attention_tc_mla_supports(int dtype, const AttnParams& p);
int launch_attention_tc_mla(const AttnParams& p, cudaStream_t s);

int gemm_tile_m(GemmImpl impl) { return impl == GEMM_TC ? 128 : 64; }
GemmImpl gemm_pick(int dtype, const GemmParams& p, int epi) {
  if (p.impl == GEMM_SIMT) return GEMM_SIMT;
  if (dtype == 1 && gemm_tc_supports(p, epi)) return GEMM_TC;
  return GEMM_SIMT;
}
int launch_gemm(int dtype, int epi, const GemmParams& p, cudaStream_t s) {
  if (gemm_pick(dtype, p, epi) == GEMM_TC) return launch_gemm_tc(epi, p, s);
  return launch_gemm_simt(dtype, epi, p, s);
}
int launch_attention(int dtype, const AttnParams& p, cudaStream_t s) {
  if (p.part_o && p.T == 1 && launch_attention_decode(dtype, p, s) == 0) return 0;
  if (attention_tc_supports(dtype, p)) return launch_attention_tc(p, s);
  if (attention_tc_mla_supports(dtype, p)) return launch_attention_tc_mla(p, s);
  if (attention_fa_supports(dtype, p)) return launch_attention_fa(p, s);
  return launch_attention_simt(dtype, p, s);
}
}  // namespace rdt

// ------------------------------------------------------------------------------------------
// C ABI
// ------------------------------------------------------------------------------------------
extern "C" {

size_t rdt_workspace_size(const rdt_config* cfg, int batch, int seq, int max_keys) {
  if (check_config(cfg) != RDT_OK || batch <= 0 || seq <= 0) return 0;
  Layout L;
  make_layout(cfg, batch, seq, std::max(max_keys, seq), &L);
  return L.total;
}

rdt_status rdt_recurrent_forward(const rdt_config* cfg, const rdt_weights* w, const float* h0, const void* e,
                                 int batch, int seq, int start_pos, int n_loops, float act_threshold,
                                 const float* halt_logit_offset, float* h_out, float* halt_weights,
                                 int32_t* expert_ids, const rdt_kv_cache* cache, const rdt_trace* trace, int flags,
                                 void* ws, size_t ws_bytes, void* stream) {
  return run_recurrent(cfg, w, h0, e, batch, seq, start_pos, nullptr, n_loops, act_threshold, halt_logit_offset,
                       h_out, halt_weights, expert_ids, cache, trace, flags, ws, ws_bytes, (cudaStream_t)stream,
                       false);
}

rdt_status rdt_recurrent_decode_step(const rdt_config* cfg, const rdt_weights* w, const float* h0, const void* e,
                                     int batch, const int32_t* cache_len, int n_loops, float act_threshold,
                                     float* h_out, float* halt_weights, int32_t* expert_ids,
                                     const rdt_kv_cache* cache, void* ws, size_t ws_bytes, void* stream) {
  return run_recurrent(cfg, w, h0, e, batch, 1, 0, cache_len, n_loops, act_threshold, nullptr, h_out, halt_weights,
                       expert_ids, cache, nullptr, 0, ws, ws_bytes, (cudaStream_t)stream, true);
}

rdt_status rdt_recurrent_decode_step_ex(const rdt_config* cfg, const rdt_weights* w, const float* h0,
                                        const void* e, int batch, const int32_t* cache_len, int n_loops,
                                        float act_threshold, const float* halt_logit_offset, float* h_out,
                                        float* halt_weights, int32_t* expert_ids, const rdt_kv_cache* cache,
                                        const rdt_trace* trace, void* ws, size_t ws_bytes, void* stream) {
  return run_recurrent(cfg, w, h0, e, batch, 1, 0, cache_len, n_loops, act_threshold, halt_logit_offset, h_out,
                       halt_weights, expert_ids, cache, trace, 0, ws, ws_bytes, (cudaStream_t)stream, true);
}

rdt_status rdt_block_forward_cached(const rdt_config* cfg, const rdt_weights* w, const float* x_in, float* x_out,
                                    int batch, int seq, int start_pos, const int32_t* cache_len,
                                    const rdt_kv_cache* cache, void* ws, size_t ws_bytes, void* stream) {
  rdt_status st = check_config(cfg);
  if (st != RDT_OK) return st;
  const bool moe = cfg->n_experts > 0;
  if ((st = check_block_weights(cfg, w, moe)) != RDT_OK) return st;
  if (!x_in || !x_out || x_in == x_out || batch <= 0 || seq <= 0 || start_pos < 0) return RDT_ERR_INVALID_ARG;
  if (!moe && cfg->n_shared_experts != 1) return RDT_ERR_INVALID_ARG;
  const bool decode = cache_len != nullptr;
  int max_keys = start_pos + seq;
  if (cache) {
    if (!cache->k || !cache->v || cache->t_max <= 0 || cache->batch < batch || cache->n_loops < 1)
      return RDT_ERR_INVALID_ARG;
    if (!decode && start_pos + seq > cache->t_max) return RDT_ERR_INVALID_ARG;
    max_keys = std::max(max_keys, cache->t_max);
  }
  if (decode && (!cache || seq != 1)) return RDT_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  ProfScope ps_block(PC_BLOCK, s);
  Ctx x;
  x.c = cfg; x.w = w; x.ws = ws; x.s = s; x.dtype = cfg->dtype;
  make_layout(cfg, batch, seq, max_keys, &x.L);
  if ((st = check_ws(ws, ws_bytes, x.L)) != RDT_OK) return st;
  x.st = at<DevStatus*>(ws, x.L.status);
  const int N = batch * seq, D = cfg->dim, F = cfg->expert_dim;
  if (cudaMemsetAsync(x.st, 0, sizeof(DevStatus), s) != cudaSuccess) return RDT_ERR_CUDA;
  launch_rope_table(at<float2*>(ws, x.L.rope), x.L.rope_pos, x.L.rope_dim, cfg->rope_theta, s);
  if (decode) launch_positions_decode(at<int*>(ws, x.L.pos), cache_len, batch, cache->t_max, x.st, s);
  else launch_positions(at<int*>(ws, x.L.pos), N, seq, start_pos, s);
  void* a = at<void*>(ws, x.L.a);
  float* x1 = at<float*>(ws, x.L.x1);
  launch_rmsnorm(1, x.dtype, x_in, D, w->attn_norm_w, a, D, N, D, cfg->norm_eps, s);
  if ((st = attention_block(x, batch, seq, x_in, a, x1, cache, 0, start_pos, decode)) != RDT_OK) return st;
  if (moe) {
    launch_iota(at<int*>(ws, x.L.run_list), at<int*>(ws, x.L.run_idx), at<int*>(ws, x.L.nrun), N, s);
    if ((st = moe_block(x, N, x1)) != RDT_OK) return st;
    CombineParams cp = combine_base(x, N);
    cp.block_only = 1; cp.out = x_out;
    launch_combine(x.dtype, cp, N, s);
  } else {
    void* f = at<void*>(ws, x.L.f);
    launch_rmsnorm(1, x.dtype, x1, D, w->ffn_norm_w, f, D, N, D, cfg->norm_eps, s);
    GemmParams up = gemm_base(x);
    up.A = f; up.lda = D; up.B = w->w13; up.ldb = D; up.M = N; up.N = F; up.K = D; up.up_off = F;
    up.C = at<void*>(ws, x.L.u); up.ldc = F;
    if (launch_gemm(x.dtype, EPI_SWIGLU_T, up, s)) return RDT_ERR_CUDA;
    GemmParams dn = gemm_base(x);
    dn.A = up.C; dn.lda = F; dn.B = w->w2; dn.ldb = F; dn.M = N; dn.N = D; dn.K = F;
    dn.C = x_out; dn.ldc = D; dn.resid = x1; dn.ld_resid = D;
    if (launch_gemm(x.dtype, EPI_RESID_F32, dn, s)) return RDT_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return RDT_ERR_CUDA;
  return RDT_OK;
}

rdt_status rdt_block_forward(const rdt_config* cfg, const rdt_weights* w, const float* x_in, float* x_out, int batch,
                             int seq, int start_pos, void* ws, size_t ws_bytes, void* stream) {
  return rdt_block_forward_cached(cfg, w, x_in, x_out, batch, seq, start_pos, nullptr, nullptr, ws, ws_bytes, stream);
}

rdt_status rdt_greedy_tokens(const float* logits, int n, int vocab, int32_t* tokens, int out_ld, void* stream) {
  if (!logits || !tokens || n <= 0 || vocab <= 0 || out_ld < 1) return RDT_ERR_INVALID_ARG;
  ProfScope ps(PC_TOKENS, (cudaStream_t)stream);
  launch_greedy(logits, n, vocab, tokens, out_ld, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
}

rdt_status rdt_to_model_dtype(const rdt_config* cfg, const float* x, void* out, long long n, void* stream) {
  if (!cfg || (cfg->dtype != 0 && cfg->dtype != 1) || !x || !out || n < 0) return RDT_ERR_INVALID_ARG;
  if (n == 0) return RDT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  ProfScope ps(PC_TOKENS, s);
  if (cfg->dtype == 0) {
    if (x != out && cudaMemcpyAsync(out, x, (size_t)n * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return RDT_ERR_CUDA;
  } else {
    launch_to_model_dtype(x, out, n, s);
  }
  return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
}

rdt_status rdt_embed(const rdt_config* cfg, const void* table, int vocab, const int32_t* ids, int n, float* out,
                     void* stream) {
  if (!cfg || cfg->dim <= 0 || (cfg->dtype != 0 && cfg->dtype != 1) || !table || !ids || !out || vocab <= 0 || n <= 0)
    return RDT_ERR_INVALID_ARG;
  ProfScope ps(PC_TOKENS, (cudaStream_t)stream);
  launch_embed(cfg->dtype, table, vocab, ids, n, cfg->dim, out, nullptr, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
}

rdt_status rdt_head_rows(const rdt_config* cfg, const float* xin, long long x_ld, int n, const float* norm_w,
                         const void* head, int vocab, float* logits, void* ws, size_t ws_bytes, void* stream) {
  rdt_status st = check_config(cfg);
  if (st != RDT_OK) return st;
  if (!xin || n <= 0 || x_ld < cfg->dim || !norm_w || !head || vocab <= 0 || !logits) return RDT_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  ProfScope ps(PC_HEAD, s);
  Layout L;
  make_layout(cfg, 1, n, n, &L);
  if ((st = check_ws(ws, ws_bytes, L)) != RDT_OK) return st;
  void* xn = at<void*>(ws, L.xn);
  launch_rmsnorm(1, cfg->dtype, xin, x_ld, norm_w, xn, cfg->dim, n, cfg->dim, cfg->norm_eps, s);
  GemmParams g;
  memset(&g, 0, sizeof(g));
  g.impl = -1;
  g.A = xn; g.lda = cfg->dim; g.B = head; g.ldb = cfg->dim; g.M = n; g.N = vocab; g.K = cfg->dim;
  g.C = logits; g.ldc = vocab; g.st = at<DevStatus*>(ws, L.status);
  if (launch_gemm(cfg->dtype, EPI_STORE_F32, g, s)) return RDT_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
}

rdt_status rdt_head(const rdt_config* cfg, const float* xin, int n, const float* norm_w, const void* head, int vocab,
                    float* logits, void* ws, size_t ws_bytes, void* stream) {
  return rdt_head_rows(cfg, xin, cfg ? cfg->dim : 0, n, norm_w, head, vocab, logits, ws, ws_bytes, stream);
}

size_t rdt_depth_batch_workspace_size(const rdt_config* cfg, int batch, int n_loops, int t_max) {
  if (check_config(cfg) != RDT_OK || batch <= 0 || n_loops <= 0 || t_max <= 0) return 0;
  Layout L;
  DepthLayout DL;
  make_depth_layout(cfg, batch, n_loops, t_max, &L, &DL);
  return DL.total;
}

rdt_status rdt_depth_batch_begin(const rdt_depth_batch* db, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  DepthCall dc;
  rdt_status st = depth_setup(db, s, &dc);
  if (st != RDT_OK) return st;
  Ctx& x = dc.x;
  const DepthParams& dp = dc.dp;
  const rdt_config* c = x.c;
  const size_t rows = (size_t)dp.B * dp.S;
  if (cudaMemsetAsync(x.st, 0, sizeof(DevStatus), s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemsetAsync(db->h_out, 0, rows * c->dim * 4, s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemsetAsync(db->halt_weights, 0, rows * dp.L * 4, s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemsetAsync(db->expert_ids, 0xFF, rows * dp.L * std::max(c->top_k, 1) * 4, s) != cudaSuccess)
    return RDT_ERR_CUDA;                                   // every id -1 until its token runs that loop
  launch_lti_A(x.w->log_A, x.w->log_dt, at<float*>(x.ws, x.L.Avec), c->dim, s);
  launch_rope_table(at<float2*>(x.ws, x.L.rope), x.L.rope_pos, x.L.rope_dim, c->rope_theta, s);
  for (int t = 0; t < dp.L; ++t) launch_loop_emb(const_cast<float*>(dp.emb_tab) + (size_t)t * dp.emb_stride,
                                                 c->loop_dim, t, c->loop_theta, s);
  launch_depth_start(x.dtype, dp, s);
  launch_iota(at<int*>(x.ws, x.L.run_list), at<int*>(x.ws, x.L.run_idx), at<int*>(x.ws, x.L.nrun), dp.B, s);
  return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
}

rdt_status rdt_depth_batch_tick(const rdt_depth_batch* db, int n_ticks, void* stream) {
  if (n_ticks < 0) return RDT_ERR_INVALID_ARG;
  DepthCall dc;
  rdt_status st = depth_setup(db, (cudaStream_t)stream, &dc);
  if (st != RDT_OK) return st;
  for (int i = 0; i < n_ticks; ++i)
    if ((st = depth_tick(db, dc)) != RDT_OK) return st;
  return cudaGetLastError() == cudaSuccess ? RDT_OK : RDT_ERR_CUDA;
}

long long rdt_depth_batch_pending(const rdt_depth_batch* db, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  DepthCall dc;
  if (depth_setup(db, s, &dc) != RDT_OK) return -1;
  int v = -1;
  if (cudaMemcpyAsync(&v, (char*)db->ws + dc.DL.pending, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return -1;
  if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
  return v;
}

rdt_status rdt_depth_batch_run(const rdt_depth_batch* db, int check_every, void* stream) {
  if (check_every <= 0) return RDT_ERR_INVALID_ARG;
  rdt_status st = rdt_depth_batch_begin(db, stream);
  if (st != RDT_OK) return st;
  // every token runs at most n_loops ticks and a slot holds one token at a time
  const long long max_ticks = (long long)db->n_tokens * db->n_loops;
  for (long long done = 0; done < max_ticks; done += check_every) {
    const int n = (int)std::min<long long>(check_every, max_ticks - done);
    if ((st = rdt_depth_batch_tick(db, n, stream)) != RDT_OK) return st;
    const long long left = rdt_depth_batch_pending(db, stream);
    if (left < 0) return RDT_ERR_CUDA;
    if (left == 0) return RDT_OK;
  }
  return rdt_depth_batch_pending(db, stream) == 0 ? RDT_OK : RDT_ERR_CUDA;
}

rdt_status rdt_read_device_status(void* ws, void* stream) {
  if (!ws) return RDT_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  DevStatus hs;
  if (cudaMemcpyAsync(&hs, ws, sizeof(hs), cudaMemcpyDeviceToHost, s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RDT_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(hs), s) != cudaSuccess) return RDT_ERR_CUDA;
  if (hs.code == ST_TIMEOUT) return RDT_ERR_DEVICE_TIMEOUT;
  if (hs.code == ST_BOUNDS) return RDT_ERR_DEVICE_BOUNDS;
  return RDT_OK;
}

const char* rdt_status_string(rdt_status s) {
  switch (s) {
    case RDT_OK: return "ok";
    case RDT_ERR_INVALID_ARG: return "invalid argument";
    case RDT_ERR_UNSUPPORTED: return "unsupported configuration";
    case RDT_ERR_WORKSPACE: return "workspace too small or misaligned";
    case RDT_ERR_CUDA: return "CUDA runtime error";
    case RDT_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case RDT_ERR_DEVICE_BOUNDS: return "device-side bounds check failed";
  }
  return "unknown status";
}

const char* rdt_version(void) { return "librdt 0.1 sm_100a"; }

}  // extern "C"
