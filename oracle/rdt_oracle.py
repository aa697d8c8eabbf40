"""CPU oracle for the looped Recurrent Block of the OpenMythos Recurrent-Depth Transformer.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package entry's smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the CUDA
library and its binding) never calls it, and it imports nothing from the product.

What it computes, and where each step comes from (page titles as extracted):
  * "OpenMythos 분석" (zero.shotlearni.ng), section "Core Structure": the model
    forward (embed -> prelude -> e = x -> recurrent -> coda -> head(norm(x))).
  * same page, section "Recurrent Block": the per-loop order -- loop-index
    embedding, norm(h_loop + e), shared block, "+ lora(trans_out, t)",
    injection(h, e, trans_out), ACT weighting into h_out.
  * same page, section "latent reasoning": LTIInjection, A = exp(-exp(clamp(log_dt +
    log_A, -20, 20))), h' = A*h + B*e + transformer_out.
  * same page, section "Repeating the parameter reduces expressiveness": loop-index
    embedding (cat(sin, cos) of t * freqs added to the first loop_dim channels) and the
    depth-wise LoRA (down(x) * scale[t] @ B; the last scale reused past max_loop_iters).
  * same page, section "MoE": softmax router, top-k on logits + router_bias, gates
    gathered from the unbiased scores and renormalised.
  * same page, section "MLA": kv_down split into c_kv / k_rope, k_rope shared by all
    heads and rotated; k_nope and v rebuilt from c_kv.
  * same page, section "RoPE & generation cache": adjacent dims as complex pairs,
    rotated by absolute position (start_pos + i).
  * same page, section "ACT": halting probability sigmoid(halt(h)); README mirror
    (runchr.com) "Attention 구현" for GQA.

Readings where the pages are silent (the full list is in the design notes):
pre-norm residual block; RMSNorm eps 1e-6; interleaved RoPE pairs, theta 10000;
loop freqs loop_theta^(-2j/loop_dim), loop_dim = dim/8; softmax scale 1/sqrt(score
dim); SwiGLU experts without biases; top-k ties broken toward the lower index;
ACT: cum += p for running rows, forced halt with the remainder at the last loop,
halted rows frozen (router/experts skipped, expert id -1); MLA in the DeepSeek-V2
layout with RMSNorm on c_q and c_kv.

Arithmetic is float64 throughout.  Weights stored in bf16 are widened exactly.
Library primitives used as single steps: matmul, a stable sort, exp/sin/cos/sqrt.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

F64 = torch.float64


def _d(t: torch.Tensor) -> torch.Tensor:
    """Exact widening to float64 on the CPU (bf16 and fp32 are subsets of fp64)."""
    return t.detach().to(device="cpu").to(F64)


# ------------------------------------------------------------------------------------------
# elementary steps
# ------------------------------------------------------------------------------------------

def rmsnorm(x: torch.Tensor, w: torch.Tensor, eps: float) -> torch.Tensor:
    """Root-mean-square norm (Zhang & Sennrich, cited in "OpenMythos 분석"):
    x / sqrt(mean(x^2) + eps) * w over the last dimension."""
    ms = (x * x).mean(dim=-1, keepdim=True)
    return x / torch.sqrt(ms + eps) * _d(w)


def silu(z: torch.Tensor) -> torch.Tensor:
    return z / (1.0 + torch.exp(-z))


def sigmoid(z: torch.Tensor) -> torch.Tensor:
    return 1.0 / (1.0 + torch.exp(-z))


def softmax(z: torch.Tensor) -> torch.Tensor:
    m = z.max(dim=-1, keepdim=True).values
    ez = torch.exp(z - m)
    return ez / ez.sum(dim=-1, keepdim=True)


def loop_embedding(t: int, loop_dim: int, dim: int, theta: float) -> torch.Tensor:
    """Loop-index embedding ("OpenMythos 분석", "Repeating the parameter ..."):
    angles = t * freqs, emb = cat(sin, cos)[:loop_dim] placed in the first loop_dim
    channels, zero elsewhere.  freqs_j = theta^(-2j/loop_dim), j < loop_dim/2."""
    emb = torch.zeros(dim, dtype=F64)
    half = loop_dim // 2
    if half == 0:
        return emb
    j = torch.arange(half, dtype=F64)
    freqs = theta ** (-2.0 * j / loop_dim)
    ang = float(t) * freqs
    emb[:half] = torch.sin(ang)
    emb[half:2 * half] = torch.cos(ang)
    return emb


def rope(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotary embedding ("OpenMythos 분석", "RoPE & generation cache"): within each
    head vector of size d, dims (2m, 2m+1) form one complex number rotated by
    angle pos * theta^(-2m/d).  x: [T, n, d]; pos: [T] absolute positions."""
    d = x.shape[-1]
    m = torch.arange(d // 2, dtype=F64)
    inv = theta ** (-2.0 * m / d)
    ang = pos.to(F64)[:, None] * inv[None, :]          # [T, d/2]
    c = torch.cos(ang)[:, None, :]
    s = torch.sin(ang)[:, None, :]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = torch.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def topk_lower_index(v: torch.Tensor, k: int) -> torch.Tensor:
    """Indices of the k largest entries of each row, in descending value order;
    equal values keep ascending index order (stable sort)."""
    order = torch.sort(v, dim=-1, descending=True, stable=True).indices
    return order[..., :k]


def expert_swiglu(w13: torch.Tensor, w2: torch.Tensor, x: torch.Tensor) -> torch.Tensor:
    """Expert(dim, hidden) as a gated-SiLU MLP without biases: W2 (silu(W1 x) * W3 x).
    w13: [2F, D] with W1 = rows [0, F), W3 = rows [F, 2F); w2: [D, F]; x: [n, D]."""
    F = w13.shape[0] // 2
    W = _d(w13)
    gate = x @ W[:F].T
    up = x @ W[F:].T
    return (silu(gate) * up) @ _d(w2).T


def lti_A(log_A: torch.Tensor, log_dt: torch.Tensor) -> torch.Tensor:
    """LTIInjection.get_A ("OpenMythos 분석", "latent reasoning")."""
    z = (_d(log_dt) + _d(log_A)).clamp(-20.0, 20.0)
    return torch.exp(-torch.exp(z))


# ------------------------------------------------------------------------------------------
# attention
# ------------------------------------------------------------------------------------------

def _causal_attend(q, k, v, q_pos, k_pos, scale):
    """q [Tq, d], k [Tk, d], v [Tk, dv]; key j visible to query i iff k_pos[j] <= q_pos[i]."""
    s = (q @ k.T) * scale
    mask = k_pos[None, :] > q_pos[:, None]
    s = s.masked_fill(mask, float("-inf"))
    p = softmax(s)
    return p @ v


def gqa_attention(cfg, W: dict, a: torch.Tensor, pos: torch.Tensor, cache: Optional[dict] = None):
    """Grouped-query attention for one sequence (README mirror, "Attention 구현").
    a: [T, D]; pos: [T] absolute positions.  Returns (o [T, H*hd], new_k, new_v)
    where new_k/new_v are the rotated keys and values of these T tokens.
    cache (optional): {"k": [C, Hkv, hd], "v": [C, Hkv, hd], "pos": [C]} keys seen before."""
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    T = a.shape[0]
    Wqkv = _d(W["w_qkv"])
    qkv = a @ Wqkv.T
    q = qkv[:, : H * hd].reshape(T, H, hd)
    k = qkv[:, H * hd: (H + Hkv) * hd].reshape(T, Hkv, hd)
    v = qkv[:, (H + Hkv) * hd:].reshape(T, Hkv, hd)
    q = rope(q, pos, cfg.rope_theta)
    k = rope(k, pos, cfg.rope_theta)
    if cache is not None:
        K = torch.cat([_d(cache["k"]), k], 0)
        V = torch.cat([_d(cache["v"]), v], 0)
        kp = torch.cat([cache["pos"].to(torch.int64), pos.to(torch.int64)], 0)
    else:
        K, V, kp = k, v, pos.to(torch.int64)
    group = H // Hkv
    out = torch.empty(T, H, hd, dtype=F64)
    for h in range(H):
        g = h // group
        out[:, h] = _causal_attend(q[:, h], K[:, g], V[:, g], pos.to(torch.int64), kp, 1.0 / math.sqrt(hd))
    return out.reshape(T, H * hd) @ _d(W["w_o"]).T, k, v


def mla_attention(cfg, W: dict, a: torch.Tensor, pos: torch.Tensor, cache: Optional[dict] = None):
    """Multi-latent attention for one sequence ("OpenMythos 분석", "MLA"; DeepSeek-V2 layout).
    q = RMSNorm(a Wqd^T) Wqu^T split per head into [nope | rope]; kv_raw = a Wkvd^T split
    into c_kv and one k_rope shared by all heads (rotated); [k_nope | v] per head =
    RMSNorm(c_kv) Wkvu^T.  Returns (o [T, D], c_kv, k_rope) -- the latent cache entries."""
    H = cfg.n_heads
    dn, dr, dv, kvr = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim, cfg.kv_lora_rank
    T = a.shape[0]
    cq = rmsnorm(a @ _d(W["w_q_down"]).T, W["q_norm_w"], cfg.norm_eps)
    q = (cq @ _d(W["w_q_up"]).T).reshape(T, H, dn + dr)
    q_nope, q_rope = q[..., :dn], rope(q[..., dn:].contiguous(), pos, cfg.rope_theta)
    kv_raw = a @ _d(W["w_kv_down"]).T
    c_kv = kv_raw[:, :kvr]
    k_rope = rope(kv_raw[:, kvr:].reshape(T, 1, dr).contiguous(), pos, cfg.rope_theta)[:, 0]
    if cache is not None:
        C_kv = torch.cat([_d(cache["c_kv"]), c_kv], 0)
        K_rope = torch.cat([_d(cache["k_rope"]), k_rope], 0)
        kp = torch.cat([cache["pos"].to(torch.int64), pos.to(torch.int64)], 0)
    else:
        C_kv, K_rope, kp = c_kv, k_rope, pos.to(torch.int64)
    kvu = (rmsnorm(C_kv, W["kv_norm_w"], cfg.norm_eps) @ _d(W["w_kv_up"]).T).reshape(-1, H, dn + dv)
    k_nope, v = kvu[..., :dn], kvu[..., dn:]
    out = torch.empty(T, H, dv, dtype=F64)
    scale = 1.0 / math.sqrt(dn + dr)
    for h in range(H):
        qh = torch.cat([q_nope[:, h], q_rope[:, h]], -1)
        kh = torch.cat([k_nope[:, h], K_rope], -1)
        out[:, h] = _causal_attend(qh, kh, v[:, h], pos.to(torch.int64), kp, scale)
    return out.reshape(T, H * dv) @ _d(W["w_o"]).T, c_kv, k_rope


def attention(cfg, W, a, pos, cache=None):
    if cfg.attn_type == "gqa":
        return gqa_attention(cfg, W, a, pos, cache)
    return mla_attention(cfg, W, a, pos, cache)


# ------------------------------------------------------------------------------------------
# MoE
# ------------------------------------------------------------------------------------------

def router(cfg, W: dict, f: torch.Tensor, forced: Optional[torch.Tensor] = None):
    """MoEFFN router ("OpenMythos 분석", "MoE"): logits = f Wr^T, scores = softmax(logits),
    idx = topk(logits + router_bias), gates = scores[idx] renormalised to sum 1.
    forced: test hook, [n, k] int64: rows with forced[i, 0] >= 0 take those experts (the
    gates are still this router's scores at them, renormalised); parity tests impose a
    route only where the two sides' biased logits differ enough to swap it.
    Returns (idx, gates, logits, biased logits, the router's own idx)."""
    k = cfg.n_experts_per_tok
    logits = f @ _d(W["w_router"]).T
    scores = softmax(logits)
    biased = logits + _d(W["router_bias"])
    own = topk_lower_index(biased, k)
    idx = own
    if forced is not None:
        use = forced[:, 0] >= 0
        idx = torch.where(use[:, None], forced.to(torch.int64), own)
    g = torch.gather(scores, -1, idx)
    g = g / g.sum(dim=-1, keepdim=True)
    return idx, g, logits, biased, own


def moe_ffn(cfg, W: dict, f: torch.Tensor, forced: Optional[torch.Tensor] = None, own: Optional[list] = None):
    """Routed top-k SwiGLU experts plus always-on shared experts (gate 1).
    forced: test hook passed to the router; own: optional list receiving the router's own idx.
    Returns (y [n, D], idx [n, k], gates [n, k], biased logits [n, E])."""
    E, S = cfg.n_experts, cfg.n_shared_experts
    idx, g, logits, biased, own_idx = router(cfg, W, f, forced)
    if own is not None:
        own.append(own_idx)
    y = torch.zeros_like(f)
    for e in torch.unique(idx).tolist():
        rows, slot = torch.nonzero(idx == e, as_tuple=True)
        y[rows] += g[rows, slot, None] * expert_swiglu(W["w13"][e], W["w2"][e], f[rows])
    for s in range(S):
        y += expert_swiglu(W["w13"][E + s], W["w2"][E + s], f)
    return y, idx, g, biased


def dense_ffn(W: dict, f: torch.Tensor):
    return expert_swiglu(W["w13"][0], W["w2"][0], f)


# ------------------------------------------------------------------------------------------
# blocks
# ------------------------------------------------------------------------------------------

def transformer_block(cfg, W: dict, x: torch.Tensor, batch: int, pos: torch.Tensor, use_moe: bool,
                      caches=None, row_mask: Optional[torch.Tensor] = None,
                      forced_ids: Optional[torch.Tensor] = None):
    """Pre-norm residual block: x1 = x + Attn(RMSNorm(x)); out = x1 + FFN(RMSNorm(x1)).
    x: [B*T, D] (sequence-major); pos: [B*T].  caches: optional per-sequence list of
    attention cache dicts (read, not modified).  row_mask (MoE only): rows whose FFN is
    evaluated; other rows get out = x1 and expert ids -1.  forced_ids: test hook, [N, k]
    routes imposed on rows with forced_ids[i, 0] >= 0 (see router).
    Returns (out, x1, info) with info holding ids/gates/biased logits/new kv per sequence
    and the router's own ids ("own_ids", -1 for rows not evaluated)."""
    N, D = x.shape
    T = N // batch
    a = rmsnorm(x, W["attn_norm_w"], cfg.norm_eps)
    attn_out = torch.empty_like(x)
    new_kv = []
    for b in range(batch):
        sl = slice(b * T, (b + 1) * T)
        o, k1, k2 = attention(cfg, W, a[sl], pos[sl], None if caches is None else caches[b])
        attn_out[sl] = o
        new_kv.append((k1, k2))
    x1 = x + attn_out
    f = rmsnorm(x1, W["ffn_norm_w"], cfg.norm_eps)
    info = {"new_kv": new_kv, "f": f}
    if not use_moe:
        return x1 + dense_ffn(W, f), x1, info
    k = cfg.n_experts_per_tok
    ids = torch.full((N, k), -1, dtype=torch.int64)
    own_ids = torch.full((N, k), -1, dtype=torch.int64)
    gates = torch.zeros(N, k, dtype=F64)
    biased = torch.zeros(N, cfg.n_experts, dtype=F64)
    rows = torch.arange(N) if row_mask is None else torch.nonzero(row_mask, as_tuple=True)[0]
    out = x1.clone()
    if rows.numel():
        own = []
        y, idx, g, bl = moe_ffn(cfg, W, f[rows], None if forced_ids is None else forced_ids[rows], own)
        out[rows] = x1[rows] + y
        ids[rows], gates[rows], biased[rows], own_ids[rows] = idx, g, bl, own[0]
    info.update(ids=ids, gates=gates, biased=biased, own_ids=own_ids)
    return out, x1, info


def lora_delta(cfg, W: dict, x: torch.Tensor, t: int) -> torch.Tensor:
    """Depth-wise LoRA ("OpenMythos 분석", "Repeating ..."): (x Wd^T * scale[t']) B with
    t' = min(t, max_loop_iters - 1) (the last scale is reused past the trained range)."""
    tt = min(t, cfg.max_loop_iters - 1)
    s = _d(W["lora_scale"])[tt]
    return ((x @ _d(W["lora_down"]).T) * s) @ _d(W["lora_B"])


def recurrent_forward(cfg, W: dict, h0: torch.Tensor, e: torch.Tensor, batch: int, n_loops: int,
                      act_threshold: float, start_pos: int = 0,
                      halt_logit_offset: Optional[torch.Tensor] = None,
                      caches: Optional[list] = None, transformer_off: bool = False,
                      record: Optional[list] = None, halt_at: Optional[torch.Tensor] = None,
                      route_ids: Optional[torch.Tensor] = None):
    """RecurrentBlock.forward ("OpenMythos 분석", "Recurrent Block") for `batch`
    sequences of T = N / batch positions each.

    Per loop t: h_loop = h + emb_t; combined = RMSNorm_rec(h_loop + e);
    trans = Block(combined) (+ LoRA delta on the block output); h_new = A*h + B*e + trans;
    rows halted before loop t stay frozen; ACT weight w (remainder when cum + p >= thr or
    at the last loop, else p) accumulates h_out += w * h_new.  With act_threshold <= 0
    ACT is off and h_out = h after the last loop.

    caches: optional per-loop list of per-sequence attention caches (decode / prefix).
    transformer_off: debug switch, trans = 0 (the pure LTI recurrence).
    record: optional list that receives per-loop dicts (h_in, f, biased logits, ids, p, cum).
    halt_at: test hook, [N] int64: -1 lets the halting rule decide; t >= 0 makes position i
    halt at loop t (weight = the remainder there) whatever cum + p is.  Parity tests set it
    only where the rule's outcome is decided by rounding (cum + p within the measured
    arithmetic drift of the threshold), so both sides then follow the same discrete path.
    route_ids: test hook, [L, N, k] int64: the routes of loop t imposed on the rows with
    route_ids[t, i, 0] >= 0 (see router); the record keeps the router's own ids.
    Returns (h_out [N, D], halt_weights [L, N], expert_ids [L, N, k], new_kv per loop)."""
    h = _d(h0).clone()
    ev = _d(e)
    N, D = h.shape
    T = N // batch
    k = cfg.n_experts_per_tok
    A = lti_A(W["log_A"], W["log_dt"])
    Bv = _d(W["inj_B"])
    pos = torch.tensor([start_pos + (i % T) for i in range(N)], dtype=torch.int64)
    h_out = torch.zeros(N, D, dtype=F64)
    cum = torch.zeros(N, dtype=F64)
    halted = torch.zeros(N, dtype=torch.bool)
    act_on = act_threshold > 0
    halt_weights = torch.zeros(n_loops, N, dtype=F64)
    expert_ids = torch.full((n_loops, N, k), -1, dtype=torch.int64)
    new_kv = []
    for t in range(n_loops):
        running = ~halted
        emb = loop_embedding(t, cfg.loop_dim, D, cfg.loop_theta)
        combined = rmsnorm(h + emb + ev, W["rec_norm_w"], cfg.norm_eps)
        rec = {"h_in": h.clone()} if record is not None else None
        if transformer_off:
            trans = torch.zeros(N, D, dtype=F64)
            new_kv.append(None)
        else:
            trans, _, info = transformer_block(cfg, W, combined, batch, pos, True,
                                               None if caches is None else caches[t], running,
                                               None if route_ids is None else route_ids[t])
            trans = trans + lora_delta(cfg, W, trans, t)
            expert_ids[t] = info["ids"]
            new_kv.append(info["new_kv"])
            if rec is not None:
                rec.update(f=info["f"], biased=info["biased"], ids=info["ids"], own_ids=info["own_ids"])
        h_new = A * h + Bv * ev + trans
        h_new[halted] = h[halted]                      # frozen rows
        if act_on:
            z = h_new @ _d(W["halt_w"]) + _d(W["halt_b"])[0]
            if halt_logit_offset is not None:
                z = z + _d(halt_logit_offset)
            p = sigmoid(z)
            last = t == n_loops - 1
            stop = (cum + p >= act_threshold) | torch.tensor(last)
            if halt_at is not None:
                forced = halt_at >= 0
                stop = torch.where(forced, halt_at == t, stop) | torch.tensor(last)
            remainder = (1.0 - cum).clamp(min=0.0)
            w = torch.where(stop, remainder, p)
            w = torch.where(running, w, torch.zeros_like(w))
            cum = torch.where(running, cum + p, cum)
            halted = halted | (running & stop)
            if rec is not None:
                rec.update(p=p, cum=cum.clone())
        else:
            w = torch.full((N,), 1.0 if t == n_loops - 1 else 0.0, dtype=F64)
        halt_weights[t] = w
        h_out = h_out + w[:, None] * h_new
        h = h_new
        if rec is not None:
            rec["h_out"] = h_new.clone()
            record.append(rec)
    return h_out, halt_weights, expert_ids, new_kv


def dense_block_forward(cfg, W: dict, x: torch.Tensor, batch: int, start_pos: int = 0):
    """A prelude/coda TransformerBlock(use_moe=False) with a dense SwiGLU FFN."""
    N = x.shape[0]
    T = N // batch
    pos = torch.tensor([start_pos + (i % T) for i in range(N)], dtype=torch.int64)
    out, _, _ = transformer_block(cfg, W, _d(x), batch, pos, False)
    return out


def model_forward(cfg, MW: dict, ids: torch.Tensor, n_loops: int, act_threshold: float,
                  route_ids: Optional[torch.Tensor] = None, record: Optional[list] = None):
    """OpenMythos.forward ("OpenMythos 분석", "Core Structure") for ids [B, T]:
    logits = head(norm(coda(recurrent(prelude(embed(ids)), e)))).
    route_ids / record: passed to the recurrent block (test hooks, see recurrent_forward).
    Returns (logits [B, T, V], recurrent outputs tuple, e)."""
    B, T = ids.shape
    x = _d(MW["embed"])[ids.reshape(-1)]
    for W in MW["prelude"]:
        x = dense_block_forward(cfg, W, x, B)
    e = x.clone()
    rec = recurrent_forward(cfg, MW["recurrent"], x, e, B, n_loops, act_threshold, record=record,
                            route_ids=route_ids)
    x = rec[0]
    for W in MW["coda"]:
        x = dense_block_forward(cfg, W, x, B)
    logits = rmsnorm(x, MW["norm_w"], cfg.norm_eps) @ _d(MW["head"]).T
    return logits.reshape(B, T, -1), rec, e


def greedy(logits: torch.Tensor) -> torch.Tensor:
    """The most likely next token per row, ties to the lowest index (the pages print the
    generation loop but not its sampling rule; greedy is the plainest reading).
    torch.argmax returns the first maximal index."""
    return torch.argmax(logits, dim=-1)


def generate(cfg, MW: dict, prompt_ids: torch.Tensor, max_new_tokens: int, n_loops: int,
             act_threshold: float = 0.0):
    """OpenMythos.generate ("OpenMythos 분석", RoPE & generation cache), by its definition:
    every new token is the greedy choice from the last position of a full forward pass
    over all tokens so far.  No cache: the library's cached steps (prompt at start_pos 0,
    then one token at position prompt_len + step - 1) must reproduce this.
    Returns (ids [B, T0 + n] int64, step logits [n, B, V])."""
    ids = prompt_ids.clone().to(torch.int64)
    step_logits = []
    for _ in range(max_new_tokens):
        logits, _, _ = model_forward(cfg, MW, ids, n_loops, act_threshold)
        last = logits[:, -1]
        step_logits.append(last)
        ids = torch.cat([ids, greedy(last)[:, None]], dim=1)
    return ids, torch.stack(step_logits)


def decode_step(cfg, W: dict, h0: torch.Tensor, e: torch.Tensor, caches: list, cache_len: list,
                n_loops: int, act_threshold: float = 0.0, halt_logit_offset: Optional[torch.Tensor] = None):
    """One KV-cached decode step of the recurrent block ("OpenMythos 분석", "RoPE &
    generation cache"): one new token per sequence b at position cache_len[b]; loop t
    attends to its own loop cache (keys 0..cache_len[b]-1) plus the new token.
    caches[t][b] = {"k": [C_b, Hkv, hd], "v": ..., "pos": [C_b]} (GQA), or
    {"c_kv": [C_b, kv_lora_rank], "k_rope": [C_b, qk_rope_head_dim], "pos": [C_b]} (MLA).
    halt_logit_offset: optional [B], added to the halting logit (as in recurrent_forward).
    Returns (h_out [B, D], halt_weights [L, B], expert_ids [L, B, k], new_kv)."""
    B = h0.shape[0]
    h = _d(h0).clone()
    ev = _d(e)
    D = h.shape[1]
    k = cfg.n_experts_per_tok
    A = lti_A(W["log_A"], W["log_dt"])
    Bv = _d(W["inj_B"])
    h_out = torch.zeros(B, D, dtype=F64)
    cum = torch.zeros(B, dtype=F64)
    halted = torch.zeros(B, dtype=torch.bool)
    halt_weights = torch.zeros(n_loops, B, dtype=F64)
    expert_ids = torch.full((n_loops, B, k), -1, dtype=torch.int64)
    new_kv = []
    for t in range(n_loops):
        running = ~halted
        emb = loop_embedding(t, cfg.loop_dim, D, cfg.loop_theta)
        combined = rmsnorm(h + emb + ev, W["rec_norm_w"], cfg.norm_eps)
        a = rmsnorm(combined, W["attn_norm_w"], cfg.norm_eps)
        attn_out = torch.empty_like(h)
        kvs = []
        for b in range(B):
            pos = torch.tensor([cache_len[b]], dtype=torch.int64)
            o, k1, k2 = attention(cfg, W, a[b:b + 1], pos, caches[t][b])
            attn_out[b] = o[0]
            kvs.append((k1, k2))
        new_kv.append(kvs)
        x1 = combined + attn_out
        f = rmsnorm(x1, W["ffn_norm_w"], cfg.norm_eps)
        trans = x1.clone()
        rows = torch.nonzero(running, as_tuple=True)[0]
        if rows.numel():
            y, idx, g, _ = moe_ffn(cfg, W, f[rows])
            trans[rows] = x1[rows] + y
            expert_ids[t, rows] = idx
        trans = trans + lora_delta(cfg, W, trans, t)
        h_new = A * h + Bv * ev + trans
        h_new[halted] = h[halted]
        if act_threshold > 0:
            z = h_new @ _d(W["halt_w"]) + _d(W["halt_b"])[0]
            if halt_logit_offset is not None:
                z = z + _d(halt_logit_offset)
            p = sigmoid(z)
            stop = (cum + p >= act_threshold) | torch.tensor(t == n_loops - 1)
            w = torch.where(stop, (1.0 - cum).clamp(min=0.0), p)
            w = torch.where(running, w, torch.zeros_like(w))
            cum = torch.where(running, cum + p, cum)
            halted = halted | (running & stop)
        else:
            w = torch.full((B,), 1.0 if t == n_loops - 1 else 0.0, dtype=F64)
        halt_weights[t] = w
        h_out = h_out + w[:, None] * h_new
        h = h_new
    return h_out, halt_weights, expert_ids, new_kv


def _append_cache(cfg, cache: dict, kv, pos: int) -> dict:
    """A sequence's loop cache extended by one position's entries (as decode_step returns
    them: rotated key and value for GQA, c_kv and rotated k_rope for MLA)."""
    k1, k2 = kv
    p = torch.tensor([pos], dtype=torch.int64)
    if cfg.attn_type == "gqa":
        return {"k": torch.cat([_d(cache["k"]), k1], 0), "v": torch.cat([_d(cache["v"]), k2], 0),
                "pos": torch.cat([cache["pos"].to(torch.int64), p])}
    return {"c_kv": torch.cat([_d(cache["c_kv"]), k1], 0), "k_rope": torch.cat([_d(cache["k_rope"]), k2], 0),
            "pos": torch.cat([cache["pos"].to(torch.int64), p])}


def decode_tokens(cfg, W: dict, h0: torch.Tensor, e: torch.Tensor, caches: list, cache_len: list, n_loops: int,
                  act_threshold: float = 0.0, halt_logit_offset: Optional[torch.Tensor] = None):
    """S successive KV-cached decode steps of each of B sequences (GeekNews summary, section
    6: continuous depth-wise batching lets each token leave the shared block at its own
    depth and new tokens take its place; it computes exactly this).  Token n of sequence b
    sits at position cache_len[b] + n; each step runs decode_step on that sequence alone and
    then appends the step's keys / values of every loop -- the loops after the token halted
    included, from its frozen state -- to the sequence's loop caches, which the next token
    reads.  h0 [B, S, D], e [B, S, D], halt_logit_offset [B, S] or None; caches[t][b] as in
    decode_step (not modified).
    Returns (h_out [B, S, D], halt_weights [B, S, L], expert_ids [B, S, L, k])."""
    B, S, D = h0.shape
    k = cfg.n_experts_per_tok
    h_out = torch.zeros(B, S, D, dtype=F64)
    hw = torch.zeros(B, S, n_loops, dtype=F64)
    ids = torch.full((B, S, n_loops, k), -1, dtype=torch.int64)
    for b in range(B):
        seq_caches = [caches[t][b] for t in range(n_loops)]
        for n in range(S):
            off = None if halt_logit_offset is None else halt_logit_offset[b, n:n + 1]
            o_h, o_hw, o_ids, new_kv = decode_step(cfg, W, h0[b, n:n + 1], e[b, n:n + 1],
                                                   [[c] for c in seq_caches], [cache_len[b] + n], n_loops,
                                                   act_threshold, off)
            h_out[b, n], hw[b, n], ids[b, n] = o_h[0], o_hw[:, 0], o_ids[:, 0]
            seq_caches = [_append_cache(cfg, seq_caches[t], new_kv[t][0], cache_len[b] + n) for t in range(n_loops)]
    return h_out, hw, ids
