"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, brute force, library routines on special cases, and invariants the
pages fix.  CPU only (no GPU marker)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

import rdt_inputs as RI
from oracle import rdt_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F64 = torch.float64


def tiny_cfg(**kw):
    return RI.get_workload("tiny_gqa_fp32").cfg.replace(**kw)


def weights(cfg, seed=0, **kw):
    return RI.block_weights(cfg, seed, **kw)


# ------------------------------------------------------------------------------------------
# 1. LTI injection: closed form, fixed point, spectral radius
# ------------------------------------------------------------------------------------------

def test_lti_closed_form_and_fixed_point():
    """With the Transformer term off, h_t = a^t h0 + b e (1 - a^t) / (1 - a) per channel
    (README mirror, "동적 시스템 관점": h_{t+1} = A h_t + B e), converging to (I - A)^-1 B e."""
    cfg = tiny_cfg()
    W = weights(cfg)
    h0, e = RI.recurrent_inputs(cfg, 2, 8, 3)
    a = torch.exp(-torch.exp(W["log_A"].double()))          # log_dt = 0
    b = W["inj_B"].double()
    for L in (1, 5, 12):
        h, hw, ids, _ = O.recurrent_forward(cfg, W, h0, e, 2, L, 0.0, transformer_off=True)
        closed = a ** L * h0.double() + b * e.double() * (1 - a ** L) / (1 - a)
        assert torch.allclose(h, closed, rtol=0, atol=1e-12)
        assert hw[-1].eq(1).all() and hw[:-1].eq(0).all()
    h, *_ = O.recurrent_forward(cfg, W, h0, e, 2, 600, 0.0, transformer_off=True)
    Amat = np.diag(a.numpy())
    fixed = np.linalg.solve(np.eye(cfg.dim) - Amat, (b * e.double()).numpy().T).T
    assert np.abs(h.numpy() - fixed).max() < 1e-10


def test_spectral_radius_below_one():
    """rho(A) < 1 by construction (README mirror "해결책"; usage script prints rho(A));
    eigenvalues of diag(A) from a general eigen-solver, including the clamp edges."""
    cfg = tiny_cfg()
    W = weights(cfg)
    A = O.lti_A(W["log_A"], W["log_dt"]).numpy()
    rho = np.abs(np.linalg.eigvals(np.diag(A))).max()
    assert 0.5 <= rho <= 0.95 + 1e-12
    # clamp edges: log_dt + log_A <= -20 still gives A < 1 in fp64; >= 20 gives A -> 0
    edge = O.lti_A(torch.tensor([-40.0, -20.0, 0.0, 20.0, 40.0]), torch.zeros(1)).numpy()
    assert (np.abs(np.linalg.eigvals(np.diag(edge))) < 1).all()
    assert edge[3] == edge[4] and edge[0] == edge[1]


# ------------------------------------------------------------------------------------------
# 2. top-k against brute force, with ties
# ------------------------------------------------------------------------------------------

def _brute_topk(row, k):
    remaining = list(range(len(row)))
    out = []
    for _ in range(k):
        best = remaining[0]
        for j in remaining:
            if row[j] > row[best]:
                best = j
        out.append(best)
        remaining.remove(best)
    return out


@pytest.mark.parametrize("E,k", [(8, 2), (8, 8), (5, 3), (16, 4)])
def test_topk_matches_bruteforce_with_ties(E, k):
    g = torch.Generator().manual_seed(E * 10 + k)
    v = torch.randint(-3, 4, (64, E), generator=g).double()       # many ties
    got = O.topk_lower_index(v, k)
    for r in range(v.shape[0]):
        assert got[r].tolist() == _brute_topk(v[r].tolist(), k)


def test_router_gates_are_softmax_of_selected_logits():
    """Gates = scores[idx] renormalised = softmax restricted to the selected logits
    (zero bias), and the biased selection changes only the chosen set."""
    cfg = tiny_cfg()
    W = weights(cfg)
    f = torch.randn(32, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(1))
    idx, g, logits, _, _ = O.router(cfg, W, f)
    sel = torch.gather(logits, 1, idx)
    assert torch.allclose(g, torch.softmax(sel, -1), atol=1e-14)
    assert torch.allclose(g.sum(-1), torch.ones(32, dtype=F64), atol=1e-14)
    # all-expert brute force: the chosen set maximises the biased logit sum
    for r in range(8):
        best = max(itertools.combinations(range(cfg.n_experts), cfg.n_experts_per_tok),
                   key=lambda c: sum(logits[r, j].item() for j in c))
        assert set(best) == set(idx[r].tolist())


# ------------------------------------------------------------------------------------------
# 3. MoE special cases reduce to dense sums (library SiLU / linear)
# ------------------------------------------------------------------------------------------

def _lib_expert(w13, w2, x):
    F = w13.shape[0] // 2
    w13 = w13.double()
    return Fn.linear(Fn.silu(Fn.linear(x, w13[:F])) * Fn.linear(x, w13[F:]), w2.double())


def test_moe_all_experts_uniform_gates_is_dense_average():
    cfg = tiny_cfg(n_experts_per_tok=8)
    W = weights(cfg)
    W["w_router"] = torch.zeros_like(W["w_router"])
    f = torch.randn(12, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(2))
    y, idx, g, _ = O.moe_ffn(cfg, W, f)
    assert torch.allclose(g, torch.full_like(g, 1 / 8), atol=1e-15)
    want = sum(_lib_expert(W["w13"][e], W["w2"][e], f) for e in range(8)) / 8
    want = want + _lib_expert(W["w13"][8], W["w2"][8], f)
    assert torch.allclose(y, want, rtol=1e-12, atol=1e-14)


def test_moe_single_expert_is_plain_swiglu():
    cfg = tiny_cfg(n_experts=1, n_experts_per_tok=1, n_shared_experts=0)
    W = weights(cfg)
    f = torch.randn(9, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(3))
    y, idx, g, _ = O.moe_ffn(cfg, W, f)
    assert torch.equal(idx, torch.zeros_like(idx)) and torch.allclose(g, torch.ones_like(g))
    assert torch.allclose(y, _lib_expert(W["w13"][0], W["w2"][0], f), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------------------------------
# 4. norms, RoPE, attention against library routines; block reduction
# ------------------------------------------------------------------------------------------

def test_rmsnorm_matches_library():
    x = torch.randn(7, 64, dtype=F64, generator=torch.Generator().manual_seed(4))
    w = torch.rand(64, dtype=torch.float32, generator=torch.Generator().manual_seed(5))
    assert torch.allclose(O.rmsnorm(x, w, 1e-6), Fn.rms_norm(x, (64,), w.double(), 1e-6), atol=1e-14)


def _rope_complex(x, pos, theta):
    """RoPE as complex phasors: pairs (2m, 2m+1) times exp(i pos theta^(-2m/d))."""
    d = x.shape[-1]
    inv = theta ** (-torch.arange(0, d, 2, dtype=F64) / d)
    ph = torch.polar(torch.ones(len(pos), d // 2, dtype=F64), pos.double()[:, None] * inv[None])
    xc = torch.view_as_complex(x.reshape(*x.shape[:-1], d // 2, 2).contiguous())
    return torch.view_as_real(xc * ph[:, None, :]).reshape(x.shape)


def test_rope_is_complex_rotation_norm_preserving_relative():
    g = torch.Generator().manual_seed(6)
    x = torch.randn(10, 3, 32, dtype=F64, generator=g)
    pos = torch.arange(10) * 7 + 3
    r = O.rope(x, pos, 10000.0)
    assert torch.allclose(r, _rope_complex(x, pos, 10000.0), atol=1e-12)
    assert torch.allclose(r.norm(dim=-1), x.norm(dim=-1), atol=1e-12)
    q = torch.randn(1, 1, 32, dtype=F64, generator=g)
    k = torch.randn(1, 1, 32, dtype=F64, generator=g)
    dots = []
    for m, n in [(5, 2), (13, 10), (103, 100)]:
        qm = O.rope(q, torch.tensor([m]), 10000.0)
        kn = O.rope(k, torch.tensor([n]), 10000.0)
        dots.append((qm * kn).sum().item())
    assert abs(dots[0] - dots[1]) < 1e-12 and abs(dots[0] - dots[2]) < 1e-12


@pytest.mark.parametrize("Hkv", [2, 8])
def test_gqa_attention_matches_sdpa(Hkv):
    cfg = tiny_cfg(n_kv_heads=Hkv)
    W = weights(cfg, attn_std=0.1)
    T = 11
    a = torch.randn(T, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(7))
    pos = torch.arange(T)
    o, k_new, v_new = O.gqa_attention(cfg, W, a, pos)
    H, hd = cfg.n_heads, cfg.head_dim
    qkv = Fn.linear(a, W["w_qkv"].double())
    q = _rope_complex(qkv[:, :H * hd].reshape(T, H, hd), pos, 10000.0)
    k = _rope_complex(qkv[:, H * hd:(H + Hkv) * hd].reshape(T, Hkv, hd), pos, 10000.0)
    v = qkv[:, (H + Hkv) * hd:].reshape(T, Hkv, hd)
    rep = H // Hkv
    att = Fn.scaled_dot_product_attention(q.transpose(0, 1), k.repeat_interleave(rep, 1).transpose(0, 1),
                                          v.repeat_interleave(rep, 1).transpose(0, 1), is_causal=True)
    want = Fn.linear(att.transpose(0, 1).reshape(T, H * hd), W["w_o"].double())
    assert torch.allclose(o, want, atol=1e-12)


def test_attention_single_token_is_wo_wv():
    """T = 1: the softmax over one key is 1, so attention = Wo Wv a."""
    cfg = tiny_cfg()
    W = weights(cfg)
    a = torch.randn(1, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(8))
    o, _, _ = O.gqa_attention(cfg, W, a, torch.tensor([5]))
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    v = (a @ W["w_qkv"].double()[(H + Hkv) * hd:].T).reshape(Hkv, hd)
    heads = torch.cat([v[h // (H // Hkv)] for h in range(H)])
    assert torch.allclose(o[0], W["w_o"].double() @ heads, atol=1e-13)


def test_block_reduction_one_loop_no_injection():
    """n_loops = 1, A = 0, B = 0, LoRA B = 0: h_1 = Block(RMSNorm_rec(h0 + emb_0 + e))."""
    cfg = tiny_cfg()
    W = weights(cfg)
    W["log_A"] = torch.full_like(W["log_A"], 30.0)        # clamp(30) -> 20 -> A = exp(-exp(20)) = 0
    W["inj_B"] = torch.zeros_like(W["inj_B"])
    W["lora_B"] = torch.zeros_like(W["lora_B"])
    assert O.lti_A(W["log_A"], W["log_dt"]).abs().max() == 0
    h0, e = RI.recurrent_inputs(cfg, 2, 6, 9)
    h1, *_ = O.recurrent_forward(cfg, W, h0, e, 2, 1, 0.0)
    emb0 = torch.zeros(cfg.dim, dtype=F64)
    emb0[cfg.loop_dim // 2:cfg.loop_dim] = 1.0                # sin(0) = 0, cos(0) = 1
    x = Fn.rms_norm(h0.double() + emb0 + e.double(), (cfg.dim,), W["rec_norm_w"].double(), 1e-6)
    pos = torch.arange(12) % 6
    blk, _, _ = O.transformer_block(cfg, W, x, 2, pos, True)
    assert torch.allclose(h1, blk, atol=1e-13)


# ------------------------------------------------------------------------------------------
# 5. causality
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("attn", ["gqa", "mla"])
def test_causality_prefix_unchanged(attn):
    """Perturbing positions > i leaves every output at positions <= i unchanged: ids
    and halting weights exactly, states to fp64 rounding (BLAS blocks row sets of
    different sizes differently, so last-bit equality is not a property of the oracle)."""
    wl = RI.get_workload("tiny_gqa_fp32" if attn == "gqa" else "tiny_mla_fp32")
    cfg = wl.cfg
    W = weights(cfg, seed=1, attn_std=0.1, halt_w_std=0.2)
    T = 10
    h0, e = RI.recurrent_inputs(cfg, 1, T, 11)
    out1 = O.recurrent_forward(cfg, W, h0, e, 1, 3, 0.99)
    h0b, eb = h0.clone(), e.clone()
    h0b[6:] += 1.0
    eb[6:] -= 0.5
    out2 = O.recurrent_forward(cfg, W, h0b, eb, 1, 3, 0.99)
    assert torch.allclose(out1[0][:6], out2[0][:6], rtol=0, atol=1e-12)
    assert torch.allclose(out1[1][:, :6], out2[1][:, :6], rtol=0, atol=1e-14)
    assert torch.equal(out1[2][:, :6], out2[2][:, :6])
    assert not torch.equal(out1[0][6:], out2[0][6:])


# ------------------------------------------------------------------------------------------
# 6. ACT
# ------------------------------------------------------------------------------------------

def test_act_weights_sum_to_one_and_halted_rows_freeze():
    wl = RI.get_workload("tiny_mla_fp32")
    cfg = wl.cfg
    W = weights(cfg, seed=1, halt_w_std=0.3)
    h0, e = RI.recurrent_inputs(cfg, 2, 16, 12)
    rec = []
    h_out, hw, ids, _ = O.recurrent_forward(cfg, W, h0, e, 2, 8, 0.99, record=rec)
    assert torch.allclose(hw.sum(0), torch.ones(32, dtype=F64), atol=1e-12)
    assert (hw >= 0).all()
    for i in range(32):
        nz = torch.nonzero(hw[:, i] > 0).flatten()
        last = int(nz.max())
        # after the halting loop: frozen state, no routing, zero weight
        for t in range(last + 1, 8):
            assert torch.equal(rec[t]["h_out"][i], rec[last]["h_out"][i])
            assert (ids[t, i] == -1).all() and hw[t, i] == 0
        # before and at the halting loop: routed
        assert (ids[: last + 1, i] >= 0).all()


def test_act_closed_form_constant_halting_probability():
    """Zero halting weight and constant p = sigmoid(b): position halts at loop
    t* = ceil(thr / p) - 1 and h_out = sum_{t<t*} p h_{t+1} + (1 - t* p) h_{t*+1},
    with h_t the LTI closed form (Transformer term off)."""
    cfg = tiny_cfg()
    W = weights(cfg)
    W["halt_w"] = torch.zeros_like(W["halt_w"])
    W["halt_b"] = torch.tensor([-1.1])                     # stored fp32, as the kernel reads it
    b = float(W["halt_b"][0])
    p = 1 / (1 + math.exp(-b))
    thr = 0.99
    tstar = math.ceil(thr / p) - 1
    L = tstar + 3
    h0, e = RI.recurrent_inputs(cfg, 1, 5, 13)
    h_out, hw, _, _ = O.recurrent_forward(cfg, W, h0, e, 1, L, thr, transformer_off=True)
    a = torch.exp(-torch.exp(W["log_A"].double()))
    bv = W["inj_B"].double() * e.double()
    hs = [a ** t * h0.double() + bv * (1 - a ** t) / (1 - a) for t in range(L + 1)]
    want = sum(p * hs[t + 1] for t in range(tstar)) + (1 - tstar * p) * hs[tstar + 1]
    assert torch.allclose(h_out, want, atol=1e-12)
    assert torch.allclose(hw[tstar], torch.full((5,), 1 - tstar * p, dtype=F64), atol=1e-14)
    assert (hw[tstar + 1:] == 0).all()


def test_halting_spread_recipe_halts_at_drawn_loop():
    cfg = tiny_cfg()
    W = weights(cfg)
    W["halt_w"] = torch.zeros_like(W["halt_w"])
    W["halt_b"] = torch.zeros(1)
    n = 40
    off, kk = RI.halting_offsets_spread(n, 4, 24, 0.9, 4)
    h0, e = RI.recurrent_inputs(cfg, 1, n, 14)
    _, hw, _, _ = O.recurrent_forward(cfg, W, h0, e, 1, 24, 0.9, halt_logit_offset=off,
                                      transformer_off=True)
    last = torch.tensor([int(torch.nonzero(hw[:, i] > 0).max()) for i in range(n)])
    assert torch.equal(last + 1, kk)


# ------------------------------------------------------------------------------------------
# 7. parameter count; golden shapes from the pages
# ------------------------------------------------------------------------------------------

def _count(w):
    if isinstance(w, list):
        return sum(_count(x) for x in w)
    return sum(v.numel() for k, v in w.items() if k != "router_bias" and not isinstance(v, list)) + \
        sum(_count(v) for v in w.values() if isinstance(v, list))


@pytest.mark.parametrize("name", ["tiny_gqa_fp32", "tiny_mla_fp32"])
def test_param_count_matches_formula(name):
    cfg = RI.get_workload(name).cfg
    MW = RI.model_weights(cfg, 0)
    assert _count(MW["recurrent"]) == RI.param_count_formula(cfg)
    total = _count(MW["recurrent"]) + _count(MW["prelude"]) + _count(MW["coda"]) + \
        MW["embed"].numel() + MW["head"].numel() + MW["norm_w"].numel()
    assert total == RI.param_count_formula(cfg, full_model=True)
    if name == "tiny_gqa_fp32":
        assert total == 1978658


def test_usage_script_shapes_and_variants():
    gold = json.load(open(os.path.join(GOLDEN, "usage_script.json")))
    for attn in ("gqa", "mla"):
        wl = RI.get_workload("tiny_gqa_fp32" if attn == "gqa" else "tiny_mla_fp32")
        for key, val in {**gold["base"], **gold[attn]}.items():
            assert getattr(wl.cfg, key) == val, key
    cfg = RI.get_workload("tiny_gqa_fp32").cfg
    MW = RI.model_weights(cfg, 0)
    ids = torch.randint(0, cfg.vocab_size, tuple(gold["ids_shape"]), generator=torch.Generator().manual_seed(0))
    logits, _, _ = O.model_forward(cfg, MW, ids, gold["forward_n_loops"], 0.0)
    assert list(logits.shape) == gold["logits_shape"]
    var = json.load(open(os.path.join(GOLDEN, "variants_table.json")))
    for wname, vname in [("rdt1b_prefill", "mythos_1b"), ("rdt3b_decode", "mythos_3b"),
                         ("rdt10b_prefill_zipf", "mythos_10b")]:
        c, v = RI.get_workload(wname).cfg, var[vname]
        assert (c.dim, c.n_experts, c.expert_dim, c.max_loop_iters) == \
            (v["dim"], v["n_experts"], v["expert_dim"], v["loop_iters"])


# ------------------------------------------------------------------------------------------
# 8. extras: LoRA clamp, loop embedding, decode == prefill, MLA absorbed form
# ------------------------------------------------------------------------------------------

def test_lora_scale_reused_past_max_loop_iters():
    cfg = tiny_cfg()
    W = weights(cfg, lora_scale_std=1.0)
    x = torch.randn(4, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(15))
    last = O.lora_delta(cfg, W, x, cfg.max_loop_iters - 1)
    for t in (cfg.max_loop_iters, cfg.max_loop_iters + 5):
        assert torch.equal(O.lora_delta(cfg, W, x, t), last)
    assert not torch.equal(O.lora_delta(cfg, W, x, 0), last)


def test_loop_embedding_values():
    e0 = O.loop_embedding(0, 32, 256, 10000.0)
    assert e0[:16].eq(0).all() and e0[16:32].eq(1).all() and e0[32:].eq(0).all()
    e3 = O.loop_embedding(3, 32, 256, 10000.0)
    assert abs(e3[0].item() - math.sin(3.0)) < 1e-15 and abs(e3[16].item() - math.cos(3.0)) < 1e-15
    assert abs(e3[1].item() - math.sin(3.0 * 10000 ** (-2 / 32))) < 1e-15
    assert torch.allclose(e3[:16] ** 2 + e3[16:32] ** 2, torch.ones(16, dtype=F64))


@pytest.mark.parametrize("act", [0.0, 0.99])
def test_decode_step_equals_prefill_of_one_more_token(act):
    """Prefill of T+1 tokens == prefill of T tokens (filling one cache per loop) followed
    by one decode step at position T ("OpenMythos 분석", "RoPE & generation cache")."""
    cfg = tiny_cfg()
    W = weights(cfg, seed=2, attn_std=0.1, halt_w_std=0.3)
    B, T, L = 2, 7, 4
    h0, e = RI.recurrent_inputs(cfg, B, T + 1, 16)
    full = O.recurrent_forward(cfg, W, h0, e, B, L, act)
    keep = torch.tensor([b * (T + 1) + i for b in range(B) for i in range(T)])
    pre = O.recurrent_forward(cfg, W, h0[keep], e[keep], B, L, act)
    caches = [[{"k": pre[3][t][b][0], "v": pre[3][t][b][1], "pos": torch.arange(T)} for b in range(B)]
              for t in range(L)]
    last = torch.tensor([b * (T + 1) + T for b in range(B)])
    dec = O.decode_step(cfg, W, h0[last], e[last], caches, [T] * B, L, act)
    assert torch.allclose(dec[0], full[0][last], atol=1e-12)
    assert torch.allclose(dec[1], full[1][:, last], atol=1e-12)
    assert torch.equal(dec[2], full[2][:, last])


@pytest.mark.parametrize("act", [0.0, 0.99])
def test_mla_decode_from_latent_cache_equals_prefill(act):
    """MLA: a decode step that reads only the latent cache (c_kv, k_rope) of the T earlier
    positions gives the prefill of T+1 tokens ("OpenMythos 분석", MLA: the cache holds the
    latent; "RoPE & generation cache")."""
    cfg = RI.get_workload("tiny_mla_fp32").cfg
    W = weights(cfg, seed=4, attn_std=0.1, halt_w_std=0.3)
    B, T, L = 2, 6, 5
    h0, e = RI.recurrent_inputs(cfg, B, T + 1, 17)
    full = O.recurrent_forward(cfg, W, h0, e, B, L, act)
    keep = torch.tensor([b * (T + 1) + i for b in range(B) for i in range(T)])
    pre = O.recurrent_forward(cfg, W, h0[keep], e[keep], B, L, act)
    caches = [[{"c_kv": pre[3][t][b][0], "k_rope": pre[3][t][b][1], "pos": torch.arange(T)} for b in range(B)]
              for t in range(L)]
    assert caches[0][0]["c_kv"].shape == (T, cfg.kv_lora_rank)
    assert caches[0][0]["k_rope"].shape == (T, cfg.qk_rope_head_dim)
    last = torch.tensor([b * (T + 1) + T for b in range(B)])
    dec = O.decode_step(cfg, W, h0[last], e[last], caches, [T] * B, L, act)
    assert torch.allclose(dec[0], full[0][last], atol=1e-12)
    assert torch.allclose(dec[1], full[1][:, last], atol=1e-12)
    assert torch.equal(dec[2], full[2][:, last])


def test_mla_absorbed_form_matches():
    """Scores via the absorbed form q_nope^T (W_uk c_kv) == q_nope . k_nope (DeepSeek-V2)."""
    wl = RI.get_workload("tiny_mla_fp32")
    cfg = wl.cfg
    W = weights(cfg, seed=3, attn_std=0.1)
    T = 9
    a = torch.randn(T, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(17))
    pos = torch.arange(T)
    o, c_kv, k_rope = O.mla_attention(cfg, W, a, pos)
    H, dn, dr, dv = cfg.n_heads, cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
    cq = Fn.rms_norm(a @ W["w_q_down"].double().T, (cfg.q_lora_rank,), W["q_norm_w"].double(), 1e-6)
    q = (cq @ W["w_q_up"].double().T).reshape(T, H, dn + dr)
    qr = _rope_complex(q[..., dn:].contiguous(), pos, 10000.0)
    ckn = Fn.rms_norm(c_kv, (cfg.kv_lora_rank,), W["kv_norm_w"].double(), 1e-6)
    Wkvu = W["w_kv_up"].double().reshape(H, dn + dv, cfg.kv_lora_rank)
    outs = []
    for h in range(H):
        q_abs = q[:, h, :dn] @ Wkvu[h, :dn]                    # [T, kv_lora]
        s = (q_abs @ ckn.T + qr[:, h] @ k_rope.T) / math.sqrt(dn + dr)
        s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
        p = torch.softmax(s, -1)
        outs.append((p @ ckn) @ Wkvu[h, dn:].T)                # absorbed value path
    want = torch.cat(outs, -1) @ W["w_o"].double().T
    assert torch.allclose(o, want, atol=1e-12)


def test_router_bias_selects_but_does_not_weight():
    """router_bias changes only the selection; gates come from the unbiased scores
    ("OpenMythos 분석", MoE section)."""
    cfg = tiny_cfg()
    W = weights(cfg)
    W["router_bias"] = torch.tensor([0, 0, 0, 0, 0, 50.0, 0, 40.0])   # force experts 5 and 7
    f = torch.randn(16, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(18))
    idx, g, logits, _, _ = O.router(cfg, W, f)
    assert (idx[:, 0] == 5).all() and (idx[:, 1] == 7).all()
    sc = torch.softmax(Fn.linear(f, W["w_router"].double()), -1)[:, [5, 7]]
    assert torch.allclose(g, sc / sc.sum(-1, keepdim=True), atol=1e-14)


def test_lora_acts_on_block_output():
    """trans_out + lora(trans_out, t) ("OpenMythos 분석", Recurrent Block): with A = 0,
    B = 0 and one loop, h_1 = T + (T Wd^T * scale[0]) B_lora, T the block output."""
    cfg = tiny_cfg()
    W = weights(cfg, lora_scale_std=1.0)
    W["log_A"] = torch.full_like(W["log_A"], 30.0)
    W["inj_B"] = torch.zeros_like(W["inj_B"])
    h0, e = RI.recurrent_inputs(cfg, 1, 6, 19)
    h1, *_ = O.recurrent_forward(cfg, W, h0, e, 1, 1, 0.0)
    emb0 = torch.zeros(cfg.dim, dtype=F64)
    emb0[cfg.loop_dim // 2:cfg.loop_dim] = 1.0
    x = Fn.rms_norm(h0.double() + emb0 + e.double(), (cfg.dim,), W["rec_norm_w"].double(), 1e-6)
    Tb, _, _ = O.transformer_block(cfg, W, x, 1, torch.arange(6), True)
    z = Fn.linear(Tb, W["lora_down"].double()) * W["lora_scale"].double()[0]
    want = Tb + z @ W["lora_B"].double()
    assert torch.allclose(h1, want, atol=1e-13)
    assert (want - Tb).abs().max() > 1e-3      # the delta is visible at this scale


def test_mla_latent_cache_entries():
    """c_kv = first kv_lora_rank outputs of kv_down; k_rope = the rest, rotated once
    and shared by all heads ("OpenMythos 분석", MLA section)."""
    cfg = RI.get_workload("tiny_mla_fp32").cfg
    W = weights(cfg, seed=3, attn_std=0.1)
    T = 9
    a = torch.randn(T, cfg.dim, dtype=F64, generator=torch.Generator().manual_seed(20))
    _, c_kv, k_rope = O.mla_attention(cfg, W, a, torch.arange(T) + 4)
    kv_raw = Fn.linear(a, W["w_kv_down"].double())
    assert torch.allclose(c_kv, kv_raw[:, :cfg.kv_lora_rank], atol=1e-15)
    want = _rope_complex(kv_raw[:, None, cfg.kv_lora_rank:].contiguous(), torch.arange(T) + 4, 10000.0)[:, 0]
    assert torch.allclose(k_rope, want, atol=1e-13)


# 9. generation
def test_generate_is_causally_consistent():
    """Causality makes a greedy generation checkable in one pass: the forward pass over the
    final sequence has, at each position T0 - 1 + s, the logits of step s and the token
    generated at step s as its argmax (a wrong start position, a non-causal mask or an
    off-by-one in the loop fails this)."""
    wl = RI.get_workload("tiny_gqa_fp32")
    cfg = wl.cfg
    MW = RI.model_weights(cfg, 3)
    prompt = torch.randint(0, cfg.vocab_size, (2, 6), generator=torch.Generator().manual_seed(4))
    ids, step_logits = O.generate(cfg, MW, prompt, 4, n_loops=3)
    assert torch.equal(ids[:, :6], prompt)
    full, _, _ = O.model_forward(cfg, MW, ids[:, :-1], 3, 0.0)
    for s in range(4):
        assert torch.allclose(full[:, 5 + s], step_logits[s], atol=1e-10)
        assert torch.equal(torch.argmax(full[:, 5 + s], -1), ids[:, 6 + s])


def test_greedy_ties_go_to_the_lowest_index():
    x = torch.tensor([[0.5, 2.0, 2.0, -1.0], [3.0, 3.0, 3.0, 3.0]], dtype=torch.float64)
    assert O.greedy(x).tolist() == [1, 0]


# ------------------------------------------------------------------------------------------
# 10. model composition ("OpenMythos 분석", Core Structure): embed -> prelude -> e = x ->
#     recurrent block -> coda -> head(norm(x)).  A block whose attention output projection
#     is zero reduces to x + FFN(RMSNorm(x)); with its FFN down-projection zero too it is
#     the identity.  The reduced blocks and the final norm / head are written with library
#     routines, and the recurrent block is the (separately pinned) oracle block.
# ------------------------------------------------------------------------------------------

def _ffn_only(W):
    """Zero the attention output projection: the block becomes x + FFN(RMSNorm(x))."""
    return {**W, "w_o": torch.zeros_like(W["w_o"])}


def _identity(W):
    return {**_ffn_only(W), "w2": torch.zeros_like(W["w2"])}


def _lib_ffn_block(W, x, eps):
    f = Fn.rms_norm(x, (x.shape[-1],), W["ffn_norm_w"].double(), eps)
    return x + _lib_expert(W["w13"][0], W["w2"][0], f)


def _model_case(prelude_layers, coda_layers, seed=5):
    cfg = tiny_cfg(prelude_layers=prelude_layers, coda_layers=coda_layers)
    MW = RI.model_weights(cfg, seed, halt_w_std=0.2)
    ids = torch.randint(0, cfg.vocab_size, (2, 7), generator=torch.Generator().manual_seed(seed))
    return cfg, MW, ids


def _lib_head(cfg, MW, x):
    return Fn.linear(Fn.rms_norm(x, (cfg.dim,), MW["norm_w"].double(), cfg.norm_eps), MW["head"].double())


def test_model_forward_with_identity_blocks_is_head_of_norm_of_recurrent():
    cfg, MW, ids = _model_case(1, 1)
    MW = {**MW, "prelude": [_identity(W) for W in MW["prelude"]], "coda": [_identity(W) for W in MW["coda"]]}
    L, thr = 3, 0.99
    logits, rec, e = O.model_forward(cfg, MW, ids, L, thr)
    x = Fn.embedding(ids.reshape(-1), MW["embed"].double())
    assert torch.equal(e, x)                                  # e is the (identity) prelude's output
    want_rec = O.recurrent_forward(cfg, MW["recurrent"], x, x, 2, L, thr)
    assert torch.allclose(rec[0], want_rec[0], rtol=0, atol=0) and torch.equal(rec[2], want_rec[2])
    want = _lib_head(cfg, MW, want_rec[0]).reshape(2, 7, -1)
    assert torch.allclose(logits, want, rtol=1e-12, atol=1e-13)


def test_model_forward_prelude_layers_in_order_and_e_after_the_prelude():
    cfg, MW, ids = _model_case(2, 1)
    MW = {**MW, "prelude": [_ffn_only(W) for W in MW["prelude"]], "coda": [_identity(W) for W in MW["coda"]]}
    L, thr = 2, 0.0
    logits, rec, e = O.model_forward(cfg, MW, ids, L, thr)
    x = Fn.embedding(ids.reshape(-1), MW["embed"].double())
    for W in MW["prelude"]:                                   # layer 0, then layer 1
        x = _lib_ffn_block(W, x, cfg.norm_eps)
    assert torch.allclose(e, x, rtol=1e-12, atol=1e-13)
    want_rec = O.recurrent_forward(cfg, MW["recurrent"], x, x, 2, L, thr)
    assert torch.allclose(rec[0], want_rec[0], rtol=1e-10, atol=1e-12)
    assert torch.allclose(logits, _lib_head(cfg, MW, want_rec[0]).reshape(2, 7, -1), rtol=1e-10, atol=1e-11)
    # the layers do not commute: the other order gives another e
    y = Fn.embedding(ids.reshape(-1), MW["embed"].double())
    for W in reversed(MW["prelude"]):
        y = _lib_ffn_block(W, y, cfg.norm_eps)
    assert (y - x).abs().max() > 1e-6


def test_model_forward_coda_layers_after_the_recurrent_block():
    cfg, MW, ids = _model_case(1, 2)
    MW = {**MW, "prelude": [_identity(W) for W in MW["prelude"]], "coda": [_ffn_only(W) for W in MW["coda"]]}
    L, thr = 3, 0.99
    logits, rec, e = O.model_forward(cfg, MW, ids, L, thr)
    x = Fn.embedding(ids.reshape(-1), MW["embed"].double())
    h = O.recurrent_forward(cfg, MW["recurrent"], x, x, 2, L, thr)[0]
    for W in MW["coda"]:
        h = _lib_ffn_block(W, h, cfg.norm_eps)
    assert torch.allclose(logits, _lib_head(cfg, MW, h).reshape(2, 7, -1), rtol=1e-10, atol=1e-11)
    # coda before the recurrent block would give other logits
    z = x
    for W in MW["coda"]:
        z = _lib_ffn_block(W, z, cfg.norm_eps)
    z = O.recurrent_forward(cfg, MW["recurrent"], z, x, 2, L, thr)[0]
    assert (_lib_head(cfg, MW, z).reshape(2, 7, -1) - logits).abs().max() > 1e-6


# ------------------------------------------------------------------------------------------
# 11. successive decode steps (what continuous depth-wise batching computes) equal the
#     prefill of the token block over the same cache prefix (causality: "OpenMythos 분석",
#     RoPE & generation cache), with tokens halting at different depths (ACT)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("attn", ["gqa", "mla"])
def test_decode_tokens_equal_prefill_of_the_token_block(attn):
    name = "tiny_gqa_fp32" if attn == "gqa" else "tiny_mla_fp32"
    cfg = RI.get_workload(name).cfg
    W = RI.block_weights(cfg, 8, attn_std=0.08, halt_w_std=0.0, halt_b=0.0)
    B, C, S, L, thr = 2, 5, 4, 6, 0.99
    g = torch.Generator().manual_seed(8)
    caches = []
    for t in range(L):
        per_seq = []
        for b in range(B):
            if attn == "gqa":
                per_seq.append({"k": torch.randn(C, cfg.n_kv_heads, cfg.head_dim, generator=g, dtype=F64),
                                "v": torch.randn(C, cfg.n_kv_heads, cfg.head_dim, generator=g, dtype=F64),
                                "pos": torch.arange(C)})
            else:
                per_seq.append({"c_kv": torch.randn(C, cfg.kv_lora_rank, generator=g, dtype=F64),
                                "k_rope": torch.randn(C, cfg.qk_rope_head_dim, generator=g, dtype=F64),
                                "pos": torch.arange(C)})
        caches.append(per_seq)
    h0, e = RI.recurrent_inputs(cfg, B, S, 8)
    off, kk = RI.halting_offsets_spread(B * S, 2, L, thr, 8)      # token i halts after kk[i] loops
    D = cfg.dim
    got_h, got_hw, got_ids = O.decode_tokens(cfg, W, h0.view(B, S, D), e.view(B, S, D), caches, [C] * B, L, thr,
                                             off.view(B, S))
    want_h, want_hw, want_ids, _ = O.recurrent_forward(cfg, W, h0, e, B, L, thr, start_pos=C,
                                                       halt_logit_offset=off, caches=caches)
    assert torch.allclose(got_h.reshape(B * S, D), want_h, rtol=1e-10, atol=1e-11)
    assert torch.allclose(got_hw.reshape(B * S, L).T, want_hw, rtol=0, atol=1e-12)
    assert torch.equal(got_ids.reshape(B * S, L, -1).transpose(0, 1), want_ids)
    # the halting spread: token i's last non-zero weight is at loop kk[i] - 1
    last = ((got_hw.reshape(B * S, L) > 0).to(torch.int64) * torch.arange(L)).max(-1).values
    assert torch.equal(last + 1, kk) and len(set(kk.tolist())) > 1
