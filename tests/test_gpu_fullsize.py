"""Full-size GPU runs in the launch configuration bench.py times, checked on outputs the
oracle can compute (a causal prefix slice, single decode sequences) and on properties
that hold at any size (halting loops, id ranges, causality, finiteness)."""
import math

import pytest
import torch

import rdt_inputs as RI
from oracle import rdt_oracle as O
from tests._helpers import (BF16_TOL, ID_MARGIN, check_route_flips, halting_loop, rel_l2, teacher_forced_ids,
                            topk_margin)

pytestmark = pytest.mark.gpu

R = pytest.importorskip("recurrent_depth_moe_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    R.load_library()


def _cpu(w):
    return {k: v.cpu() for k, v in w.items()}


def test_rdt1b_prefill_prefix_slice_matches_oracle():
    """1B-shaped prefill at full size (4 x 4096, 16 loops): rows 0..63 of sequence 0 against
    the oracle run on that causal prefix alone (exact: attention is causal, the MoE has
    no capacity coupling, ACT is per position)."""
    wl = RI.get_workload("rdt1b_prefill")
    cfg, B, T, L = wl.cfg, wl.batch, wl.seq, wl.n_loops
    dev = torch.device("cuda")
    W = RI.block_weights(cfg, wl.seed, device=dev, halt_b=wl.halt_b)
    h0, e = RI.recurrent_inputs(cfg, B, T, wl.seed, device=dev)
    blk = R.RecurrentBlock(cfg, W)
    P = 64
    tr = R.Trace.alloc(cfg, L, 0, P)
    h_out, hw, ids = blk.forward(h0, e, B, T, L, wl.act_threshold, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    Wc = _cpu(W)
    # the oracle takes the GPU's routes where they differ from its own by a near-tie that the
    # row's logit drift explains (check_route_flips), so both follow one discrete path
    rec = []
    o_h, o_hw, o_ids, _ = O.recurrent_forward(cfg, Wc, h0[:P].cpu(), e[:P].cpu(), 1, L, wl.act_threshold,
                                              record=rec, route_ids=ids[:, :P].cpu().long())
    check_route_flips(ids[:, :P], tr.biased_logits, rec)
    assert rel_l2(h_out[:P], o_h) <= BF16_TOL
    n, bad, skipped = teacher_forced_ids(cfg, Wc, tr, ids, L)
    assert n > 0 and bad == 0, f"{bad} of {n} teacher-forced rows differ ({skipped} near-ties skipped)"
    assert torch.isfinite(h_out).all()
    ids_c, hw_c = ids.cpu(), hw.cpu()
    last = ((hw_c > 0).to(torch.int64) * torch.arange(L)[:, None]).max(dim=0).values
    after = torch.arange(L)[:, None] > last[None, :]
    assert ((ids_c[~after] >= 0) & (ids_c[~after] < cfg.n_experts)).all() and (ids_c[after] == -1).all()
    assert (last == L - 1).float().mean() > 0.99             # halting bias -30: nearly every row runs 16 loops


def test_rdt1b_attention_late_key_tiles():
    """Prefill attention at the 1B shape in the launch configuration the benchmark times
    (4 x 4096, 16 heads, head dim 128): the last 128 query rows of sequence 0 attend to all
    32 key tiles, so the online softmax rescales across every tile.  One loop, checked on
    the attention branch of f = RMSNorm_ffn(x + Attn(RMSNorm_attn(x))): f minus
    RMSNorm_ffn(x), in the kernel's trace and in the oracle (peaky attention, std 0.04)."""
    wl = RI.get_workload("rdt1b_prefill")
    cfg, B, T = wl.cfg, wl.batch, wl.seq
    dev = torch.device("cuda")
    W = RI.block_weights(cfg, wl.seed, device=dev, halt_b=wl.halt_b, attn_std=0.04)
    h0, e = RI.recurrent_inputs(cfg, B, T, wl.seed, device=dev)
    blk = R.RecurrentBlock(cfg, W)
    Q = 128
    tr = R.Trace(T - Q, Q, f=torch.zeros(1, Q, cfg.dim, dtype=torch.float32, device=dev))
    blk.forward(h0, e, B, T, 1, wl.act_threshold, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    Wc = {k: W[k].cpu() for k in ("rec_norm_w", "attn_norm_w", "ffn_norm_w", "w_qkv", "w_o")}
    eps = cfg.norm_eps
    emb = O.loop_embedding(0, cfg.loop_dim, cfg.dim, cfg.loop_theta)
    comb = O.rmsnorm(h0[:T].cpu().double() + emb + e[:T].cpu().double(), Wc["rec_norm_w"], eps)
    a = O.rmsnorm(comb, Wc["attn_norm_w"], eps)
    pos = torch.arange(T)
    # rotated keys and values of positions 0 .. T - Q - 1 (the oracle's own, chunk by chunk:
    # a position's key and value depend on its row alone), then the last Q queries through
    # the oracle's cached-keys path
    ks, vs = [], []
    for c0 in range(0, T - Q, 128):
        _, kc, vc = O.gqa_attention(cfg, Wc, a[c0:c0 + 128], pos[c0:c0 + 128])
        ks.append(kc)
        vs.append(vc)
    cache = {"k": torch.cat(ks), "v": torch.cat(vs), "pos": pos[:T - Q]}
    o, _, _ = O.gqa_attention(cfg, Wc, a[T - Q:], pos[T - Q:], cache)
    f_o = O.rmsnorm(comb[T - Q:] + o, Wc["ffn_norm_w"], eps)
    f0 = O.rmsnorm(comb[T - Q:], Wc["ffn_norm_w"], eps)
    d_o = f_o - f0
    d_k = tr.f[0].cpu().double() - f0
    assert rel_l2(d_o, f_o) > 0.05, "attention barely moves f: the check would be weak"
    err = rel_l2(d_k, d_o)
    assert err <= BF16_TOL, f"relative L2 of the attention branch over the last key tiles {err:.3e}"


def test_rdt3b_mla_prefill_prefix_and_late_key_tiles():
    """MLA prefill on the tensor cores at the 3B MLA shape (24 heads, nope 128 + rope 64,
    value 128, kv_lora_rank 512), 1 x 4096, one loop: rows 0..63 against the oracle run on
    that causal prefix, and the attention branch of f for the last 128 query rows, which see
    all 32 key tiles (keys and values of the earlier positions through the oracle's own
    latent-cache path)."""
    wl = RI.get_workload("rdt3b_mla_decode")
    cfg = wl.cfg
    B, T = 1, 4096
    dev = torch.device("cuda")
    W = RI.block_weights(cfg, wl.seed, device=dev, attn_std=0.03)
    h0, e = RI.recurrent_inputs(cfg, B, T, wl.seed, device=dev)
    blk = R.RecurrentBlock(cfg, W)
    Q, P = 128, 64
    tp = R.Trace.alloc(cfg, 1, 0, P)                          # the prefix rows: routes checked
    h_out, hw, ids = blk.forward(h0, e, B, T, 1, 0.0, trace=tp)
    h_out, ids = h_out.clone(), ids.clone()
    tr = R.Trace(T - Q, Q, f=torch.zeros(1, Q, cfg.dim, dtype=torch.float32, device=dev))
    blk.forward(h0, e, B, T, 1, 0.0, trace=tr)                # the last rows: attention branch
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    Wc = _cpu(W)
    rec = []
    o_h, _, _, _ = O.recurrent_forward(cfg, Wc, h0[:P].cpu(), e[:P].cpu(), 1, 1, 0.0, record=rec,
                                       route_ids=ids[:, :P].cpu().long())
    check_route_flips(ids[:, :P], tp.biased_logits, rec)
    assert rel_l2(h_out[:P], o_h) <= BF16_TOL
    eps = cfg.norm_eps
    emb = O.loop_embedding(0, cfg.loop_dim, cfg.dim, cfg.loop_theta)
    comb = O.rmsnorm(h0.cpu().double() + emb + e.cpu().double(), Wc["rec_norm_w"], eps)
    a = O.rmsnorm(comb, Wc["attn_norm_w"], eps)
    pos = torch.arange(T)
    ck, kr = [], []
    for c0 in range(0, T - Q, 128):
        _, c, r = O.mla_attention(cfg, Wc, a[c0:c0 + 128], pos[c0:c0 + 128])
        ck.append(c)
        kr.append(r)
    cache = {"c_kv": torch.cat(ck), "k_rope": torch.cat(kr), "pos": pos[:T - Q]}
    o, _, _ = O.mla_attention(cfg, Wc, a[T - Q:], pos[T - Q:], cache)
    f_o = O.rmsnorm(comb[T - Q:] + o, Wc["ffn_norm_w"], eps)
    f0 = O.rmsnorm(comb[T - Q:], Wc["ffn_norm_w"], eps)
    d_o, d_k = f_o - f0, tr.f[0].cpu().double() - f0
    assert rel_l2(d_o, f_o) > 0.05, "attention barely moves f: the check would be weak"
    err = rel_l2(d_k, d_o)
    assert err <= BF16_TOL, f"relative L2 of the MLA attention branch over the last key tiles {err:.3e}"


def test_rdt3b_decode_sequences_match_oracle():
    """3B-shaped decode at full size (64 sequences, per-loop 4096-token random caches):
    sequences 0 and 37 against the oracle decode step."""
    wl = RI.get_workload("rdt3b_decode")
    cfg, B, L = wl.cfg, wl.batch, wl.n_loops
    dev = torch.device("cuda")
    t_max = wl.cache_len + 8
    W = RI.block_weights(cfg, wl.seed, device=dev)
    k, v = RI.random_kv_cache(cfg, L, B, t_max, wl.cache_len, wl.seed, device=dev)
    h0, e = RI.decode_inputs(cfg, B, 0, wl.seed, device=dev)
    blk = R.RecurrentBlock(cfg, W)
    cache = R.KVCache(k, v)
    clen = torch.full((B,), wl.cache_len, dtype=torch.int32, device=dev)
    tr = R.Trace.alloc(cfg, L, 0, B)
    d_h, d_hw, d_ids = blk.decode_step(h0, e, clen, cache, L, wl.act_threshold, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    Wc = _cpu(W)
    # every sequence's routes in every loop, teacher-forced on the step's own router input
    n, bad, skipped = teacher_forced_ids(cfg, Wc, tr, d_ids, L)
    assert n > 0 and bad == 0, f"{bad} of {n} teacher-forced decode rows differ ({skipped} near-ties skipped)"
    for b in (0, 37):
        caches = [[{"k": k[t, b, :, :wl.cache_len].permute(1, 0, 2).cpu(),
                    "v": v[t, b, :, :wl.cache_len].permute(1, 0, 2).cpu(),
                    "pos": torch.arange(wl.cache_len)}] for t in range(L)]
        o_h, o_hw, o_ids, _ = O.decode_step(cfg, Wc, h0[b:b + 1].cpu(), e[b:b + 1].cpu(), caches, [wl.cache_len],
                                            L, wl.act_threshold)
        assert rel_l2(d_h[b:b + 1], o_h) <= BF16_TOL


def test_rdt10b_zipf_prefill_matches_oracle():
    """10B-shaped load-imbalanced prefill at full size (2 x 8192, 24 loops, 128 experts
    top-8, Zipf router bias, halting spread over 4..24 loops): rows 0..31 of sequence 0
    against the oracle run on that causal prefix alone (all 24 loops, the same bias and
    halting offsets); every position halts at exactly its drawn loop, halted positions
    report id -1 and zero weight, routed ids are exact teacher-forced on the traced rows,
    and the output is finite."""
    wl = RI.get_workload("rdt10b_prefill_zipf")
    cfg, B, T, L = wl.cfg, wl.batch, wl.seq, wl.n_loops
    N = B * T
    dev = torch.device("cuda")
    bias = RI.zipf_router_bias(cfg.n_experts, cfg.dim, wl.zipf_s, wl.seed)
    W = RI.block_weights(cfg, wl.seed, device=dev, router_bias=bias, halt_w_std=0.0, halt_b=0.0)
    off, kk = RI.halting_offsets_spread(N, wl.halt_spread[0], wl.halt_spread[1], wl.act_threshold, wl.seed)
    h0, e = RI.recurrent_inputs(cfg, B, T, wl.seed, device=dev)
    blk = R.RecurrentBlock(cfg, W)
    P = 32
    tr = R.Trace.alloc(cfg, L, 0, P)
    h_out, hw, ids = blk.forward(h0, e, B, T, L, wl.act_threshold, halt_logit_offset=off.to(dev), trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    hw_c, ids_c = hw.cpu(), ids.cpu()
    last = ((hw_c > 0).to(torch.int64) * torch.arange(L)[:, None]).max(dim=0).values
    assert torch.equal(last + 1, kk), "halting loop differs from the drawn k_i"
    assert torch.allclose(hw_c.sum(0), torch.ones(N), atol=1e-5)
    after = torch.arange(L)[:, None] > last[None, :]
    assert (ids_c[after] == -1).all() and (hw_c[after] == 0).all()
    assert ((ids_c[~after] >= 0) & (ids_c[~after] < cfg.n_experts)).all()
    assert torch.isfinite(h_out).all()
    n, bad, skipped = teacher_forced_ids(cfg, _cpu({"w_router": W["w_router"], "router_bias": W["router_bias"]}),
                                         tr, ids, L)
    assert n > 0 and bad == 0, f"{bad} of {n} teacher-forced rows differ ({skipped} near-ties skipped)"
    # the Zipf bias makes the load imbalanced: popular experts take far more than E / k share
    counts = torch.bincount(ids_c[0][ids_c[0] >= 0].flatten(), minlength=cfg.n_experts).double()
    assert counts.max() / counts.mean() > 3.0
    # values: the causal prefix of sequence 0 through the oracle (halting is fixed by the
    # offsets, p_i = 0.9 / (k_i - 0.5), so both sides halt at the same loops)
    h_p = h_out[:P].cpu()
    Wc = _cpu(W)
    del W, blk
    torch.cuda.empty_cache()
    rec = []
    o_h, o_hw, o_ids, _ = O.recurrent_forward(cfg, Wc, h0[:P].cpu(), e[:P].cpu(), 1, L, wl.act_threshold,
                                              halt_logit_offset=off[:P], record=rec,
                                              route_ids=ids_c[:, :P].long())
    n_flip = check_route_flips(ids_c[:, :P], tr.biased_logits, rec)
    assert torch.equal(halting_loop(o_hw), last[:P])
    err = rel_l2(h_p, o_h)
    assert err <= BF16_TOL, f"relative L2 of h_out over the prefix {err:.3e} ({n_flip} near-tie routes aligned)"


def test_rdt3b_mla_decode_sequence_matches_oracle():
    """3B-shaped decode with multi-latent attention at full size (64 sequences, per-loop
    4096-token random latent caches, kv_lora_rank 512): sequence 37 against the oracle
    decode step, and the new latent entries of every loop."""
    wl = RI.get_workload("rdt3b_mla_decode")
    cfg, B, L = wl.cfg, wl.batch, wl.n_loops
    dev = torch.device("cuda")
    t_max = wl.cache_len + 8
    W = RI.block_weights(cfg, wl.seed, device=dev)
    ckv, kr = RI.random_latent_cache(cfg, L, B, t_max, wl.cache_len, wl.seed, device=dev)
    h0, e = RI.decode_inputs(cfg, B, 0, wl.seed, device=dev)
    blk = R.RecurrentBlock(cfg, W)
    cache = R.KVCache(ckv, kr)
    clen = torch.full((B,), wl.cache_len, dtype=torch.int32, device=dev)
    tr = R.Trace.alloc(cfg, L, 0, B)
    d_h, d_hw, d_ids = blk.decode_step(h0, e, clen, cache, L, wl.act_threshold, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    assert torch.isfinite(d_h).all()
    Wc = _cpu(W)
    n, bad, skipped = teacher_forced_ids(cfg, Wc, tr, d_ids, L)
    assert n > 0 and bad == 0, f"{bad} of {n} teacher-forced decode rows differ ({skipped} near-ties skipped)"
    b = 37
    caches = [[{"c_kv": ckv[t, b, :wl.cache_len].cpu(), "k_rope": kr[t, b, :wl.cache_len].cpu(),
                "pos": torch.arange(wl.cache_len)}] for t in range(L)]
    o_h, o_hw, o_ids, new_kv = O.decode_step(cfg, Wc, h0[b:b + 1].cpu(), e[b:b + 1].cpu(), caches, [wl.cache_len],
                                             L, wl.act_threshold)
    assert rel_l2(d_h[b:b + 1], o_h) <= BF16_TOL
    for t in range(L):
        assert rel_l2(ckv[t, b, wl.cache_len], new_kv[t][0][0][0]) <= BF16_TOL


# model shapes of generation: (workload whose block shape is used, loops, ACT threshold,
# halting bias).  The 1B model is the generation workload itself; the 3B and 10B models
# take the decode and prefill workloads' block shapes with one prelude and one coda dense
# layer (dense hidden 4 dim / 3: 4096 at dim 3072, 5461 at dim 4096, which the binding pads
# to 5504), ACT off; the 10B model runs 4 of its loops to bound the oracle's time.
GEN_SHAPES = {"rdt1b": ("rdt1b_generate", None, None, None), "rdt3b": ("rdt3b_decode", 16, 0.0, 0.0),
              "rdt10b": ("rdt10b_prefill_zipf", 4, 0.0, 0.0)}


@pytest.mark.parametrize("shape", ["rdt1b", "rdt3b", "rdt10b"])
def test_generation_teacher_forced(shape):
    """Generation with the 1B / 3B / 10B-shaped model (1 prelude + 1 coda layer; vocabulary
    reduced to 4096 here, since it only sizes the embedding and the head): the oracle's
    forward pass over the GPU's own sequence gives, at every generated step, logits within
    the bf16 tolerance and the GPU's token as its argmax up to near-ties."""
    name, loops, thr, halt_b = GEN_SHAPES[shape]
    wl = RI.get_workload(name)
    cfg = wl.cfg.replace(vocab_size=4096, prelude_layers=1, coda_layers=1)
    L = loops or wl.n_loops
    thr = wl.act_threshold if thr is None else thr
    halt_b = wl.halt_b if halt_b is None else halt_b
    dev = torch.device("cuda")
    MW = RI.model_weights(cfg, wl.seed, device=dev, halt_b=halt_b)
    B, T0, new = 2, 24, 3
    prompt = torch.randint(0, cfg.vocab_size, (B, T0), generator=torch.Generator().manual_seed(11))
    gen = R.Generator(cfg, MW, B, T0, new, L, thr, trace=True)
    gen.prefill(prompt.to(device=dev, dtype=torch.int32).contiguous())
    b = 0
    logits = [gen.logits.clone()]
    # the recurrent block's routes and biased logits of sequence b at every position
    routes = [gen.rec_out[2][:, b * T0:(b + 1) * T0].clone()]
    biased = [gen.trace_prefill.biased_logits[:, b * T0:(b + 1) * T0].clone()]
    for s in range(1, new):
        gen.decode(s)
        logits.append(gen.logits.clone())
        routes.append(gen.dec_out[2][:, b:b + 1].clone())
        biased.append(gen.trace_decode.biased_logits[:, b:b + 1].clone())
    torch.cuda.synchronize()
    toks = gen.tokens.t().cpu().long()
    seq = torch.cat([prompt, toks], dim=1)
    MWc = {k: ([{kk: vv.cpu() for kk, vv in blk.items()} for blk in v] if isinstance(v, list) else
               ({kk: vv.cpu() for kk, vv in v.items()} if isinstance(v, dict) else v.cpu())) for k, v in MW.items()}
    del gen, MW
    torch.cuda.empty_cache()
    route_ids = torch.cat(routes, 1).cpu().long()           # [L, T0 + new - 1, k]
    rec = []
    full, _, _ = O.model_forward(cfg, MWc, seq[b:b + 1, :-1], L, thr, route_ids=route_ids, record=rec)
    check_route_flips(route_ids, torch.cat(biased, 1), rec)
    for s in range(new):
        ol = full[0, T0 - 1 + s]
        gl = logits[s][b].cpu()
        assert rel_l2(gl, ol) <= BF16_TOL, s
        gap = float(ol.max() - ol[toks[b, s]])
        assert gap <= 2e-2 * float(ol.max() - ol.min()), s
