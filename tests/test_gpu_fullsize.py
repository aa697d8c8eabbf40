"""Full-size GPU runs in the launch configuration bench.py times, checked on outputs the
oracle can compute (a causal prefix slice, single decode sequences) and on properties
that hold at any size (halting loops, id ranges, causality, finiteness)."""
import math

import pytest
import torch

import rdt_inputs as RI
from oracle import rdt_oracle as O
from tests._helpers import BF16_TOL, ID_MARGIN, rel_l2, teacher_forced_ids, topk_margin

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
    o_h, o_hw, o_ids, _ = O.recurrent_forward(cfg, Wc, h0[:P].cpu(), e[:P].cpu(), 1, L, wl.act_threshold)
    assert rel_l2(h_out[:P], o_h) <= BF16_TOL
    n, bad, skipped = teacher_forced_ids(cfg, Wc, tr, ids, L)
    assert n > 0 and bad == 0, f"{bad} of {n} teacher-forced rows differ ({skipped} near-ties skipped)"
    assert torch.isfinite(h_out).all()
    ids_c, hw_c = ids.cpu(), hw.cpu()
    last = ((hw_c > 0).to(torch.int64) * torch.arange(L)[:, None]).max(dim=0).values
    after = torch.arange(L)[:, None] > last[None, :]
    assert ((ids_c[~after] >= 0) & (ids_c[~after] < cfg.n_experts)).all() and (ids_c[after] == -1).all()
    assert (last == L - 1).float().mean() > 0.99             # halting bias -30: nearly every row runs 16 loops


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
    d_h, d_hw, d_ids = blk.decode_step(h0, e, clen, cache, L, wl.act_threshold)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    Wc = _cpu(W)
    for b in (0, 37):
        caches = [[{"k": k[t, b, :, :wl.cache_len].permute(1, 0, 2).cpu(),
                    "v": v[t, b, :, :wl.cache_len].permute(1, 0, 2).cpu(),
                    "pos": torch.arange(wl.cache_len)}] for t in range(L)]
        o_h, o_hw, o_ids, _ = O.decode_step(cfg, Wc, h0[b:b + 1].cpu(), e[b:b + 1].cpu(), caches, [wl.cache_len],
                                            L, wl.act_threshold)
        assert rel_l2(d_h[b:b + 1], o_h) <= BF16_TOL


def test_rdt10b_zipf_prefill_properties():
    """10B-shaped load-imbalanced prefill at full size (2 x 8192, 24 loops, 128 experts
    top-8, Zipf router bias, halting spread over 4..24 loops): every position halts at
    exactly its drawn loop, halted positions report id -1 and zero weight, routed ids are
    exact teacher-forced on sampled rows, and the output is finite."""
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
    d_h, d_hw, d_ids = blk.decode_step(h0, e, clen, cache, L, wl.act_threshold)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    assert torch.isfinite(d_h).all()
    Wc = _cpu(W)
    b = 37
    caches = [[{"c_kv": ckv[t, b, :wl.cache_len].cpu(), "k_rope": kr[t, b, :wl.cache_len].cpu(),
                "pos": torch.arange(wl.cache_len)}] for t in range(L)]
    o_h, o_hw, o_ids, new_kv = O.decode_step(cfg, Wc, h0[b:b + 1].cpu(), e[b:b + 1].cpu(), caches, [wl.cache_len],
                                             L, wl.act_threshold)
    assert rel_l2(d_h[b:b + 1], o_h) <= BF16_TOL
    for t in range(L):
        assert rel_l2(ckv[t, b, wl.cache_len], new_kv[t][0][0][0]) <= BF16_TOL


def test_rdt1b_generation_teacher_forced():
    """Generation with the 1B-shaped model (16 loops, 64 experts, 1 prelude + 1 coda layer;
    vocabulary reduced to 4096 here, since it only sizes the embedding and the head): the
    oracle's forward pass over the GPU's own sequence gives, at every generated step,
    logits within the bf16 tolerance and the GPU's token as its argmax up to near-ties."""
    wl = RI.get_workload("rdt1b_generate")
    cfg = wl.cfg.replace(vocab_size=4096)
    dev = torch.device("cuda")
    MW = RI.model_weights(cfg, wl.seed, device=dev, halt_b=wl.halt_b)
    B, T0, new, L = 2, 24, 3, wl.n_loops
    prompt = torch.randint(0, cfg.vocab_size, (B, T0), generator=torch.Generator().manual_seed(11))
    gen = R.Generator(cfg, MW, B, T0, new, L, wl.act_threshold)
    gen.prefill(prompt.to(device=dev, dtype=torch.int32).contiguous())
    logits = [gen.logits.clone()]
    for s in range(1, new):
        gen.decode(s)
        logits.append(gen.logits.clone())
    torch.cuda.synchronize()
    toks = gen.tokens.t().cpu().long()
    seq = torch.cat([prompt, toks], dim=1)
    MWc = {k: ([{kk: vv.cpu() for kk, vv in blk.items()} for blk in v] if isinstance(v, list) else
               ({kk: vv.cpu() for kk, vv in v.items()} if isinstance(v, dict) else v.cpu())) for k, v in MW.items()}
    b = 0
    full, _, _ = O.model_forward(cfg, MWc, seq[b:b + 1, :-1], L, wl.act_threshold)
    for s in range(new):
        ol = full[0, T0 - 1 + s]
        gl = logits[s][b].cpu()
        assert rel_l2(gl, ol) <= BF16_TOL, s
        gap = float(ol.max() - ol[toks[b, s]])
        assert gap <= 2e-2 * float(ol.max() - ol.min()), s
