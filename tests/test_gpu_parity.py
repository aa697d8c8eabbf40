"""GPU (librdt) against the CPU oracle on the same seeded inputs.

fp32 mode: max relative error <= 1e-4, ids exact.  bf16 mode: relative L2 <= 2e-2 on
h_out (and logits), ids teacher-forced with the 1e-3 margin rule."""
import math

import pytest
import torch

import rdt_inputs as RI
from oracle import rdt_oracle as O
from tests._helpers import (BF16_TOL, FP32_TOL, halting_loop, max_rel, oracle_following_halts, rel_l2,
                            teacher_forced_ids, to_dev)

pytestmark = pytest.mark.gpu

R = pytest.importorskip("recurrent_depth_moe_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    R.load_library()


def _recurrent_case(name, n_loops=None, seq=None, batch=None, **wkw):
    wl = RI.get_workload(name)
    cfg = wl.cfg
    B = batch or wl.batch
    T = seq or wl.seq
    L = n_loops or wl.n_loops
    W = RI.block_weights(cfg, wl.seed, **wkw)
    h0, e = RI.recurrent_inputs(cfg, B, T, wl.seed)
    return wl, cfg, W, h0, e, B, T, L


@pytest.mark.parametrize("name", ["tiny_gqa_fp32", "tiny_mla_fp32", "mid_gqa_fp32"])
def test_recurrent_fp32_matches_oracle(name):
    wl, cfg, W, h0, e, B, T, L = _recurrent_case(name, attn_std=0.08, halt_w_std=0.2, lora_scale_std=1.0)
    thr = wl.act_threshold
    blk = R.RecurrentBlock(cfg, to_dev(W))
    tr = R.Trace.alloc(cfg, L, 0, B * T)
    h_out, hw, ids = blk.forward(h0.cuda(), e.cuda(), B, T, L, thr, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    o_h, o_hw, o_ids, _ = O.recurrent_forward(cfg, W, h0, e, B, L, thr)
    assert max_rel(h_out, o_h) <= FP32_TOL
    assert max_rel(hw, o_hw) <= FP32_TOL
    assert torch.equal(ids.cpu().long(), o_ids)


@pytest.mark.parametrize("dim,rank", [(512, 5), (4096, 4), (4096, 8), (4096, 16)])
def test_combine_lora_staging_modes_fp32(dim, rank):
    """The combine kernel's LoRA paths ("OpenMythos 분석", Recurrent Block: the depth-wise LoRA
    of the transformer output) at row widths 512 and 4096 in fp32: both matrices staged in
    shared memory (rank 5 at 512, odd, so the last pair of ranks has one live rank; rank 4 at
    4096), the down projection alone (rank 8 at 4096: 128 KB) and neither (rank 16: 256 KB
    each).  320 rows take the persistent row-group kernel; halting rows freeze along the way.
    Max relative error <= 1e-4 against the oracle, ids exact.  The attention and halting
    weights' scale shrinks as 1 / sqrt(dim) so that the query-key and halting logits keep one
    scale at every width: unscaled, at dim 4096 the oracle's own steps taken in fp32 already
    drift 2.7e-4 from fp64, past what a 1e-4 bar can separate from a fault; scaled, the drift
    is below 4e-5 on h_out and the halting weights at every case here."""
    cfg = RI.RDTConfig(dim=dim, n_heads=dim // 128, n_kv_heads=max(dim // 512, 1), max_seq_len=512,
                       max_loop_iters=4, n_experts=8, n_shared_experts=1, n_experts_per_tok=2, expert_dim=128,
                       lora_rank=rank, dtype="fp32")
    sc = math.sqrt(512 / dim)
    W = RI.block_weights(cfg, 300 + rank, attn_std=0.08 * sc, halt_w_std=0.2 * sc, lora_scale_std=1.0)
    B, T, L, thr = 1, 320, 3, 0.99
    h0, e = RI.recurrent_inputs(cfg, B, T, 301)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    h_out, hw, ids = blk.forward(h0.cuda(), e.cuda(), B, T, L, thr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    o_h, o_hw, o_ids, _ = O.recurrent_forward(cfg, W, h0, e, B, L, thr)
    assert max_rel(h_out, o_h) <= FP32_TOL
    assert max_rel(hw, o_hw) <= FP32_TOL
    assert torch.equal(ids.cpu().long(), o_ids)
    assert (halting_loop(o_hw) < L - 1).any(), "some rows halt before the last loop"


def test_tiny_gqa_fp32_model_logits():
    """The usage script's tiny GQA model end to end: logits (2, 16, 1000)."""
    wl = RI.get_workload("tiny_gqa_fp32")
    cfg = wl.cfg
    MW = RI.model_weights(cfg, wl.seed)
    ids = torch.randint(0, cfg.vocab_size, (wl.batch, wl.seq), generator=torch.Generator().manual_seed(wl.seed))
    logits, rec = R.model_forward(cfg, to_dev(MW), ids.cuda(), wl.n_loops, wl.act_threshold)
    o_logits, o_rec, _ = O.model_forward(cfg, MW, ids, wl.n_loops, wl.act_threshold)
    assert tuple(logits.shape) == (2, 16, 1000)
    assert max_rel(logits, o_logits) <= FP32_TOL
    assert max_rel(rec[0], o_rec[0]) <= FP32_TOL
    assert torch.equal(rec[2].cpu().long(), o_rec[2])


def test_tiny_mla_fp32_model_logits():
    wl = RI.get_workload("tiny_mla_fp32")
    cfg = wl.cfg
    MW = RI.model_weights(cfg, wl.seed)
    ids = torch.randint(0, cfg.vocab_size, (wl.batch, wl.seq), generator=torch.Generator().manual_seed(wl.seed))
    logits, rec = R.model_forward(cfg, to_dev(MW), ids.cuda(), wl.n_loops, wl.act_threshold)
    o_logits, o_rec, _ = O.model_forward(cfg, MW, ids, wl.n_loops, wl.act_threshold)
    assert max_rel(logits, o_logits) <= FP32_TOL
    assert max_rel(rec[1], o_rec[1]) <= FP32_TOL
    assert torch.equal(rec[2].cpu().long(), o_rec[2])


def _bf16_compare(cfg, W, h_out, hw, ids, tr, o_h, L):
    """bf16 parity, end to end: relative L2 over every position (the oracle follows the
    GPU's halting loop where that decision was a near-tie, see oracle_following_halts);
    ids exact teacher-forced (the kernel's own router input) wherever the top-k margin is
    >= 1e-3.  End-to-end routes are not compared: a near-tie flip at one position changes
    that position's state, hence its keys and values, hence every later position's
    attention."""
    err = rel_l2(h_out.cpu(), o_h)
    assert err <= BF16_TOL, f"relative L2 {err:.3e}"
    n, nbad, skipped = teacher_forced_ids(cfg, W, tr, ids, L)
    assert n > 0 and nbad == 0, f"{nbad} of {n} teacher-forced id rows differ ({skipped} near-ties skipped)"


def _teacher_forced_states(cfg, W, tr, e, B, L, ids, hw):
    """One loop of the oracle from the kernel's own state entering loop t, against the
    kernel's state entering loop t + 1 (no compounding across loops).  Rows running in
    loop t are compared, except where the kernel's route differs from the oracle's at a
    near-tie (margin < DECISION_MARGIN).  Returns the per-loop relative L2 errors."""
    from tests._helpers import DECISION_MARGIN, topk_margin
    hl = halting_loop(hw)
    errs = []
    for t in range(L - 1):
        h_in = tr.h_in[t].cpu()
        got = tr.h_in[t + 1].cpu().double()
        h_new, o_ids, biased = _one_loop(cfg, W, h_in, e, B, t)
        rows = hl >= t
        diff = (ids[t].cpu().long() != o_ids).any(-1) & rows
        near = topk_margin(biased, cfg.n_experts_per_tok) < DECISION_MARGIN
        assert not (diff & ~near).any(), f"loop {t}: routes differ away from near-ties"
        keep = rows & ~diff
        errs.append(rel_l2(got[keep], h_new[keep]))
    return errs


def _one_loop(cfg, W, h, e, B, t):
    """Oracle state update of loop t from state h (Transformer + LoRA + injection).
    Returns (h_new, expert ids, biased router logits)."""
    emb = O.loop_embedding(t, cfg.loop_dim, cfg.dim, cfg.loop_theta)
    hd = h.double()
    comb = O.rmsnorm(hd + emb + e.double(), W["rec_norm_w"], cfg.norm_eps)
    T = h.shape[0] // B
    pos = torch.arange(h.shape[0]) % T
    trans, _, info = O.transformer_block(cfg, W, comb, B, pos, True)
    trans = trans + O.lora_delta(cfg, W, trans, t)
    A = O.lti_A(W["log_A"], W["log_dt"])
    return A * hd + W["inj_B"].double() * e.double() + trans, info["ids"], info["biased"]


STRONG = dict(attn_std=0.08, halt_w_std=0.2, lora_scale_std=1.0)   # peaky attention, visible LoRA and ACT


@pytest.mark.parametrize("variant", ["literal", "strong"])
@pytest.mark.parametrize("name", ["tiny_mla_bf16", "mid_gqa_bf16", "mid_e64_bf16", "mid_e128_bf16", "mid_t392_bf16"])
def test_recurrent_bf16_matches_oracle(name, variant):
    wl, cfg, W, h0, e, B, T, L = _recurrent_case(name, **(STRONG if variant == "strong" else {}))
    thr = wl.act_threshold
    blk = R.RecurrentBlock(cfg, to_dev(W))
    tr = R.Trace.alloc(cfg, L, 0, B * T)
    h_out, hw, ids = blk.forward(h0.cuda(), e.cuda(), B, T, L, thr, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    run = lambda halt_at, rec: O.recurrent_forward(cfg, W, h0, e, B, L, thr, record=rec, halt_at=halt_at)
    (o_h, o_hw, o_ids, _), rec, n_forced, margin = oracle_following_halts(run, ids, tr.p, thr)
    _bf16_compare(cfg, W, h_out, hw, ids, tr, o_h, L)
    errs = _teacher_forced_states(cfg, W, tr, e, B, L, ids, hw)
    assert max(errs) <= BF16_TOL, f"per-loop teacher-forced relative L2 {errs}"


def test_tiny_mla_bf16_model_logits():
    wl = RI.get_workload("tiny_mla_bf16")
    cfg = wl.cfg
    MW = RI.model_weights(cfg, wl.seed)
    ids = torch.randint(0, cfg.vocab_size, (wl.batch, wl.seq), generator=torch.Generator().manual_seed(wl.seed))
    logits, rec = R.model_forward(cfg, to_dev(MW), ids.cuda(), wl.n_loops, wl.act_threshold)
    o_logits, o_rec, _ = O.model_forward(cfg, MW, ids, wl.n_loops, wl.act_threshold)
    assert rel_l2(rec[0], o_rec[0]) <= BF16_TOL
    assert rel_l2(logits, o_logits) <= BF16_TOL


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_lti_closed_form_on_gpu(dtype):
    """Transformer term off: h_L = a^L h0 + b e (1 - a^L)/(1 - a) (README mirror, 동적 시스템 관점)."""
    wl = RI.get_workload("mid_gqa_fp32")
    cfg = wl.cfg.replace(dtype=dtype)
    W = RI.block_weights(cfg, 3)
    h0, e = RI.recurrent_inputs(cfg, 1, 40, 3)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    L = 9
    h, hw, ids = blk.forward(h0.cuda(), e.cuda(), 1, 40, L, 0.0, flags=R.RDT_FLAG_TRANSFORMER_OFF)
    a = torch.exp(-torch.exp(W["log_A"].double()))
    closed = a ** L * h0.double() + W["inj_B"].double() * e.double() * (1 - a ** L) / (1 - a)
    assert max_rel(h, closed) <= 1e-5
    assert (ids.cpu() == -1).all() and torch.equal(hw.cpu()[-1], torch.ones(40))


@pytest.mark.parametrize("name", ["mid_gqa_fp32", "mid_gqa_bf16"])
def test_causality_bit_exact_on_gpu(name):
    """Perturbing later positions leaves earlier rows bit-identical (fixed reduction order,
    no split across rows)."""
    wl, cfg, W, h0, e, B, T, L = _recurrent_case(name, attn_std=0.08, halt_w_std=0.2)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    out1 = [t.clone() for t in blk.forward(h0.cuda(), e.cuda(), B, T, L, wl.act_threshold)]
    h0b, eb = h0.clone(), e.clone()
    cut = 150
    for b in range(B):
        h0b[b * T + cut:(b + 1) * T] += 0.5
        eb[b * T + cut:(b + 1) * T] = (eb[b * T + cut:(b + 1) * T].float() * -1.0).to(eb.dtype)
    out2 = blk.forward(h0b.cuda(), eb.cuda(), B, T, L, wl.act_threshold)
    for b in range(B):
        sl = slice(b * T, b * T + cut)
        assert torch.equal(out1[0][sl], out2[0][sl])
        assert torch.equal(out1[1][:, sl], out2[1][:, sl])
        assert torch.equal(out1[2][:, sl], out2[2][:, sl])


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_decode_step_matches_oracle_and_prefill(dtype):
    """Prefill T tokens filling per-loop caches, then one decode step at position T:
    equals the oracle decode step, and the prefill of T + 1 tokens."""
    wl = RI.get_workload("mid_gqa_fp32")
    cfg = wl.cfg.replace(dtype=dtype)
    W = RI.block_weights(cfg, 7, attn_std=0.08, halt_w_std=0.2)
    B, T, L, thr = 3, 37, 3, 0.99
    h0, e = RI.recurrent_inputs(cfg, B, T + 1, 7)
    keep = torch.tensor([b * (T + 1) + i for b in range(B) for i in range(T)])
    last = torch.tensor([b * (T + 1) + T for b in range(B)])
    blk = R.RecurrentBlock(cfg, to_dev(W))
    t_max = 64
    k = torch.zeros(L, B, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=cfg.torch_dtype, device="cuda")
    cache = R.KVCache(k, torch.zeros_like(k))
    blk.forward(h0[keep].cuda(), e[keep].cuda(), B, T, L, thr, cache=cache)
    clen = torch.full((B,), T, dtype=torch.int32, device="cuda")
    tr = R.Trace.alloc(cfg, L, 0, B)
    d_h, d_hw, d_ids = blk.decode_step(h0[last].cuda(), e[last].cuda(), clen, cache, L, thr, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    full = O.recurrent_forward(cfg, W, h0, e, B, L, thr)
    if dtype == "fp32":
        assert max_rel(d_h, full[0][last]) <= FP32_TOL
        assert torch.equal(d_ids.cpu().long(), full[2][:, last])
    else:
        assert rel_l2(d_h, full[0][last]) <= BF16_TOL
    # the decode step's routes, teacher-forced on its own router input
    n, bad, skipped = teacher_forced_ids(cfg, W, tr, d_ids, L)
    assert n > 0 and bad == 0, f"{bad} of {n} teacher-forced decode rows differ ({skipped} near-ties skipped)"
    # GPU prefill of T + 1 tokens gives the same last rows as GPU prefill + decode
    p_h, p_hw, p_ids = blk.forward(h0.cuda(), e.cuda(), B, T + 1, L, thr)
    tol = 1e-5 if dtype == "fp32" else 1e-2
    assert rel_l2(d_h, p_h[last.cuda()]) <= tol


def test_invalid_arguments_return_errors():
    wl = RI.get_workload("tiny_gqa_fp32")
    cfg = wl.cfg
    W = to_dev(RI.block_weights(cfg, 0))
    blk = R.RecurrentBlock(cfg, W)
    h0, e = RI.recurrent_inputs(cfg, 1, 8, 0)
    h0, e = h0.cuda(), e.cuda()
    with pytest.raises(R.RdtError) as ei:
        blk.forward(h0, e, 1, 8, 0, 0.0)                 # n_loops = 0
    assert ei.value.code == 1
    with pytest.raises(R.RdtError) as ei:
        blk.forward(h0, e, 1, 8, 2, float("nan"))        # NaN threshold
    assert ei.value.code == 1
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(R.RdtError) as ei:
        blk.forward(h0, e, 1, 8, 2, 0.0, workspace=small)
    assert ei.value.code == 3
    bad = dict(W)
    bad.pop("w_router")
    with pytest.raises(R.RdtError) as ei:
        R.RecurrentBlock(cfg, bad).forward(h0, e, 1, 8, 2, 0.0)
    assert ei.value.code == 1


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_decode_rescales_as_key_scores_grow(dtype):
    """Decode attention whose running maximum keeps rising: the cached keys are scaled by
    1 + j / 32 at position j (fp32), so a query's largest score grows about 30-fold along a
    1000-key cache and passes the previous maximum by more than the lazy-rescale threshold
    (2^8) on 6-9 of its 16 tiles; every rescale of the running sum and output must hold.
    bf16 takes 1 + j / 160 (3-4 raises, scores up to about 30): at scores near 100 the bf16
    rounding of the query alone moves a score by about 0.2, which the 2e-2 bar would not
    separate from a fault.  Ragged lengths (1000, 600, 129 keys) put the growth in one key
    range and across ranges."""
    cfg = RI.RDTConfig(dim=768, n_heads=6, n_kv_heads=2, max_seq_len=1100, max_loop_iters=2, n_experts=8,
                       n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, dtype=dtype)
    W = RI.block_weights(cfg, 24, attn_std=0.05)
    B, L, t_max = 3, 2, 1100
    lens = [1000, 600, 129]
    k, v = RI.random_kv_cache(cfg, L, B, t_max, max(lens), 25)
    grow = (1.0 + torch.arange(t_max, dtype=torch.float64) / (32 if dtype == "fp32" else 160)).to(k.dtype)
    k = k * grow[None, None, None, :, None]
    for b, n in enumerate(lens):
        k[:, b, :, n:] = 0
        v[:, b, :, n:] = 0
    h0, e = RI.decode_inputs(cfg, B, 0, 26)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = R.KVCache(k.cuda(), v.cuda())
    clen = torch.tensor(lens, dtype=torch.int32, device="cuda")
    d_h, d_hw, d_ids = blk.decode_step(h0.cuda(), e.cuda(), clen, cache, L, 0.0)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    caches = [[{"k": k[t, b, :, :lens[b]].permute(1, 0, 2), "v": v[t, b, :, :lens[b]].permute(1, 0, 2),
                "pos": torch.arange(lens[b])} for b in range(B)] for t in range(L)]
    o_h, o_hw, o_ids, _ = O.decode_step(cfg, W, h0, e, caches, lens, L, 0.0)
    if dtype == "fp32":
        assert max_rel(d_h, o_h) <= FP32_TOL
    else:
        for b in range(B):
            assert rel_l2(d_h[b], o_h[b]) <= BF16_TOL, b


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_decode_random_cache_ragged_lengths(dtype):
    """Decode step against random per-loop caches (the 3B decode workload's structure:
    GQA group 3, one cache per loop) with a different cache length per sequence."""
    cfg = RI.RDTConfig(dim=768, n_heads=6, n_kv_heads=2, max_seq_len=160, max_loop_iters=3, n_experts=8,
                       n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, dtype=dtype)
    W = RI.block_weights(cfg, 21, attn_std=0.05)
    B, L, t_max = 4, 3, 160
    lens = [37, 100, 64, 5]
    k, v = RI.random_kv_cache(cfg, L, B, t_max, max(lens), 22)
    for b, n in enumerate(lens):                       # positions >= len are not part of the cache
        k[:, b, :, n:] = 0
        v[:, b, :, n:] = 0
    h0, e = RI.decode_inputs(cfg, B, 0, 23)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = R.KVCache(k.cuda(), v.cuda())
    clen = torch.tensor(lens, dtype=torch.int32, device="cuda")
    tr = R.Trace.alloc(cfg, L, 0, B)
    d_h, d_hw, d_ids = blk.decode_step(h0.cuda(), e.cuda(), clen, cache, L, 0.0, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    n, bad, skipped = teacher_forced_ids(cfg, W, tr, d_ids, L)
    assert n > 0 and bad == 0, f"{bad} of {n} teacher-forced decode rows differ ({skipped} near-ties skipped)"
    caches = [[{"k": k[t, b, :, :lens[b]].permute(1, 0, 2), "v": v[t, b, :, :lens[b]].permute(1, 0, 2),
                "pos": torch.arange(lens[b])} for b in range(B)] for t in range(L)]
    o_h, o_hw, o_ids, new_kv = O.decode_step(cfg, W, h0, e, caches, lens, L, 0.0)
    if dtype == "fp32":
        assert max_rel(d_h, o_h) <= FP32_TOL
        assert torch.equal(d_ids.cpu().long(), o_ids)
    else:
        assert rel_l2(d_h, o_h) <= BF16_TOL
    # the new keys / values were appended at cache_len[b] in every loop cache
    kc = cache.k.cpu()
    for t in range(L):
        for b in range(B):
            got = kc[t, b, :, lens[b]].double()
            want = new_kv[t][b][0][0].double()
            assert rel_l2(got, want) <= (1e-5 if dtype == "fp32" else 2e-2)
