"""Continuous depth-wise batching of decode steps (rdt_depth_batch_*): each sequence's tokens
leave the shared block at their own depth and the next token takes the slot.  The results
must equal successive decode steps per sequence: the oracle's decode_tokens (fp32: max
relative error <= 1e-4, ids exact; bf16: relative L2 <= 2e-2), and the library's own
lockstep decode steps with the same halting-logit offsets.  The loop caches must hold every
token's keys / values at every loop, the loops after it halted included."""
import pytest
import torch

import rdt_inputs as RI
from oracle import rdt_oracle as O
from tests._helpers import BF16_TOL, FP32_TOL, max_rel, rel_l2, to_dev

pytestmark = pytest.mark.gpu

R = pytest.importorskip("recurrent_depth_moe_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    R.load_library()


def _case(dtype, L=6, S=4, lens=(5, 20, 11), act=True, seed=81):
    cfg = RI.RDTConfig(dim=512, n_heads=4, n_kv_heads=2, max_seq_len=64, max_loop_iters=4, n_experts=8,
                       n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, dtype=dtype)
    # zero halting head: the per-token offsets alone decide the halting loop (spread 2..L)
    W = RI.block_weights(cfg, seed, attn_std=0.08, halt_w_std=0.0, halt_b=0.0, lora_scale_std=1.0)
    B = len(lens)
    t_max = max(lens) + S + 3
    k, v = RI.random_kv_cache(cfg, L, B, t_max, max(lens), seed + 1)
    for b, n in enumerate(lens):
        k[:, b, :, n:] = 0
        v[:, b, :, n:] = 0
    h0, e = RI.recurrent_inputs(cfg, B, S, seed + 2)
    h0, e = h0.view(B, S, cfg.dim), e.view(B, S, cfg.dim)
    thr = 0.99 if act else 0.0
    off, kk = RI.halting_offsets_spread(B * S, 2, max(L, 2), 0.99, seed + 3)
    return cfg, W, list(lens), k, v, h0, e, off.view(B, S), kk.view(B, S), thr, L


def _oracle(cfg, W, lens, k, v, h0, e, off, thr, L):
    B = len(lens)
    caches = [[{"k": k[t, b, :, :lens[b]].permute(1, 0, 2), "v": v[t, b, :, :lens[b]].permute(1, 0, 2),
                "pos": torch.arange(lens[b])} for b in range(B)] for t in range(L)]
    return O.decode_tokens(cfg, W, h0, e, caches, lens, L, thr, off if thr > 0 else None)


def _depth(cfg, W, lens, k, v, h0, e, off, thr, L, check_every=3, cuda_graph=False):
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = R.KVCache(k.cuda(), v.cuda())
    clen = torch.tensor(lens, dtype=torch.int32, device="cuda")
    db = R.DepthBatch(blk, h0.cuda().contiguous(), e.cuda().contiguous(), clen, cache, L, thr,
                      off.cuda().contiguous() if thr > 0 else None)
    out = db.run(check_every=check_every, cuda_graph=cuda_graph)
    torch.cuda.synchronize()
    assert db.read_status() == 0
    assert db.pending() == 0
    return [o.cpu() for o in out], cache


def _lockstep(cfg, W, lens, k, v, h0, e, off, thr, L):
    """The library's lockstep decode steps: token n of every sequence, all L loops."""
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = R.KVCache(k.cuda(), v.cuda())
    B, S = h0.shape[:2]
    outs = []
    for n in range(S):
        clen = torch.tensor([x + n for x in lens], dtype=torch.int32, device="cuda")
        o = blk.decode_step(h0[:, n].cuda().contiguous(), e[:, n].cuda().contiguous(), clen, cache, L, thr,
                            halt_logit_offset=off[:, n].cuda().contiguous() if thr > 0 else None)
        outs.append([x.clone() for x in o])
    torch.cuda.synchronize()
    h = torch.stack([o[0].cpu() for o in outs], 1)                    # [B, S, D]
    hw = torch.stack([o[1].cpu() for o in outs], 1).permute(2, 1, 0)  # [L, S, B] -> [B, S, L]
    ids = torch.stack([o[2].cpu() for o in outs], 1).permute(2, 1, 0, 3)
    return (h, hw, ids), cache


def test_depth_batch_fp32_matches_successive_decode_steps():
    cfg, W, lens, k, v, h0, e, off, kk, thr, L = _case("fp32")
    (h, hw, ids), cache = _depth(cfg, W, lens, k, v, h0, e, off, thr, L)
    oh, ohw, oids = _oracle(cfg, W, lens, k, v, h0, e, off, thr, L)
    assert max_rel(h, oh) <= FP32_TOL
    assert max_rel(hw, ohw) <= FP32_TOL
    assert torch.equal(ids.long(), oids)
    last = ((hw > 0).to(torch.int64) * torch.arange(L)).max(-1).values
    assert torch.equal(last + 1, kk), "tokens halt at their drawn depth"
    assert len(set(kk.flatten().tolist())) > 1, "the halting spread makes the depths differ"
    # every token's keys / values at every loop (the loops after its halt come from the fill)
    (lh, lhw, lids), lcache = _lockstep(cfg, W, lens, k, v, h0, e, off, thr, L)
    for b, n0 in enumerate(lens):
        sl = slice(n0, n0 + h0.shape[1])
        assert max_rel(cache.k[:, b, :, sl].cpu(), lcache.k[:, b, :, sl].cpu()) <= 1e-5
        assert max_rel(cache.v[:, b, :, sl].cpu(), lcache.v[:, b, :, sl].cpu()) <= 1e-5
    assert max_rel(h, lh) <= 1e-5 and torch.equal(ids, lids)


def test_depth_batch_act_off_every_token_runs_all_loops():
    cfg, W, lens, k, v, h0, e, off, kk, thr, L = _case("fp32", L=3, S=3, act=False, seed=91)
    (h, hw, ids), _ = _depth(cfg, W, lens, k, v, h0, e, off, thr, L, check_every=2)
    oh, ohw, oids = _oracle(cfg, W, lens, k, v, h0, e, off, thr, L)
    assert max_rel(h, oh) <= FP32_TOL
    assert torch.equal(ids.long(), oids)
    assert torch.equal(hw[..., -1], torch.ones(hw.shape[:2])) and (hw[..., :-1] == 0).all()


def test_depth_batch_bf16_matches_oracle_and_lockstep():
    cfg, W, lens, k, v, h0, e, off, kk, thr, L = _case("bf16", L=8, S=5, lens=(7, 30, 19, 3), seed=101)
    (h, hw, ids), cache = _depth(cfg, W, lens, k, v, h0, e, off, thr, L)
    oh, ohw, oids = _oracle(cfg, W, lens, k, v, h0, e, off, thr, L)
    assert rel_l2(h, oh) <= BF16_TOL
    last = ((hw > 0).to(torch.int64) * torch.arange(L)).max(-1).values
    assert torch.equal(last + 1, kk)
    (lh, lhw, lids), lcache = _lockstep(cfg, W, lens, k, v, h0, e, off, thr, L)
    assert rel_l2(h, lh) <= 5e-3
    assert (ids == lids).all(-1).float().mean() >= 0.98
    for b, n0 in enumerate(lens):
        sl = slice(n0, n0 + h0.shape[1])
        assert rel_l2(cache.k[:, b, :, sl].float().cpu(), lcache.k[:, b, :, sl].float().cpu()) <= 5e-3


def test_depth_batch_graph_replay_equals_eager():
    cfg, W, lens, k, v, h0, e, off, kk, thr, L = _case("bf16", L=6, S=6, lens=(4, 9), seed=111)
    (h1, hw1, ids1), c1 = _depth(cfg, W, lens, k, v, h0, e, off, thr, L, check_every=2)
    (h2, hw2, ids2), c2 = _depth(cfg, W, lens, k, v, h0, e, off, thr, L, check_every=2, cuda_graph=True)
    assert torch.equal(h1, h2) and torch.equal(hw1, hw2) and torch.equal(ids1, ids2)
    assert torch.equal(c1.k, c2.k) and torch.equal(c1.v, c2.v)


def test_depth_batch_one_loop_one_token():
    cfg, W, lens, k, v, h0, e, off, kk, thr, L = _case("fp32", L=1, S=1, act=False, seed=121)
    (h, hw, ids), _ = _depth(cfg, W, lens, k, v, h0, e, off, thr, L, check_every=1)
    oh, ohw, oids = _oracle(cfg, W, lens, k, v, h0, e, off, thr, L)
    assert max_rel(h, oh) <= FP32_TOL and torch.equal(ids.long(), oids)
