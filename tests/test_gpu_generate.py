"""Generation on the GPU ("OpenMythos 분석", RoPE & generation cache): prelude / coda
blocks with their own caches, the recurrent block with one cache per loop, greedy tokens.
Compared with the oracle's generate, which recomputes the whole sequence every step."""
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


@pytest.mark.parametrize("name", ["tiny_gqa_fp32", "tiny_mla_fp32"])
def test_cached_block_prefill_then_decode_equals_longer_prefill(name):
    """A prelude block: prefill of T tokens into its cache, then one decode step at T,
    equals the prefill of T + 1 tokens (rows T of each sequence)."""
    cfg = RI.get_workload(name).cfg
    W = to_dev(RI.dense_block_weights(cfg, 5))
    B, T, t_max = 3, 21, 32
    x = torch.randn(B * (T + 1), cfg.dim, generator=torch.Generator().manual_seed(6)).cuda()
    keep = torch.tensor([b * (T + 1) + i for b in range(B) for i in range(T)]).cuda()
    last = torch.tensor([b * (T + 1) + T for b in range(B)]).cuda()
    blk = R.Block(cfg, W)
    from recurrent_depth_moe_b200.api import _layer_cache
    cache = _layer_cache(cfg, 1, B, t_max)
    blk.forward(x[keep].contiguous(), B, T, 0, cache=cache)
    clen = torch.full((B,), T, dtype=torch.int32, device="cuda")
    d = blk.forward(x[last].contiguous(), B, 1, 0, cache=cache, cache_len=clen)
    full = blk.forward(x, B, T + 1)
    assert max_rel(d, full[last]) <= FP32_TOL
    # and the oracle's dense block agrees with the longer prefill
    o = O.dense_block_forward(cfg, {k: v.cpu() for k, v in W.items()}, x.cpu().double(), B)
    assert max_rel(full, o) <= FP32_TOL


def _gpu_generate(cfg, MW, prompt, new, L, thr):
    gen = R.Generator(cfg, MW, prompt.shape[0], prompt.shape[1], new, L, thr)
    ids = prompt.to(device="cuda", dtype=torch.int32).contiguous()
    gen.prefill(ids)
    logits = [gen.logits.clone()]
    for s in range(1, new):
        gen.decode(s)
        logits.append(gen.logits.clone())
    torch.cuda.synchronize()
    return gen.tokens.t().cpu().long(), torch.stack(logits).cpu()


@pytest.mark.parametrize("name,L", [("tiny_gqa_fp32", 8), ("tiny_mla_fp32", 8)])
def test_generate_fp32_matches_oracle(name, L):
    """The usage script's generation (prompt 2 x 16, 8 new tokens, n_loops 8 > max_loop_iters):
    the same tokens and the same logits at every step."""
    wl = RI.get_workload(name)
    cfg = wl.cfg
    MW = RI.model_weights(cfg, wl.seed)
    prompt = torch.randint(0, cfg.vocab_size, (2, 16), generator=torch.Generator().manual_seed(wl.seed))
    new = 8
    toks, logits = _gpu_generate(cfg, to_dev(MW), prompt, new, L, wl.act_threshold)
    o_ids, o_logits = O.generate(cfg, MW, prompt, new, L, wl.act_threshold)
    for s in range(new):
        assert max_rel(logits[s], o_logits[s]) <= FP32_TOL, s
        top2 = torch.topk(o_logits[s], 2, dim=-1).values
        if ((top2[:, 0] - top2[:, 1]) < 1e-4).any():
            break                                      # a near-tie: later steps may follow another token
        assert torch.equal(toks[:, s], o_ids[:, 16 + s]), s


def test_generate_bf16_teacher_forced():
    """bf16 MLA generation: the oracle run over the GPU's own sequence gives, at every
    step, logits within the bf16 tolerance and the GPU's token as its argmax up to
    near-ties (the oracle's top logit minus the chosen one under 2e-2 of the logit range)."""
    wl = RI.get_workload("tiny_mla_bf16")
    cfg = wl.cfg
    MW = RI.model_weights(cfg, wl.seed)
    prompt = torch.randint(0, cfg.vocab_size, (2, 16), generator=torch.Generator().manual_seed(7))
    new = 8
    toks, logits = _gpu_generate(cfg, to_dev(MW), prompt, new, 8, wl.act_threshold)
    seq = torch.cat([prompt, toks], dim=1)
    full, _, _ = O.model_forward(cfg, MW, seq[:, :-1], 8, wl.act_threshold)
    for s in range(new):
        ol = full[:, 15 + s]
        assert rel_l2(logits[s], ol) <= BF16_TOL, s
        gap = ol.max(-1).values - ol.gather(1, toks[:, s:s + 1])[:, 0]
        span = ol.max(-1).values - ol.min(-1).values
        assert (gap <= 2e-2 * span).all(), s


@pytest.mark.parametrize("name", ["tiny_gqa_fp32", "tiny_mla_bf16"])
def test_graph_replay_equals_eager(name):
    """The Generator's CUDA-graph replay of the decode step gives the eager steps' tokens
    and logits bit for bit (same kernels, same fixed buffers; the step's inputs are copied
    into place before each replay)."""
    wl = RI.get_workload(name)
    cfg = wl.cfg
    MW = to_dev(RI.model_weights(cfg, wl.seed))
    prompt = torch.randint(0, cfg.vocab_size, (2, 16), generator=torch.Generator().manual_seed(9))
    ids = prompt.to(device="cuda", dtype=torch.int32).contiguous()
    runs = []
    for graph in (False, True):
        gen = R.Generator(cfg, MW, 2, 16, 8, 8, wl.act_threshold, cuda_graph=graph)
        gen.prefill(ids)
        logits = []
        for s in range(1, 8):
            gen.decode(s)
            logits.append(gen.logits.clone())
        torch.cuda.synchronize()
        runs.append((gen.tokens.clone(), torch.stack(logits), gen._graph is not None, gen.graph_launches))
    assert not runs[0][2] and runs[1][2] and runs[1][3] > 0
    assert torch.equal(runs[0][0], runs[1][0])
    assert torch.equal(runs[0][1], runs[1][1])
