"""CUDA-graph replay of the decode step (DecodeGraph) against eager decode steps: the same
outputs and the same cache contents, bit for bit, over several steps (same kernels, same
inputs; the graph reads its inputs from fixed buffers and advances the cache length
itself).  GQA and MLA (latent cache, absorbed attention) blocks."""
import pytest
import torch

import rdt_inputs as RI
from tests._helpers import to_dev

pytestmark = pytest.mark.gpu

R = pytest.importorskip("recurrent_depth_moe_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    R.load_library()


def _mla_cfg():
    return RI.RDTConfig(dim=512, n_heads=4, n_kv_heads=4, max_seq_len=256, max_loop_iters=4, n_experts=8,
                        n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, attn_type="mla",
                        kv_lora_rank=128, q_lora_rank=192, qk_rope_head_dim=32, qk_nope_head_dim=64,
                        v_head_dim=64, dtype="bf16")


@pytest.mark.parametrize("kind", ["gqa", "mla"])
def test_decode_graph_equals_eager_steps(kind):
    cfg = RI.get_workload("mid_gqa_bf16").cfg if kind == "gqa" else _mla_cfg()
    W = to_dev(RI.block_weights(cfg, 71, attn_std=0.05))
    B, L, t_max, filled, n_steps = 4, 3, 64, 20, 6
    make = RI.random_kv_cache if kind == "gqa" else RI.random_latent_cache
    k, v = make(cfg, L, B, t_max, filled, 72)
    inputs = [RI.decode_inputs(cfg, B, st, 73) for st in range(n_steps)]
    blk = R.RecurrentBlock(cfg, W)

    cache_a = R.KVCache(k.clone().cuda(), v.clone().cuda())
    clen_a = torch.full((B,), filled, dtype=torch.int32, device="cuda")
    eager = []
    for h, e in inputs:
        o = blk.decode_step(h.cuda(), e.cuda(), clen_a, cache_a, L, 0.0)
        eager.append(tuple(t.clone() for t in o))
        clen_a.add_(1)

    cache_b = R.KVCache(k.clone().cuda(), v.clone().cuda())
    clen_b = torch.full((B,), filled, dtype=torch.int32, device="cuda")
    dg = R.DecodeGraph(blk, B, cache_b, clen_b, L, 0.0)
    graphed = []
    for h, e in inputs:
        o = dg.step(h.cuda(), e.cuda())
        graphed.append(tuple(t.clone() for t in o))
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    assert dg._graph is not None and dg.graph_launches > 0
    for st in range(n_steps):
        for a, b in zip(eager[st], graphed[st]):
            assert torch.equal(a, b), f"step {st}"
    assert torch.equal(clen_a, clen_b)
    assert torch.equal(cache_a.k, cache_b.k) and torch.equal(cache_a.v, cache_b.v)
