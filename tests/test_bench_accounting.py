"""The bench's roofline accounting (algorithmic FLOPs and bytes), checked against the sizes
of the tensors the workloads actually allocate rather than against its own formulas."""
import os
import sys

import torch

import rdt_inputs as RI

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
import bench  # noqa: E402  (the module only defines; main() runs under __main__)


def _bytes(*ts, elem=2):
    return sum(t.numel() for t in ts) * elem


def test_attention_weight_bytes_match_the_weight_tensors():
    for name, keys in (("tiny_gqa_fp32", ("w_qkv", "w_o")),
                       ("tiny_mla_fp32", ("w_q_down", "w_q_up", "w_kv_down", "w_kv_up", "w_o"))):
        cfg = RI.get_workload(name).cfg
        W = RI.block_weights(cfg, 1)
        assert bench.attn_weight_bytes(cfg) == _bytes(*(W[k] for k in keys)), name


def test_cache_bytes_per_key_match_the_cache_tensors():
    cfg = RI.get_workload("mid_gqa_bf16").cfg
    k, v = RI.random_kv_cache(cfg, 2, 3, 16, 4, 1)          # [L, B, Hkv, t_max, hd]
    per_key = (k[0, 0, :, 0].numel() + v[0, 0, :, 0].numel()) * k.element_size()
    assert bench.cache_bytes_per_key(cfg) == per_key
    mla = RI.get_workload("tiny_mla_bf16").cfg
    c, r = RI.random_latent_cache(mla, 2, 3, 16, 4, 1)      # [L, B, t_max, kvr], [L, B, t_max, dr]
    assert bench.cache_bytes_per_key(mla) == (c[0, 0, 0].numel() + r[0, 0, 0].numel()) * c.element_size()


def test_expert_up_flops_count_two_flops_per_weight_per_row():
    wl = RI.get_workload("rdt1b_prefill")
    cfg = wl.cfg
    per_expert_w13 = 2 * cfg.expert_dim * cfg.dim             # gate and up rows of one expert
    rows = 16384 * (cfg.n_experts_per_tok + cfg.n_shared_experts)
    assert bench.expert_up_flops(wl, 16384) == 2.0 * rows * per_expert_w13
    assert bench.expert_up_flops(wl, 16384) == 1374389534720.0


def test_decode_bytes_follow_the_realised_routing():
    cfg = RI.get_workload("tiny_gqa_fp32").cfg.replace(dtype="bf16")
    W = RI.block_weights(cfg, 1)
    expert = _bytes(W["w13"][0], W["w2"][0])
    fixed = _bytes(W["w_qkv"], W["w_o"]) + _bytes(W["w_router"], W["lora_down"], W["lora_B"])
    k, _ = RI.random_kv_cache(cfg, 1, 1, 4, 1, 1)
    per_key = 2 * k[0, 0, :, 0].numel() * 2
    lens = torch.tensor([5, 9, 0])
    # loop 0 touches experts {1, 4}; loop 1 only {4}; -1 marks a halted row
    ids = torch.tensor([[[1, 4], [4, 1], [1, 1]],
                        [[4, 4], [-1, -1], [4, 4]]])
    got = bench.decode_algorithmic_bytes(cfg, ids, lens)
    kv = (5 + 1 + 9 + 1 + 0 + 1) * per_key
    S = cfg.n_shared_experts
    want = (2 + S) * expert + fixed + kv + (1 + S) * expert + fixed + kv
    assert got == want
    # a halted row adds nothing; repeating an expert adds nothing
    ids2 = ids.clone()
    ids2[1, 0] = -1
    assert bench.decode_algorithmic_bytes(cfg, ids2, lens) == got


def test_attention_flops_count_the_keys_each_running_row_sees():
    """Brute force over (loop, row, key): a row at position p that runs loop t sees keys
    0 .. p; each (query, key) pair costs (score dim + value dim) multiply-adds per head."""
    for name in ("mid_gqa_bf16", "tiny_mla_bf16"):
        cfg = RI.get_workload(name).cfg
        T, L = 5, 3
        last = torch.tensor([2, 0, 1, 2, 2, 0, 0, 1, 2, 1])    # two sequences of 5; last loop each row ran
        d = (2 * cfg.head_dim) if cfg.attn_type == "gqa" else \
            (cfg.qk_nope_head_dim + cfg.qk_rope_head_dim + cfg.v_head_dim)
        want = 0
        for t in range(L):
            for i in range(last.numel()):
                if t <= int(last[i]):
                    for key in range(i % T + 1):
                        want += 2 * cfg.n_heads * d
        assert bench.attention_flops_executed(cfg, last, T) == float(want), name
