"""Prefill attention at sequence lengths around its 128-query / 128-key tiles (head dim
128, bf16: the tcgen05 kernel when T is a multiple of 8, the mma.sync kernel otherwise).
Checked for one loop, teacher-forced: from the kernel's own state entering the loop, the
attention branch's share of the FFN input f = RMSNorm_ffn(x + Attn(RMSNorm_attn(x))), i.e.
f minus RMSNorm_ffn(x), in the oracle and in the kernel's trace of f ("OpenMythos 분석", Core
Structure: causal self-attention inside the pre-norm block).
Peaky attention weights (std 0.08) so that the softmax is far from uniform."""
import pytest
import torch

import rdt_inputs as RI
from oracle import rdt_oracle as O
from tests._helpers import BF16_TOL, rel_l2, to_dev

pytestmark = pytest.mark.gpu

R = pytest.importorskip("recurrent_depth_moe_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    R.load_library()


# 8: one short query tile; 120 / 128 / 136: around one tile; 256 / 264: one full pair and a
# pair plus 8 rows; 392: two pairs, the last tile 8 rows; 520: five tiles (a pair with one
# tile); 100: not a multiple of 8 (the mma.sync kernel)
@pytest.mark.parametrize("T", [8, 120, 128, 136, 256, 264, 392, 520, 100])
def test_attention_tile_edges(T):
    cfg = RI.get_workload("mid_gqa_bf16").cfg
    W = RI.block_weights(cfg, 31, attn_std=0.08)
    B, L = 2, 1
    h0, e = RI.recurrent_inputs(cfg, B, T, 32)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    tr = R.Trace.alloc(cfg, L, 0, B * T)
    blk.forward(h0.cuda(), e.cuda(), B, T, L, 0.99, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    h_in = tr.h_in[0].cpu().double()
    emb = O.loop_embedding(0, cfg.loop_dim, cfg.dim, cfg.loop_theta)
    comb = O.rmsnorm(h_in + emb + e.double(), W["rec_norm_w"], cfg.norm_eps)
    pos = torch.arange(B * T) % T
    _, _, info = O.transformer_block(cfg, W, comb, B, pos, True)
    # the attention branch's share of f: f with the branch minus f without it
    f0 = O.rmsnorm(comb, W["ffn_norm_w"], cfg.norm_eps)
    d_o = info["f"] - f0
    d_k = tr.f[0].cpu().double() - f0
    assert rel_l2(d_o, info["f"]) > 0.05, "attention barely moves f: the check would be weak"
    for b in range(B):   # every sequence on its own
        rows = slice(b * T, (b + 1) * T)
        err = rel_l2(d_k[rows], d_o[rows])
        assert err <= BF16_TOL, f"sequence {b}: relative L2 of the attention branch {err:.3e}"
    # the last query row of each sequence sees every key: compare it on its own too
    last = [b * T + T - 1 for b in range(B)]
    assert rel_l2(d_k[last], d_o[last]) <= BF16_TOL


def test_attention_rescales_at_the_diagonal_tile():
    """The tensor-core prefill attention's lazy rescale, forced: each query head's projection
    is 0.3 x its group's key projection, and the second half of every sequence carries one
    common direction, so a query there scores its own (diagonal) key tile about 13 log2 units
    above the random keys before it, past the 2^8 threshold: its running maximum is raised
    and the O accumulator rescaled in TMEM (checked on the oracle's scores below).  T = 512:
    two key tiles before the raise."""
    import math
    cfg = RI.get_workload("mid_gqa_bf16").cfg
    H, Hkv, hd, D = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.dim
    G = H // Hkv
    W = RI.block_weights(cfg, 41, attn_std=0.08)
    wq = W["w_qkv"].clone()
    for h in range(H):
        g = h // G
        wq[h * hd:(h + 1) * hd] = (0.3 * wq[(H + g) * hd:(H + g + 1) * hd].float()).to(wq.dtype)
    W["w_qkv"] = wq
    B, T, L = 2, 512, 1
    h0, e = RI.recurrent_inputs(cfg, B, T, 42)
    u = torch.randn(D, generator=torch.Generator().manual_seed(43))
    h0 = h0.view(B, T, D).clone()
    h0[:, T // 2:] = 20 * u + 0.1 * h0[:, T // 2:]
    h0 = h0.view(B * T, D)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    tr = R.Trace.alloc(cfg, L, 0, B * T)
    blk.forward(h0.cuda(), e.cuda(), B, T, L, 0.99, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    h_in = tr.h_in[0].cpu().double()
    emb = O.loop_embedding(0, cfg.loop_dim, cfg.dim, cfg.loop_theta)
    comb = O.rmsnorm(h_in + emb + e.double(), W["rec_norm_w"], cfg.norm_eps)
    # the construction works: every query of the second half raises its running maximum (log2
    # units, 128-key tiles in order) by more than 8 at its diagonal tile, head 0 of sequence 0
    a = O.rmsnorm(comb[:T], W["attn_norm_w"], cfg.norm_eps)
    qkv = a @ W["w_qkv"].double().T
    pos = torch.arange(T)
    q = O.rope(qkv[:, :H * hd].view(T, H, hd), pos, cfg.rope_theta)[:, 0]
    k = O.rope(qkv[:, H * hd:(H + Hkv) * hd].view(T, Hkv, hd), pos, cfg.rope_theta)[:, 0]
    sc = (q @ k.T) * (1.4426950408889634 / math.sqrt(hd))
    for i in range(T // 2, T):
        m0 = float(sc[i, :T // 2].max())
        assert float(sc[i, (i // 128) * 128:i + 1].max()) > m0 + 8
    pos_all = torch.arange(B * T) % T
    _, _, info = O.transformer_block(cfg, W, comb, B, pos_all, True)
    f0 = O.rmsnorm(comb, W["ffn_norm_w"], cfg.norm_eps)
    d_o = info["f"] - f0
    d_k = tr.f[0].cpu().double() - f0
    for b in range(B):
        hot = slice(b * T + T // 2, (b + 1) * T)
        err = rel_l2(d_k[hot], d_o[hot])
        assert err <= BF16_TOL, f"sequence {b}: relative L2 of the attention branch over the raised rows {err:.3e}"
        rows = slice(b * T, (b + 1) * T)
        assert rel_l2(d_k[rows], d_o[rows]) <= BF16_TOL


def _mla_wide(H=24):
    # DeepSeek-V2 head widths (nope 128, rope 64, value 128, kv_lora_rank 512): the
    # tensor-core MLA prefill kernel's shape
    return RI.RDTConfig(dim=1536, n_heads=H, n_kv_heads=H, max_seq_len=1024, max_loop_iters=2, n_experts=8,
                        n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, attn_type="mla",
                        kv_lora_rank=512, q_lora_rank=256, qk_rope_head_dim=64, qk_nope_head_dim=128,
                        v_head_dim=128, dtype="bf16")


# MLA prefill on the tensor cores (one 128-query tile per CTA, keys [k_nope | shared k_rope],
# values read in place): around one tile, several tiles with a ragged last one
@pytest.mark.parametrize("T", [8, 128, 136, 300, 520])
def test_mla_attention_tile_edges(T):
    cfg = _mla_wide()
    W = RI.block_weights(cfg, 33, attn_std=0.05)
    B, L = 2, 1
    h0, e = RI.recurrent_inputs(cfg, B, T, 34)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    tr = R.Trace.alloc(cfg, L, 0, B * T)
    blk.forward(h0.cuda(), e.cuda(), B, T, L, 0.99, trace=tr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    h_in = tr.h_in[0].cpu().double()
    emb = O.loop_embedding(0, cfg.loop_dim, cfg.dim, cfg.loop_theta)
    comb = O.rmsnorm(h_in + emb + e.double(), W["rec_norm_w"], cfg.norm_eps)
    pos = torch.arange(B * T) % T
    _, _, info = O.transformer_block(cfg, W, comb, B, pos, True)
    f0 = O.rmsnorm(comb, W["ffn_norm_w"], cfg.norm_eps)
    d_o = info["f"] - f0
    d_k = tr.f[0].cpu().double() - f0
    assert rel_l2(d_o, info["f"]) > 0.05, "attention barely moves f: the check would be weak"
    for b in range(B):
        rows = slice(b * T, (b + 1) * T)
        err = rel_l2(d_k[rows], d_o[rows])
        assert err <= BF16_TOL, f"sequence {b}: relative L2 of the MLA attention branch {err:.3e}"
