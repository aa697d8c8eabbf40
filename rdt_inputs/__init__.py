"""Seeded synthetic inputs for the looped Recurrent Block (OpenMythos RDT).

This module is shared by the CPU oracle and the CUDA path as *data only*: it
holds the workload configurations and draws weights and activations from
seeded generators.  It contains none of the method's arithmetic (no norm, no
attention, no routing, no injection, no halting); the two consumers compute
those independently.

Shapes follow the model-variant table and the tiny usage script of the
OpenMythos README mirror (runchr.com "OpenMythos", sections "사용법" and
"모델 변형"), and the workload recipes stated in the design notes.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Optional

import torch

__all__ = [
    "RDTConfig", "Workload", "WORKLOADS", "get_workload",
    "block_weights", "dense_block_weights", "model_weights",
    "unit_rms_rows", "recurrent_inputs", "decode_inputs", "random_kv_cache",
    "halting_offsets_spread", "zipf_router_bias", "param_count_formula",
]


@dataclass
class RDTConfig:
    """Mirror of ``MythosConfig`` fields (README usage script) plus the
    constants the pages leave open (fixed readings: loop_dim = dim // 8,
    loop_theta = rope_theta = 10000, norm_eps = 1e-6)."""
    vocab_size: int = 1000
    dim: int = 256
    n_heads: int = 8
    n_kv_heads: int = 2
    max_seq_len: int = 128
    max_loop_iters: int = 4
    prelude_layers: int = 1
    coda_layers: int = 1
    n_experts: int = 8
    n_shared_experts: int = 1
    n_experts_per_tok: int = 2
    expert_dim: int = 64
    lora_rank: int = 8
    attn_type: str = "gqa"          # "gqa" | "mla"
    kv_lora_rank: int = 0
    q_lora_rank: int = 0
    qk_rope_head_dim: int = 0
    qk_nope_head_dim: int = 0
    v_head_dim: int = 0
    rope_theta: float = 10000.0
    loop_theta: float = 10000.0
    loop_dim: Optional[int] = None   # None -> dim // 8
    norm_eps: float = 1e-6
    dtype: str = "fp32"              # "fp32" | "bf16": storage of matrices, e, GEMM inputs

    def __post_init__(self):
        if self.loop_dim is None:
            self.loop_dim = self.dim // 8

    @property
    def head_dim(self) -> int:
        return self.dim // self.n_heads

    @property
    def dense_hidden(self) -> int:
        # Prelude/Coda FFN is Expert(dim, dim * 4 // 3) ("OpenMythos 분석", MoE section)
        return self.dim * 4 // 3

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def replace(self, **kw) -> "RDTConfig":
        return dataclasses.replace(self, **kw)


@dataclass
class Workload:
    name: str
    cfg: RDTConfig
    batch: int
    seq: int
    n_loops: int
    seed: int
    act_threshold: float            # <= 0: ACT off
    kind: str = "prefill"           # "prefill" | "decode" | "model" | "generate"
    halt_b: float = 0.0             # halting-head bias
    halt_spread: Optional[tuple] = None   # (lo, hi): per-position halting loop via logit offset
    zipf_s: Optional[float] = None  # router bias giving Zipf-like popularity
    cache_len: int = 0              # decode: tokens already in each loop's cache
    decode_steps: int = 0
    device_weights: bool = False    # draw weights with a device generator (too large for host)
    notes: str = ""


def _tiny_base(**kw) -> RDTConfig:
    base = dict(vocab_size=1000, dim=256, n_heads=8, max_seq_len=128, max_loop_iters=4,
                prelude_layers=1, coda_layers=1, n_experts=8, n_shared_experts=1,
                n_experts_per_tok=2, expert_dim=64, lora_rank=8)
    base.update(kw)
    return RDTConfig(**base)


WORKLOADS = {
    # Tiny RDT, fp32, GQA: the README usage script's config; batch 2 x seq 16; ACT off.
    "tiny_gqa_fp32": Workload("tiny_gqa_fp32", _tiny_base(n_kv_heads=2, dtype="fp32"),
                              batch=2, seq=16, n_loops=4, seed=0, act_threshold=0.0, kind="model"),
    # Tiny RDT with MLA, fp32 and bf16; batch 8 x seq 128; 8 loops > max_loop_iters 4; ACT 0.99.
    "tiny_mla_fp32": Workload("tiny_mla_fp32", _tiny_base(
        attn_type="mla", n_kv_heads=8, kv_lora_rank=32, q_lora_rank=64, qk_rope_head_dim=16,
        qk_nope_head_dim=16, v_head_dim=16, dtype="fp32"),
        batch=8, seq=128, n_loops=8, seed=1, act_threshold=0.99, kind="model"),
    "tiny_mla_bf16": Workload("tiny_mla_bf16", _tiny_base(
        attn_type="mla", n_kv_heads=8, kv_lora_rank=32, q_lora_rank=64, qk_rope_head_dim=16,
        qk_nope_head_dim=16, v_head_dim=16, dtype="bf16"),
        batch=8, seq=128, n_loops=8, seed=1, act_threshold=0.99, kind="model"),
    # 1B-shaped recurrent block prefill (mythos_1b: dim 2048, 64 experts, expert_dim 2048, 16 loops).
    "rdt1b_prefill": Workload("rdt1b_prefill", RDTConfig(
        dim=2048, n_heads=16, n_kv_heads=4, max_seq_len=4096, max_loop_iters=16,
        n_experts=64, n_shared_experts=1, n_experts_per_tok=4, expert_dim=2048, lora_rank=16,
        dtype="bf16"), batch=4, seq=4096, n_loops=16, seed=2, act_threshold=0.99, halt_b=-30.0,
        device_weights=True),
    # 3B-shaped KV-cached decode (mythos_3b: dim 3072, 64 experts, expert_dim 4096, 16 loops).
    "rdt3b_decode": Workload("rdt3b_decode", RDTConfig(
        dim=3072, n_heads=24, n_kv_heads=8, max_seq_len=4096 + 128, max_loop_iters=16,
        n_experts=64, n_shared_experts=1, n_experts_per_tok=4, expert_dim=4096, lora_rank=16,
        dtype="bf16"), batch=64, seq=1, n_loops=16, seed=3, act_threshold=0.0, kind="decode",
        cache_len=4096, decode_steps=128, device_weights=True),
    # The same decode with multi-latent attention: the pages fix MLA dims only for the tiny
    # model, so the latent widths are DeepSeek-V2's (the MLA design the pages cite):
    # kv_lora_rank 512, q_lora_rank 1536, rope 64, nope 128, v 128.  Per loop and token the
    # latent cache holds (512 + 64) x 2 bytes against 2 x 8 x 128 x 2 for the GQA cache.
    "rdt3b_mla_decode": Workload("rdt3b_mla_decode", RDTConfig(
        dim=3072, n_heads=24, n_kv_heads=24, max_seq_len=4096 + 128, max_loop_iters=16,
        n_experts=64, n_shared_experts=1, n_experts_per_tok=4, expert_dim=4096, lora_rank=16,
        attn_type="mla", kv_lora_rank=512, q_lora_rank=1536, qk_rope_head_dim=64, qk_nope_head_dim=128,
        v_head_dim=128, dtype="bf16"), batch=64, seq=1, n_loops=16, seed=5, act_threshold=0.0, kind="decode",
        cache_len=4096, decode_steps=128, device_weights=True),
    # MLA prefill at the 3B MLA shape (the widths of rdt3b_mla_decode): 1 x 4096, 16 loops,
    # halting bias -30 as in the 1B prefill; the workload of the tensor-core MLA prefill line.
    "rdt3b_mla_prefill": Workload("rdt3b_mla_prefill", RDTConfig(
        dim=3072, n_heads=24, n_kv_heads=24, max_seq_len=4096, max_loop_iters=16,
        n_experts=64, n_shared_experts=1, n_experts_per_tok=4, expert_dim=4096, lora_rank=16,
        attn_type="mla", kv_lora_rank=512, q_lora_rank=1536, qk_rope_head_dim=64, qk_nope_head_dim=128,
        v_head_dim=128, dtype="bf16"), batch=1, seq=4096, n_loops=16, seed=12, act_threshold=0.99, halt_b=-30.0,
        device_weights=True),
    # The 3B-shaped decode with ACT on and a per-token halting spread over 4..16 loops (zero
    # halting head, per-token logit offsets as in the 10B prefill): the workload on which
    # continuous depth-wise batching is compared with lockstep decode steps.  64 sequences,
    # 64 new tokens each.
    "rdt3b_decode_halting": Workload("rdt3b_decode_halting", RDTConfig(
        dim=3072, n_heads=24, n_kv_heads=8, max_seq_len=4096 + 128, max_loop_iters=16,
        n_experts=64, n_shared_experts=1, n_experts_per_tok=4, expert_dim=4096, lora_rank=16,
        dtype="bf16"), batch=64, seq=1, n_loops=16, seed=9, act_threshold=0.99, kind="decode",
        halt_spread=(4, 16), cache_len=4096, decode_steps=64, device_weights=True),
    # Greedy generation with the 1B-shaped model: the recurrent block of rdt1b_prefill, one
    # prelude and one coda layer (the usage script's counts; the variant table gives none)
    # and the vocabulary of the tokenizer the pages name (openai/gpt-oss-20b: 201,088
    # tokens).  64 sequences, 128-token prompts, 128 new tokens each.
    "rdt1b_generate": Workload("rdt1b_generate", RDTConfig(
        vocab_size=201088, dim=2048, n_heads=16, n_kv_heads=4, max_seq_len=4096, max_loop_iters=16,
        prelude_layers=1, coda_layers=1, n_experts=64, n_shared_experts=1, n_experts_per_tok=4,
        expert_dim=2048, lora_rank=16, dtype="bf16"), batch=64, seq=128, n_loops=16, seed=8,
        act_threshold=0.99, halt_b=-30.0, kind="generate", decode_steps=128, device_weights=True),
    # Profiling case for the latent attention: the attention of rdt3b_mla_decode (same
    # heads, latent widths, batch and cache length) with a small MoE and 2 loops, so that
    # well under 1 GB is held on the device.
    "mla_decode_attn_small": Workload("mla_decode_attn_small", RDTConfig(
        dim=3072, n_heads=24, n_kv_heads=24, max_seq_len=4096 + 128, max_loop_iters=2,
        n_experts=8, n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=16,
        attn_type="mla", kv_lora_rank=512, q_lora_rank=1536, qk_rope_head_dim=64, qk_nope_head_dim=128,
        v_head_dim=128, dtype="bf16"), batch=64, seq=1, n_loops=2, seed=6, act_threshold=0.0, kind="decode",
        cache_len=4096, decode_steps=8, device_weights=True),
    # Profiling case for the GQA decode attention: the attention of rdt3b_decode (24 heads,
    # 8 kv heads, 64 sequences, 4096-token caches) with a small MoE and 2 loops (about 2.2 GB
    # of caches on the device).
    "decode_attn_small": Workload("decode_attn_small", RDTConfig(
        dim=3072, n_heads=24, n_kv_heads=8, max_seq_len=4096 + 128, max_loop_iters=2,
        n_experts=8, n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=16,
        dtype="bf16"), batch=64, seq=1, n_loops=2, seed=10, act_threshold=0.0, kind="decode",
        cache_len=4096, decode_steps=8, device_weights=True),
    # Profiling case for the decode expert GEMMs and routing: the MoE of rdt3b_decode (64
    # routed + 1 shared experts of width 4096, top-4, 64 sequences) with 1 loop and short
    # caches (about 5 GB of expert weights on the device).
    "decode_moe_small": Workload("decode_moe_small", RDTConfig(
        dim=3072, n_heads=24, n_kv_heads=8, max_seq_len=512, max_loop_iters=1,
        n_experts=64, n_shared_experts=1, n_experts_per_tok=4, expert_dim=4096, lora_rank=16,
        dtype="bf16"), batch=64, seq=1, n_loops=1, seed=11, act_threshold=0.0, kind="decode",
        cache_len=256, decode_steps=8, device_weights=True),
    # 10B-shaped prefill, load-imbalanced (mythos_10b: dim 4096, 128 experts, expert_dim 5632, 24 loops).
    "rdt10b_prefill_zipf": Workload("rdt10b_prefill_zipf", RDTConfig(
        dim=4096, n_heads=32, n_kv_heads=8, max_seq_len=8192, max_loop_iters=24,
        n_experts=128, n_shared_experts=1, n_experts_per_tok=8, expert_dim=5632, lora_rank=16,
        dtype="bf16"), batch=2, seq=8192, n_loops=24, seed=4, act_threshold=0.9,
        halt_spread=(4, 24), zipf_s=1.1, device_weights=True),
    # Test-only mid-size block: several GEMM tiles with ragged tails, hd 128 attention.
    "mid_gqa_bf16": Workload("mid_gqa_bf16", RDTConfig(
        dim=512, n_heads=4, n_kv_heads=2, max_seq_len=512, max_loop_iters=2,
        n_experts=8, n_shared_experts=1, n_experts_per_tok=2, expert_dim=256, lora_rank=8,
        dtype="bf16"), batch=2, seq=200, n_loops=3, seed=5, act_threshold=0.99),
    # Test-only: router widths of the 1B / 10B shapes (fused tensor-core routing), ragged expert segments.
    "mid_e64_bf16": Workload("mid_e64_bf16", RDTConfig(
        dim=512, n_heads=4, n_kv_heads=2, max_seq_len=512, max_loop_iters=2,
        n_experts=64, n_shared_experts=1, n_experts_per_tok=4, expert_dim=128, lora_rank=16,
        dtype="bf16"), batch=2, seq=200, n_loops=3, seed=6, act_threshold=0.99),
    "mid_e128_bf16": Workload("mid_e128_bf16", RDTConfig(
        dim=512, n_heads=4, n_kv_heads=1, max_seq_len=512, max_loop_iters=2,
        n_experts=128, n_shared_experts=1, n_experts_per_tok=8, expert_dim=128, lora_rank=16,
        dtype="bf16"), batch=1, seq=300, n_loops=2, seed=7, act_threshold=0.9),
    # Test-only: several query-tile pairs with a ragged last tile (tensor-core attention), GQA group 4.
    "mid_t392_bf16": Workload("mid_t392_bf16", RDTConfig(
        dim=512, n_heads=4, n_kv_heads=1, max_seq_len=512, max_loop_iters=2,
        n_experts=8, n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8,
        dtype="bf16"), batch=2, seq=392, n_loops=2, seed=8, act_threshold=0.99),
    "mid_gqa_fp32": Workload("mid_gqa_fp32", RDTConfig(
        dim=512, n_heads=4, n_kv_heads=2, max_seq_len=512, max_loop_iters=2,
        n_experts=8, n_shared_experts=1, n_experts_per_tok=2, expert_dim=256, lora_rank=8,
        dtype="fp32"), batch=2, seq=200, n_loops=3, seed=5, act_threshold=0.99),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


# --------------------------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------------------------

def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, g, dtype, device):
    return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)


def _attn_weights(cfg: RDTConfig, g, dt, device, std: float) -> dict:
    D, H = cfg.dim, cfg.n_heads
    w = {}
    if cfg.attn_type == "gqa":
        hd, Hkv = cfg.head_dim, cfg.n_kv_heads
        w["w_qkv"] = _normal(((H + 2 * Hkv) * hd, D), std, g, dt, device)
        w["w_o"] = _normal((D, H * hd), std, g, dt, device)
    else:
        dn, dr, dv = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
        w["w_q_down"] = _normal((cfg.q_lora_rank, D), std, g, dt, device)
        w["q_norm_w"] = torch.ones(cfg.q_lora_rank, dtype=torch.float32, device=device)
        w["w_q_up"] = _normal((H * (dn + dr), cfg.q_lora_rank), std, g, dt, device)
        w["w_kv_down"] = _normal((cfg.kv_lora_rank + dr, D), std, g, dt, device)
        w["kv_norm_w"] = torch.ones(cfg.kv_lora_rank, dtype=torch.float32, device=device)
        w["w_kv_up"] = _normal((H * (dn + dv), cfg.kv_lora_rank), std, g, dt, device)
        w["w_o"] = _normal((D, H * dv), std, g, dt, device)
    return w


def block_weights(cfg: RDTConfig, seed: int, device="cpu", *, std: float = 0.02,
                  attn_std: Optional[float] = None, lora_scale_std: Optional[float] = None,
                  a_range=(0.5, 0.95), inj_b: float = 0.1, halt_b: float = 0.0,
                  halt_w_std: Optional[float] = None, router_bias=None) -> dict:
    """Recurrent-block weights.  Linear weights N(0, std); norm weights 1;
    LTI: a_i ~ U[a_range], log_dt = 0, log_A = log(-log a_i) (so exp(-exp(log_A)) = a_i);
    injection B = inj_b * 1; halting head N(0, std) weight and constant bias."""
    D, E, S, F, r = cfg.dim, cfg.n_experts, cfg.n_shared_experts, cfg.expert_dim, cfg.lora_rank
    dt = cfg.torch_dtype
    g = _gen(seed, device)
    f32 = torch.float32
    w = {
        "rec_norm_w": torch.ones(D, dtype=f32, device=device),
        "attn_norm_w": torch.ones(D, dtype=f32, device=device),
        "ffn_norm_w": torch.ones(D, dtype=f32, device=device),
    }
    w.update(_attn_weights(cfg, g, dt, device, attn_std if attn_std is not None else std))
    w["w_router"] = _normal((E, D), std, g, dt, device)
    if router_bias is None:
        w["router_bias"] = torch.zeros(E, dtype=f32, device=device)
    else:
        w["router_bias"] = router_bias.to(device=device, dtype=f32)
    w13 = torch.empty((E + S, 2 * F, D), dtype=dt, device=device)
    w2 = torch.empty((E + S, D, F), dtype=dt, device=device)
    for x in range(E + S):   # per expert, so device memory for fp32 draws stays small
        w13[x] = _normal((2 * F, D), std, g, dt, device)
        w2[x] = _normal((D, F), std, g, dt, device)
    w["w13"], w["w2"] = w13, w2
    w["lora_down"] = _normal((r, D), std, g, dt, device)
    w["lora_B"] = _normal((r, D), std, g, dt, device)
    w["lora_scale"] = _normal((cfg.max_loop_iters, r),
                              lora_scale_std if lora_scale_std is not None else std, g, f32, device)
    a = torch.rand(D, generator=g, device=device, dtype=torch.float64) * (a_range[1] - a_range[0]) + a_range[0]
    w["log_A"] = torch.log(-torch.log(a)).to(f32)
    w["log_dt"] = torch.zeros(1, dtype=f32, device=device)
    w["inj_B"] = torch.full((D,), inj_b, dtype=f32, device=device)
    w["halt_w"] = _normal((D,), halt_w_std if halt_w_std is not None else std, g, f32, device)
    w["halt_b"] = torch.full((1,), halt_b, dtype=f32, device=device)
    return w


def dense_block_weights(cfg: RDTConfig, seed: int, device="cpu", std: float = 0.02) -> dict:
    """Prelude/Coda block: pre-norm attention + dense SwiGLU Expert(dim, dim*4//3)."""
    D, Fd = cfg.dim, cfg.dense_hidden
    dt = cfg.torch_dtype
    g = _gen(seed, device)
    w = {"attn_norm_w": torch.ones(D, dtype=torch.float32, device=device),
         "ffn_norm_w": torch.ones(D, dtype=torch.float32, device=device)}
    w.update(_attn_weights(cfg, g, dt, device, std))
    w["w13"] = _normal((1, 2 * Fd, D), std, g, dt, device)
    w["w2"] = _normal((1, D, Fd), std, g, dt, device)
    return w


def model_weights(cfg: RDTConfig, seed: int, device="cpu", std: float = 0.02, **block_kw) -> dict:
    """Full tiny model: embedding, prelude blocks, recurrent block, coda blocks,
    final norm and an untied LM head."""
    g = _gen(seed + 1000, device)
    dt = cfg.torch_dtype
    return {
        "embed": _normal((cfg.vocab_size, cfg.dim), std, g, dt, device),
        "prelude": [dense_block_weights(cfg, seed * 100 + 10 + i, device, std) for i in range(cfg.prelude_layers)],
        "recurrent": block_weights(cfg, seed, device, std=std, **block_kw),
        "coda": [dense_block_weights(cfg, seed * 100 + 50 + i, device, std) for i in range(cfg.coda_layers)],
        "norm_w": torch.ones(cfg.dim, dtype=torch.float32, device=device),
        "head": _normal((cfg.vocab_size, cfg.dim), std, g, dt, device),
    }


def unit_rms_rows(x: torch.Tensor) -> torch.Tensor:
    """Input recipe: scale each row of an N(0,1) draw to unit root-mean-square."""
    x64 = x.double()
    return (x64 / torch.sqrt((x64 * x64).mean(-1, keepdim=True))).float()


def recurrent_inputs(cfg: RDTConfig, batch: int, seq: int, seed: int, device="cpu"):
    """h0 (fp32) and e (model dtype), rows drawn N(0,1) then scaled to unit RMS."""
    g = _gen(seed + 7, device)
    N = batch * seq
    h0 = unit_rms_rows(torch.randn(N, cfg.dim, generator=g, device=device))
    e = unit_rms_rows(torch.randn(N, cfg.dim, generator=g, device=device)).to(cfg.torch_dtype)
    return h0, e


def decode_inputs(cfg: RDTConfig, batch: int, step: int, seed: int, device="cpu"):
    """One decode step's new-token h0 / e rows (unit RMS), seeded per step."""
    return recurrent_inputs(cfg, batch, 1, seed * 100003 + step, device)


def random_kv_cache(cfg: RDTConfig, n_loops: int, batch: int, t_max: int, filled: int,
                    seed: int, device="cpu"):
    """One random GQA cache per recurrent loop: K, V [n_loops, B, Hkv, t_max, hd]
    (model dtype), N(0,1) in positions [0, filled), zero beyond."""
    g = _gen(seed + 31, device)
    shape = (n_loops, batch, cfg.n_kv_heads, t_max, cfg.head_dim)
    k = torch.zeros(shape, dtype=cfg.torch_dtype, device=device)
    v = torch.zeros(shape, dtype=cfg.torch_dtype, device=device)
    for t in range(n_loops):
        k[t, :, :, :filled] = torch.randn(batch, cfg.n_kv_heads, filled, cfg.head_dim,
                                          generator=g, device=device).to(cfg.torch_dtype)
        v[t, :, :, :filled] = torch.randn(batch, cfg.n_kv_heads, filled, cfg.head_dim,
                                          generator=g, device=device).to(cfg.torch_dtype)
    return k, v


def random_latent_cache(cfg: RDTConfig, n_loops: int, batch: int, t_max: int, filled: int,
                        seed: int, device="cpu"):
    """One random MLA latent cache per recurrent loop: c_kv [n_loops, B, t_max, kv_lora_rank]
    and k_rope [n_loops, B, t_max, qk_rope_head_dim] (model dtype), N(0,1) in positions
    [0, filled), zero beyond."""
    g = _gen(seed + 37, device)
    ckv = torch.zeros(n_loops, batch, t_max, cfg.kv_lora_rank, dtype=cfg.torch_dtype, device=device)
    kr = torch.zeros(n_loops, batch, t_max, cfg.qk_rope_head_dim, dtype=cfg.torch_dtype, device=device)
    for t in range(n_loops):
        ckv[t, :, :filled] = torch.randn(batch, filled, cfg.kv_lora_rank, generator=g,
                                         device=device).to(cfg.torch_dtype)
        kr[t, :, :filled] = torch.randn(batch, filled, cfg.qk_rope_head_dim, generator=g,
                                        device=device).to(cfg.torch_dtype)
    return ckv, kr


def halting_offsets_spread(n: int, lo: int, hi: int, threshold: float, seed: int):
    """Per-position halting-logit offsets that make position i halt after exactly
    k_i loops, k_i ~ U{lo..hi}: with a zero halting weight and bias, the halting
    probability is constant p_i = threshold / (k_i - 0.5), i.e. logit(p_i).
    Returns (offsets fp32 [n], k int64 [n])."""
    g = _gen(seed + 97, "cpu")
    k = torch.randint(lo, hi + 1, (n,), generator=g)
    p = threshold / (k.double() - 0.5)
    off = torch.log(p / (1.0 - p)).float()
    return off, k


def zipf_router_bias(n_experts: int, dim: int, s: float, seed: int, std: float = 0.02):
    """Router bias making expert popularity roughly Zipf(s): bias_e = -s * ln(rank_e) * sigma,
    rank a seeded permutation of 1..E, sigma = std * sqrt(dim) (router-logit std for unit-RMS input)."""
    g = _gen(seed + 13, "cpu")
    rank = torch.randperm(n_experts, generator=g).double() + 1.0
    sigma = std * math.sqrt(dim)
    return (-s * torch.log(rank) * sigma).float()


def param_count_formula(cfg: RDTConfig, full_model: bool = False) -> int:
    """Parameter count of the recurrent block under the fixed readings (and, optionally,
    the full model with untied embedding and head).  ``router_bias`` is a buffer, not a
    parameter ("OpenMythos 분석", MoE section), so it is not counted."""
    D, H, E, S, F, r = cfg.dim, cfg.n_heads, cfg.n_experts, cfg.n_shared_experts, cfg.expert_dim, cfg.lora_rank
    if cfg.attn_type == "gqa":
        hd, Hkv = cfg.head_dim, cfg.n_kv_heads
        attn = D * H * hd + 2 * D * Hkv * hd + H * hd * D
    else:
        dn, dr, dv = cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim
        attn = (cfg.q_lora_rank * D + cfg.q_lora_rank + H * (dn + dr) * cfg.q_lora_rank
                + (cfg.kv_lora_rank + dr) * D + cfg.kv_lora_rank + H * (dn + dv) * cfg.kv_lora_rank
                + D * H * dv)
    rec = (3 * D + attn + E * D + 3 * D * F * (E + S) + 2 * D * r + r * cfg.max_loop_iters
           + 2 * D + 1 + D + 1)
    if not full_model:
        return rec
    Fd = cfg.dense_hidden
    dense = 2 * D + attn + 3 * D * Fd
    return rec + 2 * cfg.vocab_size * D + D + (cfg.prelude_layers + cfg.coda_layers) * dense
