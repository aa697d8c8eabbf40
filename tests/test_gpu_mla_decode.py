"""MLA with a latent cache on the GPU: prefill fills one (c_kv, k_rope) cache per loop; a
single-row call (decode step, or one token at start_pos > 0) reads it in the
weight-absorbed form (bf16) or by rebuilding the per-head keys and values (fp32), and a
later prefill chunk rebuilds them ("OpenMythos 분석", MLA; "RoPE & generation cache").
Compared with the oracle's decode step (which takes the same latent cache), with its
prefill of the whole sequence, and with the GPU's own prefill."""
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


def _tiny(dtype):
    return RI.get_workload("tiny_mla_fp32").cfg.replace(dtype=dtype)


def _mid(dtype):
    # wider latent (128) and head dims (nope 64, rope 32, v 64): GEMMs large enough for the tensor-core path
    return RI.RDTConfig(dim=512, n_heads=4, n_kv_heads=4, max_seq_len=256, max_loop_iters=4, n_experts=8,
                        n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, attn_type="mla",
                        kv_lora_rank=128, q_lora_rank=192, qk_rope_head_dim=32, qk_nope_head_dim=64,
                        v_head_dim=64, dtype=dtype)


def _latent_cache(cfg, L, B, t_max):
    z = lambda w: torch.zeros(L, B, t_max, w, dtype=cfg.torch_dtype, device="cuda")
    return R.KVCache(z(cfg.kv_lora_rank), z(cfg.qk_rope_head_dim))


def _close(got, want, dtype):
    if dtype == "fp32":
        assert max_rel(got, want) <= FP32_TOL
    else:
        assert rel_l2(got, want) <= BF16_TOL


@pytest.mark.parametrize("make", [_tiny, _mid])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_mla_prefill_then_decode_matches_oracle_and_prefill(make, dtype):
    cfg = make(dtype)
    W = RI.block_weights(cfg, 51, attn_std=0.08, halt_w_std=0.2)
    B, T, L, thr, t_max = 3, 37, 3, 0.99, 64
    h0, e = RI.recurrent_inputs(cfg, B, T + 1, 52)
    keep = torch.tensor([b * (T + 1) + i for b in range(B) for i in range(T)])
    last = torch.tensor([b * (T + 1) + T for b in range(B)])
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = _latent_cache(cfg, L, B, t_max)
    blk.forward(h0[keep].cuda(), e[keep].cuda(), B, T, L, thr, cache=cache)
    clen = torch.full((B,), T, dtype=torch.int32, device="cuda")
    d_h, d_hw, d_ids = blk.decode_step(h0[last].cuda(), e[last].cuda(), clen, cache, L, thr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    full = O.recurrent_forward(cfg, W, h0, e, B, L, thr)
    _close(d_h, full[0][last], dtype)
    assert max_rel(d_hw, full[1][:, last]) <= (FP32_TOL if dtype == "fp32" else 2e-2)
    if dtype == "fp32":
        assert torch.equal(d_ids.cpu().long(), full[2][:, last])
    # the cache now holds the latent entries of all T + 1 positions of every loop
    for t in range(L):
        for b in range(B):
            c_kv, k_rope = full[3][t][b]
            _close(cache.k[t, b, :T + 1], c_kv, dtype)
            _close(cache.v[t, b, :T + 1], k_rope, dtype)
    assert not cache.k[:, :, T + 1:].any()              # nothing written past the new token
    p_h, p_hw, p_ids = blk.forward(h0.cuda(), e.cuda(), B, T + 1, L, thr)
    assert rel_l2(d_h, p_h[last.cuda()]) <= (1e-5 if dtype == "fp32" else 1e-2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_mla_decode_random_latent_cache_ragged_lengths(dtype):
    """Decode against random per-loop latent caches with a different length per sequence."""
    cfg = _mid(dtype)
    W = RI.block_weights(cfg, 53, attn_std=0.05)
    B, L, t_max = 4, 3, 160
    lens = [37, 100, 64, 5]
    ckv, kr = RI.random_latent_cache(cfg, L, B, t_max, max(lens), 54)
    for b, n in enumerate(lens):                       # positions >= len are not part of the cache
        ckv[:, b, n:] = 0
        kr[:, b, n:] = 0
    h0, e = RI.decode_inputs(cfg, B, 0, 55)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = R.KVCache(ckv.cuda(), kr.cuda())
    clen = torch.tensor(lens, dtype=torch.int32, device="cuda")
    d_h, d_hw, d_ids = blk.decode_step(h0.cuda(), e.cuda(), clen, cache, L, 0.0)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    caches = [[{"c_kv": ckv[t, b, :lens[b]], "k_rope": kr[t, b, :lens[b]], "pos": torch.arange(lens[b])}
               for b in range(B)] for t in range(L)]
    o_h, o_hw, o_ids, new_kv = O.decode_step(cfg, W, h0, e, caches, lens, L, 0.0)
    _close(d_h, o_h, dtype)
    if dtype == "fp32":
        assert torch.equal(d_ids.cpu().long(), o_ids)
    for t in range(L):
        for b in range(B):
            _close(cache.k[t, b, lens[b]], new_kv[t][b][0][0], dtype)
            _close(cache.v[t, b, lens[b]], new_kv[t][b][1][0], dtype)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_mla_chunked_prefill_reads_the_latent_cache(dtype):
    """A second prefill chunk at start_pos = T1 attends to the first chunk through the
    latent cache: its rows equal the oracle's prefill of the whole T1 + T2 tokens."""
    cfg = _mid(dtype)
    W = RI.block_weights(cfg, 56, attn_std=0.08, halt_w_std=0.2)
    B, T1, T2, L, thr, t_max = 2, 40, 24, 3, 0.99, 80
    h0, e = RI.recurrent_inputs(cfg, B, T1 + T2, 57)
    first = torch.tensor([b * (T1 + T2) + i for b in range(B) for i in range(T1)])
    second = torch.tensor([b * (T1 + T2) + T1 + i for b in range(B) for i in range(T2)])
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = _latent_cache(cfg, L, B, t_max)
    blk.forward(h0[first].cuda(), e[first].cuda(), B, T1, L, thr, cache=cache)
    c_h, c_hw, c_ids = blk.forward(h0[second].cuda(), e[second].cuda(), B, T2, L, thr, start_pos=T1, cache=cache)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    full = O.recurrent_forward(cfg, W, h0, e, B, L, thr)
    _close(c_h, full[0][second], dtype)
    if dtype == "fp32":
        assert torch.equal(c_ids.cpu().long(), full[2][:, second])


def _wide(H):
    # DeepSeek-V2 latent widths (kv_lora_rank 512, rope 64); the heads are the 8-wide MMA
    # columns: H 4, 12 and 20 leave padded columns inside a tile, H 32 fills four
    return RI.RDTConfig(dim=1536, n_heads=H, n_kv_heads=H, max_seq_len=1024, max_loop_iters=4, n_experts=8,
                        n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, attn_type="mla",
                        kv_lora_rank=512, q_lora_rank=256, qk_rope_head_dim=64, qk_nope_head_dim=128,
                        v_head_dim=128, dtype="bf16")


@pytest.mark.parametrize("H", [4, 8, 12, 16, 20, 24, 32])
def test_mla_absorbed_decode_wide_latent_ragged(H):
    """Absorbed decode at kv_lora_rank 512 against the oracle's decode step, with ragged
    cache lengths: several key ranges, a tile-aligned length + 1, an empty cache (the new
    token alone) and a single cached token."""
    _wide_case(H, 720, [300, 700, 64, 0, 1])


@pytest.mark.parametrize("t_max,lens", [(100, [99, 40, 0]), (128, [127, 5, 64])])
def test_mla_absorbed_decode_wide_latent_short_caches(t_max, lens):
    """Caches shorter than one 128-key tile (the mma.sync kernel at kv_lora_rank 512) and
    exactly one tile (the tensor-core kernel: a full tile, and short sequences whose tile
    starts before key 0 and reads zeros there)."""
    _wide_case(24, t_max, lens)


def test_mla_absorbed_decode_rescales_as_rope_scores_grow():
    """The tensor-core latent attention with a running maximum that keeps rising: k_rope is
    scaled by 1 + j / 32 at position j (the latent part is scale-free: its RMSNorm factor r_j
    cancels any scaling of c_j), so the rope scores grow along the cache and pass the previous
    maximum by more than the lazy-rescale threshold (2^8) tile after tile; the rescales of the
    running sums and of U^T in TMEM must hold."""
    _wide_case(24, 720, [700, 300, 129, 1], rope_growth=True)


def _wide_case(H, t_max, lens, rope_growth=False):
    cfg = _wide(H)
    W = RI.block_weights(cfg, 60 + H, attn_std=0.05)
    B, L = len(lens), 2
    ckv, kr = RI.random_latent_cache(cfg, L, B, t_max, max(lens), 61)
    if rope_growth:
        kr = kr * (1.0 + torch.arange(t_max, dtype=torch.float64) / 32).to(kr.dtype)[None, None, :, None]
    for b, n in enumerate(lens):
        ckv[:, b, n:] = 0
        kr[:, b, n:] = 0
    h0, e = RI.decode_inputs(cfg, B, 0, 62)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = R.KVCache(ckv.cuda(), kr.cuda())
    clen = torch.tensor(lens, dtype=torch.int32, device="cuda")
    d_h, d_hw, d_ids = blk.decode_step(h0.cuda(), e.cuda(), clen, cache, L, 0.0)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    caches = [[{"c_kv": ckv[t, b, :lens[b]], "k_rope": kr[t, b, :lens[b]], "pos": torch.arange(lens[b])}
               for b in range(B)] for t in range(L)]
    o_h, o_hw, o_ids, new_kv = O.decode_step(cfg, W, h0, e, caches, lens, L, 0.0)
    for b in range(B):                                  # every sequence on its own, not just on average
        assert rel_l2(d_h[b], o_h[b]) <= BF16_TOL, b
    for t in range(L):                                  # the new token's latent entry, every loop
        for b in range(B):
            assert rel_l2(cache.k[t, b, lens[b]], new_kv[t][b][0][0]) <= BF16_TOL


def test_mla_single_token_prefill_through_the_cache():
    """rdt_recurrent_forward with one token at start_pos > 0 reads the latent cache the
    same way as the decode step."""
    cfg = _mid("bf16")
    W = RI.block_weights(cfg, 63, attn_std=0.08, halt_w_std=0.2)
    B, T, L, thr, t_max = 2, 20, 3, 0.99, 32
    h0, e = RI.recurrent_inputs(cfg, B, T + 1, 64)
    keep = torch.tensor([b * (T + 1) + i for b in range(B) for i in range(T)])
    last = torch.tensor([b * (T + 1) + T for b in range(B)])
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = _latent_cache(cfg, L, B, t_max)
    blk.forward(h0[keep].cuda(), e[keep].cuda(), B, T, L, thr, cache=cache)
    s_h, s_hw, s_ids = blk.forward(h0[last].cuda(), e[last].cuda(), B, 1, L, thr, start_pos=T, cache=cache)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    full = O.recurrent_forward(cfg, W, h0, e, B, L, thr)
    assert rel_l2(s_h, full[0][last]) <= BF16_TOL
