"""The library's error paths, exercised without faulting the GPU context.

* A tensor-core GEMM whose TMA producer issues no loads (a test-only flag): its MMA and
  epilogue waits never see their barriers complete, give up at their bound, record
  RDT_ERR_DEVICE_TIMEOUT in the device status word and free TMEM with nothing in
  flight.  The next normal call in the same process still matches the oracle.
* A decode position out of range (cache_len = t_max): it is recorded as
  RDT_ERR_DEVICE_BOUNDS and clamped before any table or cache access, so the outputs stay
  finite and the other sequences of the batch are unaffected.
* Rows with more than 32 expert slots (top_k + shared > 32) take the CTA-per-row combine
  kernel and still match the oracle."""
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


def test_gemm_timeout_is_recorded_and_the_context_stays_usable():
    from recurrent_depth_moe_b200 import _native as N
    wl = RI.get_workload("mid_gqa_bf16")
    cfg = wl.cfg
    B, T, L = 1, 160, 2
    W = RI.block_weights(cfg, wl.seed, attn_std=0.08, halt_w_std=0.2)
    h0, e = RI.recurrent_inputs(cfg, B, T, wl.seed)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    blk.forward(h0.cuda(), e.cuda(), B, T, L, wl.act_threshold, flags=N.RDT_FLAG_TEST_GEMM_TIMEOUT)
    assert blk.read_status() == N.RDT_ERR_DEVICE_TIMEOUT
    assert blk.read_status() == N.RDT_OK                 # reading clears the word
    # the same process, the same workspace: a normal call is unaffected
    h, hw, ids = blk.forward(h0.cuda(), e.cuda(), B, T, L, wl.act_threshold)
    torch.cuda.synchronize()
    assert blk.read_status() == N.RDT_OK
    oh, _, _, _ = O.recurrent_forward(cfg, W, h0, e, B, L, wl.act_threshold)
    assert rel_l2(h, oh) <= BF16_TOL


def test_mla_attention_timeout_is_recorded_and_the_context_stays_usable():
    """The tensor-core MLA latent attention with its TMA producers idle (test flag): its
    score-MMA thread's bounded wait gives up, every other warp role sees the abort and
    leaves with nothing in flight, TMEM is freed, and the status word reads
    RDT_ERR_DEVICE_TIMEOUT; a normal decode step in the same process then matches the
    oracle ("OpenMythos 분석", MLA)."""
    from recurrent_depth_moe_b200 import _native as N
    cfg = RI.RDTConfig(dim=1536, n_heads=24, n_kv_heads=24, max_seq_len=1024, max_loop_iters=4, n_experts=8,
                       n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, attn_type="mla",
                       kv_lora_rank=512, q_lora_rank=256, qk_rope_head_dim=64, qk_nope_head_dim=128,
                       v_head_dim=128, dtype="bf16")
    W = RI.block_weights(cfg, 71, attn_std=0.05)
    B, L, t_max, n = 2, 2, 720, 700
    ckv, kr = RI.random_latent_cache(cfg, L, B, t_max, n, 72)
    h0, e = RI.decode_inputs(cfg, B, 0, 73)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    cache = R.KVCache(ckv.cuda(), kr.cuda())
    blk.forward(h0.cuda(), e.cuda(), B, 1, L, 0.0, start_pos=n, cache=cache, flags=N.RDT_FLAG_TEST_MLA_ATTN_TIMEOUT)
    torch.cuda.synchronize()
    assert blk.read_status() == N.RDT_ERR_DEVICE_TIMEOUT
    assert blk.read_status() == N.RDT_OK                 # reading clears the word
    # the same process, the same block: a normal decode step is unaffected (the flagged call
    # wrote this step's latent entries at position n; the decode step rewrites them)
    cache = R.KVCache(ckv.cuda(), kr.cuda())
    clen = torch.full((B,), n, dtype=torch.int32, device="cuda")
    d_h, _, _ = blk.decode_step(h0.cuda(), e.cuda(), clen, cache, L, 0.0)
    torch.cuda.synchronize()
    assert blk.read_status() == N.RDT_OK
    caches = [[{"c_kv": ckv[t, b, :n], "k_rope": kr[t, b, :n], "pos": torch.arange(n)} for b in range(B)]
              for t in range(L)]
    o_h, _, _, _ = O.decode_step(cfg, W, h0, e, caches, [n] * B, L, 0.0)
    for b in range(B):
        assert rel_l2(d_h[b], o_h[b]) <= BF16_TOL, b


def test_decode_position_out_of_range_is_recorded_and_clamped():
    from recurrent_depth_moe_b200 import _native as N
    cfg = RI.RDTConfig(dim=512, n_heads=4, n_kv_heads=2, max_seq_len=96, max_loop_iters=2, n_experts=8,
                       n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, dtype="bf16")
    W = to_dev(RI.block_weights(cfg, 61))
    B, L, t_max = 4, 2, 96
    k0, v0 = RI.random_kv_cache(cfg, L, B, t_max, 80, 62, device="cuda")
    h0, e = RI.decode_inputs(cfg, B, 0, 63, device="cuda")
    blk = R.RecurrentBlock(cfg, W)
    good = torch.tensor([10, 80, 33, 50], dtype=torch.int32, device="cuda")
    bad = good.clone()
    bad[1] = t_max                                       # one past the cache
    ref = blk.decode_step(h0, e, good, R.KVCache(k0.clone(), v0.clone()), L)
    torch.cuda.synchronize()
    assert blk.read_status() == N.RDT_OK
    out = blk.decode_step(h0, e, bad, R.KVCache(k0.clone(), v0.clone()), L)
    torch.cuda.synchronize()
    assert blk.read_status() == N.RDT_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out[0]).all()
    others = torch.tensor([0, 2, 3])
    assert max_rel(out[0][others], ref[0][others]) <= 1e-5
    bad[1] = -1                                          # before the cache
    out = blk.decode_step(h0, e, bad, R.KVCache(k0.clone(), v0.clone()), L)
    torch.cuda.synchronize()
    assert blk.read_status() == N.RDT_ERR_DEVICE_BOUNDS
    assert torch.isfinite(out[0]).all()


def test_more_than_32_expert_slots_per_row_match_oracle():
    """top_k 30 + 4 shared experts = 34 slots per row (fp32, ids exact)."""
    cfg = RI.RDTConfig(dim=256, n_heads=4, n_kv_heads=2, max_seq_len=32, max_loop_iters=2, n_experts=40,
                       n_shared_experts=4, n_experts_per_tok=30, expert_dim=32, lora_rank=4, dtype="fp32")
    W = RI.block_weights(cfg, 71, attn_std=0.08, halt_w_std=0.2, lora_scale_std=1.0)
    B, T, L, thr = 2, 24, 2, 0.99
    h0, e = RI.recurrent_inputs(cfg, B, T, 71)
    blk = R.RecurrentBlock(cfg, to_dev(W))
    h, hw, ids = blk.forward(h0.cuda(), e.cuda(), B, T, L, thr)
    torch.cuda.synchronize()
    assert blk.read_status() == 0
    oh, ohw, oids, _ = O.recurrent_forward(cfg, W, h0, e, B, L, thr)
    assert max_rel(h, oh) <= FP32_TOL
    assert max_rel(hw, ohw) <= FP32_TOL
    assert torch.equal(ids.cpu().long(), oids)
