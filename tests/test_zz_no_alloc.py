"""rdt_recurrent_decode_step_static: the decode step for callers that cannot allocate
device memory (its scratch is a static array inside the library).  Called through the
C ABI and compared, on two calls in a row, with rdt_recurrent_decode_step given a
caller workspace.  Kept in its own file so that pytest collects it last."""
import ctypes

import pytest
import torch

import rdt_inputs as RI
from tests._helpers import BF16_TOL, FP32_TOL, max_rel, rel_l2, to_dev

pytestmark = pytest.mark.gpu

R = pytest.importorskip("recurrent_depth_moe_b200")


def _lib():
    from recurrent_depth_moe_b200 import _native as N
    lib = N.load()
    P = ctypes.c_void_p
    fn = lib.rdt_recurrent_decode_step_static
    fn.argtypes = [ctypes.POINTER(N.rdt_config), ctypes.POINTER(N.rdt_weights), P, P, ctypes.c_int, P, ctypes.c_int,
                   ctypes.c_float, P, P, P, ctypes.POINTER(N.rdt_kv_cache), P]
    fn.restype = ctypes.c_int
    lib.rdt_read_static_status.argtypes = [P]
    lib.rdt_read_static_status.restype = ctypes.c_int
    return lib, N


def _cfg(dtype):
    return RI.RDTConfig(dim=768, n_heads=6, n_kv_heads=2, max_seq_len=160, max_loop_iters=3, n_experts=8,
                        n_shared_experts=1, n_experts_per_tok=2, expert_dim=128, lora_rank=8, dtype=dtype)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_static_scratch_decode_matches_workspace_decode(dtype):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib, N = _lib()
    cfg = _cfg(dtype)
    W = to_dev(RI.block_weights(cfg, 41, attn_std=0.05, halt_w_std=0.2))
    B, L, t_max, thr = 4, 3, 160, 0.99
    lens = torch.tensor([37, 100, 64, 5], dtype=torch.int32, device="cuda")
    k0, v0 = RI.random_kv_cache(cfg, L, B, t_max, 100, 42, device="cuda")
    blk = R.RecurrentBlock(cfg, W)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):                              # two calls in a row, fresh inputs each time
        h0, e = RI.decode_inputs(cfg, B, call, 43, device="cuda")
        ref_cache = R.KVCache(k0.clone(), v0.clone())
        ref = blk.decode_step(h0, e, lens, ref_cache, L, thr)
        st_cache = R.KVCache(k0.clone(), v0.clone())
        cs = st_cache.struct()
        out = (torch.empty(B, cfg.dim, dtype=torch.float32, device="cuda"),
               torch.empty(L, B, dtype=torch.float32, device="cuda"),
               torch.empty(L, B, cfg.n_experts_per_tok, dtype=torch.int32, device="cuda"))
        rc = lib.rdt_recurrent_decode_step_static(ctypes.byref(blk.cs), ctypes.byref(blk.w.struct), h0.data_ptr(),
                                                  e.data_ptr(), B, lens.data_ptr(), L, thr, out[0].data_ptr(),
                                                  out[1].data_ptr(), out[2].data_ptr(), ctypes.byref(cs), stream)
        assert rc == 0, N.STATUS.get(rc, rc)
        # the device status word of the static scratch: no bounds violation, no timeout
        assert lib.rdt_read_static_status(stream) == 0
        assert blk.read_status() == 0
        torch.cuda.synchronize()
        if dtype == "fp32":
            assert max_rel(out[0], ref[0]) <= FP32_TOL
            assert max_rel(st_cache.k, ref_cache.k) <= FP32_TOL
            assert max_rel(st_cache.v, ref_cache.v) <= FP32_TOL
        else:
            assert rel_l2(out[0], ref[0]) <= BF16_TOL
            assert rel_l2(st_cache.k.float(), ref_cache.k.float()) <= BF16_TOL
            assert rel_l2(st_cache.v.float(), ref_cache.v.float()) <= BF16_TOL
        assert max_rel(out[1], ref[1]) <= FP32_TOL
        assert torch.equal(out[2], ref[2])


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib, N = _lib()
    cfg = _cfg("bf16")
    W = to_dev(RI.block_weights(cfg, 44))
    blk = R.RecurrentBlock(cfg, W)
    B, L, t_max = 4096, 1, 256                        # workspace well beyond 32 MiB
    assert R.workspace_size(blk.cs, B, 1, t_max) > (32 << 20)
    k = torch.zeros(L, 1, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    cs = N.rdt_kv_cache()
    cs.k, cs.v, cs.n_loops, cs.batch, cs.t_max = k.data_ptr(), k.data_ptr(), L, B, t_max
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    rc = lib.rdt_recurrent_decode_step_static(ctypes.byref(blk.cs), ctypes.byref(blk.w.struct), dummy.data_ptr(),
                                              dummy.data_ptr(), B, dummy.data_ptr(), L, 0.0, dummy.data_ptr(),
                                              dummy.data_ptr(), dummy.data_ptr(), ctypes.byref(cs),
                                              torch.cuda.current_stream().cuda_stream)
    assert rc == N.RDT_ERR_WORKSPACE
