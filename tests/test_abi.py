"""The C-ABI library builds for sm_100a, loads without a GPU, and exports every
entry point include/rdt.h declares; host-only calls behave (no kernel launches)."""
import ctypes
import os
import re

import pytest

import rdt_inputs as RI

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "rdt.h")).read()
    return re.findall(r"RDT_API\s+[\w\s\*]+?\b(rdt_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def lib():
    from recurrent_depth_moe_b200 import build as B
    B.build()
    from recurrent_depth_moe_b200 import _native
    return _native.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    from recurrent_depth_moe_b200 import _native
    assert set(_native.EXPORTS) <= set(names)


def test_status_strings_and_version(lib):
    assert lib.rdt_version().startswith(b"librdt")
    for code in range(7):
        assert lib.rdt_status_string(code)


def test_workspace_size_host_logic(lib):
    from recurrent_depth_moe_b200 import api
    for name in ["tiny_gqa_fp32", "tiny_mla_fp32", "rdt1b_prefill", "rdt3b_decode", "rdt10b_prefill_zipf"]:
        wl = RI.get_workload(name)
        cs = api.config_struct(wl.cfg)
        n = api.workspace_size(cs, wl.batch, wl.seq, wl.seq + wl.cache_len)
        assert n > 0 and n % 256 == 0
        # monotone in the number of sequences
        assert api.workspace_size(cs, wl.batch * 2, wl.seq, wl.seq + wl.cache_len) > n
    bad = api.config_struct(RI.get_workload("tiny_gqa_fp32").cfg)
    bad.n_kv_heads = 3                       # 8 heads not divisible by 3
    assert api.workspace_size(bad, 2, 16, 16) == 0
    bad = api.config_struct(RI.get_workload("tiny_gqa_fp32").cfg)
    bad.top_k = 9                            # more than n_experts
    assert api.workspace_size(bad, 2, 16, 16) == 0
    bad = api.config_struct(RI.get_workload("tiny_gqa_fp32").cfg)
    bad.loop_dim = 31                        # odd loop_dim
    assert api.workspace_size(bad, 2, 16, 16) == 0


def test_no_cuda_means_loud_failure():
    import torch
    if torch.cuda.is_available():
        pytest.skip("CUDA present")
    import recurrent_depth_moe_b200 as R
    wl = RI.get_workload("tiny_gqa_fp32")
    with pytest.raises(RuntimeError):
        R.RecurrentBlock(wl.cfg, RI.block_weights(wl.cfg, 0))
