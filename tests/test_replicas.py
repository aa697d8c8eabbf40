"""Replica plumbing on 2 gloo ranks (CPU): sequence shards partition the batch, the
job time is the max over ranks, the work the sum, and replicas share weights but draw
different sequences."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import rdt_inputs as RI
from recurrent_depth_moe_b200 import replicas as REP


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world_size, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world_size)
    try:
        r, ws = REP.world()
        shard = REP.shard_sequences(7, r, ws)
        t = REP.max_over_ranks(10.0 + r)             # rank 1 is slower
        work = REP.sum_over_ranks(100.0 * (r + 1))
        cfg = RI.get_workload("tiny_gqa_fp32").cfg
        W = RI.block_weights(cfg, 0)
        h0, e = RI.recurrent_inputs(cfg, 1, 4, REP.replica_input_seed(0, r))
        g = [torch.zeros(2, dtype=torch.float64) for _ in range(ws)]
        dist.all_gather(g, torch.tensor([float(W["w_qkv"].double().sum()), float(h0.double().sum())], dtype=torch.float64))
        out[r] = (r, ws, list(shard), t, work, [x.tolist() for x in g])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replica_plumbing():
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    r0, r1 = out[0], out[1]
    assert r0[1] == r1[1] == 2
    assert r0[2] + r1[2] == list(range(7)) and len(r0[2]) == 4 and len(r1[2]) == 3
    assert r0[3] == r1[3] == 11.0                    # max of 10 and 11
    assert r0[4] == r1[4] == 300.0                   # 100 + 200
    g = r0[5]
    assert g[0][0] == g[1][0]                        # identical weights on every replica
    assert g[0][1] != g[1][1]                        # different sequences per replica


def test_single_process_defaults():
    assert REP.world() == (0, 1)
    assert REP.max_over_ranks(3.5) == 3.5 and REP.sum_over_ranks(2.0) == 2.0
    assert list(REP.shard_sequences(5, 0, 1)) == list(range(5))
