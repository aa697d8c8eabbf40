"""Benchmark of the looped Recurrent Block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full recurrent-block forward (all loops, every kernel of the path) over
one batch of the 10B-shaped load-imbalanced prefill workload (dim 4096, 32 heads GQA with
8 kv heads, 128 routed + 1 shared SwiGLU experts, top-8, expert_dim 5632, lora_rank 16,
24 loops, batch 2 x seq 8192, bf16, router bias giving Zipf(1.1) expert popularity,
per-position halting spread over 4-24 loops).  The value counts executed token-loops.
The same line carries the 1B-shaped prefill (and its literal halting-bias variant), the
3B-shaped KV-cached decode (GQA and MLA) and the 1B-shaped greedy generation.  Weights
and inputs are seeded synthetic draws.

Multi-GPU (torchrun, one process per GPU): each rank runs an independent replica on
its own batch (sequences shard with no exchange); the time is the max over ranks.

Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle instead (on
bounded samples of the same workload, host cores only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import rdt_inputs as RI  # noqa: E402
from recurrent_depth_moe_b200 import replicas as REP  # noqa: E402

METRIC = "recurrent-block token·loops/s prefill; decode tokens/s; % roofline, 1×B200"
UNIT = "token·loops/s"
WORKLOAD = "rdt10b_prefill_zipf"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def workload_desc(wl):
    c = wl.cfg
    shape = {"rdt1b_prefill": "1B-shaped recurrent block prefill",
             "rdt10b_prefill_zipf": "10B-shaped load-imbalanced recurrent block prefill",
             "rdt3b_mla_prefill": "3B-shaped MLA recurrent block prefill"}.get(wl.name, wl.name)
    attn = (f"{c.n_heads} heads GQA ({c.n_kv_heads} kv)" if c.attn_type == "gqa" else
            f"{c.n_heads} heads MLA (kv_lora_rank {c.kv_lora_rank}, q_lora_rank {c.q_lora_rank}, nope "
            f"{c.qk_nope_head_dim}, rope {c.qk_rope_head_dim}, v {c.v_head_dim})")
    extra = ""
    if wl.zipf_s:
        extra += f", Zipf(s={wl.zipf_s}) router bias"
    if wl.halt_spread:
        extra += f", halting spread over {wl.halt_spread[0]}-{wl.halt_spread[1]} loops"
    return (f"{wl.name}: {shape}, dim {c.dim}, {attn}, "
            f"{c.n_experts} routed + {c.n_shared_experts} shared SwiGLU experts top-{c.n_experts_per_tok}, "
            f"expert_dim {c.expert_dim}, lora_rank {c.lora_rank}, {wl.n_loops} loops, batch {wl.batch} x seq {wl.seq}, "
            f"{c.dtype}, ACT {wl.act_threshold} (halting bias {wl.halt_b}){extra}")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.idx), "-lms", "200"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "power_w_max": max(power) if power else None}


# DRAM traffic of one full-size expert-up launch of a workload, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum, 1 pass), valid only while the GEMM's
# sources are the ones it was captured from (sha256 of k_gemm_tc.cu + tc_common.cuh).
EXPERT_UP_TRAFFIC = {
    # mean over the 16 expert-up launches of one step (ncu --metrics dram__bytes_read.sum,
    # dram__bytes_write.sum on the default prefill command of each workload)
    "rdt1b_prefill": {"batch": 4, "n_loops": 16, "bytes": 1738791616,
                      "sha256": "20988b66acaa3c9ae7884b4054f06d19dff31b3b5c797b65bf83a17772fb436f"},
    # mean over the 24 expert-up launches of one step
    "rdt10b_prefill_zipf": {"batch": 2, "n_loops": 24, "bytes": 13418124843,
                            "sha256": "20988b66acaa3c9ae7884b4054f06d19dff31b3b5c797b65bf83a17772fb436f"},
}


def expert_up_traffic(wl):
    import hashlib
    rec = EXPERT_UP_TRAFFIC.get(wl.name)
    if rec is None or wl.batch != rec["batch"] or wl.n_loops != rec["n_loops"]:
        return None
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "recurrent_depth_moe_b200", "csrc")
    h = hashlib.sha256()
    for f in ("k_gemm_tc.cu", "tc_common.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return rec["bytes"] if h.hexdigest() == rec["sha256"] else None


def attention_flops_executed(cfg, last: torch.Tensor, T: int) -> float:
    """Causal prefill attention of the rows that run, summed over the loops: a row at position
    p running loop t attends to p + 1 keys, (score dim + value dim) * 2 FLOPs per head and key
    (a halted row's query is not computed).  last[i] = the last loop row i ran."""
    if cfg.attn_type == "gqa":
        dqk = dv = cfg.head_dim
    else:
        dqk, dv = cfg.qk_nope_head_dim + cfg.qk_rope_head_dim, cfg.v_head_dim
    pos = torch.arange(last.numel(), device=last.device) % T
    return float(2.0 * cfg.n_heads * (dqk + dv) * ((last + 1).double() * (pos + 1).double()).sum().item())


def expert_up_flops(wl, n_running: float) -> float:
    c = wl.cfg
    rows = n_running * (c.n_experts_per_tok + c.n_shared_experts)
    return 2.0 * rows * c.dim * 2 * c.expert_dim


# ------------------------------------------------------------------------------------------
# CPU oracle sample (reference arm and cpu_baseline)
# ------------------------------------------------------------------------------------------

ORACLE_SAMPLE = {"rdt1b_prefill": (32, 4), "rdt10b_prefill_zipf": (8, 2)}   # positions, loops per reference step
# the cpu_baseline leg of the default line: one sample of about 10-15 s of host work
CPU_BASELINE_SAMPLE = {"rdt1b_prefill": (128, 16), "rdt10b_prefill_zipf": (24, 8)}


def oracle_sample(wl, W_cpu, h0, e, positions: int, loops: int, halt_off=None):
    """Time the CPU oracle on sequence 0, positions [0, positions), `loops` loops.
    Causal prefix slices are exact (attention is causal, routing per token)."""
    from oracle import rdt_oracle as O
    t0 = time.perf_counter()
    O.recurrent_forward(wl.cfg, W_cpu, h0[:positions], e[:positions], 1, loops, wl.act_threshold,
                        halt_logit_offset=None if halt_off is None else halt_off[:positions])
    dt = time.perf_counter() - t0
    return positions * loops / dt, dt


def workload_weights(wl, device, halt_b=None):
    """Weights of a prefill workload (Zipf router bias and halting spread where the
    workload names them) and its per-position halting-logit offsets (or None)."""
    cfg = wl.cfg
    if wl.zipf_s or wl.halt_spread:
        bias = RI.zipf_router_bias(cfg.n_experts, cfg.dim, wl.zipf_s, wl.seed) if wl.zipf_s else None
        W = RI.block_weights(cfg, wl.seed, device=device, router_bias=bias,
                             halt_w_std=0.0 if wl.halt_spread else None, halt_b=0.0 if wl.halt_spread else wl.halt_b)
    else:
        W = RI.block_weights(cfg, wl.seed, device=device, halt_b=wl.halt_b if halt_b is None else halt_b)
    off = None
    if wl.halt_spread:
        off, _ = RI.halting_offsets_spread(wl.batch * wl.seq, wl.halt_spread[0], wl.halt_spread[1],
                                           wl.act_threshold, wl.seed)
        off = off.to(device)
    return W, off


def run_reference(args, wl, rank, world):
    """The oracle as it stands, on the host cores, on a bounded causal-prefix sample of the
    workload per step.  Large workloads draw their weights with the device generator (as
    the GPU arm does, so both see the same numbers) and copy them to the host once."""
    if rank != 0:
        return
    torch.manual_seed(0)
    dev = "cuda" if (wl.device_weights and torch.cuda.is_available()) else "cpu"
    W, off = workload_weights(wl, dev)
    W = {k: v.cpu() for k, v in W.items()}
    off = None if off is None else off.cpu()
    if dev == "cuda":
        torch.cuda.empty_cache()
    pos, loops = ORACLE_SAMPLE.get(wl.name, (32, 4))
    h0, e = RI.recurrent_inputs(wl.cfg, 1, pos, wl.seed)
    for _ in range(args.warmup):
        oracle_sample(wl, W, h0, e, pos, 1, off)
    total = 0.0
    for _ in range(args.steps):
        _, dt = oracle_sample(wl, W, h0, e, pos, loops, off)
        total += dt
    value = args.steps * pos * loops / total
    cores = torch.get_num_threads()
    sample = f"sequence 0, positions 0-{pos - 1}, loops 0-{loops - 1} of {wl.name} (fp64 oracle, per step)"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": workload_desc(wl), "batch": wl.batch, "seq_len": wl.seq, "n_loops": wl.n_loops},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------

def run_prefill(args, wl, rank, world, local_rank, *, steps=None, e2e=True, cpu_baseline=False, halt_b=None):
    """Time `steps` recurrent-block forwards of a prefill workload (inputs resident in HBM),
    with the per-class event profile inside the timed region; optionally the same through
    the public API with host buffers (e2e) and the CPU oracle on a bounded sample."""
    import recurrent_depth_moe_b200 as R
    from recurrent_depth_moe_b200 import _native as NAT
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = wl.cfg
    B, T, L = wl.batch, wl.seq, wl.n_loops
    N = B * T
    steps = steps or args.steps
    # weights: identical replica on every rank; inputs: a different batch per rank
    W, halt_off = workload_weights(wl, dev, halt_b)
    h0, e = RI.recurrent_inputs(cfg, B, T, REP.replica_input_seed(wl.seed, rank), device=dev)
    blk = R.RecurrentBlock(cfg, W)
    ws = blk.workspace(B, T, T)
    out = (torch.empty(N, cfg.dim, dtype=torch.float32, device=dev),
           torch.empty(L, N, dtype=torch.float32, device=dev),
           torch.empty(L, N, cfg.n_experts_per_tok, dtype=torch.int32, device=dev))
    stream = torch.cuda.current_stream()

    def step():
        blk.forward(h0, e, B, T, L, wl.act_threshold, halt_logit_offset=halt_off, out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert blk.read_status() == 0, "device status word set during warm-up"

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[local_rank]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local_rank
    clocks = ClockSampler(gpu_index)
    clocks.start()
    time.sleep(0.3)
    NAT.profile_start()
    n0 = NAT.launch_count()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    launches = NAT.launch_count() - n0
    prof = NAT.profile_stop()
    clk = clocks.stop()
    assert blk.read_status() == 0, "device status word set during the timed steps"
    ms = ev0.elapsed_time(ev1) / steps
    ms_max = REP.max_over_ranks(ms, device=dev)

    # executed token-loops of one step (positions that halt early run fewer loops)
    hw = out[1]
    last = ((hw > 0).to(torch.int64) * torch.arange(L, device=dev)[:, None]).max(dim=0).values
    executed = float((last + 1).sum().item())
    executed_all = REP.sum_over_ranks(executed, device=dev)
    value = executed_all / (ms_max / 1e3)
    ids = out[2][0].cpu()
    load = torch.bincount(ids[ids >= 0].flatten().long(), minlength=cfg.n_experts).double()

    res = {"value": value, "ms_per_step": ms_max, "steps": steps, "executed_token_loops_per_step": executed_all,
           "mean_loops": executed / N, "gpu_launches": launches, "clocks": clk,
           "expert_load_max_over_mean_loop0": float(load.max() / load.mean()),
           "kernel_ms_per_step": {k: {"launches": v[0], "ms_per_step": v[1] / steps} for k, v in sorted(prof.items())}}
    if e2e:
        # end to end through the public API: every step copies its inputs from pinned host
        # memory and its results back to pinned host memory, inside the timed region.  The
        # copies run on their own streams with two device buffers, so step n + 1's inputs
        # and step n's results cross the host link while step n + 1 / n computes.
        h0_h = h0.cpu().pin_memory()
        e_h = e.cpu().pin_memory()
        h0_d = [torch.empty_like(h0) for _ in range(2)]
        e_d = [torch.empty_like(e) for _ in range(2)]
        outs = [out, tuple(torch.empty_like(o) for o in out)]
        outs_h = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in out]
        h2d = h0_h.numel() * h0_h.element_size() + e_h.numel() * e_h.element_size()
        d2h = sum(o.numel() * o.element_size() for o in out)
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event()
        in_ready, c_done, d_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]        # a buffer's previous step (its compute and read-back) is enqueued

        def h2d_into(k):
            with torch.cuda.stream(s_in):
                if used[k]:
                    s_in.wait_event(c_done[k])        # the compute that read buffer k is done
                h0_d[k].copy_(h0_h, non_blocking=True)
                e_d[k].copy_(e_h, non_blocking=True)
                in_ready[k].record(s_in)

        def run_e2e(n_steps):
            h2d_into(0)
            for n in range(n_steps):
                k = n % 2
                stream.wait_event(in_ready[k])
                if used[k]:
                    stream.wait_event(d_done[k])      # step n - 2's results are read back
                blk.forward(h0_d[k], e_d[k], B, T, L, wl.act_threshold, halt_logit_offset=halt_off,
                            out=outs[k], workspace=ws)
                c_done[k].record(stream)
                used[k] = True
                if n + 1 < n_steps:
                    h2d_into(1 - k)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(c_done[k])
                    for oh, od in zip(outs_h, outs[k]):
                        oh.copy_(od, non_blocking=True)
                    d_done[k].record(s_out)
            stream.wait_event(d_done[(n_steps - 1) % 2])

        run_e2e(1)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_stream(stream)
        run_e2e(steps)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = REP.max_over_ranks(e0.elapsed_time(e1) / steps, device=dev)
        res["e2e"] = {"value": executed_all / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h,
                      "overlap": "copy streams: step n+1's inputs and step n's results cross the host link "
                                 "while the neighbouring step computes (two device buffers)"}
        del h0_d, e_d, outs, outs_h

    pk, pk_kind = peaks()
    up = prof.get("expert_up_swiglu", (0, 0.0))
    achieved = None
    mean_running = executed / L        # rows routed per launch, averaged over the loops
    if up[0]:
        achieved = expert_up_flops(wl, mean_running) / (up[1] / up[0] / 1e3) / 1e12
    peak_t = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    att = prof.get("attention", (0, 0.0))
    if att[0]:
        att_flops = attention_flops_executed(cfg, last, T) / L   # per launch, the loops' average
        att_tf = att_flops / (att[1] / att[0] / 1e3) / 1e12
        res["attention_roofline"] = {
            "bound": "tensor", "achieved": att_tf, "peak": peak_t, "unit": "TFLOP/s", "frac": att_tf / peak_t,
            "flops_per_launch": att_flops, "ms_per_launch": att[1] / att[0],
            "kernel": ("k_attn_tc (tcgen05, GQA)" if cfg.attn_type == "gqa" else
                       "k_attn_tc (tcgen05, MLA: keys [k_nope | k_rope], values read in place)")}
    res["roofline"] = {"bound": "tensor", "kernel": "expert_up_swiglu (tcgen05 grouped GEMM, SwiGLU epilogue)",
                       "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
                       "frac": (achieved / peak_t) if achieved else None,
                       "peak_kind": f"{pk_kind} bf16 sustained (kernel timed inside a long step)",
                       "traffic": expert_up_traffic(wl), "flops_per_launch": expert_up_flops(wl, mean_running)}
    # host copy for the CPU-oracle baseline, then the GPU workload is freed
    W_cpu = None
    if cpu_baseline and rank == 0 and world == 1:
        W_cpu = {k: v.cpu() for k, v in W.items()}
        pos, loops = CPU_BASELINE_SAMPLE.get(wl.name, (32, 4))
        h0_c, e_c = h0[:pos].cpu(), e[:pos].cpu()
        off_c = None if halt_off is None else halt_off[:pos].cpu()
    del blk, ws, W, out, h0, e
    torch.cuda.empty_cache()
    if W_cpu is not None:
        rate, dt = oracle_sample(wl, W_cpu, h0_c, e_c, pos, loops, off_c)
        res["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
                               "sample": f"sequence 0, positions 0-{pos - 1}, loops 0-{loops - 1} of {wl.name} "
                                         f"(fp64 oracle, {dt:.1f} s)"}
        del W_cpu
    return res


def run_ours(args, wl, rank, world, local_rank):
    """The headline line: the largest single-GPU prefill workload (the 10B-shaped
    load-imbalanced prefill) at the top level; the 1B-shaped prefill (with its literal
    halting-bias variant), the 3B-shaped decode (GQA and MLA) and the 1B-shaped generation
    alongside, with their headline figures also as flat top-level keys."""
    head = run_prefill(args, wl, rank, world, local_rank, e2e=True, cpu_baseline=not args.no_cpu_baseline)
    side = literal = None
    if not args.no_secondary and wl.name != "rdt1b_prefill":
        wl1 = RI.get_workload("rdt1b_prefill")
        side = run_prefill(args, wl1, rank, world, local_rank, e2e=False)
        # the literal reading of the 1B config: halting bias 0, so positions halt after 2-3 loops
        literal = run_prefill(args, wl1, rank, world, local_rank, steps=min(args.steps, 5), e2e=False, halt_b=0.0)
    mla_prefill = None
    if not args.no_secondary:
        mla_prefill = run_prefill(args, RI.get_workload("rdt3b_mla_prefill"), rank, world, local_rank,
                                  steps=min(args.steps, 5), e2e=False)
    decode_res = None if args.no_decode else run_decode(args, rank, world, local_rank)
    mla_res = None if args.no_decode or args.no_mla_decode else run_decode(args, rank, world, local_rank,
                                                                             "rdt3b_mla_decode")
    gen_res = None if args.no_decode or args.no_generate else run_generate(args, rank, world, local_rank)
    depth_res = None if args.no_decode or args.no_depth else run_depth_decode(args, rank, world, local_rank)
    if rank != 0:
        return
    cfg = wl.cfg
    res = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded N(0,0.02) weights, unit-RMS h0/e rows)",
           "config": {"workload": workload_desc(wl), "batch": wl.batch * world, "seq_len": wl.seq,
                      "n_loops": wl.n_loops,
                      "parallelism": f"replicas x{world} (sequence-sharded, no collective)",
                      "l2": f"inputs larger than L2 ({3 * cfg.dim * cfg.expert_dim * (cfg.n_experts + cfg.n_shared_experts) * 2 / 1e9:.2f} GB of expert weights streamed per loop)"},
           "executed_token_loops_per_step": head["executed_token_loops_per_step"],
           "mean_loops_per_position": head["mean_loops"],
           "expert_load_max_over_mean_loop0": head["expert_load_max_over_mean_loop0"],
           "roofline": head["roofline"], "expert_up_frac": head["roofline"]["frac"],
           "gpu_launches": head["gpu_launches"], "kernel_ms_per_step": head["kernel_ms_per_step"],
           "e2e": head["e2e"], "clocks": head["clocks"]}
    if "cpu_baseline" in head:
        res["cpu_baseline"] = head["cpu_baseline"]
    if side is not None:
        res["rdt1b_prefill"] = {"workload": workload_desc(RI.get_workload("rdt1b_prefill")), **side}
        res["rdt1b_prefill_token_loops_per_s"] = side["value"]
        res["rdt1b_prefill_ms_per_step"] = side["ms_per_step"]
        res["rdt1b_expert_up_frac"] = side["roofline"]["frac"]
    if literal is not None:
        res["rdt1b_prefill_literal_halt_b0"] = {
            "workload": "rdt1b_prefill with halting bias 0 (the config's literal reading: N(0, 0.02) halting "
                        "weights, positions halt after 2-3 of the 16 loops)", **literal}
        res["rdt1b_literal_token_loops_per_s"] = literal["value"]
        res["rdt1b_literal_mean_loops"] = literal["mean_loops"]
    if "attention_roofline" in head:
        res["attention_frac"] = head["attention_roofline"]["frac"]
    if side is not None and "attention_roofline" in side:
        res["rdt1b_attention_frac"] = side["attention_roofline"]["frac"]
    if mla_prefill is not None:
        res["rdt3b_mla_prefill"] = {"workload": workload_desc(RI.get_workload("rdt3b_mla_prefill")), **mla_prefill}
        res["rdt3b_mla_prefill_token_loops_per_s"] = mla_prefill["value"]
        if "attention_roofline" in mla_prefill:
            res["mla_prefill_attention_tflops"] = mla_prefill["attention_roofline"]["achieved"]
            res["mla_prefill_attention_frac"] = mla_prefill["attention_roofline"]["frac"]
    if decode_res is not None:
        res["decode"] = decode_res
        res["decode_tokens_per_s"] = decode_res["value"]
        res["decode_hbm_frac"] = decode_res["roofline"]["frac"]
        res["decode_attention_hbm_frac"] = decode_res["attention_roofline"]["frac"]
    if mla_res is not None:
        res["decode_mla"] = mla_res
        res["decode_mla_tokens_per_s"] = mla_res["value"]
        res["decode_mla_hbm_frac"] = mla_res["roofline"]["frac"]
        res["decode_mla_attention_hbm_frac"] = mla_res["attention_roofline"]["frac"]
    if depth_res is not None:
        res["depth_batch"] = depth_res
        res["depth_batch_tokens_per_s"] = depth_res["depth_batch_tokens_per_s"]
        res["depth_batch_lockstep_tokens_per_s"] = depth_res["lockstep_tokens_per_s"]
        res["depth_batch_speedup"] = depth_res["speedup"]
    if gen_res is not None:
        res["generate"] = gen_res
        res["generate_tokens_per_s"] = gen_res["value"]
        res["generate_decode_hbm_frac"] = gen_res["decode_roofline"]["frac"]
    print(json.dumps(res), flush=True)


def attn_weight_bytes(cfg) -> int:
    """bf16 bytes of one loop's attention weights."""
    D, H = cfg.dim, cfg.n_heads
    if cfg.attn_type == "gqa":
        hd, Hkv = cfg.head_dim, cfg.n_kv_heads
        return ((H + 2 * Hkv) * hd * D + D * H * hd) * 2
    dn, dr, dv, kvr, ql = (cfg.qk_nope_head_dim, cfg.qk_rope_head_dim, cfg.v_head_dim, cfg.kv_lora_rank,
                           cfg.q_lora_rank)
    return (ql * D + H * (dn + dr) * ql + (kvr + dr) * D + H * (dn + dv) * kvr + D * H * dv) * 2


def cache_bytes_per_key(cfg) -> int:
    """bf16 bytes one cached position holds per loop: K and V of every kv head (GQA), or
    the latent c_kv plus one k_rope shared by all heads (MLA)."""
    if cfg.attn_type == "gqa":
        return 2 * cfg.n_kv_heads * cfg.head_dim * 2
    return (cfg.kv_lora_rank + cfg.qk_rope_head_dim) * 2


def decode_algorithmic_bytes(cfg, ids: torch.Tensor, lens: torch.Tensor) -> float:
    """HBM bytes one decode step must move at minimum: every expert a loop touches is
    streamed once (routed experts by the realised routing, plus the shared ones), the
    attention / router / LoRA weights once per loop, each sequence's cache of that loop
    read once (cache_len + 1 positions) and one new cache row written."""
    D, F, E, S = cfg.dim, cfg.expert_dim, cfg.n_experts, cfg.n_shared_experts
    expert_bytes = 3 * D * F * 2
    attn_bytes = attn_weight_bytes(cfg)
    small = (E * D + 2 * cfg.lora_rank * D) * 2
    L = ids.shape[0]
    kv = float((lens.double() + 1).sum()) * cache_bytes_per_key(cfg)
    total = 0.0
    for t in range(L):
        distinct = int(torch.unique(ids[t][ids[t] >= 0]).numel())
        total += (distinct + S) * expert_bytes + attn_bytes + small + kv
    return total


def run_decode(args, rank, world, local_rank, name="rdt3b_decode"):
    """3B-shaped KV-cached decode: 64 sequences with 4096-token random caches per loop
    (GQA K/V, or the MLA latent cache), one new token per sequence per step over
    `decode_steps` steps."""
    import recurrent_depth_moe_b200 as R
    from recurrent_depth_moe_b200 import _native as NAT
    dev = torch.device("cuda", local_rank)
    wl = RI.get_workload(name)
    cfg = wl.cfg
    B, L, steps = wl.batch, wl.n_loops, args.decode_steps
    n_prof = min(steps, 32)                 # eager, profiled steps after the timed ones
    t_max = wl.cache_len + args.warmup + 2 + steps + n_prof
    W = RI.block_weights(cfg, wl.seed, device=dev)
    make_cache = RI.random_kv_cache if cfg.attn_type == "gqa" else RI.random_latent_cache
    k, v = make_cache(cfg, L, B, t_max, wl.cache_len, REP.replica_input_seed(wl.seed, rank), device=dev)
    h0s, es = [], []
    for st in range(steps + args.warmup):
        h, e = RI.decode_inputs(cfg, B, st, REP.replica_input_seed(wl.seed, rank), device=dev)
        h0s.append(h)
        es.append(e)
    blk = R.RecurrentBlock(cfg, W)
    cache = R.KVCache(k, v)
    ws = blk.workspace(B, 1, t_max)
    clen = torch.full((B,), wl.cache_len, dtype=torch.int32, device=dev)
    out = (torch.empty(B, cfg.dim, dtype=torch.float32, device=dev), torch.empty(L, B, dtype=torch.float32, device=dev),
           torch.empty(L, B, cfg.n_experts_per_tok, dtype=torch.int32, device=dev))
    # the step through the library's DecodeGraph: eager once, then captured and replayed
    dg = R.DecodeGraph(blk, B, cache, clen, L, wl.act_threshold, workspace=ws, out=out)
    for st in range(args.warmup):
        dg.step(h0s[st], es[st])
    while dg._graph is None:                # fewer than 2 warm-up steps: capture before timing
        dg.step(h0s[0], es[0])
    torch.cuda.synchronize()
    assert blk.read_status() == 0, "device status word set during decode warm-up"
    stream = torch.cuda.current_stream()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for st in range(steps):
        dg.step(h0s[args.warmup + st], es[args.warmup + st])
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    assert blk.read_status() == 0, "device status word set during the timed decode steps"
    ms = e0.elapsed_time(e1) / steps
    ms_max = REP.max_over_ranks(ms, device=dev)
    # algorithmic bytes of the last timed step (its routing and cache lengths)
    bytes_step = decode_algorithmic_bytes(cfg, out[2].cpu(), (clen - 1).cpu())
    pk, pk_kind = peaks()
    gbs = bytes_step / (ms / 1e3) / 1e9
    # per-class breakdown, attention roofline and launch count: n_prof more steps, eagerly
    # (the profiler's events are recorded at launch time, so DecodeGraph does not replay
    # while profiling); not part of the timed numbers
    lens0 = clen.clone()
    NAT.profile_start()
    n0 = NAT.launch_count()
    for st in range(n_prof):
        dg.step(h0s[st], es[st])
    torch.cuda.synchronize()
    launches = (NAT.launch_count() - n0) * steps // n_prof
    prof = NAT.profile_stop()
    # attention alone: the cache bytes of the profiled steps over the attention kernels' time
    keys_read = float(n_prof * (lens0.double() + 1).sum() + B * n_prof * (n_prof - 1) / 2) * L
    attn_ms = prof.get("attention", (0, 0.0))[1] / n_prof
    attn_bytes = keys_read / n_prof * cache_bytes_per_key(cfg)
    attn_gbs = attn_bytes / (attn_ms / 1e3) / 1e9 if attn_ms else None
    if cfg.attn_type == "gqa":
        attn_desc = f"{cfg.n_heads} heads GQA ({cfg.n_kv_heads} kv, head dim {cfg.head_dim})"
        attn_kernel = "k_attn_decode_mma + k_attn_decode_combine (split-KV, mma.sync)"
    else:
        attn_desc = (f"{cfg.n_heads} heads MLA (kv_lora_rank {cfg.kv_lora_rank}, q_lora_rank {cfg.q_lora_rank}, "
                     f"rope {cfg.qk_rope_head_dim}, nope {cfg.qk_nope_head_dim}, v {cfg.v_head_dim}; latent cache, "
                     f"absorbed)")
        attn_kernel = "k_mla_q_absorb + k_mla_attn_tc + k_mla_out (split-KV latent attention; tcgen05 at kv_lora_rank 512)"
    res = {"metric": "decode tokens/s", "value": B * world / (ms_max / 1e3), "unit": "tokens/s",
           "ms_per_step": ms_max, "steps": steps,
           "workload": (f"{wl.name}: 3B-shaped KV-cached decode, dim {cfg.dim}, {attn_desc}, "
                        f"{cfg.n_experts} routed + {cfg.n_shared_experts} shared experts "
                        f"top-{cfg.n_experts_per_tok}, expert_dim {cfg.expert_dim}, {L} loops, batch {B} sequences "
                        f"with {wl.cache_len}-token random caches per loop, 1 new token per step, bf16, ACT off"),
           "cache_bytes_per_token_loop": cache_bytes_per_key(cfg),
           "attention_roofline": {"bound": "hbm", "kernel": attn_kernel, "achieved": attn_gbs,
                                  "peak": pk.get("hbm_gbs"), "unit": "GB/s",
                                  "frac": attn_gbs / pk.get("hbm_gbs") if attn_gbs else None,
                                  "ms_per_step": attn_ms, "cache_bytes_per_step": attn_bytes,
                                  "peak_kind": f"{pk_kind} HBM copy bandwidth"},
           "roofline": {"bound": "hbm", "kernel": "whole decode step (expert weights + caches streamed)",
                        "achieved": gbs, "peak": pk.get("hbm_gbs"), "unit": "GB/s",
                        "frac": gbs / pk.get("hbm_gbs"), "peak_kind": f"{pk_kind} HBM copy bandwidth",
                        "algorithmic_bytes_per_step": bytes_step, "traffic": None},
           "gpu_launches": launches,
           "cuda_graph": {"decode_step_replayed": dg._graph is not None, "launches_per_step": dg.graph_launches},
           "kernel_ms_per_step_eager": {k2: {"launches": v2[0] / n_prof, "ms_per_step": v2[1] / n_prof}
                                        for k2, v2 in sorted(prof.items())}}
    del k, v, cache, W, blk, ws, dg
    torch.cuda.empty_cache()
    return res


def run_depth_decode(args, rank, world, local_rank, name="rdt3b_decode_halting"):
    """Continuous depth-wise batching against lockstep decode steps on the 3B-shaped decode
    with a 4..16-loop halting spread: 64 sequences decode S tokens each, first as S lockstep
    steps (every step runs all 16 loops; halted rows skip the experts but keep their slot;
    replayed from a CUDA graph), then through DepthBatch (a token leaves its slot when it
    halts and the sequence's next token takes it; ticks replayed from a CUDA graph).  Both
    write the same caches; the outputs are compared."""
    import recurrent_depth_moe_b200 as R
    from recurrent_depth_moe_b200 import _native as NAT
    dev = torch.device("cuda", local_rank)
    wl = RI.get_workload(name)
    cfg = wl.cfg
    B, L, S, thr = wl.batch, wl.n_loops, args.depth_tokens or wl.decode_steps, wl.act_threshold
    t_max = wl.cache_len + S + 8
    seed = REP.replica_input_seed(wl.seed, rank)
    W = RI.block_weights(cfg, wl.seed, device=dev, halt_w_std=0.0, halt_b=0.0)
    k, v = RI.random_kv_cache(cfg, L, B, t_max, wl.cache_len, seed, device=dev)
    h0, e = RI.recurrent_inputs(cfg, B, S, seed, device=dev)
    h0, e = h0.view(B, S, cfg.dim), e.view(B, S, cfg.dim)
    off, kk = RI.halting_offsets_spread(B * S, wl.halt_spread[0], wl.halt_spread[1], thr, seed)
    off = off.view(B, S).to(dev)
    steps_in = [(h0[:, n].contiguous(), e[:, n].contiguous(), off[:, n].contiguous()) for n in range(S)]
    blk = R.RecurrentBlock(cfg, W)
    cache = R.KVCache(k, v)
    stream = torch.cuda.current_stream()
    # lockstep decode steps
    clen = torch.full((B,), wl.cache_len, dtype=torch.int32, device=dev)
    dg = R.DecodeGraph(blk, B, cache, clen, L, thr, halt_logit_offset=True)
    for n in range(2):                       # eager step, then the captured one
        dg.step(*steps_in[n])
    torch.cuda.synchronize()
    clen.fill_(wl.cache_len)
    lock_h = torch.empty(B, S, cfg.dim, dtype=torch.float32, device=dev)
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for n in range(S):
        lock_h[:, n].copy_(dg.step(*steps_in[n])[0])
    e1.record(stream)
    torch.cuda.synchronize()
    lock_ms = REP.max_over_ranks(e0.elapsed_time(e1), device=dev)
    assert blk.read_status() == 0
    # depth-batched
    clen0 = torch.full((B,), wl.cache_len, dtype=torch.int32, device=dev)
    db = R.DepthBatch(blk, h0, e, clen0, cache, L, thr, off)
    check_every = 16
    db.run(check_every=check_every, cuda_graph=True)             # warm-up (captures the tick graph)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    out = db.run(check_every=check_every, cuda_graph=True)
    e3.record(stream)
    torch.cuda.synchronize()
    depth_ms = REP.max_over_ranks(e2.elapsed_time(e3), device=dev)
    assert db.read_status() == 0
    ticks = db.ticks
    diff = float((out[0] - lock_h).norm() / lock_h.norm())
    # per-class breakdown of the depth-batched run (eager, profiled; not timed)
    NAT.profile_start()
    n0 = NAT.launch_count()
    db.run(check_every=check_every)
    torch.cuda.synchronize()
    launches = NAT.launch_count() - n0
    prof = NAT.profile_stop()
    mean_loops = float(kk.double().mean())
    tokens = B * S * world
    res = {"metric": "decode tokens/s, continuous depth-wise batching vs lockstep steps",
           "workload": (f"{wl.name}: 3B-shaped KV-cached decode (dim {cfg.dim}, {cfg.n_heads} heads GQA "
                        f"({cfg.n_kv_heads} kv), {cfg.n_experts} routed + {cfg.n_shared_experts} shared experts "
                        f"top-{cfg.n_experts_per_tok}, expert_dim {cfg.expert_dim}, {L} loops), {B} sequences "
                        f"with {wl.cache_len}-token random caches per loop, {S} new tokens each, bf16, ACT "
                        f"{thr} with per-token halting spread over {wl.halt_spread[0]}-{wl.halt_spread[1]} loops "
                        f"(mean {mean_loops:.2f})"),
           "depth_batch_tokens_per_s": tokens / (depth_ms / 1e3), "depth_batch_ms": depth_ms,
           "depth_batch_ticks": ticks, "depth_batch_ms_per_tick": depth_ms / max(ticks, 1),
           "lockstep_tokens_per_s": tokens / (lock_ms / 1e3), "lockstep_ms": lock_ms,
           "lockstep_ms_per_step": lock_ms / S,
           "speedup": lock_ms / depth_ms, "ideal_speedup": L / mean_loops,
           "mean_loops_per_token": mean_loops, "executed_token_loops": float(kk.sum()) * world,
           "max_rel_l2_depth_vs_lockstep_h_out": diff,
           "cuda_graph": {"ticks_per_replay": check_every, "launches_per_replay": db.graph_launches,
                          "lockstep_launches_per_step": dg.graph_launches},
           "gpu_launches_eager_run": launches,
           "kernel_ms_eager_run": {k2: {"launches": v2[0], "ms": v2[1]} for k2, v2 in sorted(prof.items())}}
    del db, dg, cache, k, v, W, blk
    torch.cuda.empty_cache()
    return res


def run_generate(args, rank, world, local_rank):
    """1B-shaped greedy generation through the library's Generator: the prompt pass
    (embedding, prelude, 16-loop recurrent prefill filling the caches, coda, head of the
    last positions), then one decode step per new token.  End to end: the prompt ids are
    copied in from pinned host memory and the generated ids copied out, inside the timed
    region."""
    import recurrent_depth_moe_b200 as R
    from recurrent_depth_moe_b200 import _native as NAT
    dev = torch.device("cuda", local_rank)
    wl = RI.get_workload("rdt1b_generate")
    cfg = wl.cfg
    B, T0, new, L = wl.batch, wl.seq, args.generate_new or wl.decode_steps, wl.n_loops
    MW = RI.model_weights(cfg, wl.seed, device=dev, halt_b=wl.halt_b)
    g = torch.Generator().manual_seed(REP.replica_input_seed(wl.seed, rank))
    prompts = [torch.randint(0, cfg.vocab_size, (B, T0), generator=g, dtype=torch.int32).pin_memory()
               for _ in range(2)]
    gen = R.Generator(cfg, MW, B, T0, new, L, wl.act_threshold)
    ids_d = torch.empty(B, T0, dtype=torch.int32, device=dev)
    out_h = torch.empty(new, B, dtype=torch.int32).pin_memory()
    stream = torch.cuda.current_stream()

    def one(prompt):
        ids_d.copy_(prompt, non_blocking=True)
        gen.prefill(ids_d)
        for step in range(1, new):
            gen.decode(step)
        out_h.copy_(gen.tokens, non_blocking=True)

    one(prompts[0])                                    # warm-up: a whole generation (captures the step graph)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record(stream)
    ids_d.copy_(prompts[1], non_blocking=True)
    gen.prefill(ids_d)
    e1.record(stream)
    for step in range(1, new):
        gen.decode(step)
    out_h.copy_(gen.tokens, non_blocking=True)
    e2.record(stream)
    torch.cuda.synchronize()
    # per-class breakdown and launch count: the same generation again, eagerly (the
    # profiler's events are recorded at launch time, so the Generator does not replay its
    # graph while profiling); not part of the timed numbers
    NAT.profile_start()
    n0 = NAT.launch_count()
    one(prompts[1])
    torch.cuda.synchronize()
    launches = NAT.launch_count() - n0
    prof = NAT.profile_stop()
    total_ms = REP.max_over_ranks(e0.elapsed_time(e2), device=dev)
    prefill_ms = e0.elapsed_time(e1)
    decode_ms = e1.elapsed_time(e2) / (new - 1)
    # algorithmic bytes of one decode step: the recurrent block's (16 loops, realised
    # routing of the last step), the prelude / coda blocks' weights and caches, the head
    D, Hkv, hd = cfg.dim, cfg.n_kv_heads, cfg.head_dim
    lens = torch.full((B,), T0 + new - 2)
    rec_bytes = decode_algorithmic_bytes(cfg, gen.dec_out[2].cpu(), lens)
    Fd = cfg.dim * 4 // 3
    block_bytes = (cfg.prelude_layers + cfg.coda_layers) * (
        attn_weight_bytes(cfg) + 3 * D * Fd * 2 + float((lens + 1).sum()) * cache_bytes_per_key(cfg))
    head_bytes = cfg.vocab_size * D * 2 + B * D * 2
    step_bytes = rec_bytes + block_bytes + head_bytes
    pk, pk_kind = peaks()
    gbs = step_bytes / (decode_ms / 1e3) / 1e9
    gen_graph, gen_graph_launches = gen._graph is not None, gen.graph_launches
    del gen, MW
    torch.cuda.empty_cache()
    return {"metric": "generated tokens/s (greedy, prompt pass included)", "value": B * new * world / (total_ms / 1e3),
            "unit": "tokens/s", "ms_per_generation": total_ms, "prefill_ms": prefill_ms,
            "decode_ms_per_token_step": decode_ms,
            "workload": (f"{wl.name}: 1B-shaped model (dim {D}, {cfg.n_heads} heads GQA ({Hkv} kv), "
                         f"{cfg.n_experts} routed + {cfg.n_shared_experts} shared experts top-{cfg.n_experts_per_tok}, "
                         f"expert_dim {cfg.expert_dim}, {L} loops, {cfg.prelude_layers} prelude + {cfg.coda_layers} "
                         f"coda dense layers, vocab {cfg.vocab_size}), batch {B} sequences, {T0}-token prompts, "
                         f"{new} new tokens, bf16, ACT 0.99 (halting bias -30)"),
            "e2e": {"h2d_bytes_per_generation": B * T0 * 4, "d2h_bytes_per_generation": new * B * 4},
            "decode_roofline": {"bound": "hbm", "kernel": "whole decode step (weights, caches and head streamed)",
                                "achieved": gbs, "peak": pk.get("hbm_gbs"), "unit": "GB/s",
                                "frac": gbs / pk.get("hbm_gbs"), "algorithmic_bytes_per_step": step_bytes,
                                "peak_kind": f"{pk_kind} HBM copy bandwidth"},
            "gpu_launches": launches,
            "cuda_graph": {"decode_step_replayed": gen_graph, "launches_per_step": gen_graph_launches},
            "kernel_ms_per_generation_eager": {k: {"launches": v[0], "ms": v[1]} for k, v in sorted(prof.items())}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the 1B-shaped prefill lines")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=128)
    ap.add_argument("--no-mla-decode", action="store_true", help="skip the multi-latent-attention decode line")
    ap.add_argument("--no-generate", action="store_true", help="skip the 1B-shaped generation line")
    ap.add_argument("--no-depth", action="store_true", help="skip the depth-wise batching decode line")
    ap.add_argument("--depth-only", action="store_true", help="profiling: run only the depth-wise batching line")
    ap.add_argument("--depth-tokens", type=int, default=None, help="tokens per sequence of the depth-wise line")
    ap.add_argument("--generate-only", action="store_true", help="profiling: run only the generation line")
    ap.add_argument("--generate-new", type=int, default=None, help="profiling: new tokens per generation")
    ap.add_argument("--decode-only", default=None,
                    choices=["rdt3b_decode", "rdt3b_mla_decode", "mla_decode_attn_small", "decode_attn_small",
                             "decode_moe_small"],
                    help="profiling: run only this decode workload and print its line")
    ap.add_argument("--workload", default=WORKLOAD, choices=["rdt1b_prefill", "rdt10b_prefill_zipf"])
    ap.add_argument("--batch", type=int, default=None, help="override the sequences per step (small profiling cases)")
    ap.add_argument("--loops", type=int, default=None, help="override n_loops (small profiling cases)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override the routed expert count (small profiling cases: the same row shapes in a few GB)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        log("warm-up raised to 3 steps")
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = RI.get_workload(args.workload)
    if args.batch or args.loops or args.experts:
        import dataclasses
        wl = dataclasses.replace(wl, batch=args.batch or wl.batch, n_loops=args.loops or wl.n_loops,
                                 cfg=wl.cfg.replace(n_experts=args.experts) if args.experts else wl.cfg)
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    from recurrent_depth_moe_b200 import build as BLD
    if rank == 0:
        BLD.build()
    if world > 1:
        torch.distributed.barrier()
    try:
        if args.decode_only or args.generate_only or args.depth_only:
            res = (run_generate(args, rank, world, local_rank) if args.generate_only else
                   run_depth_decode(args, rank, world, local_rank) if args.depth_only else
                   run_decode(args, rank, world, local_rank, args.decode_only))
            if rank == 0:
                print(json.dumps(res), flush=True)
        else:
            run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
