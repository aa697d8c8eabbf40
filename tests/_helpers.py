"""Shared helpers of the parity tests: device copies of seeded inputs, metrics,
and the teacher-forced router check."""
from __future__ import annotations

import math

import torch

import rdt_inputs as RI
from oracle import rdt_oracle as O

F64 = torch.float64


def to_dev(w, device="cuda"):
    if isinstance(w, dict):
        return {k: to_dev(v, device) for k, v in w.items()}
    if isinstance(w, list):
        return [to_dev(v, device) for v in w]
    return w.to(device).contiguous()


def to_cpu(w):
    if isinstance(w, dict):
        return {k: to_cpu(v) for k, v in w.items()}
    if isinstance(w, list):
        return [to_cpu(v) for v in w]
    return w.detach().cpu()


def max_rel(g: torch.Tensor, o: torch.Tensor) -> float:
    """fp32-mode metric: max |g - o| / max |o| over the tensor."""
    g, o = g.detach().cpu().double(), o.detach().cpu().double()
    return float((g - o).abs().max() / o.abs().max().clamp_min(1e-30))


def rel_l2(g: torch.Tensor, o: torch.Tensor) -> float:
    """bf16-mode metric: ||g - o||_2 / ||o||_2."""
    g, o = g.detach().cpu().double(), o.detach().cpu().double()
    return float((g - o).norm() / o.norm().clamp_min(1e-30))


FP32_TOL = 1e-4      # max relative error, fp32 mode
BF16_TOL = 2e-2      # relative L2, bf16 mode
ID_MARGIN = 1e-3     # router ties below this biased-logit margin may differ


def topk_margin(biased: torch.Tensor, k: int) -> torch.Tensor:
    """Smallest gap between consecutive entries among the k + 1 largest biased logits:
    below it, either the chosen set (k-th vs (k+1)-th) or the emitted order (a tie
    inside the top k) can flip under rounding.  inf when nothing can flip."""
    s = torch.sort(biased, dim=-1, descending=True).values
    m = min(k + 1, s.shape[-1])
    if m < 2:
        return torch.full(s.shape[:-1], math.inf, dtype=s.dtype)
    return (s[..., : m - 1] - s[..., 1:m]).min(dim=-1).values


def teacher_forced_ids(cfg, W, trace, ids_gpu: torch.Tensor, n_loops: int):
    """Recompute top-k in fp64 on the kernel's own router input (trace.f) and compare
    with the kernel's ids wherever the margin is >= ID_MARGIN.
    Returns (n_compared, n_mismatch, n_skipped)."""
    k = cfg.n_experts_per_tok
    Wr = W["w_router"].detach().cpu().double()
    bias = W["router_bias"].detach().cpu().double()
    r0, n = trace.row0, trace.n_rows
    compared = mism = skipped = 0
    for t in range(n_loops):
        ids_t = ids_gpu[t, r0:r0 + n].cpu().long()
        run = ids_t[:, 0] >= 0
        if not run.any():
            continue
        f = trace.f[t].cpu().double()[run]
        biased = f @ Wr.T + bias
        want = O.topk_lower_index(biased, k)
        marg = topk_margin(biased, k)
        ok = marg >= ID_MARGIN
        got = ids_t[run]
        compared += int(ok.sum())
        skipped += int((~ok).sum())
        # compare as sets in the kernel's order: the kernel emits descending biased order too
        mism += int((got[ok] != want[ok]).any(dim=-1).sum())
    return compared, mism, skipped


DECISION_MARGIN = 5e-2   # bf16 teacher-forced: a route may differ only where the oracle's margin is below this


def halting_loop(hw: torch.Tensor) -> torch.Tensor:
    """Index of the last loop with a non-zero ACT weight, per position."""
    L = hw.shape[0]
    nz = (hw.cpu() > 0).to(torch.int64) * torch.arange(L)[:, None]
    return nz.max(dim=0).values


def halting_loop_ids(ids: torch.Tensor) -> torch.Tensor:
    """Index of the last loop a position ran its experts in, per position (ids [L, N, k]; a
    halted position reports -1 from the next loop on).  Unlike the last non-zero ACT weight
    this is exact even where the remainder weight at the halting loop is 0."""
    L = ids.shape[0]
    ran = (ids.cpu()[..., 0] >= 0).to(torch.int64) * torch.arange(L)[:, None]
    return ran.max(dim=0).values


def check_route_flips(ids_gpu: torch.Tensor, biased_gpu: torch.Tensor, record: list) -> int:
    """Routes the oracle took from the GPU (route_ids) against the oracle's own top-k of the
    same run (record[t]["own_ids"]), per loop and running row.  Top-k picks the k largest
    biased logits ("OpenMythos 분석", MoE), so a route can differ only if some expert a the
    oracle picked and some expert b the GPU picked (or an order inside the top k) swap
    between the two sides' logits: with eps = max_e |l_gpu - l_oracle| of that row,
    l_oracle[a] - l_oracle[b] <= 2 eps.  Any difference not explained so fails.
    ids_gpu [L, N, k], biased_gpu [L, N, E] (the GPU's traced biased logits).
    Returns the number of (loop, row) routes that differ."""
    n = 0
    for t, r in enumerate(record):
        own = r["own_ids"]
        got = ids_gpu[t].cpu().long()
        run = (own[:, 0] >= 0) & (got[:, 0] >= 0)
        diff = torch.nonzero((own != got).any(-1) & run)[:, 0]
        for i in diff.tolist():
            lo = r["biased"][i]
            eps = float((lo - biased_gpu[t, i].cpu().double()).abs().max())
            o, g = own[i].tolist(), got[i].tolist()
            if set(o) != set(g):
                pairs = [(a, b) for a in set(o) - set(g) for b in set(g) - set(o)]
            else:   # same experts in another order: the pairs the GPU emitted in the oracle's wrong order
                pairs = [(g[y], g[x]) for x in range(len(g)) for y in range(x + 1, len(g))
                         if float(lo[g[x]]) < float(lo[g[y]])]
            worst = max(float(lo[a] - lo[b]) for a, b in pairs)
            assert worst <= 2 * eps + 1e-9, (f"loop {t} row {i}: route {g} vs the oracle's {o} with a logit "
                                             f"gap {worst:.3e} beyond the row's drift 2 x {eps:.3e}")
            n += 1
    return n


MAX_FORCED_FRAC = 0.02   # bf16: at most this share of positions may halt one loop apart from the oracle


def halt_margin(p_gpu: torch.Tensor, p_oracle: torch.Tensor, halt_loop: torch.Tensor) -> float:
    """How far apart the two sides' cumulative halting sums can drift by rounding alone:
    the number of loops times the largest |p_gpu - p_oracle| seen on any position and any
    loop it ran (t <= its halting loop), both sides on the same discrete path.  The ACT
    rule ("OpenMythos 분석", ACT) halts when cum + p >= thr with cum the running sum of p,
    so two computations of cum differ by at most the sum of their per-loop differences."""
    L = p_gpu.shape[0]
    ran = torch.arange(L)[:, None] <= halt_loop[None, :]
    d = (p_gpu.cpu().double() - p_oracle.cpu().double()).abs()[ran]
    return L * float(d.max()) if d.numel() else 0.0


def check_forced_halts(forced: torch.Tensor, t_star: torch.Tensor, cum_oracle: torch.Tensor, thr: float,
                       margin: float, n_positions: int, max_frac: float = MAX_FORCED_FRAC):
    """A position may halt at another loop than the oracle's only where the oracle's
    cum + p at the earlier of the two loops (t_star) is within `margin` of the threshold,
    and only for a small share of the positions.  forced: positions; cum_oracle [L, N]."""
    if forced.numel() == 0:
        return
    assert forced.numel() <= max(1, int(max_frac * n_positions)), \
        f"{forced.numel()} of {n_positions} positions halt at another loop than the oracle"
    dist = (cum_oracle[t_star, forced] - thr).abs()
    far = dist > margin
    assert not far.any(), (f"{int(far.sum())} positions halt at another loop with cum + p "
                           f"{dist[far].min():.3e} from the threshold (margin {margin:.3e})")


def oracle_following_halts(run, ids_gpu: torch.Tensor, p_gpu: torch.Tensor, thr: float, max_rounds: int = 10):
    """Run the oracle (`run(halt_at, record)` -> (h_out, hw, ids, kv)) so that it takes the
    GPU's halting loop at the positions where the halting decision was decided by rounding.

    A halted position is frozen but its keys and values are recomputed every loop, so a
    position that halts one loop apart changes what every later position of its sequence
    attends to; instead of leaving those positions out, the oracle is rerun with the GPU's
    halting loop imposed on the disagreeing positions (halt_at), which keeps every position
    comparable end to end.  Each imposed position must have been a near-tie: the oracle's
    cum + p within the rounding drift (halt_margin, measured on the aligned run) of thr.
    Halting loops are read from the expert ids (halting_loop_ids).
    Returns (oracle outputs, record, number of imposed positions, margin)."""
    hg = halting_loop_ids(ids_gpu)
    N = hg.numel()
    halt_at = torch.full((N,), -1, dtype=torch.int64)
    t_star = torch.zeros(N, dtype=torch.int64)
    cum_first = None
    for _ in range(max_rounds):
        rec = []
        out = run(halt_at if (halt_at >= 0).any() else None, rec)
        ho = halting_loop_ids(out[2])
        cum = torch.stack([r["cum"] for r in rec])
        if cum_first is None:
            cum_first = cum
        new = (ho != hg) & (halt_at < 0)
        if not new.any():
            break
        t_star[new] = torch.minimum(hg, ho)[new]
        halt_at[new] = hg[new]
    forced = torch.nonzero(halt_at >= 0)[:, 0]
    ho = halting_loop_ids(out[2])
    left = ho != hg
    assert not left.any(), (f"the oracle still halts {int(left.sum())} positions at another loop after imposing "
                            f"{int((halt_at >= 0).sum())} (forced still differing: {int((left & (halt_at >= 0)).sum())})")
    margin = halt_margin(p_gpu, torch.stack([r["p"] for r in rec]), hg)
    check_forced_halts(forced, t_star[forced], cum, thr, margin, N)
    return out, rec, int(forced.numel()), margin
