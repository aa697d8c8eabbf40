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


HALT_MARGIN = 2e-2   # bf16: a position may halt at another loop only where the oracle's cum + p is this close to thr


def same_halting_rows(hw_gpu: torch.Tensor, hw_oracle: torch.Tensor, record: list, thr: float,
                      seq: int = 0) -> torch.Tensor:
    """ACT halts a position when cum + p reaches the threshold ("OpenMythos 분석", ACT), a
    decision taken on a float: within rounding of the threshold bf16 and fp64 may halt one
    loop apart, as a top-k near-tie may route apart.  Asserts that every position whose
    halting loop differs had, in the oracle, cum + p within HALT_MARGIN of thr at the
    earlier of the two loops.  Returns the mask of positions whose result is still
    determined: a halted row is frozen but its keys and values are recomputed every loop,
    so a position that halts at another loop changes what every later position of its
    sequence attends to.  With seq > 0 (rows sequence-major, seq positions each) those
    later positions are left out as well; with seq = 0 only the position itself."""
    hg, ho = halting_loop(hw_gpu), halting_loop(hw_oracle)
    diff = hg != ho
    if diff.any():
        t_first = torch.minimum(hg, ho)[diff]
        cum = torch.stack([r["cum"] for r in record])            # [L, N] oracle cum after loop t
        near = (cum[t_first, torch.nonzero(diff)[:, 0]] - thr).abs() < HALT_MARGIN
        assert near.all(), f"{int((~near).sum())} positions halt at another loop away from the threshold"
    if seq <= 0:
        return ~diff
    d = diff.view(-1, seq).to(torch.int64)
    downstream = torch.cumsum(d, dim=1) > 0                     # at or after the first disagreement
    return ~downstream.reshape(-1)
