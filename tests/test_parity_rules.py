"""The parity tests' rules for float-decided discrete outcomes, checked on planted cases."""
import math

import pytest
import torch

from tests._helpers import (check_forced_halts, check_route_flips, halt_margin, halting_loop, halting_loop_ids,
                            oracle_following_halts, topk_margin)


def _hw(loops, L=3):
    """ACT weights with position i halting at loop loops[i]."""
    hw = torch.zeros(L, len(loops))
    for i, t in enumerate(loops):
        hw[: t + 1, i] = 1.0 / (t + 1)
    return hw


def test_halt_margin_is_loops_times_the_largest_drift_on_loops_run():
    p_o = torch.full((3, 4), 0.3, dtype=torch.float64)
    p_g = p_o.clone()
    p_g[0, 1] += 0.002          # ran: counts
    p_g[2, 0] += 0.5            # position 0 halted at loop 1: loop 2 is not compared
    assert halt_margin(p_g, p_o, torch.tensor([1, 2, 2, 2])) == pytest.approx(3 * 0.002)


def test_forced_halt_near_the_threshold_is_accepted():
    thr = 0.99
    cum = torch.tensor([[0.2, 0.6, 0.3], [0.5, thr + 0.004, 0.6], [1.1, 1.2, 1.0]], dtype=torch.float64)
    check_forced_halts(torch.tensor([1]), torch.tensor([1]), cum, thr, margin=0.005, n_positions=100)


def test_forced_halt_away_from_the_threshold_fails():
    thr = 0.99
    cum = torch.tensor([[0.2, 0.5, 0.3], [0.5, 0.99, 0.6], [1.1, 1.2, 1.0]], dtype=torch.float64)
    with pytest.raises(AssertionError):
        check_forced_halts(torch.tensor([1]), torch.tensor([0]), cum, thr, margin=0.005, n_positions=100)


def test_too_many_forced_halts_fail():
    thr = 0.99
    cum = torch.full((3, 10), thr, dtype=torch.float64)
    with pytest.raises(AssertionError):
        check_forced_halts(torch.tensor([1, 2, 3]), torch.tensor([1, 1, 1]), cum, thr, margin=0.1, n_positions=10,
                           max_frac=0.2)


def _ids(loops, L=3):
    """Expert ids [L, N, 1] of positions halting at loop loops[i] (-1 after the halt)."""
    ids = torch.full((L, len(loops), 1), -1, dtype=torch.int64)
    for i, t in enumerate(loops):
        ids[: t + 1, i] = 0
    return ids


def test_halting_loop_from_ids_is_exact_with_a_zero_remainder():
    hw = torch.tensor([[0.6], [0.5], [0.0]])          # halts at loop 2 with remainder max(1 - 1.1, 0) = 0
    assert halting_loop(hw).tolist() == [1]
    assert halting_loop_ids(_ids([2])).tolist() == [2]


def test_route_flip_within_the_row_drift_is_accepted_and_beyond_it_fails():
    record = [{"own_ids": torch.tensor([[0, 1], [2, 3]]),
               "biased": torch.tensor([[3.0, 2.0, 1.99, 0.0], [0.0, 0.0, 5.0, 4.0]], dtype=torch.float64)}]
    gpu_ids = torch.tensor([[[0, 2], [2, 3]]])            # row 0: expert 2 instead of 1 (oracle gap 0.01)
    near = torch.tensor([[[3.0, 2.0, 2.0049, 0.0], [0.0, 0.0, 5.0, 4.0]]])   # row drift 0.0051: explained
    assert check_route_flips(gpu_ids, near, record) == 1
    far = torch.tensor([[[3.0, 2.0, 1.9920, 0.0], [0.0, 0.0, 5.0, 4.0]]])    # drift 0.002 < gap / 2
    with pytest.raises(AssertionError):
        check_route_flips(gpu_ids, far, record)
    swapped = torch.tensor([[[1, 0], [2, 3]]])           # same experts, order inverted (gap 1.0)
    with pytest.raises(AssertionError):
        check_route_flips(swapped, near, record)


def test_oracle_route_hook_imposes_the_given_experts():
    import rdt_inputs as RI
    from oracle import rdt_oracle as O
    cfg = RI.get_workload("tiny_gqa_fp32").cfg
    W = RI.block_weights(cfg, 4)
    h0, e = RI.recurrent_inputs(cfg, 1, 6, 4)
    rec = []
    base = O.recurrent_forward(cfg, W, h0, e, 1, 3, 0.0, record=rec)
    same = O.recurrent_forward(cfg, W, h0, e, 1, 3, 0.0, route_ids=base[2])
    assert torch.equal(base[0], same[0]) and torch.equal(base[2], same[2])
    route = base[2].clone()
    route[1, 2] = torch.tensor([7, 6])                   # loop 1, position 2: other experts
    rec2 = []
    moved = O.recurrent_forward(cfg, W, h0, e, 1, 3, 0.0, record=rec2, route_ids=route)
    assert moved[2][1, 2].tolist() == [7, 6] and torch.equal(rec2[1]["own_ids"][2], base[2][1, 2])
    assert not torch.equal(moved[0][2], base[0][2])
    # earlier positions untouched (causal; the expert matmuls group rows differently, hence
    # agreement to rounding rather than bit for bit)
    assert torch.allclose(moved[0][:2], base[0][:2], rtol=1e-12, atol=1e-12)


def test_oracle_is_rerun_on_the_gpu_halting_loop_of_a_near_tie():
    """A planted oracle whose position 1 reaches the threshold at loop 1 by 0.001 while the
    GPU halts it at loop 2: the helper reruns it with that halt imposed."""
    thr, L = 0.99, 3
    calls = []

    def run(halt_at, rec):
        calls.append(None if halt_at is None else halt_at.clone())
        loops = [2, 1, 2] if halt_at is None else [2, int(halt_at[1]), 2]
        p = torch.tensor([[0.3, 0.5, 0.3], [0.3, 0.491, 0.3], [0.3, 0.3, 0.3]], dtype=torch.float64)
        cum = torch.cumsum(p, 0)
        for t in range(L):
            rec.append({"p": p[t], "cum": cum[t]})
        return None, _hw(loops), _ids(loops), None

    p_gpu = torch.tensor([[0.3, 0.5, 0.3], [0.3, 0.4895, 0.3], [0.3, 0.3, 0.3]], dtype=torch.float64)
    out, rec, n_forced, margin = oracle_following_halts(run, _ids([2, 2, 2]), p_gpu, thr)
    assert n_forced == 1 and calls[0] is None and calls[1].tolist() == [-1, 2, -1]
    assert margin == pytest.approx(3 * 0.0015)
    assert halting_loop(out[1]).tolist() == [2, 2, 2]


def test_oracle_halt_at_hook_imposes_the_halting_loop():
    """The oracle's test hook: halt_at[i] = t halts position i at loop t with the remainder as
    its weight (ACT weights still sum to one); -1 everywhere is the plain rule."""
    import rdt_inputs as RI
    from oracle import rdt_oracle as O
    cfg = RI.get_workload("tiny_gqa_fp32").cfg
    W = RI.block_weights(cfg, 3, halt_w_std=0.0, halt_b=-3.0)      # p = sigmoid(-3): no early halt
    h0, e = RI.recurrent_inputs(cfg, 1, 6, 3)
    L = 4
    base = O.recurrent_forward(cfg, W, h0, e, 1, L, 0.99)
    same = O.recurrent_forward(cfg, W, h0, e, 1, L, 0.99, halt_at=torch.full((6,), -1, dtype=torch.int64))
    assert torch.equal(base[0], same[0]) and torch.equal(base[1], same[1])
    assert halting_loop(base[1]).tolist() == [L - 1] * 6
    forced = O.recurrent_forward(cfg, W, h0, e, 1, L, 0.99, halt_at=torch.tensor([-1, 1, -1, -1, 0, -1]))
    assert halting_loop(forced[1]).tolist() == [3, 1, 3, 3, 0, 3]
    assert torch.allclose(forced[1].sum(0), torch.ones(6, dtype=torch.float64), atol=1e-12)
    p = 1.0 / (1.0 + math.exp(3.0))
    assert float(forced[1][1, 1]) == pytest.approx(1.0 - p)             # remainder after one loop of p
    assert (forced[2][2:, 1] == -1).all()                                # frozen after its halt


def test_topk_margin_counts_order_swaps_inside_the_top_k():
    s = torch.tensor([[3.0, 2.9995, 1.0, 0.0]], dtype=torch.float64)        # top-2 order is a near-tie
    assert float(topk_margin(s, 2)[0]) == pytest.approx(5e-4)
    s = torch.tensor([[3.0, 2.0, 1.0, 0.999]], dtype=torch.float64)          # the 3rd / 4th near-tie is outside top-2 + 1
    assert float(topk_margin(s, 2)[0]) == pytest.approx(1.0)


def test_dense_padding_keeps_the_block_function():
    """The binding pads a dense FFN's hidden width to a multiple of 128 (SwiGLU tile, TMA rows)
    with zero rows and columns; the SwiGLU FFN computes the same function (fp64, 4 dim / 3
    widths of the 1B and tiny configs)."""
    import torch.nn.functional as Fn
    from recurrent_depth_moe_b200.api import dense_padded
    g = torch.Generator().manual_seed(9)
    for D in (256, 2048):
        F = D * 4 // 3
        w = {"w13": torch.randn(1, 2 * F, D, generator=g, dtype=torch.float64),
             "w2": torch.randn(1, D, F, generator=g, dtype=torch.float64)}
        p, Fp = dense_padded(w)
        assert Fp % 128 == 0 and Fp >= F and Fp - F < 128
        x = torch.randn(5, D, generator=g, dtype=torch.float64)

        def ffn(w13, w2, h):
            return (Fn.silu(x @ w13[0, :h].T) * (x @ w13[0, h:].T)) @ w2[0].T
        assert torch.allclose(ffn(w["w13"], w["w2"], F), ffn(p["w13"], p["w2"], Fp), rtol=1e-12, atol=1e-12)
