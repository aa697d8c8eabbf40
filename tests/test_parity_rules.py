"""The parity tests' rules for float-decided discrete outcomes, checked on planted cases."""
import pytest
import torch

from tests._helpers import HALT_MARGIN, same_halting_rows, topk_margin


def _hw(loops):
    """ACT weights with position i halting at loop loops[i] (L = 3)."""
    hw = torch.zeros(3, len(loops))
    for i, t in enumerate(loops):
        hw[: t + 1, i] = 1.0 / (t + 1)
    return hw


def test_halting_disagreement_near_the_threshold_is_accepted():
    thr = 0.99
    record = [{"cum": torch.tensor([0.2, 0.6, 0.3])},
              {"cum": torch.tensor([0.5, thr + HALT_MARGIN / 2, 0.6])},   # the oracle just reaches thr
              {"cum": torch.tensor([1.1, 1.2, 1.0])}]
    keep = same_halting_rows(_hw([2, 2, 2]), _hw([2, 1, 2]), record, thr)   # position 1: oracle halts at loop 1
    assert keep.tolist() == [True, False, True]


def test_halting_disagreement_away_from_the_threshold_fails():
    thr = 0.99
    record = [{"cum": torch.tensor([0.2, 0.5, 0.3])},
              {"cum": torch.tensor([0.5, 0.99, 0.6])},
              {"cum": torch.tensor([1.1, 1.2, 1.0])}]
    with pytest.raises(AssertionError):
        same_halting_rows(_hw([2, 0, 2]), _hw([2, 1, 2]), record, thr)   # loop 0: cum 0.5, far from 0.99


def test_topk_margin_counts_order_swaps_inside_the_top_k():
    s = torch.tensor([[3.0, 2.9995, 1.0, 0.0]], dtype=torch.float64)        # top-2 order is a near-tie
    assert float(topk_margin(s, 2)[0]) == pytest.approx(5e-4)
    s = torch.tensor([[3.0, 2.0, 1.0, 0.999]], dtype=torch.float64)          # the 3rd / 4th near-tie is outside top-2 + 1
    assert float(topk_margin(s, 2)[0]) == pytest.approx(1.0)


def test_positions_after_a_halting_disagreement_are_left_out_of_their_sequence():
    thr = 0.99
    # two sequences of 3 positions; position 1 of sequence 0 halts one loop apart
    record = [{"cum": torch.tensor([0.2, 0.6, 0.3, 0.2, 0.2, 0.2])},
              {"cum": torch.tensor([0.5, thr + HALT_MARGIN / 2, 0.6, 0.5, 0.5, 0.5])},
              {"cum": torch.tensor([1.1, 1.2, 1.0, 1.0, 1.0, 1.0])}]
    keep = same_halting_rows(_hw([2, 2, 2, 2, 2, 2]), _hw([2, 1, 2, 2, 2, 2]), record, thr, seq=3)
    assert keep.tolist() == [True, False, False, True, True, True]


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
