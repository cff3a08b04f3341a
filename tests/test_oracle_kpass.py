"""Pins for the oracle's k-pass composition (nested windows), against constructions that share none of
its code: the pinned two-pass oracle (k = 2), torch SDPA over all tokens (k = 1), and dense masked
attention built from token coordinates with torch float64 autograd (k = 3), plus invariants and the
cost model's structure. No GPU.
"""
import numpy as np
import pytest
import torch

from oracle import squad_oracle as orc

ORDERS = [orc.KPASS_FORWARD, orc.KPASS_REVERSE]


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _same_group_masks(grid, levels):
    """Pass p's 'same sequence' relation from coordinates: two tokens share a pass-p sequence when
    their rows agree above level p (y // (h_1...h_p)) and below it (y mod (h_1...h_{p-1})), likewise
    their columns, and, except for the first pass, their frames."""
    T, H, W = grid
    t, y, x = np.unravel_index(np.arange(T * H * W), (T, H, W))
    masks = []
    for p in range(len(levels)):
        below_h = int(np.prod([a for a, _ in levels[:p]]))
        below_w = int(np.prod([b for _, b in levels[:p]]))
        upto_h, upto_w = below_h * levels[p][0], below_w * levels[p][1]

        def eq(v):
            return v[:, None] == v[None, :]

        m = eq(y // upto_h) & eq(y % below_h) & eq(x // upto_w) & eq(x % below_w)
        if p > 0:
            m &= eq(t)
        masks.append(m)
    return masks


def _torch_chain(q, k, v, masks, order_idx, scale):
    x = v
    for p in order_idx:
        x = torch.nn.functional.scaled_dot_product_attention(q, k, x, attn_mask=torch.from_numpy(masks[p]),
                                                             scale=scale)
    return x


@pytest.mark.parametrize("order,two_pass", [(orc.KPASS_FORWARD, orc.LOCAL_THEN_GLOBAL),
                                            (orc.KPASS_REVERSE, orc.GLOBAL_THEN_LOCAL)])
def test_two_levels_are_squad(order, two_pass):
    """k = 2 with levels (h_1, w_1), (H/h_1, W/w_1) is SQuad with window (T, h_1, w_1), forward and
    backward, in the matching order."""
    grid, levels, window = (3, 4, 6), [(2, 3), (2, 2)], (3, 2, 3)
    n, d = 72, 6
    q, k, v, do = (_rand((1, 2, n, d), s) for s in (1, 2, 3, 4))
    np.testing.assert_allclose(orc.kpass_fwd(q, k, v, grid, levels, order),
                               orc.squad_attn_fwd(q, k, v, grid, window, two_pass), rtol=0, atol=1e-13)
    for got, ref in zip(orc.kpass_bwd(q, k, v, do, grid, levels, order),
                        orc.squad_attn_bwd(q, k, v, do, grid, window, two_pass)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_one_level_is_full_attention():
    grid = (2, 3, 4)
    n, d = 24, 5
    q, k, v = (_rand((1, 3, n, d), s) for s in (5, 6, 7))
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v))).numpy()
    np.testing.assert_allclose(orc.kpass_fwd(q, k, v, grid, [(3, 4)]), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("grid,levels", [((2, 8, 12), [(2, 2), (2, 3), (2, 2)]),
                                         ((1, 12, 8), [(3, 2), (2, 2), (2, 2)]),
                                         ((3, 4, 6), [(1, 3), (2, 1), (2, 2)])])
def test_three_levels_are_masked_attention_chain(order, grid, levels):
    """k = 3 forward against a chain of torch SDPA calls restricted by coordinate masks, and the
    backward against torch autograd through that chain (float64)."""
    T, H, W = grid
    n, d = T * H * W, 4
    masks = _same_group_masks(grid, levels)
    order_idx = [0, 1, 2] if order == orc.KPASS_FORWARD else [2, 1, 0]
    q, k, v, do = (_rand((1, 2, n, d), s) for s in (21, 22, 23, 24))
    sc = 0.6
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    to = _torch_chain(tq, tk, tv, masks, order_idx, sc)
    np.testing.assert_allclose(orc.kpass_fwd(q, k, v, grid, levels, order, scale=sc), to.detach().numpy(),
                               rtol=1e-12, atol=1e-12)
    to.backward(torch.from_numpy(do))
    for got, ref in zip(orc.kpass_bwd(q, k, v, do, grid, levels, order, scale=sc), (tq.grad, tk.grad, tv.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("order", ORDERS)
def test_three_levels_reach_every_token(order):
    """k hops connect every source to every target: the composed n x n weight matrix is row-stochastic
    with every entry positive; the two orders give different operators."""
    grid, levels = (2, 4, 4), [(1, 2), (2, 1), (2, 2)]
    n = 32
    q, k = (_rand((1, 1, n, 3), s) for s in (31, 32))
    m = orc.kpass_composed_matrix(q, k, grid, levels, order)
    np.testing.assert_allclose(m.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (m > 0).all()
    other = orc.KPASS_REVERSE if order == orc.KPASS_FORWARD else orc.KPASS_FORWARD
    assert np.abs(m - orc.kpass_composed_matrix(q, k, grid, levels, other)).max() > 1e-3


def test_constant_values_are_returned():
    grid, levels = (2, 4, 6), [(2, 1), (1, 3), (2, 2)]
    n = 48
    q, k = (_rand((2, 1, n, 5), s) for s in (41, 42))
    v = np.broadcast_to(_rand((2, 1, 1, 7), 43), (2, 1, n, 7))
    for order in ORDERS:
        np.testing.assert_allclose(orc.kpass_fwd(q, k, v, grid, levels, order), v, rtol=0, atol=1e-13)


@pytest.mark.parametrize("grid,levels", [((2, 8, 12), [(2, 2), (2, 3), (2, 2)]), ((3, 4, 6), [(1, 3), (2, 1), (2, 2)])])
def test_groups_partition_the_tokens_and_vary_one_level(grid, levels):
    masks = _same_group_masks(grid, levels)
    n = grid[0] * grid[1] * grid[2]
    for p in range(len(levels)):
        g = orc.level_groups(grid, levels, p)
        assert np.array_equal(np.sort(g.ravel()), np.arange(n))
        same = np.zeros((n, n), dtype=bool)
        for row in g:
            same[np.ix_(row, row)] = True
        assert np.array_equal(same, masks[p])


def test_flops_reduce_and_follow_the_sequences():
    B, h, d = 1, 3, 16
    # k = 2 is the two-pass cost, k = 1 full attention
    assert orc.kpass_flops(B, h, d, (21, 22, 40), [(2, 4), (11, 10)]) == orc.squad_flops(B, h, d, 18480, 168)
    assert orc.kpass_flops(B, h, d, (3, 4, 6), [(4, 6)]) == orc.full_flops(B, h, d, 72)
    # balanced levels m_p = n^(1/k): 4 k h d n^(1 + 1/k); (T, H, W) = (4, 4, 4), k = 3, m_p = 4
    n = 64
    assert orc.kpass_flops(B, h, d, (4, 4, 4), [(1, 1), (2, 2), (2, 2)]) == pytest.approx(
        4 * 3 * B * h * d * n ** (4 / 3), rel=1e-12)
    # and the sum over the oracle's own sequences of 4 s^2 d
    grid, levels = (2, 8, 12), [(2, 2), (2, 3), (2, 2)]
    total = sum(4.0 * B * h * d * g.shape[0] * g.shape[1] ** 2
                for g in (orc.level_groups(grid, levels, p) for p in range(3)))
    assert orc.kpass_flops(B, h, d, grid, levels) == total


def test_levels_must_factor_the_grid():
    with pytest.raises(ValueError):
        orc.level_groups((2, 4, 6), [(2, 3), (3, 2)], 0)
    with pytest.raises(ValueError):
        orc.level_groups((2, 4, 6), [], 0)
    with pytest.raises(ValueError):
        orc.kpass_fwd(np.zeros((1, 1, 48, 2)), np.zeros((1, 1, 48, 2)), np.zeros((1, 1, 48, 2)), (2, 4, 6),
                      [(4, 6)], order="sideways")
