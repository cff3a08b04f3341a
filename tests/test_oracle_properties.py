"""Property tests of the oracle over random small grids and windows (no GPU): the invariants the pins
check on fixed shapes hold on every drawn shape. Composed weights are row-stochastic and positive, the
two passes partition the tokens, constant values come back unchanged, and k = 2 nested levels are
the two-pass method, in both orders."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import squad_oracle as orc


def _divisors(x):
    return [a for a in range(1, x + 1) if x % a == 0]


@st.composite
def grid_and_window(draw):
    T = draw(st.integers(1, 3))
    H = draw(st.integers(1, 6))
    W = draw(st.integers(1, 6))
    hw = draw(st.sampled_from(_divisors(H)))
    ww = draw(st.sampled_from(_divisors(W)))
    return (T, H, W), (T, hw, ww)


ORDERS = [orc.LOCAL_THEN_GLOBAL, orc.GLOBAL_THEN_LOCAL]


@settings(max_examples=40, deadline=None)
@given(grid_and_window(), st.sampled_from(ORDERS), st.integers(0, 2 ** 31 - 1))
def test_composed_matrix_is_row_stochastic_and_positive(gw, order, seed):
    grid, window = gw
    n = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((1, 1, n, 3)), rng.standard_normal((1, 1, n, 3))
    m = orc.composed_matrix(q, k, grid, window, order)
    np.testing.assert_allclose(m.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (m > 0).all()


@settings(max_examples=40, deadline=None)
@given(grid_and_window())
def test_local_and_global_sequences_partition_the_tokens(gw):
    grid, window = gw
    n = grid[0] * grid[1] * grid[2]
    table = orc.window_partition(*grid, *window)
    assert np.array_equal(np.sort(table.ravel()), np.arange(n))
    # a window and a slot share exactly one token
    for c in range(table.shape[0]):
        for j in range(table.shape[1]):
            assert len(set(table[c]) & set(table[:, j])) == 1


@settings(max_examples=30, deadline=None)
@given(grid_and_window(), st.sampled_from(ORDERS + [orc.LOCAL_ONLY, orc.GLOBAL_ONLY]), st.integers(0, 2 ** 31 - 1))
def test_constant_values_come_back(gw, order, seed):
    grid, window = gw
    n = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((1, 2, n, 4)), rng.standard_normal((1, 2, n, 4))
    v = np.broadcast_to(rng.standard_normal((1, 2, 1, 5)), (1, 2, n, 5))
    np.testing.assert_allclose(orc.squad_attn_fwd(q, k, v, grid, window, order), v, rtol=0, atol=1e-12)


@settings(max_examples=30, deadline=None)
@given(grid_and_window(), st.integers(0, 2 ** 31 - 1))
def test_two_levels_are_the_two_pass_method(gw, seed):
    (T, H, W), (_, hw, ww) = gw
    n = T * H * W
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((1, 1, n, 4)) for _ in range(3))
    levels = [(hw, ww), (H // hw, W // ww)]
    for kp, two in ((orc.KPASS_FORWARD, orc.LOCAL_THEN_GLOBAL), (orc.KPASS_REVERSE, orc.GLOBAL_THEN_LOCAL)):
        np.testing.assert_allclose(orc.kpass_fwd(q, k, v, (T, H, W), levels, kp),
                                   orc.squad_attn_fwd(q, k, v, (T, H, W), (T, hw, ww), two), rtol=0, atol=1e-12)


@st.composite
def grid_and_levels(draw):
    """A small grid factored into three levels per axis (every pass over at least two tokens)."""
    T = draw(st.integers(1, 2))
    hs = [draw(st.integers(1, 3)) for _ in range(3)]
    ws = [draw(st.integers(1, 3)) for _ in range(3)]
    levels = list(zip(hs, ws))
    if T * hs[0] * ws[0] < 2:
        levels[0] = (hs[0], 2)
    for i in (1, 2):
        if levels[i][0] * levels[i][1] < 2:
            levels[i] = (2, levels[i][1])
    H = int(np.prod([a for a, _ in levels]))
    W = int(np.prod([b for _, b in levels]))
    return (T, H, W), levels


@settings(max_examples=25, deadline=None)
@given(grid_and_levels(), st.sampled_from([orc.KPASS_FORWARD, orc.KPASS_REVERSE]), st.integers(0, 2 ** 31 - 1))
def test_three_levels_reach_every_token_and_keep_constants(gl, order, seed):
    grid, levels = gl
    n = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((1, 1, n, 3)), rng.standard_normal((1, 1, n, 3))
    m = orc.kpass_composed_matrix(q, k, grid, levels, order)
    np.testing.assert_allclose(m.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (m > 0).all()
    v = np.broadcast_to(rng.standard_normal((1, 1, 1, 4)), (1, 1, n, 4))
    np.testing.assert_allclose(orc.kpass_fwd(q, k, v, grid, levels, order), v, rtol=0, atol=1e-12)
