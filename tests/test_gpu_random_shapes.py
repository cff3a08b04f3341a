"""Seeded random shapes through every path (needs a B200): grid, window (dividing or not), order, dtype,
head dim, batch and heads drawn from a fixed seed; forward and backward against the fp64 oracle."""
import numpy as np
import pytest
import torch

from test_gpu_parity import run_bwd, run_fwd

pytestmark = pytest.mark.gpu

ORDERS = ["local_then_global", "global_then_local", "local_only", "global_only"]


def _cases(n_cases=12, seed=20261202):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n_cases:
        T = int(rng.integers(1, 7))
        hw, ww = int(rng.integers(1, 5)), int(rng.integers(1, 5))
        H = hw * int(rng.integers(1, 5)) + int(rng.integers(0, hw))     # sometimes not a multiple
        W = ww * int(rng.integers(1, 5)) + int(rng.integers(0, ww))
        if H < hw or W < ww or T * H * W > 700:
            continue
        dtype = torch.bfloat16 if rng.random() < 0.6 else torch.float32
        d = 128 if rng.random() < 0.7 else 64
        cases.append((int(rng.integers(1, 3)), int(rng.integers(1, 4)), d, (T, H, W), (T, hw, ww),
                      ORDERS[int(rng.integers(0, 4))], dtype))
    return cases


@pytest.mark.parametrize("B,h,d,grid,window,order,dtype", _cases())
def test_random_shape_forward_and_backward(B, h, d, grid, window, order, dtype):
    run_fwd(B, h, d, grid, window, order, dtype)
    run_bwd(B, h, d, grid, window, order, dtype)
