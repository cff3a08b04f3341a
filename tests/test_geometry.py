"""The kernels' index arithmetic, checked on the CPU (no GPU): a host build of csrc/geometry.cuh
walks every TMA chunk box as the hardware traverses it and must reproduce the oracle's window and
slot tables exactly (rows of the window table = local sequences, its columns = global sequences)."""
import subprocess

import numpy as np
import pytest

from oracle import squad_oracle as orc


@pytest.fixture(scope="module")
def checker(geometry_checker):
    return geometry_checker


CASES = [
    (1, 2, (21, 22, 40), (2, 4)), (1, 1, (21, 30, 52), (2, 4)), (1, 1, (21, 44, 80), (4, 4)),
    (2, 3, (21, 4, 8), (2, 4)), (1, 2, (5, 12, 20), (2, 4)), (1, 1, (21, 8, 8), (4, 4)),
    (1, 3, (3, 30, 52), (2, 4)), (1, 2, (1, 16, 16), (4, 4)), (1, 2, (2, 8, 8), (8, 8)),
    (1, 1, (7, 6, 10), (3, 5)), (1, 4, (5, 8, 8), (2, 2)),
]


@pytest.mark.parametrize("B,h,grid,win", CASES)
def test_boxes_match_oracle_tables(checker, B, h, grid, win):
    T, H, W = grid
    r = subprocess.run([checker, str(B), str(h), str(T), str(H), str(W), str(win[0]), str(win[1])],
                       capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]
    tables = {0: [], 1: []}
    for line in r.stdout.splitlines():
        if line.startswith("seq "):
            head, toks = line.split(":")
            kind = int(head.split()[1])
            tables[kind].append([int(t) for t in toks.split()])
    ref = orc.window_partition(T, H, W, T, *win)
    np.testing.assert_array_equal(np.array(tables[0]), ref)
    np.testing.assert_array_equal(np.array(tables[1]), ref.T)


def test_fast_division(checker):
    r = subprocess.run([checker, "div"], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]
