"""Sequence-parallel SQuad (one all-to-all between the passes), world sizes 2, 3 and 4 over gloo on the CPU.

Each rank holds a band of window rows; the per-rank compute is the fp64 oracle's single-pass functions and
the block reordering around the exchanges a plain torch statement of it (test doubles for the library
calls, which tests/test_gpu_seqpar.py checks against the same statement), so this checks the exchange and
the composition of the passes against the oracle's whole-grid result, forward and backward, in both
orders."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200.seqpar import SeqParallelSquad, band_of

ORC = {"local_only": orc.LOCAL_ONLY, "global_only": orc.GLOBAL_ONLY}


def _fwd(q, k, v, grid, window, order):
    o = orc.squad_attn_fwd(q.numpy(), k.numpy(), v.numpy(), grid, window, ORC[order])
    return torch.from_numpy(o), None


def _bwd(q, k, v, o, do, ws, grid, window, order):
    g = orc.squad_attn_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), grid, window, ORC[order])
    return tuple(torch.from_numpy(x) for x in g)


# Axis order of the block index (b, head, r, tg) in each layout of the split (a block is Hb*W*d contiguous
# elements): the library's squad_seqpar_reorder moves blocks between these layouts.
AXES = {"band": "bhrt", "frames": "bhtr", "chunks": "rbht"}


def torch_reorder(x, grid, R, src, dst, add=None):
    """Plain torch statement of the split's block reordering (the test double of squad_seqpar_reorder)."""
    T, H, W = grid
    d = x.shape[-1]
    B, h = (x.shape[1], x.shape[2]) if src == "chunks" else (x.shape[0], x.shape[1])
    size = {"b": B, "h": h, "r": R, "t": T // R}
    blocks = x.reshape(*(size[a] for a in AXES[src]), (H // R) * W * d)
    y = blocks.permute(*(AXES[src].index(a) for a in AXES[dst]), 4).contiguous()
    y = y.reshape((R, B, h, -1, d) if dst == "chunks" else (B, h, -1, d))
    return y if add is None else y + add


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, grid, window, order, result):
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, H, W = grid
        rng = np.random.default_rng(5)
        q, k, v, do = (torch.from_numpy(rng.standard_normal((1, 2, T * H * W, 4))) for _ in range(4))
        sp = SeqParallelSquad(grid, window, fwd=_fwd, bwd=_bwd, reorder=torch_reorder)
        o_b, ctx = sp.forward(band_of(q, grid, rank, world), band_of(k, grid, rank, world),
                              band_of(v, grid, rank, world), order)
        grads = sp.backward(ctx, band_of(do, grid, rank, world))
        pieces = [o_b] + list(grads)
        gathered = [[torch.empty_like(x) for _ in range(world)] for x in pieces]
        for g, x in zip(gathered, pieces):
            dist.all_gather(g, x.contiguous())
        if rank == 0:
            result.update({name: [t.numpy() for t in g] for name, g in zip(("o", "dq", "dk", "dv"), gathered)})
            result["inputs"] = (q.numpy(), k.numpy(), v.numpy(), do.numpy())
    finally:
        dist.destroy_process_group()


def _assemble(bands, grid):
    T, H, W = grid
    R = len(bands)
    B, h, _, d = bands[0].shape
    parts = [b.reshape(B, h, T, H // R, W, d) for b in bands]
    return np.concatenate(parts, axis=3).reshape(B, h, T * H * W, d)


SPLITS = [
    # (world, grid, window): T % R == 0 and (H / hw) % R == 0
    (2, (4, 8, 6), (4, 2, 3)),     # two row bands of two window rows, two frames per group
    (3, (3, 6, 6), (3, 2, 3)),     # a world size that is not a power of two: one window row per band
    (4, (4, 8, 6), (4, 2, 3)),     # one frame per group: the global pass's window is one frame deep
]


@pytest.mark.parametrize("world,grid,window", SPLITS)
@pytest.mark.parametrize("order", ["local_then_global", "global_then_local"])
def test_sequence_parallel_matches_whole_grid(order, world, grid, window):
    with mp.get_context("spawn").Manager() as m:
        result = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), grid, window, order, result), nprocs=world, join=True)
        res = dict(result)
    q, k, v, do = res["inputs"]
    oo = {"local_then_global": orc.LOCAL_THEN_GLOBAL, "global_then_local": orc.GLOBAL_THEN_LOCAL}[order]
    ref_o = orc.squad_attn_fwd(q, k, v, grid, window, oo)
    ref_g = orc.squad_attn_bwd(q, k, v, do, grid, window, oo)
    np.testing.assert_allclose(_assemble(res["o"], grid), ref_o, rtol=1e-10, atol=1e-12)
    for name, ref in zip(("dq", "dk", "dv"), ref_g):
        np.testing.assert_allclose(_assemble(res[name], grid), ref, rtol=1e-9, atol=1e-11)


def test_sequence_parallel_rejects_bad_splits():
    class G:   # a stand-in group of 2 for the shape checks (no communication happens)
        pass
    import unittest.mock as um
    with um.patch.object(dist, "get_world_size", return_value=2), um.patch.object(dist, "get_rank", return_value=0):
        with pytest.raises(ValueError):
            SeqParallelSquad((3, 8, 6), (3, 2, 3), group=G(), fwd=_fwd, bwd=_bwd, reorder=torch_reorder)  # T % R
        with pytest.raises(ValueError):
            SeqParallelSquad((4, 6, 6), (4, 2, 3), group=G(), fwd=_fwd, bwd=_bwd, reorder=torch_reorder)  # (H / hw) % R


def test_reorder_moves_nothing_when_the_layouts_order_blocks_alike():
    """The premise of the library's shortcut (a view instead of a copy): with one rank every pair of
    layouts, and with any R a layout and itself, order the blocks alike."""
    B, h, d = 2, 3, 4
    for R, grid in ((1, (4, 6, 5)), (2, (4, 6, 5)), (3, (6, 9, 5))):
        n = grid[0] * grid[1] * grid[2]
        pairs = [(a, b) for a in AXES for b in AXES] if R == 1 else [(a, a) for a in AXES]
        for src, dst in pairs:
            shape = (R, B, h, n // (R * R), d) if src == "chunks" else (B, h, n // R, d)
            x = torch.arange(B * h * n // R * d, dtype=torch.float64).reshape(shape)
            assert torch.equal(torch_reorder(x, grid, R, src, dst).flatten(), x.flatten()), (R, src, dst)
    # and with more than one rank, different layouts do move blocks
    x = torch.arange(B * h * 120 // 2 * d, dtype=torch.float64).reshape(B, h, 60, d)
    assert not torch.equal(torch_reorder(x, (4, 6, 5), 2, "band", "frames").flatten(), x.flatten())
