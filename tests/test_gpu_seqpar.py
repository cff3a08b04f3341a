"""Sequence-parallel SQuad with the CUDA kernels on one GPU (a one-rank NCCL group), forward and backward
against the fp64 oracle (needs a B200): the one-rank shortcut (the fused launch), and the split path
forced with explicit compute functions (single-pass launches around the exchanges, which are the
identity at one rank); and the library's block reordering around the exchanges against its plain torch
statement."""
import itertools
import os
import socket

import pytest
import torch
import torch.distributed as dist

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200.inputs import make_inputs
from sub_quadratic_two_squad_b200 import squad_seqpar_reorder
from sub_quadratic_two_squad_b200.seqpar import SeqParallelSquad
from test_gpu_parity import _dev, _host, check_bf16
from test_seqpar import torch_reorder

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def one_rank_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("order", ["local_then_global", "global_then_local"])
def test_sequence_parallel_one_rank(one_rank_group, order, split):
    grid, window = (21, 4, 8), (21, 2, 4)
    n = 21 * 4 * 8
    x = make_inputs(2, 2, n, 128, dtype="bf16", with_dout=True)
    q, k, v, do = (_dev(x[s], torch.bfloat16) for s in ("q", "k", "v", "do"))
    if split:
        from sub_quadratic_two_squad_b200 import squad_attn_bwd, squad_attn_fwd
        sp = SeqParallelSquad(grid, window, fwd=lambda q, k, v, g, w, o: squad_attn_fwd(q, k, v, g, w, o),
                              bwd=lambda q, k, v, out, do, ws, g, w, o: squad_attn_bwd(q, k, v, out, do, ws, g, w, o))
        assert not sp.whole
    else:
        sp = SeqParallelSquad(grid, window)
        assert sp.whole
    o, ctx = sp.forward(q, k, v, order)
    dq, dk, dv = sp.backward(ctx, do)
    oo = {"local_then_global": orc.LOCAL_THEN_GLOBAL, "global_then_local": orc.GLOBAL_THEN_LOCAL}[order]
    check_bf16(_host(o), orc.squad_attn_fwd(x["q"], x["k"], x["v"], grid, window, oo), "O")
    for name, mine, ref in zip(("dQ", "dK", "dV"), (dq, dk, dv),
                               orc.squad_attn_bwd(x["q"], x["k"], x["v"], x["do"], grid, window, oo)):
        check_bf16(_host(mine), ref, name)


LAYOUTS = ("band", "frames", "chunks")


def _layout_shape(layout, B, h, n, d, R):
    return (R, B, h, n // (R * R), d) if layout == "chunks" else (B, h, n // R, d)


@pytest.mark.parametrize("B,h,d,grid,R,dtype", [
    (2, 3, 128, (2, 3, 5), 1, torch.bfloat16),
    (2, 3, 128, (4, 6, 5), 2, torch.bfloat16),
    (2, 3, 64, (6, 9, 5), 3, torch.float32),
    (1, 2, 128, (8, 8, 6), 4, torch.float32),
    (1, 12, 128, (21, 30, 52), 3, torch.bfloat16),   # the 1.3B grid over 3 ranks: 252 blocks of 10x52 tokens
])
def test_seqpar_reorder_matches_torch(B, h, d, grid, R, dtype):
    """squad_seqpar_reorder bit for bit against the torch statement of the block reordering, for every
    pair of layouts, with and without the fused sum (fp32, rounded once)."""
    n = grid[0] * grid[1] * grid[2]
    gen = torch.Generator(device="cuda").manual_seed(17 * R + d)
    for src, dst in itertools.product(LAYOUTS, repeat=2):
        x = torch.randn(_layout_shape(src, B, h, n, d, R), device="cuda", generator=gen).to(dtype)
        add = torch.randn(_layout_shape(dst, B, h, n, d, R), device="cuda", generator=gen).to(dtype)
        assert torch.equal(squad_seqpar_reorder(x, grid, R, src, dst), torch_reorder(x, grid, R, src, dst)), (src, dst)
        assert torch.equal(squad_seqpar_reorder(x, grid, R, src, dst, add=add),
                           torch_reorder(x, grid, R, src, dst, add=add)), (src, dst, "add")
