"""Repeatability under different scratch contents (needs a B200): the same inputs, three forward and
backward calls, every output and workspace byte filled beforehand with a different pattern (0xFF:
NaN in bf16 and fp32; 0x7F: a large finite value; 0x00). The results must be bitwise identical and
finite. The shapes give every persistent CTA several work items, so the paths between items (the next
item's loads while the previous one is written out, accumulator columns reused across items, the
fused launch's per-head hand-off) are exercised: a read of scratch before it is written, or of an
item's data after the next item's loads replaced it, changes the bits from one call to the next."""
import pytest
import torch

from sub_quadratic_two_squad_b200 import (make_params, squad_attn_bwd, squad_attn_bwd_kernels,
                                          squad_attn_bwd_workspace_bytes, squad_attn_fwd,
                                          squad_attn_fwd_workspace_bytes)
from sub_quadratic_two_squad_b200.inputs import make_inputs
from test_gpu_parity import _dev

pytestmark = pytest.mark.gpu

CASES = [
    # (B, h, grid, window, order, backward kernels expected): items per CTA > 1 on 148 SMs
    (1, 4, (21, 22, 40), (21, 2, 4), "local_then_global", ("tc_whole", "tc_whole")),      # 440 windows, 672 slots
    (1, 4, (21, 22, 40), (21, 2, 4), "global_then_local", ("tc_whole", "tc_whole")),
    (1, 24, (21, 8, 16), (21, 4, 4), "local_then_global", ("tc_chunked", "tc_whole")),    # 576 chunk items
    (1, 24, (2, 32, 64), (2, 2, 4), "local_then_global", ("tc_whole", "tc_chunked")),     # 256-token slots
]


@pytest.mark.parametrize("B,h,grid,window,order,kernels", CASES)
def test_forward_backward_bitwise_repeatable(B, h, grid, window, order, kernels):
    d = 128
    n = grid[0] * grid[1] * grid[2]
    assert tuple(squad_attn_bwd_kernels(B, h, d, grid, window, order)) == kernels
    x = make_inputs(B, h, n, d, dtype="bf16", heavy_tail=True, with_dout=True, seed=123)
    q, k, v, do = (_dev(x[s], torch.bfloat16) for s in ("q", "k", "v", "do"))
    prm = make_params(B, h, d, grid, window, order, torch.bfloat16)
    fwd_bytes, bwd_bytes = squad_attn_fwd_workspace_bytes(prm), squad_attn_bwd_workspace_bytes(prm)
    results = []
    for fill in (0xFF, 0x7F, 0x00):
        def filled(shape):
            t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
            t.view(torch.uint8).fill_(fill)
            return t
        o = filled(q.shape)
        ws = torch.full((fwd_bytes,), fill, dtype=torch.uint8, device="cuda")
        squad_attn_fwd(q, k, v, grid, window, order, out=o, workspace=ws)
        dq, dk, dv = filled(q.shape), filled(q.shape), filled(q.shape)
        bws = torch.full((bwd_bytes,), fill, dtype=torch.uint8, device="cuda")
        squad_attn_bwd(q, k, v, o, do, ws, grid, window, order, dq=dq, dk=dk, dv=dv, workspace=bws)
        torch.cuda.synchronize()
        for name, t in zip(("o", "dq", "dk", "dv"), (o, dq, dk, dv)):
            assert torch.isfinite(t.float()).all(), f"{name}: non-finite elements after a 0x{fill:02X} fill"
        results.append([t.view(torch.int16).clone() for t in (o, dq, dk, dv)])
    for i in (1, 2):
        for name, a, b in zip(("o", "dq", "dk", "dv"), results[0], results[i]):
            assert torch.equal(a, b), f"{name} differs between call 0 and call {i}"
