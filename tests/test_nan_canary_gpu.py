"""NaN canaries (needs a B200): every output and workspace byte is set to 0xFF before the call (NaN as
bf16 and as fp32), so an element the kernels leave unwritten, or a read of scratch before it is
written, shows up as a non-finite or wrong result. Covers each launch path: the fused two-pass kernel,
a single pass, a padded grid, the fp32 CUDA-core kernels, the chunked kernel (336-token windows) and
the k-pass chain, forward and backward."""
import ctypes

import pytest
import torch

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import (make_kpass_params, make_params, squad_attn_bwd, squad_attn_bwd_workspace_bytes,
                                          squad_attn_fwd, squad_attn_fwd_workspace_bytes, squad_kpass_bwd,
                                          squad_kpass_fwd)
from sub_quadratic_two_squad_b200 import _lib
from sub_quadratic_two_squad_b200.inputs import make_inputs
from test_gpu_parity import ORC_ORDER, _dev, _host, check_bf16, check_fp32

pytestmark = pytest.mark.gpu


def _canary(shape_or_bytes, dtype, device="cuda"):
    if dtype == torch.uint8:
        return torch.full((shape_or_bytes,), 0xFF, dtype=torch.uint8, device=device)
    return torch.full(shape_or_bytes, float("nan"), dtype=dtype, device=device)


CASES = [
    # (B, h, d, grid, window, order, dtype): the launch path it exercises
    (1, 2, 128, (21, 4, 8), (21, 2, 4), "local_then_global", torch.bfloat16),   # fused two-pass kernel
    (1, 2, 128, (21, 4, 8), (21, 2, 4), "global_then_local", torch.bfloat16),
    (2, 1, 128, (5, 12, 20), (5, 2, 4), "local_only", torch.bfloat16),          # one pass, short kernel
    (1, 2, 128, (5, 7, 9), (5, 2, 4), "local_then_global", torch.bfloat16),     # padded grid
    (1, 2, 64, (5, 8, 8), (5, 2, 2), "local_then_global", torch.float32),       # CUDA-core kernels
    (1, 1, 128, (21, 8, 8), (21, 4, 4), "local_then_global", torch.bfloat16),   # 336-token windows: chunked
]


@pytest.mark.parametrize("B,h,d,grid,window,order,dtype", CASES)
def test_squad_outputs_and_workspaces_fully_written(B, h, d, grid, window, order, dtype):
    n = grid[0] * grid[1] * grid[2]
    x = make_inputs(B, h, n, d, dtype="bf16" if dtype == torch.bfloat16 else "fp32", with_dout=True, seed=99)
    q, k, v, do = (_dev(x[s], dtype) for s in ("q", "k", "v", "do"))
    prm = make_params(B, h, d, grid, window, order, dtype)
    o = _canary(q.shape, dtype)
    ws = _canary(squad_attn_fwd_workspace_bytes(prm), torch.uint8)
    squad_attn_fwd(q, k, v, grid, window, order, out=o, workspace=ws)
    dq, dk, dv = (_canary(q.shape, dtype) for _ in range(3))
    bws = _canary(squad_attn_bwd_workspace_bytes(prm), torch.uint8)
    squad_attn_bwd(q, k, v, o, do, ws, grid, window, order, dq=dq, dk=dk, dv=dv, workspace=bws)
    torch.cuda.synchronize()
    check = check_bf16 if dtype == torch.bfloat16 else check_fp32
    outs = [_host(t) for t in (o, dq, dk, dv)]
    refs = [orc.squad_attn_fwd(x["q"], x["k"], x["v"], grid, window, ORC_ORDER[order])]
    refs += list(orc.squad_attn_bwd(x["q"], x["k"], x["v"], x["do"], grid, window, ORC_ORDER[order]))
    for name, got, ref in zip(("o", "dq", "dk", "dv"), outs, refs):
        assert torch.isfinite(torch.from_numpy(got)).all(), f"{name}: unwritten or NaN-polluted elements"
        check(got, ref, name)


def test_kpass_outputs_and_workspaces_fully_written():
    B, h, d, grid, levels = 1, 2, 128, (2, 8, 12), [(2, 2), (2, 3), (2, 2)]
    n = 2 * 8 * 12
    x = make_inputs(B, h, n, d, dtype="bf16", with_dout=True, seed=98)
    q, k, v, do = (_dev(x[s], torch.bfloat16) for s in ("q", "k", "v", "do"))
    prm = make_kpass_params(B, h, d, grid, levels)
    lib = _lib.load()
    o = _canary(q.shape, torch.bfloat16)
    ws = _canary(lib.squad_kpass_fwd_workspace_bytes(ctypes.byref(prm)), torch.uint8)
    squad_kpass_fwd(q, k, v, grid, levels, out=o, workspace=ws)
    dq, dk, dv = (_canary(q.shape, torch.bfloat16) for _ in range(3))
    bws = _canary(lib.squad_kpass_bwd_workspace_bytes(ctypes.byref(prm)), torch.uint8)
    squad_kpass_bwd(q, k, v, o, do, ws, grid, levels, dq=dq, dk=dk, dv=dv, workspace=bws)
    torch.cuda.synchronize()
    refs = [orc.kpass_fwd(x["q"], x["k"], x["v"], grid, levels)]
    refs += list(orc.kpass_bwd(x["q"], x["k"], x["v"], x["do"], grid, levels))
    for name, t, ref in zip(("o", "dq", "dk", "dv"), (o, dq, dk, dv), refs):
        got = _host(t)
        assert torch.isfinite(torch.from_numpy(got)).all(), f"{name}: unwritten or NaN-polluted elements"
        check_bf16(got, ref, name)
