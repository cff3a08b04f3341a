"""k composed nested-window passes on the CUDA path vs the fp64 oracle, element by element, on the same
seeded inputs (needs a B200). Tolerances as for the two-pass method: fp32 normwise <= 1e-5; bf16 max
abs <= 1e-2 max|ref| and mean abs <= 1e-3 max|ref|, for o and for dq, dk, dv separately."""
import pytest
import torch

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import squad_kpass_bwd, squad_kpass_fwd, squad_kpass_status
from sub_quadratic_two_squad_b200.inputs import make_inputs
from test_gpu_parity import _dev, _host, check_bf16, check_fp32

pytestmark = pytest.mark.gpu

BF16, FP32 = torch.bfloat16, torch.float32
ORC = {"forward": orc.KPASS_FORWARD, "reverse": orc.KPASS_REVERSE}

CASES = [
    # (B, h, d, grid, levels, dtype): what it exercises
    (1, 2, 128, (2, 8, 12), [(2, 2), (2, 3), (2, 2)], BF16),        # k = 3 on the tensor cores; the middle
                                                                   # pass adds to the fp32 dQ/dK shares
    (1, 2, 64, (2, 8, 12), [(2, 2), (2, 3), (2, 2)], FP32),         # k = 3 on the CUDA cores (exact path)
    (1, 2, 128, (21, 8, 16), [(2, 4), (2, 2), (2, 2)], BF16),       # 168-token windows, 4-token outer levels
    (2, 1, 128, (1, 16, 16), [(2, 2), (2, 2), (2, 2), (2, 2)], BF16),  # k = 4, T = 1
    (1, 2, 128, (3, 8, 8), [(8, 8)], BF16),                         # k = 1: full attention over 192 tokens
    (1, 3, 128, (21, 4, 8), [(2, 4), (2, 2)], BF16),                # k = 2: the two-pass problem
    (1, 1, 128, (2, 20, 40), [(2, 2), (10, 10), (1, 2)], BF16),     # a 100-token middle level, 2-token outer
    (1, 2, 128, (21, 16, 16), [(4, 4), (2, 2), (2, 2)], BF16),      # 336-token first level: chunked backward
    (1, 2, 128, (2, 32, 32), [(2, 2), (16, 16)], BF16),             # 256-token outer level: chunked backward
]


@pytest.mark.parametrize("order", ["forward", "reverse"])
@pytest.mark.parametrize("B,h,d,grid,levels,dtype", CASES)
def test_kpass_forward_and_backward(B, h, d, grid, levels, dtype, order):
    n = grid[0] * grid[1] * grid[2]
    x = make_inputs(B, h, n, d, dtype="bf16" if dtype == BF16 else "fp32", with_dout=True, seed=4321)
    q, k, v, do = (_dev(x[s], dtype) for s in ("q", "k", "v", "do"))
    o, ws = squad_kpass_fwd(q, k, v, grid, levels, order)
    assert squad_kpass_status(ws, q, grid, levels, order) == 0
    check = check_bf16 if dtype == BF16 else check_fp32
    check(_host(o), orc.kpass_fwd(x["q"], x["k"], x["v"], grid, levels, ORC[order]), "o")
    dq, dk, dv = squad_kpass_bwd(q, k, v, o, do, ws, grid, levels, order)
    torch.cuda.synchronize()
    refs = orc.kpass_bwd(x["q"], x["k"], x["v"], x["do"], grid, levels, ORC[order])
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        check(_host(got), ref, name)
