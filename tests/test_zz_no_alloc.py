"""squad_attn_fwd_noalloc: the forward for callers that cannot allocate device memory (a framework that
owns the whole memory pool, latency-critical loops, plugins that only see the tensors). Its scratch is
a fixed device array inside the library; these tests check that it gives exactly the results of the
workspace entry point (the same kernels run on the same inputs, so bit for bit), call after call, that
those results meet the oracle's tolerance, and that it refuses problems larger than that array.

Collected last on purpose: run after the rest of the suite, and alone in a fresh process, it must
pass either way.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import _lib, make_params, squad_attn_fwd, squad_attn_fwd_workspace_bytes
from sub_quadratic_two_squad_b200.build import build
from sub_quadratic_two_squad_b200.inputs import make_inputs


def _noalloc(lib, prm, q, k, v, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return lib.squad_attn_fwd_noalloc(ctypes.byref(prm), ptr(q), ptr(k), ptr(v), ptr(out), stream)


def test_noalloc_rejects_problems_beyond_its_scratch():
    build()
    lib = _lib.load()
    big = make_params(1, 40, 128, (21, 44, 80), (21, 4, 4))   # needs far more than the fixed scratch
    assert squad_attn_fwd_workspace_bytes(big) > _lib.SQUAD_NOALLOC_MAX_WORKSPACE_BYTES
    p16 = ctypes.c_void_p(16)
    assert lib.squad_attn_fwd_noalloc(ctypes.byref(big), p16, p16, p16, p16, None) == _lib.SQUAD_ERR_UNSUPPORTED


# (B, h, d, grid, window, dtype, oracle heads): the Wan-2.2-5B block (fused two-pass kernel), a small
# batched grid, a grid the window does not divide (reflect padding: the scratch also holds the padded
# q, k, v and output), and the fp32 CUDA-core path.
CASES = [
    (1, 24, 128, (21, 22, 40), (21, 2, 4), torch.bfloat16, (0, 23)),
    (2, 3, 128, (21, 4, 8), (21, 2, 4), torch.bfloat16, (0, 1, 2)),
    (1, 4, 128, (21, 5, 9), (21, 2, 4), torch.bfloat16, (0, 3)),
    (1, 4, 64, (5, 8, 8), (5, 2, 2), torch.float32, (0, 1, 2, 3)),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,h,d,grid,window,dtype,heads", CASES)
def test_noalloc_matches_workspace_forward_on_two_calls(B, h, d, grid, window, dtype, heads):
    build()
    lib = _lib.load()
    n = grid[0] * grid[1] * grid[2]
    prm = make_params(B, h, d, grid, window, dtype=dtype)
    assert squad_attn_fwd_workspace_bytes(prm) <= _lib.SQUAD_NOALLOC_MAX_WORKSPACE_BYTES
    kind = "bf16" if dtype == torch.bfloat16 else "fp32"
    for seed in (11, 12):   # two calls in a row through the same scratch
        x = make_inputs(B, h, n, d, dtype=kind, heavy_tail=True, seed=seed)
        q, k, v = (torch.from_numpy(x[s]).to("cuda", dtype) for s in "qkv")
        ref, _ = squad_attn_fwd(q, k, v, grid, window)
        out = torch.full_like(q, float("nan"))
        assert _noalloc(lib, prm, q, k, v, out) == _lib.SQUAD_OK
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical bits
        assert torch.equal(out.view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                           ref.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))
        a = out.double().cpu().numpy()
        for hh in heads:
            sl = (slice(None), slice(hh, hh + 1))
            r = orc.squad_attn_fwd(x["q"][sl], x["k"][sl], x["v"][sl], grid, window)
            err, scale = np.abs(a[sl] - r), np.abs(r).max()
            assert np.isfinite(a[sl]).all()
            if dtype == torch.bfloat16:
                assert err.max() <= 1e-2 * scale and err.mean() <= 1e-3 * scale
            else:
                assert err.max() <= 1e-5 * scale
