"""squad_attn_fwd_noalloc: the forward for callers that cannot allocate device memory (a framework that
owns the whole memory pool, latency-critical loops, plugins that only see the tensors). Its scratch is
a fixed device array inside the library; these tests check that it gives the results of the
workspace entry point, call after call, and that it refuses problems larger than that array.

Collected last on purpose: run after the rest of the suite, and alone in a fresh process, it must
pass either way.
"""
import ctypes

import numpy as np
import pytest
import torch

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


@pytest.mark.gpu
@pytest.mark.parametrize("B,h,grid,window", [(1, 24, (21, 22, 40), (21, 2, 4)), (2, 3, (21, 4, 8), (21, 2, 4))])
def test_noalloc_matches_workspace_forward_on_two_calls(B, h, grid, window):
    build()
    lib = _lib.load()
    n = grid[0] * grid[1] * grid[2]
    prm = make_params(B, h, 128, grid, window)
    assert squad_attn_fwd_workspace_bytes(prm) <= _lib.SQUAD_NOALLOC_MAX_WORKSPACE_BYTES
    for seed in (11, 12):   # two calls in a row through the same scratch
        x = make_inputs(B, h, n, 128, dtype="bf16", heavy_tail=True, seed=seed)
        q, k, v = (torch.from_numpy(x[s]).to("cuda", torch.bfloat16) for s in "qkv")
        ref, _ = squad_attn_fwd(q, k, v, grid, window)
        out = torch.full_like(q, float("nan"))
        assert _noalloc(lib, prm, q, k, v, out) == _lib.SQUAD_OK
        torch.cuda.synchronize()
        a, r = out.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.isfinite(a).all()
        err, scale = np.abs(a - r), np.abs(r).max()
        assert err.max() <= 1e-2 * scale and err.mean() <= 1e-3 * scale
