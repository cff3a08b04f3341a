"""The k-pass entry points without a GPU: the library's own level-to-pass mapping (squad_kpass_pass_params)
reproduces the oracle's nested-window definition when each reported single-pass problem is run by the
oracle on the reshaped buffers; argument checks, workspace sizes and FLOP counts."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import _lib, make_kpass_params, squad_kpass_pass_params
from sub_quadratic_two_squad_b200.api import SquadError
from sub_quadratic_two_squad_b200.build import build

ORDERS = {"forward": orc.KPASS_FORWARD, "reverse": orc.KPASS_REVERSE}
SINGLE = {_lib.SQUAD_LOCAL_ONLY: orc.LOCAL_ONLY, _lib.SQUAD_GLOBAL_ONLY: orc.GLOBAL_ONLY}


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _library_passes(B, h, d, grid, levels, order):
    """The single-pass problems the library runs, in execution order: (shape, grid, window, order)."""
    prm = make_kpass_params(B, h, d, grid, levels, order, dtype=_lib.SQUAD_FP32)
    idx = list(range(len(levels)))
    seq = idx if order == "forward" else idx[::-1]
    out = []
    for lv in seq:
        s = squad_kpass_pass_params(prm, lv)
        assert (s.d, s.dtype) == (d, _lib.SQUAD_FP32)
        out.append(((s.B, s.h, s.T * s.H * s.W, s.d), (s.T, s.H, s.W), (s.tw, s.hw, s.ww), SINGLE[s.order]))
    return out


CASES = [
    ((2, 8, 12), [(2, 2), (2, 3), (2, 2)]),
    ((3, 4, 6), [(1, 3), (2, 1), (2, 2)]),
    ((1, 12, 8), [(3, 2), (2, 2), (2, 2)]),
    ((2, 4, 8), [(2, 2), (2, 4)]),
    ((2, 4, 6), [(4, 6)]),
    ((1, 8, 8), [(2, 2), (2, 1), (1, 2), (2, 2)]),
]


@pytest.mark.parametrize("order", ["forward", "reverse"])
@pytest.mark.parametrize("grid,levels", CASES)
def test_library_mapping_reproduces_the_definition(lib, order, grid, levels):
    """Run each pass the library reports, with the oracle's single-pass functions on the same memory
    reshaped to that pass's [B', h', n', d], chaining values and summing gradient shares; the result
    is the oracle's k-pass forward and backward."""
    B, h, d = 2, 2, 64
    n = grid[0] * grid[1] * grid[2]
    q, k, v, do = (_rand((B, h, n, d), s) for s in (1, 2, 3, 4))
    passes = _library_passes(B, h, d, grid, levels, order)

    x, values = v, []
    for shape, g, w, o in passes:
        values.append(x)
        x = orc.squad_attn_fwd(q.reshape(shape), k.reshape(shape), x.reshape(shape), g, w, o).reshape(q.shape)
    np.testing.assert_allclose(x, orc.kpass_fwd(q, k, v, grid, levels, ORDERS[order]), rtol=0, atol=1e-12)

    dq, dk, g_in = np.zeros_like(q), np.zeros_like(k), do
    for (shape, g, w, o), val in zip(passes[::-1], values[::-1]):
        a, b, c = orc.squad_attn_bwd(q.reshape(shape), k.reshape(shape), val.reshape(shape), g_in.reshape(shape),
                                     g, w, o)
        dq += a.reshape(q.shape)
        dk += b.reshape(q.shape)
        g_in = c.reshape(q.shape)
    for got, ref in zip((dq, dk, g_in), orc.kpass_bwd(q, k, v, do, grid, levels, ORDERS[order])):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11)


def test_two_levels_are_the_two_pass_problem(lib):
    """k = 2: level 0 is the local pass with window (T, h_1, w_1); level 1 the global pass over the same
    windows (heads and frames folded into the batch); the FLOPs are the two-pass count."""
    grid, levels = (21, 22, 40), [(2, 4), (11, 10)]
    prm = make_kpass_params(1, 24, 128, grid, levels)
    s0, s1 = squad_kpass_pass_params(prm, 0), squad_kpass_pass_params(prm, 1)
    assert (s0.B, s0.h, s0.T, s0.H, s0.W, s0.tw, s0.hw, s0.ww, s0.order) == \
        (1, 24, 21, 22, 40, 21, 2, 4, _lib.SQUAD_LOCAL_ONLY)
    assert (s1.B, s1.h, s1.T, s1.H, s1.W, s1.tw, s1.hw, s1.ww, s1.order) == \
        (24 * 21, 1, 1, 22, 40, 1, 2, 4, _lib.SQUAD_GLOBAL_ONLY)
    assert lib.squad_kpass_flops(ctypes.byref(prm)) == pytest.approx(orc.squad_flops(1, 24, 128, 18480, 168), rel=1e-12)


@pytest.mark.parametrize("grid,levels", CASES + [((21, 44, 80), [(2, 4), (2, 2), (11, 10)])])
def test_flops_match_the_oracle(lib, grid, levels):
    prm = make_kpass_params(1, 3, 64, grid, levels)
    assert lib.squad_kpass_flops(ctypes.byref(prm)) == pytest.approx(orc.kpass_flops(1, 3, 64, grid, levels),
                                                                     rel=1e-12)


def _align(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("dtype,eb", [(_lib.SQUAD_BF16, 2), (_lib.SQUAD_FP32, 4)])
@pytest.mark.parametrize("levels", [[(4, 6)], [(2, 2), (2, 3)], [(2, 2), (2, 3), (1, 2)], [(2, 1), (1, 3), (2, 2), (1, 2)]])
def test_workspace_sizes(lib, dtype, eb, levels):
    grid = (3, int(np.prod([a for a, _ in levels])), int(np.prod([b for _, b in levels])))
    B, h, d = 2, 3, 64
    prm = make_kpass_params(B, h, d, grid, levels, dtype=dtype)
    k = len(levels)
    bhn = B * h * grid[0] * grid[1] * grid[2]
    t, f, l = _align(bhn * d * eb), _align(bhn * d * 4), _align(bhn * 4)
    assert lib.squad_kpass_fwd_workspace_bytes(ctypes.byref(prm)) == 256 + (k - 1) * t + k * l
    assert lib.squad_kpass_bwd_workspace_bytes(ctypes.byref(prm)) == 256 + 2 * f + l + min(k - 1, 2) * t


def _kp(**kw):
    a = dict(B=1, h=2, d=128, grid=(2, 8, 12), levels=[(2, 2), (2, 3), (2, 2)], order="forward", dtype=0)
    a.update(kw)
    return make_kpass_params(a["B"], a["h"], a["d"], a["grid"], a["levels"], a["order"], a["dtype"], a.get("scale"))


@pytest.mark.parametrize("kw,status", [
    (dict(levels=[(2, 2), (3, 3), (2, 2)]), _lib.SQUAD_ERR_INVALID_ARG),           # does not factor H x W
    (dict(levels=[(2, 2), (2, 3)]), _lib.SQUAD_ERR_INVALID_ARG),                   # product short of the grid
    (dict(levels=[(2, 2), (2, 3), (2, 0)]), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(order=2), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(d=96), _lib.SQUAD_ERR_UNSUPPORTED),
    (dict(B=0), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(scale=-2.0), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(grid=(2, 8, 12), levels=[(2, 2), (1, 1), (4, 6)]), _lib.SQUAD_ERR_UNSUPPORTED),   # a one-token pass
    (dict(grid=(1, 8, 12), levels=[(1, 1), (8, 12)]), _lib.SQUAD_ERR_UNSUPPORTED),
])
def test_bad_params_rejected_before_launch(lib, kw, status):
    prm = _kp(**kw)
    p16, p256 = ctypes.c_void_p(16), ctypes.c_void_p(256)
    assert lib.squad_kpass_fwd(ctypes.byref(prm), p16, p16, p16, p16, p256, None) == status
    assert lib.squad_kpass_fwd_workspace_bytes(ctypes.byref(prm)) == 0
    assert lib.squad_kpass_bwd_workspace_bytes(ctypes.byref(prm)) == 0
    assert lib.squad_kpass_flops(ctypes.byref(prm)) == 0.0
    out = _lib.SquadParams()
    assert lib.squad_kpass_pass_params(ctypes.byref(prm), 0, ctypes.byref(out)) == status


def test_k_out_of_range_and_bad_level_index(lib):
    prm = _kp()
    out = _lib.SquadParams()
    for lv in (-1, 3):
        assert lib.squad_kpass_pass_params(ctypes.byref(prm), lv, ctypes.byref(out)) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_kpass_pass_params(ctypes.byref(prm), 0, None) == _lib.SQUAD_ERR_INVALID_ARG
    for k in (0, _lib.SQUAD_KPASS_MAX_LEVELS + 1):
        prm.k = k
        assert lib.squad_kpass_fwd_workspace_bytes(ctypes.byref(prm)) == 0
    with pytest.raises(ValueError):
        make_kpass_params(1, 1, 64, (1, 32, 32), [(2, 2)] * 5)
    with pytest.raises(SquadError):
        squad_kpass_pass_params(_kp(levels=[(2, 2), (3, 3), (2, 2)]), 0)


def test_bad_pointers_rejected(lib):
    prm = _kp()
    p16, p8, p128, p256 = (ctypes.c_void_p(x) for x in (16, 8, 128, 256))
    assert lib.squad_kpass_fwd(ctypes.byref(prm), None, p16, p16, p16, p256, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_kpass_fwd(ctypes.byref(prm), p8, p16, p16, p16, p256, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_kpass_fwd(ctypes.byref(prm), p16, p16, p16, p16, p128, None) == _lib.SQUAD_ERR_INVALID_ARG
    args = [p16] * 5 + [p256] + [p16] * 3 + [p256, None]
    args[4] = None
    assert lib.squad_kpass_bwd(ctypes.byref(prm), *args) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_kpass_status(ctypes.byref(prm), p128, None) == _lib.SQUAD_ERR_INVALID_ARG


def _checker_tables(exe, s):
    r = subprocess.run([exe, str(s.B), str(s.h), str(s.T), str(s.H), str(s.W), str(s.hw), str(s.ww)],
                       capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]
    tables = {0: [], 1: []}
    for line in r.stdout.splitlines():
        if line.startswith("seq "):
            head, toks = line.split(":")
            tables[int(head.split()[1])].append(frozenset(int(t) for t in toks.split()))
    return tables


@pytest.mark.parametrize("grid,levels", CASES)
def test_kernel_boxes_of_each_view_are_the_level_groups(lib, geometry_checker, grid, levels):
    """The kernels' own box arithmetic (a host build of csrc/geometry.cuh) on each level's reported view:
    every token is covered once per pass, and the sequences of the view's first head are the oracle's
    level groups that lie in the first n' tokens of the buffer (the view's first head)."""
    B, h = 2, 2
    prm = make_kpass_params(B, h, 128, grid, levels)
    for lv in range(len(levels)):
        s = squad_kpass_pass_params(prm, lv)
        kind = 0 if s.order == _lib.SQUAD_LOCAL_ONLY else 1
        got = set(_checker_tables(geometry_checker, s)[kind])
        n_view = s.T * s.H * s.W
        ref = {frozenset(int(t) for t in g) for g in orc.level_groups(grid, levels, lv) if g.max() < n_view}
        assert got == ref


def test_chain_schedule(tmp_path):
    """A host build of csrc/kpass_plan.h: the forward and backward schedules the library executes pass
    values, log-sum-exps and value gradients along the chain (tests/kpass_check.cpp)."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = str(tmp_path / "kpass_check")
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(root, "include"),
                    "-I", os.path.join(root, "sub_quadratic_two_squad_b200", "csrc"),
                    os.path.join(root, "tests", "kpass_check.cpp"), "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:]
    bwd3 = [l for l in r.stdout.splitlines() if l.startswith("bwd k=3 order=0")]
    assert [l.split()[6:8] for l in bwd3] == [["g_in=-3", "g_out=0"], ["g_in=0", "g_out=1"], ["g_in=1", "g_out=-4"]]
