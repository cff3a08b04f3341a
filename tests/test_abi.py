"""The C-ABI library without a GPU: it loads, exports every symbol include/squad_attn.h declares, and
rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest
import torch

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import _lib, make_params
from sub_quadratic_two_squad_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"^SQUAD_API[^;(]*?(\w+)\s*\(", text, flags=re.M))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert {"squad_attn_fwd", "squad_attn_bwd", "full_attn_fwd"} <= names
    for name in names:
        assert hasattr(lib, name), name
    assert set(_lib.SIGNATURES) == names


def test_status_strings(lib):
    for s in range(5):
        assert lib.squad_status_string(s)
    assert lib.squad_status_string(99) == b"unknown status"
    assert lib.squad_attn_abi_version() >= 1


P5B = dict(B=1, h=24, d=128, grid=(21, 22, 40), window=(21, 2, 4))


def _p(**kw):
    a = dict(P5B)
    a.update(kw)
    return make_params(a["B"], a["h"], a["d"], a["grid"], a["window"], a.get("order", "local_then_global"),
                       a.get("dtype", 0), a.get("scale"))


def _fwd(lib, prm, ptr=16):
    p = ctypes.c_void_p(ptr)
    return lib.squad_attn_fwd(ctypes.byref(prm), p, p, p, p, ctypes.c_void_p(ptr * 16), None)


@pytest.mark.parametrize("kw,status", [
    (dict(window=(20, 2, 4)), _lib.SQUAD_ERR_UNSUPPORTED),      # window must span all frames
    (dict(window=(21, 0, 4)), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(window=(22, 2, 4)), _lib.SQUAD_ERR_INVALID_ARG),      # larger than the grid
    (dict(d=96), _lib.SQUAD_ERR_UNSUPPORTED),
    (dict(d=0), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(B=0), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(order=7), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(order=4), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(order=-1), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(dtype=5), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(scale=-1.0), _lib.SQUAD_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.SQUAD_ERR_INVALID_ARG),
])
def test_bad_params_rejected_before_launch(lib, kw, status):
    assert _fwd(lib, _p(**kw)) == status
    assert lib.squad_attn_fwd_workspace_bytes(ctypes.byref(_p(**kw))) == 0


def test_bad_pointers_rejected(lib):
    prm = _p()
    assert lib.squad_attn_fwd(ctypes.byref(prm), None, None, None, None, None, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert _fwd(lib, prm, ptr=8) == _lib.SQUAD_ERR_INVALID_ARG           # 16-byte alignment
    p16 = ctypes.c_void_p(16)
    assert lib.squad_attn_fwd(ctypes.byref(prm), p16, p16, p16, p16, ctypes.c_void_p(128), None) == \
        _lib.SQUAD_ERR_INVALID_ARG                                          # workspace 256-byte alignment
    assert lib.full_attn_fwd(ctypes.byref(prm), None, p16, p16, p16, None, None) == _lib.SQUAD_ERR_INVALID_ARG
    args = [p16] * 5 + [ctypes.c_void_p(256)] + [p16] * 3 + [ctypes.c_void_p(256), None]
    args[4] = None
    assert lib.squad_attn_bwd(ctypes.byref(prm), *args) == _lib.SQUAD_ERR_INVALID_ARG


@pytest.mark.parametrize("cfg", [
    (1, 24, 128, (21, 22, 40), (21, 2, 4)), (1, 12, 128, (21, 30, 52), (21, 2, 4)),
    (1, 24, 128, (21, 44, 80), (21, 4, 4)), (1, 4, 64, (5, 8, 8), (5, 2, 2))])
def test_flops_match_the_oracle_cost_model(lib, cfg):
    B, h, d, grid, window = cfg
    prm = make_params(B, h, d, grid, window)
    n, w = grid[0] * grid[1] * grid[2], window[0] * window[1] * window[2]
    assert lib.squad_attn_flops(ctypes.byref(prm)) == pytest.approx(orc.squad_flops(B, h, d, n, w), rel=1e-12)
    assert lib.full_attn_flops(ctypes.byref(prm)) == pytest.approx(orc.full_flops(B, h, d, n), rel=1e-12)


@pytest.mark.parametrize("cfg", [(1, 24, 128, (21, 22, 40), (21, 2, 4)), (1, 4, 64, (5, 8, 8), (5, 2, 2))])
def test_single_pass_orders_accepted_and_counted(lib, cfg):
    """local_only / global_only: one pass each, so their FLOPs are the two terms of the two-pass count."""
    B, h, d, grid, window = cfg
    n, w = grid[0] * grid[1] * grid[2], window[0] * window[1] * window[2]
    fl = {}
    for order in ("local_only", "global_only"):
        prm = make_params(B, h, d, grid, window, order)
        assert lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm)) > 0
        assert lib.squad_attn_bwd_workspace_bytes(ctypes.byref(prm)) > 0
        fl[order] = lib.squad_attn_flops(ctypes.byref(prm))
    assert fl["local_only"] == pytest.approx(4.0 * B * h * d * n * w, rel=1e-12)
    assert fl["local_only"] + fl["global_only"] == pytest.approx(orc.squad_flops(B, h, d, n, w), rel=1e-12)


@pytest.mark.parametrize("grid", [(21, 22, 40), (21, 30, 52), (21, 44, 80), (21, 60, 104), (13, 17, 29), (5, 8, 8),
                                  (1, 1, 1), (3, 1, 50), (7, 31, 2), (21, 23, 46), (5, 17, 17), (9, 31, 93), (21, 29, 29)])
def test_window_solver_matches_the_oracle(lib, grid):
    tw, hw, ww = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    assert lib.squad_window_solve(*grid, ctypes.byref(tw), ctypes.byref(hw), ctypes.byref(ww)) == _lib.SQUAD_OK
    assert (tw.value, hw.value, ww.value) == orc.window_solve(*grid)


def test_window_solver_rejects_bad_arguments(lib):
    x = ctypes.c_int()
    assert lib.squad_window_solve(0, 4, 4, ctypes.byref(x), ctypes.byref(x), ctypes.byref(x)) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_window_solve(4, 4, 4, None, ctypes.byref(x), ctypes.byref(x)) == _lib.SQUAD_ERR_INVALID_ARG


@pytest.mark.parametrize("window", [(21, 3, 4), (21, 2, 3), (21, 5, 7), (21, 22, 39)])
def test_non_dividing_windows_run_on_the_padded_grid(lib, window):
    """Accepted (reflect padding): the workspaces grow by the padded tensors and the FLOP count is the
    cost of the padded grid."""
    grid = (21, 22, 40)
    prm = make_params(1, 24, 128, grid, window)
    hp, wp = -(-22 // window[1]) * window[1], -(-40 // window[2]) * window[2]
    n_p, w = 21 * hp * wp, window[0] * window[1] * window[2]
    fwd = lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm))
    assert fwd >= 5 * 24 * n_p * 128 * 2 + 2 * 24 * n_p * 4   # O1 + padded q, k, v, o + LSEs
    assert lib.squad_attn_bwd_workspace_bytes(ctypes.byref(prm)) >= 3 * 24 * n_p * 128 * 4 + 4 * 24 * n_p * 128 * 2
    assert lib.squad_attn_flops(ctypes.byref(prm)) == pytest.approx(orc.squad_flops(1, 24, 128, n_p, w), rel=1e-12)


def test_wait_selftest_rejects_bad_arguments(lib):
    assert lib.squad_wait_selftest(None, 1000, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_wait_selftest(ctypes.c_void_p(2), 1000, None) == _lib.SQUAD_ERR_INVALID_ARG      # alignment
    assert lib.squad_wait_selftest(ctypes.c_void_p(256), 0, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_wait_selftest(ctypes.c_void_p(256), 2_000_000_000, None) == _lib.SQUAD_ERR_INVALID_ARG


def test_workspace_sizes(lib):
    prm = _p()
    n = 21 * 22 * 40
    fwd = lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm))
    assert fwd >= 24 * n * 128 * 2 + 2 * 24 * n * 4
    bwd = lib.squad_attn_bwd_workspace_bytes(ctypes.byref(prm))
    assert bwd >= 3 * 24 * n * 128 * 4 + 24 * n * 4


def test_size_limits(lib):
    """n = T H W up to 2^30 tokens and B h n below 2^31 rows are accepted (workspace sizes computed in
    64 bits); one past either limit is refused as unsupported before any launch."""
    # n = 2^30 exactly: grid (1, 2^15, 2^15), one head
    prm = make_params(1, 1, 128, (1, 1 << 15, 1 << 15), (1, 2, 4))
    fwd = lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm))
    assert fwd >= (1 << 30) * 128 * 2 + 2 * (1 << 30) * 4          # O1 (bf16) + two LSEs, no 32-bit wrap
    assert lib.squad_attn_bwd_workspace_bytes(ctypes.byref(prm)) >= 3 * (1 << 30) * 128 * 4
    # n = 2^30 + one row of tokens: refused
    prm = make_params(1, 1, 128, (1, (1 << 15) + 1, 1 << 15), (1, 1, 4))
    assert lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm)) == 0
    assert _fwd(lib, prm) == _lib.SQUAD_ERR_UNSUPPORTED
    # h = 2 heads of 2^30 tokens are 2^31 rows, one past the limit
    prm = make_params(1, 2, 128, (1, 1 << 15, 1 << 15), (1, 2, 4))
    assert lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm)) == 0
    assert _fwd(lib, prm) == _lib.SQUAD_ERR_UNSUPPORTED
    # the padded grid counts: 32767 x 32769 = 2^30 - 1 tokens is accepted as it is, but a window of
    # height 2 pads it to 32768 x 32769 > 2^30 tokens and is refused
    grid = (1, (1 << 15) - 1, (1 << 15) + 1)
    assert lib.squad_attn_fwd_workspace_bytes(ctypes.byref(make_params(1, 1, 128, grid, (1, 1, 1)))) > 0
    prm = make_params(1, 1, 128, grid, (1, 2, 1))
    assert lib.squad_attn_fwd_workspace_bytes(ctypes.byref(prm)) == 0
    assert _fwd(lib, prm) == _lib.SQUAD_ERR_UNSUPPORTED


def test_host_forward_rejects_bad_arguments_before_enqueueing(lib):
    prm = _p()
    assert lib.squad_attn_fwd_host_workspace_bytes(ctypes.byref(prm), 4) > 0
    assert lib.squad_attn_fwd_host_workspace_bytes(ctypes.byref(prm), 0) == 0
    assert lib.squad_attn_fwd_host_workspace_bytes(ctypes.byref(prm), 25) == 0    # more runs than heads
    assert lib.squad_attn_fwd_host_workspace_bytes(ctypes.byref(prm), 65) == 0
    # a run's workspace is that of its heads only
    one = lib.squad_attn_fwd_host_workspace_bytes(ctypes.byref(prm), 24)
    assert one == lib.squad_attn_fwd_workspace_bytes(ctypes.byref(_p(h=1)))
    host, dev, ws = ctypes.c_void_p(4096), ctypes.c_void_p(16), ctypes.c_void_p(256)

    def call(prm=prm, groups=4, h=host, d=dev, w=ws):
        return lib.squad_attn_fwd_host(ctypes.byref(prm), h, h, h, h, d, d, d, d, w, groups, None, None, None)

    assert call(groups=0) == _lib.SQUAD_ERR_INVALID_ARG
    assert call(prm=_p(window=(20, 2, 4))) == _lib.SQUAD_ERR_INVALID_ARG
    assert call(h=ctypes.c_void_p(0)) == _lib.SQUAD_ERR_INVALID_ARG
    assert call(d=ctypes.c_void_p(8)) == _lib.SQUAD_ERR_INVALID_ARG             # not 16-byte aligned
    assert call(w=ctypes.c_void_p(128)) == _lib.SQUAD_ERR_INVALID_ARG           # not 256-byte aligned


@pytest.mark.parametrize("grid,window,order,dtype,d,expect", [
    ((21, 22, 40), (21, 2, 4), "local_then_global", 0, 128, (1, 1)),   # 168- and 110-token sequences: whole
    ((21, 44, 80), (21, 4, 4), "local_then_global", 0, 128, (2, 2)),   # 336-token windows, 220-token slots
    ((21, 8, 8), (21, 4, 4), "global_then_local", 0, 128, (1, 2)),     # 4-token slots, 336-token windows
    ((5, 48, 48), (5, 2, 2), "global_only", 0, 128, (2, 0)),           # 576-token slot sequences
    ((21, 22, 40), (21, 3, 4), "local_then_global", 0, 128, (2, 1)),   # padded to 21x24x40: 252-token windows
    ((21, 22, 40), (21, 2, 4), "local_then_global", 0, 64, (3, 3)),    # d = 64: CUDA cores
    ((5, 8, 8), (5, 2, 2), "local_then_global", 1, 128, (3, 3)),       # fp32: CUDA cores
])
def test_backward_kernel_selection(lib, grid, window, order, dtype, d, expect):
    """Which backward kernel each pass takes is decided on the host from the parameters alone."""
    ks = (ctypes.c_int * 2)()
    prm = make_params(1, 2, d, grid, window, order, dtype)
    assert lib.squad_attn_bwd_kernels(ctypes.byref(prm), ks) == _lib.SQUAD_OK
    assert (ks[0], ks[1]) == expect
    assert lib.squad_attn_bwd_kernels(ctypes.byref(prm), None) == _lib.SQUAD_ERR_INVALID_ARG
    assert lib.squad_attn_bwd_kernels(ctypes.byref(make_params(1, 2, d, grid, (4, 2, 4), order, dtype)), ks) != 0


def test_bwd_workspace_carries_pds_scratch_only_where_the_whole_sequence_kernel_needs_it():
    """The whole-sequence backward (129-208 tokens) keeps each sequence's P and dS in one scratch slot per
    resident CTA (160 slots of 8 panels of the sequence rounded to 16 rows x 128 bytes); other passes
    need none. Same n, so the rest of the workspace is the same size."""
    lib = _lib.load()

    def ws(window, order="local_then_global", dtype=torch.bfloat16):
        prm = make_params(1, 24, 128, (21, 22, 40), window, order, dtype)
        return lib.squad_attn_bwd_workspace_bytes(ctypes.byref(prm))

    slot = 8 * 176 * 128                                   # 168-token windows: 176-row panels
    base = ws((21, 1, 4))                                  # 84-token windows, 220-token slots: no scratch
    assert ws((21, 2, 4)) == base + 160 * slot             # local pass of 168 tokens
    assert ws((21, 2, 4), "local_only") == base + 160 * slot
    assert ws((21, 2, 4), "global_only") == base           # 110-token slots: the one-tile kernel
    assert ws((21, 2, 4), dtype=torch.float32) == ws((21, 1, 4), dtype=torch.float32)   # CUDA-core kernels


def test_seqpar_reorder_rejects_bad_arguments(lib):
    """Argument errors come back before anything is launched (no GPU needed)."""
    prm = make_params(1, 2, 128, (4, 6, 5), (4, 1, 1))
    a, b, c = ctypes.c_void_p(4096), ctypes.c_void_p(8192), ctypes.c_void_p(12288)
    bad = ctypes.c_void_p(4104)   # 8-byte aligned only
    reorder = lib.squad_seqpar_reorder
    assert reorder(None, 2, 0, 2, a, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert reorder(ctypes.byref(prm), 0, 0, 2, a, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG     # R < 1
    assert reorder(ctypes.byref(prm), 3, 0, 2, a, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG     # H % R (T = 4)
    assert reorder(ctypes.byref(prm), 4, 0, 2, a, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG     # T % R ok, H % R
    assert reorder(ctypes.byref(prm), 2, 0, 3, a, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG     # layout
    assert reorder(ctypes.byref(prm), 2, -1, 2, a, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert reorder(ctypes.byref(prm), 2, 0, 2, a, None, a, None) == _lib.SQUAD_ERR_INVALID_ARG     # y == x
    assert reorder(ctypes.byref(prm), 2, 0, 2, a, b, b, None) == _lib.SQUAD_ERR_INVALID_ARG        # y == add
    assert reorder(ctypes.byref(prm), 2, 0, 2, bad, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG   # alignment
    assert reorder(ctypes.byref(prm), 2, 0, 2, a, bad, c, None) == _lib.SQUAD_ERR_INVALID_ARG
    assert reorder(ctypes.byref(prm), 2, 0, 2, a, None, None, None) == _lib.SQUAD_ERR_INVALID_ARG
    odd = make_params(1, 2, 96, (4, 6, 5), (4, 1, 1))
    assert reorder(ctypes.byref(odd), 2, 0, 2, a, None, b, None) == _lib.SQUAD_ERR_INVALID_ARG     # d
