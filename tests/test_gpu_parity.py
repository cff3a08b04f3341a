"""CUDA path vs the fp64 oracle, element by element, on the same seeded inputs (needs a B200).

Tolerances (the acceptance bounds of this library against the fp64 oracle):
  fp32 mode: normwise max |gpu - ref| / max |ref| <= 1e-5.
  bf16 mode (fp32 accumulation): max |gpu - ref| <= 1e-2 * max |ref| and mean |gpu - ref| <= 1e-3 * max |ref|,
  applied to O, and to dQ, dK, dV separately.
The bf16 oracle runs on the bf16-rounded inputs (upcast to fp64), so only the kernel's own rounding
(P and the pass-1 output in bf16, fp32 accumulation) is measured.
"""
import numpy as np
import pytest
import torch

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import (full_attn_fwd, squad_attn_bwd, squad_attn_bwd_kernels, squad_attn_fwd,
                                          squad_attn_fwd_status)
from sub_quadratic_two_squad_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

LG, GL = "local_then_global", "global_then_local"
LO, GO = "local_only", "global_only"
ORC_ORDER = {LG: orc.LOCAL_THEN_GLOBAL, GL: orc.GLOBAL_THEN_LOCAL, LO: orc.LOCAL_ONLY, GO: orc.GLOBAL_ONLY}


def _dev(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


def check_bf16(gpu, ref, what=""):
    err = np.abs(gpu - ref)
    scale = np.abs(ref).max()
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert err.max() <= 1e-2 * scale, f"{what}: max abs err {err.max():.3e} > 1e-2 * {scale:.3e}"
    assert err.mean() <= 1e-3 * scale, f"{what}: mean abs err {err.mean():.3e} > 1e-3 * {scale:.3e}"


def check_fp32(gpu, ref, what=""):
    rel = np.abs(gpu - ref).max() / np.abs(ref).max()
    assert rel <= 1e-5, f"{what}: normwise relative error {rel:.3e} > 1e-5"


def run_fwd(B, h, d, grid, window, order, dtype, heavy_tail=False, heads=None, seed=1234):
    n = grid[0] * grid[1] * grid[2]
    x = make_inputs(B, h, n, d, dtype="bf16" if dtype == torch.bfloat16 else "fp32", heavy_tail=heavy_tail, seed=seed)
    q, k, v = (_dev(x[s], dtype) for s in "qkv")
    out, ws = squad_attn_fwd(q, k, v, grid, window, order)
    assert squad_attn_fwd_status(ws, q, grid, window, order) == 0
    gpu = _host(out)
    heads = range(h) if heads is None else heads
    for hh in heads:
        sl = (slice(None), slice(hh, hh + 1))
        ref = orc.squad_attn_fwd(x["q"][sl], x["k"][sl], x["v"][sl], grid, window, ORC_ORDER[order])
        (check_bf16 if dtype == torch.bfloat16 else check_fp32)(gpu[sl], ref, f"head {hh}")
    return x, gpu


# ------------------------------------------------------------------------------------------------
# tiny oracle case (fp32) and the single-window special case
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("order", [LG, GL])
def test_tiny_fp32(order):
    run_fwd(1, 4, 64, (5, 8, 8), (5, 2, 2), order, torch.float32)


def test_tiny_fp32_single_window_equals_full_attention():
    x, gpu = run_fwd(1, 4, 64, (5, 8, 8), (5, 8, 8), LG, torch.float32)
    ref, _ = orc.full_attn_fwd(x["q"], x["k"], x["v"])
    check_fp32(gpu, ref)


# ------------------------------------------------------------------------------------------------
# tensor-core path: shapes that exercise every chunking case at small n
# ------------------------------------------------------------------------------------------------

SMALL_BF16 = [
    # (B, h, grid, window): what it exercises
    (2, 3, (21, 4, 8), (21, 2, 4)),     # local 168 = 128 + 40 rows (shared K/V pair); global 4-token slots
    (1, 2, (5, 12, 20), (5, 2, 4)),     # single-chunk sequences in both passes (40 and 30 tokens)
    (1, 1, (21, 8, 8), (21, 4, 4)),     # local 336 = 128 + 128 + 80 rows: mixed shared/unshared pairs
    (1, 3, (3, 30, 52), (3, 2, 4)),     # global 195 = 117 + 78 rows (line-aligned chunks), odd tile count
    (1, 2, (1, 16, 16), (1, 4, 4)),     # T = 1
    (1, 2, (2, 8, 8), (2, 8, 8)),       # one window: local 128 rows exactly, global sequences of 1 token
    (1, 1, (7, 6, 10), (7, 3, 5)),      # rows not a multiple of 16 anywhere (105-token windows, 4-token slots)
]


@pytest.mark.parametrize("B,h,grid,window", SMALL_BF16)
@pytest.mark.parametrize("order", [LG, GL])
def test_small_bf16(B, h, grid, window, order):
    run_fwd(B, h, 128, grid, window, order, torch.bfloat16, heavy_tail=True)


def test_single_window_bf16_equals_full_attention():
    x, gpu = run_fwd(1, 2, 128, (2, 8, 8), (2, 8, 8), LG, torch.bfloat16)
    ref, _ = orc.full_attn_fwd(x["q"], x["k"], x["v"])
    check_bf16(gpu, ref)


def test_bf16_d64_cuda_core_path():
    run_fwd(1, 2, 64, (5, 8, 8), (5, 2, 2), LG, torch.bfloat16)


# ------------------------------------------------------------------------------------------------
# the Wan-shaped workloads at full size
# ------------------------------------------------------------------------------------------------

def test_wan22_5b_forward():
    run_fwd(1, 24, 128, (21, 22, 40), (21, 2, 4), LG, torch.bfloat16, heavy_tail=True)


@pytest.mark.parametrize("order", [LG, GL])
def test_wan21_1p3b_forward_both_orders(order):
    run_fwd(1, 12, 128, (21, 30, 52), (21, 2, 4), order, torch.bfloat16, heavy_tail=True)


def test_hires_5b_forward_sampled_heads():
    run_fwd(1, 24, 128, (21, 44, 80), (21, 4, 4), LG, torch.bfloat16, heavy_tail=True, heads=[0, 11, 23])


# ------------------------------------------------------------------------------------------------
# full attention
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("n,dtype", [(1000, torch.bfloat16), (300, torch.float32), (128, torch.bfloat16)])
def test_full_attention_small(n, dtype):
    d = 128 if dtype == torch.bfloat16 else 64
    x = make_inputs(2, 2, n, d, dtype="bf16" if dtype == torch.bfloat16 else "fp32", heavy_tail=True)
    q, k, v = (_dev(x[s], dtype) for s in "qkv")
    lse = torch.empty((2, 2, n), dtype=torch.float32, device="cuda")
    out = full_attn_fwd(q, k, v, lse=lse)
    ref, ref_lse = orc.full_attn_fwd(x["q"], x["k"], x["v"])
    (check_bf16 if dtype == torch.bfloat16 else check_fp32)(_host(out), ref)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=1e-3 if dtype == torch.bfloat16 else 1e-5)


@pytest.mark.parametrize("case", ["short_kernel", "chunked_local", "full"])
def test_late_large_keys_raise_the_softmax_reference(case):
    """Keys late in each sequence scaled by 64 (a power of two, exact in bf16), so that later columns'
    scores exceed the first chunk's maximum by far more than the kernels' headroom: the one-pass
    softmax must raise its reference, rescale what it already wrote and take the chunk again.
    168-token windows (short kernel, third chunk), 336-token windows (chunked kernel, second and third
    key blocks) and full attention over 384 tokens (third key block, the output rescaled too)."""
    if case == "full":
        n = 384
        x = make_inputs(1, 2, n, 128, dtype="bf16")
        x["k"][:, :, 200:, :] *= 64.0
        q, k, v = (_dev(x[s], torch.bfloat16) for s in "qkv")
        lse = torch.empty((1, 2, n), dtype=torch.float32, device="cuda")
        out = full_attn_fwd(q, k, v, lse=lse)
        ref, ref_lse = orc.full_attn_fwd(x["q"], x["k"], x["v"])
        check_bf16(_host(out), ref, "full")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=1e-5, atol=1e-2)
        return
    grid, window, first_late = {"short_kernel": ((21, 4, 8), (21, 2, 4), 128),
                                "chunked_local": ((21, 8, 8), (21, 4, 4), 192)}[case]
    order = LG if case == "short_kernel" else LO
    n = grid[0] * grid[1] * grid[2]
    x = make_inputs(1, 2, n, 128, dtype="bf16")
    late = orc.window_partition(*grid, *window)[:, first_late:].ravel()
    x["k"][:, :, late, :] *= 64.0
    q, k, v = (_dev(x[s], torch.bfloat16) for s in "qkv")
    out, ws = squad_attn_fwd(q, k, v, grid, window, order)
    assert squad_attn_fwd_status(ws, q, grid, window, order) == 0
    ref = orc.squad_attn_fwd(x["q"], x["k"], x["v"], grid, window, ORC_ORDER[order])
    check_bf16(_host(out), ref, case)


@pytest.mark.parametrize("grid", [(21, 22, 40), (21, 44, 80)])
def test_full_attention_wan_sizes_sampled_rows(grid):
    n = grid[0] * grid[1] * grid[2]
    x = make_inputs(1, 24, n, 128, dtype="bf16", heavy_tail=True)
    q, k, v = (_dev(x[s], torch.bfloat16) for s in "qkv")
    gpu = _host(full_attn_fwd(q, k, v, grid=grid))
    rows = np.random.default_rng(0).choice(n, 256, replace=False)
    for hh in (0, 23):
        sl = (slice(None), slice(hh, hh + 1))
        ref, _ = orc.full_attn_fwd(x["q"][sl], x["k"][sl], x["v"][sl], rows=rows)
        check_bf16(gpu[sl][:, :, rows], ref, f"head {hh}")


# ------------------------------------------------------------------------------------------------
# backward
# ------------------------------------------------------------------------------------------------

def run_bwd(B, h, d, grid, window, order, dtype, heads=None):
    n = grid[0] * grid[1] * grid[2]
    x = make_inputs(B, h, n, d, dtype="bf16" if dtype == torch.bfloat16 else "fp32", with_dout=True)
    q, k, v, do = (_dev(x[s], dtype) for s in ("q", "k", "v", "do"))
    out, ws = squad_attn_fwd(q, k, v, grid, window, order)
    dq, dk, dv = squad_attn_bwd(q, k, v, out, do, ws, grid, window, order)
    g = [_host(t) for t in (dq, dk, dv)]
    o = _host(out)
    heads = range(h) if heads is None else heads
    check = check_bf16 if dtype == torch.bfloat16 else check_fp32
    for hh in heads:
        sl = (slice(None), slice(hh, hh + 1))
        check(o[sl], orc.squad_attn_fwd(x["q"][sl], x["k"][sl], x["v"][sl], grid, window, ORC_ORDER[order]),
              f"O head {hh}")
        ref = orc.squad_attn_bwd(x["q"][sl], x["k"][sl], x["v"][sl], x["do"][sl], grid, window, ORC_ORDER[order])
        for name, mine, r in zip(("dQ", "dK", "dV"), g, ref):
            check(mine[sl], r, f"{name} head {hh}")


@pytest.mark.parametrize("order", [LG, GL])
def test_backward_tiny_fp32(order):
    run_bwd(1, 4, 64, (5, 8, 8), (5, 2, 2), order, torch.float32)


@pytest.mark.parametrize("order", [LG, GL])
def test_backward_small_bf16(order):
    run_bwd(2, 2, 128, (21, 4, 8), (21, 2, 4), order, torch.bfloat16)


def _bwd_kernels(h, grid, window, order):
    return squad_attn_bwd_kernels(1, h, 128, grid, window, order, torch.bfloat16)


@pytest.mark.parametrize("B,h,grid,window", [
    (1, 2, (3, 2, 43), (3, 1, 43)),     # local 129 = 128 + 1 rows (scratch panels of 144 rows); global 2
    (2, 1, (2, 43, 6), (2, 1, 2)),      # global 129 (43 x 3 slot boxes); local 4
    (1, 2, (3, 30, 52), (3, 2, 4)),     # global 195: 13 rows past the sequence in 208-row panels
    (1, 2, (13, 4, 32), (13, 2, 8)),    # local 208 = 13 x 16: no padding row, dQ over dP's columns
    (2, 1, (2, 13, 32), (2, 1, 2)),     # global 208
    (1, 2, (11, 4, 6), (11, 3, 6)),     # local 198 on a reflect-padded grid (H 4 -> 6)
])
@pytest.mark.parametrize("order", [LG, GL])
def test_backward_whole_sequence_kernel_length_range(B, h, grid, window, order):
    """The whole-sequence backward at the ends of its two-tile range (129-208 tokens): a one-row second
    tile, rows past the sequence up to the 16-row rounding, and sequences long enough (over 192 tokens)
    that dQ shares tensor-memory columns with dP instead of having its own."""
    assert _bwd_kernels(h, grid, window, order) == ("tc_whole", "tc_whole")
    run_bwd(B, h, 128, grid, window, order, torch.bfloat16)


@pytest.mark.parametrize("B,h,grid,window", [
    (1, 2, (4, 3, 22), (4, 1, 11)),     # local 44: two 48-row bands per packed tile; global 6
    (1, 2, (4, 8, 8), (4, 4, 4)),       # local 64: two 64-row bands; global 4
    (1, 2, (5, 2, 26), (5, 1, 13)),     # local 65: one 72-row band, products over 80 rows; global 4
    (1, 2, (3, 2, 80), (3, 1, 40)),     # local 120: products read 8 rows past the 120-row panels
    (1, 2, (2, 16, 16), (2, 2, 2)),     # global 64; local 8
    (2, 1, (2, 16, 18), (2, 2, 2)),     # global 72; local 8
    (1, 2, (3, 20, 20), (3, 2, 2)),     # global 100 (a 104-row band); local 12
    (1, 1, (1, 120, 2), (1, 1, 2)),     # global 120; local 2
])
@pytest.mark.parametrize("order", [LG, GL, LO, GO])
def test_one_tile_sequence_lengths(B, h, grid, window, order):
    """Sequences of 44-120 tokens: the packed one-tile backward (and the packed single-pass forward) with
    two sequences per tile, and the unpacked one where the band (the length rounded to 8 rows) is not a
    multiple of 16, so its products read 8 rows past the panel, which meet only zero P and dS."""
    assert all(k == "tc_whole" for k in _bwd_kernels(h, grid, window, order) if k is not None)
    run_bwd(B, h, 128, grid, window, order, torch.bfloat16)


@pytest.mark.parametrize("grid,window,long_pass", [
    ((2, 64, 32), (2, 4, 2), "global"),    # slot sequences of 256 tokens (O over the second half of S); windows of 16
    ((15, 8, 16), (15, 4, 4), "local"),    # windows of 240 = 128 + 112 rows; slot sequences of 8
])
@pytest.mark.parametrize("order", [LG, GL])
def test_fused_forward_longest_short_sequences(grid, window, long_pass, order):
    """The fused two-pass forward at the top of the short kernel's range (221-256 tokens; heavy-tailed
    keys for the forward), and its backward, whose long pass runs on the chunked kernels."""
    run_fwd(1, 2, 128, grid, window, order, torch.bfloat16, heavy_tail=True)
    ks = _bwd_kernels(2, grid, window, order)
    first_is_long = (order == LG) == (long_pass == "local")
    assert ks == (("tc_chunked", "tc_whole") if first_is_long else ("tc_whole", "tc_chunked"))
    run_bwd(1, 2, 128, grid, window, order, torch.bfloat16)


@pytest.mark.parametrize("order", [LG, GL])
def test_backward_bf16_long_windows_chunked_tensor_cores(order):
    """336-token windows (3 chunks of 8, 8 and 5 lines of 16 tokens) on the chunked tensor-core kernels;
    the 4-token slot sequences on the whole-sequence one."""
    ks = _bwd_kernels(1, (21, 8, 8), (21, 4, 4), order)
    assert ks == (("tc_chunked", "tc_whole") if order == LG else ("tc_whole", "tc_chunked"))
    run_bwd(1, 1, 128, (21, 8, 8), (21, 4, 4), order, torch.bfloat16)


@pytest.mark.parametrize("order,B,h", [(GO, 1, 2), (LG, 1, 2), (GO, 2, 1)])
def test_backward_bf16_long_slot_sequences_chunked(order, B, h):
    """576-token slot sequences (24 lines of 24 tokens: chunks of 5 lines, the last one 4) on the chunked
    kernels, alone and after a 20-token local pass; two batches of one head."""
    ks = _bwd_kernels(h, (5, 48, 48), (5, 2, 2), order)
    assert ks == (("tc_chunked", None) if order == GO else ("tc_whole", "tc_chunked"))
    run_bwd(B, h, 128, (5, 48, 48), (5, 2, 2), order, torch.bfloat16)


def test_backward_hires_5b_chunked():
    """The high-resolution 5B block (21x44x80, window 21x4x4): 336-token windows and 220-token slot
    sequences, both passes on the chunked tensor-core kernels (2 heads, every element)."""
    assert _bwd_kernels(2, (21, 44, 80), (21, 4, 4), LG) == ("tc_chunked", "tc_chunked")
    run_bwd(1, 2, 128, (21, 44, 80), (21, 4, 4), LG, torch.bfloat16)


def test_backward_padded_window_21x3x4_chunked():
    """The 5B grid with a 21x3x4 window, reflect-padded to 21x24x40: 252-token windows in chunks of 10,
    10 and 1 lines of 12 tokens (a 12-row last chunk)."""
    assert _bwd_kernels(2, (21, 22, 40), (21, 3, 4), LG) == ("tc_chunked", "tc_whole")
    run_bwd(1, 2, 128, (21, 22, 40), (21, 3, 4), LG, torch.bfloat16)


def test_backward_wan21_14b():
    run_bwd(1, 40, 128, (21, 22, 40), (21, 2, 4), LG, torch.bfloat16, heads=[0, 13, 27, 39])


# ------------------------------------------------------------------------------------------------
# single-pass variants (one pass alone)
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("order", [LO, GO])
def test_single_pass_tiny_fp32(order):
    run_fwd(1, 4, 64, (5, 8, 8), (5, 2, 2), order, torch.float32)
    run_bwd(1, 4, 64, (5, 8, 8), (5, 2, 2), order, torch.float32)


@pytest.mark.parametrize("order", [LO, GO])
def test_single_pass_small_bf16(order):
    run_fwd(2, 2, 128, (21, 4, 8), (21, 2, 4), order, torch.bfloat16)
    run_bwd(2, 2, 128, (21, 4, 8), (21, 2, 4), order, torch.bfloat16)


@pytest.mark.parametrize("order", [LO, GO])
def test_single_pass_wan22_5b_shape(order):
    """Windows of 168 and slot sequences of 110 tokens, one pass, forward and backward (2 heads)."""
    run_fwd(1, 24, 128, (21, 22, 40), (21, 2, 4), order, torch.bfloat16, heavy_tail=True, heads=[0, 23])
    run_bwd(1, 2, 128, (21, 22, 40), (21, 2, 4), order, torch.bfloat16)


@pytest.mark.parametrize("order,B,h", [(LO, 1, 3), (GO, 1, 3), (LO, 2, 2)])
def test_single_pass_short_sequences_packed(order, B, h):
    """21-token windows (five per 128-row tile) and 8-token slot sequences (sixteen per tile), tiles that
    span heads and batches, the last tile of each launch partly filled; forward and backward."""
    run_fwd(B, h, 128, (3, 4, 14), (3, 1, 7), order, torch.bfloat16)
    run_bwd(B, h, 128, (3, 4, 14), (3, 1, 7), order, torch.bfloat16)


# ------------------------------------------------------------------------------------------------
# grids the window does not divide (reflect padding, both passes on the padded grid, crop)
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("order", [LG, GL, LO, GO])
def test_padded_tiny_fp32(order):
    """5x7x9 with a 5x2x4 window: padded to 5x8x12 (one row, three columns reflected)."""
    run_fwd(1, 2, 64, (5, 7, 9), (5, 2, 4), order, torch.float32)
    run_bwd(1, 2, 64, (5, 7, 9), (5, 2, 4), order, torch.float32)


@pytest.mark.parametrize("order", [LG, GL])
def test_padded_small_bf16(order):
    run_fwd(1, 2, 128, (21, 5, 9), (21, 2, 4), order, torch.bfloat16)
    run_bwd(1, 2, 128, (21, 5, 9), (21, 2, 4), order, torch.bfloat16)


def test_padded_odd_resolution_bf16():
    """The 5B block with one more latent row and column (21x23x41, padded to 21x24x44)."""
    run_fwd(1, 24, 128, (21, 23, 41), (21, 2, 4), LG, torch.bfloat16, heavy_tail=True, heads=[0, 23])
    run_bwd(1, 2, 128, (21, 23, 41), (21, 2, 4), LG, torch.bfloat16)
