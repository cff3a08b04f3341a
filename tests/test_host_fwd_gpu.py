"""squad_attn_fwd_host (needs a B200): the forward from pinned host buffers through the C entry point,
split over runs of heads with the copies overlapped on three streams, gives the bits of one device call
on the same inputs, across back-to-back calls on alternating inputs (the calls' event joins order each
run's copies and forward between calls)."""
import numpy as np
import pytest
import torch

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import HostRunner, squad_attn_fwd
from sub_quadratic_two_squad_b200.inputs import make_inputs
from test_gpu_parity import check_bf16

pytestmark = pytest.mark.gpu


def _pinned(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("groups", [1, 4, 6])
def test_host_forward_gives_the_device_call_bits(groups):
    B, h, d, grid, window = 1, 6, 128, (21, 4, 8), (21, 2, 4)
    n = 21 * 4 * 8
    xs = [make_inputs(B, h, n, d, dtype="bf16", heavy_tail=True, seed=s) for s in (11, 12)]
    hosts = [tuple(_pinned(x[s]) for s in "qkv") for x in xs]
    refs = []
    for x in xs:
        q, k, v = (torch.from_numpy(x[s]).to("cuda", torch.bfloat16) for s in "qkv")
        refs.append(squad_attn_fwd(q, k, v, grid, window)[0].cpu())
    runner = HostRunner(B, h, d, grid, window, groups=groups)
    outs = [torch.empty((B, h, n, d), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    runner.start(start)
    for i, o in enumerate(outs):
        runner(*hosts[i % 2], o)
    runner.end(end)
    end.synchronize()
    assert start.elapsed_time(end) > 0
    for i, o in enumerate(outs):
        assert torch.equal(o, refs[i % 2]), f"call {i}"
    check_bf16(outs[0].float().numpy().astype(np.float64),
               orc.squad_attn_fwd(xs[0]["q"], xs[0]["k"], xs[0]["v"], grid, window), "o")


def test_host_forward_padded_grid_and_batches():
    """Runs that split batches and a grid the window does not divide (each run pads its own heads)."""
    B, h, d, grid, window = 2, 3, 128, (21, 5, 9), (21, 2, 4)
    n = 21 * 5 * 9
    x = make_inputs(B, h, n, d, dtype="bf16", heavy_tail=True, seed=21)
    q, k, v = (torch.from_numpy(x[s]).to("cuda", torch.bfloat16) for s in "qkv")
    ref = squad_attn_fwd(q, k, v, grid, window)[0].cpu()
    runner = HostRunner(B, h, d, grid, window, groups=4)
    o = torch.empty((B, h, n, d), dtype=torch.bfloat16).pin_memory()
    runner(*(_pinned(x[s]) for s in "qkv"), o)
    torch.cuda.synchronize()
    assert torch.equal(o, ref)
