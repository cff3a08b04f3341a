"""The autograd wrappers (needs a B200): gradients through torch autograd are the library's backward,
and match the fp64 oracle within the bf16 bounds."""
import pytest
import torch

from oracle import squad_oracle as orc
from sub_quadratic_two_squad_b200 import squad_attention, squad_attn_bwd, squad_attn_fwd, squad_kpass_attention
from sub_quadratic_two_squad_b200.inputs import make_inputs
from test_gpu_parity import _dev, _host, check_bf16

pytestmark = pytest.mark.gpu


def test_squad_attention_autograd():
    grid, window = (21, 4, 8), (21, 2, 4)
    n = 21 * 4 * 8
    x = make_inputs(1, 2, n, 128, dtype="bf16", with_dout=True, seed=77)
    q, k, v = (_dev(x[s], torch.bfloat16).requires_grad_(True) for s in "qkv")
    do = _dev(x["do"], torch.bfloat16)
    o = squad_attention(q, k, v, grid, window)
    o.backward(do)
    # the same kernels called directly give the same bits
    o2, ws = squad_attn_fwd(q.detach(), k.detach(), v.detach(), grid, window)
    g2 = squad_attn_bwd(q.detach(), k.detach(), v.detach(), o2, do, ws, grid, window)
    assert torch.equal(o.detach(), o2)
    for a, b in zip((q.grad, k.grad, v.grad), g2):
        assert torch.equal(a, b)
    check_bf16(_host(o.detach()), orc.squad_attn_fwd(x["q"], x["k"], x["v"], grid, window), "o")
    for name, got, ref in zip(("dq", "dk", "dv"), (q.grad, k.grad, v.grad),
                              orc.squad_attn_bwd(x["q"], x["k"], x["v"], x["do"], grid, window)):
        check_bf16(_host(got), ref, name)


def test_kpass_attention_autograd():
    grid, levels = (2, 8, 12), [(2, 2), (2, 3), (2, 2)]
    n = 2 * 8 * 12
    x = make_inputs(1, 2, n, 128, dtype="bf16", with_dout=True, seed=78)
    q, k, v = (_dev(x[s], torch.bfloat16).requires_grad_(True) for s in "qkv")
    o = squad_kpass_attention(q, k, v, grid, levels)
    o.backward(_dev(x["do"], torch.bfloat16))
    check_bf16(_host(o.detach()), orc.kpass_fwd(x["q"], x["k"], x["v"], grid, levels), "o")
    for name, got, ref in zip(("dq", "dk", "dv"), (q.grad, k.grad, v.grad),
                              orc.kpass_bwd(x["q"], x["k"], x["v"], x["do"], grid, levels)):
        check_bf16(_host(got), ref, name)
