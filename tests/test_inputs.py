"""The synthetic input recipe (no GPU): seeded Philox streams per tensor, bf16 rounding that matches
torch's round-to-nearest-even, and the heavy-tailed keys (exactly round(0.02 n) rows per head, x4)."""
import numpy as np
import pytest
import torch

from sub_quadratic_two_squad_b200 import inputs


def test_deterministic_and_one_stream_per_tensor():
    a = inputs.make_inputs(1, 2, 96, 16, with_dout=True, seed=5)
    b = inputs.make_inputs(1, 2, 96, 16, with_dout=True, seed=5)
    for name in ("q", "k", "v", "do"):
        assert np.array_equal(a[name], b[name])
    assert not np.array_equal(a["q"], a["k"]) and not np.array_equal(a["k"], a["v"])
    # the stream of tensor i is Philox(seed + 7 i)
    ref = np.random.Generator(np.random.Philox(5 + 7 * 2)).standard_normal((1, 2, 96, 16), dtype=np.float32)
    assert np.array_equal(inputs.round_to_bf16(ref), a["v"])


def test_bf16_rounding_is_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000).astype(np.float32) * np.float32(1e3)
    # exact halfway cases: low 16 bits 0x8000, with even and odd kept parts (ties go to the even one)
    halves = (np.arange(1000, dtype=np.uint32) * np.uint32(0x10000) + np.uint32(0x3F808000)).view(np.float32)
    x = np.concatenate([x, halves, -halves])
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(inputs.round_to_bf16(x), ref)


def test_bf16_mode_is_representable_and_fp32_mode_is_not_rounded():
    a = inputs.make_inputs(1, 1, 64, 32, dtype="bf16")
    for name in ("q", "k", "v"):
        assert np.array_equal(torch.from_numpy(a[name]).to(torch.bfloat16).float().numpy(), a[name])
    f = inputs.make_inputs(1, 1, 64, 32, dtype="fp32")
    assert not np.array_equal(inputs.round_to_bf16(f["q"]), f["q"])
    with pytest.raises(ValueError):
        inputs.make_inputs(1, 1, 4, 4, dtype="fp16")


@pytest.mark.parametrize("n", [168, 18480 // 24, 1000])
def test_heavy_tail_scales_exactly_two_percent_of_keys_by_four(n):
    B, h, d = 2, 3, 8
    plain = inputs.make_inputs(B, h, n, d, heavy_tail=False, seed=9)
    heavy = inputs.make_inputs(B, h, n, d, heavy_tail=True, seed=9)
    m = int(round(0.02 * n))
    for name in ("q", "v"):
        assert np.array_equal(plain[name], heavy[name])
    for b in range(B):
        for hh in range(h):
            scaled = ~np.all(plain["k"][b, hh] == heavy["k"][b, hh], axis=1)
            assert scaled.sum() == m
            assert np.array_equal(heavy["k"][b, hh][scaled], 4.0 * plain["k"][b, hh][scaled])
            assert set(np.flatnonzero(scaled)) == set(inputs.heavy_tail_rows(B, h, n, seed=9)[b, hh])
