"""Seeded synthetic inputs for SQuad-Attention, shared by the tests, the bench and smoke().

This module draws numbers and nothing else: it holds none of the attention arithmetic, so the fp64
oracle and the CUDA path can both be fed from it without sharing any of the method's code.

Recipe (one Philox stream per tensor, counter-based and platform independent):

* Q, K, V, dO ~ N(0, 1), float32, seed = ``seed + 7 * tensor_id`` with Q=0, K=1, V=2, dO=3.
* bf16 mode: every value is rounded to the nearest bfloat16 (ties to even) *before* either side sees
  it, so the oracle (fp64) and the kernels (bf16 operands) start from identical numbers.
* Heavy tail (the Wan-shaped forward workloads): for every (b, head), round(0.02 * n) key tokens,
  drawn without replacement from a seeded permutation, have their K row multiplied by 4. The pages
  describe video-DiT attention maps as sparse, with most of each row's weight on a handful of keys
  (agihunt.info digest, the paragraph on the motivating observation); scaling 2 % of the
  keys by 4 gives logits with a standard deviation of 4 on those keys and of 1 elsewhere, which
  reproduces that shape. Multiplying by 4 is exact in bf16.

Layout of every tensor: [B, h, n, d] row-major, token index n = (t * H + y) * W + x.
"""
from __future__ import annotations

import numpy as np

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}
DEFAULT_SEED = 1234
HEAVY_TAIL_FRACTION = 0.02
HEAVY_TAIL_FACTOR = 4.0


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(seed))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16, ties to even; returns float32 holding them."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def normal(shape, tensor: str, seed: int = DEFAULT_SEED) -> np.ndarray:
    """N(0,1) float32 array for one named tensor ("q", "k", "v" or "do")."""
    return _rng(seed + 7 * TENSOR_IDS[tensor]).standard_normal(shape, dtype=np.float32)


def heavy_tail_rows(B: int, h: int, n: int, seed: int = DEFAULT_SEED) -> np.ndarray:
    """Indices [B, h, m] of the key tokens scaled by HEAVY_TAIL_FACTOR, m = round(0.02 n)."""
    m = int(round(HEAVY_TAIL_FRACTION * n))
    rng = _rng(seed + 7 * TENSOR_IDS["k"] + 1)
    out = np.empty((B, h, m), dtype=np.int64)
    for b in range(B):
        for hh in range(h):
            out[b, hh] = rng.permutation(n)[:m]
    return out


def make_inputs(B: int, h: int, n: int, d: int, dtype: str = "bf16", heavy_tail: bool = False,
                with_dout: bool = False, seed: int = DEFAULT_SEED) -> dict:
    """Q, K, V (and dO) as float32 numpy arrays of shape [B, h, n, d].

    With dtype == "bf16" every value is bf16-representable; with "fp32" they are plain float32.
    """
    if dtype not in ("bf16", "fp32"):
        raise ValueError(f"dtype must be 'bf16' or 'fp32', got {dtype!r}")
    shape = (B, h, n, d)
    names = ["q", "k", "v"] + (["do"] if with_dout else [])
    out = {}
    for name in names:
        x = normal(shape, name, seed)
        if dtype == "bf16":
            x = round_to_bf16(x)
        out[name] = x
    if heavy_tail:
        rows = heavy_tail_rows(B, h, n, seed)
        k = out["k"]
        for b in range(B):
            for hh in range(h):
                k[b, hh, rows[b, hh], :] *= np.float32(HEAVY_TAIL_FACTOR)
    return out
