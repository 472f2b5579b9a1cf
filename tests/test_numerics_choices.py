"""CPU pins for two numerical choices of the attention kernels (no GPU).

1. The weights P of the P.V product are multiplied as two 16-bit terms
   (hi = RNE(p), lo = RNE(p - hi)).  One 16-bit rounding of p cannot hold the
   2e-3 gate: with two visible keys of weights w and 1 - w the output error
   reaches about 2^-9 |v0 - v1| for bf16.  Emulated here with torch's bf16 /
   fp16 rounding against the float64 oracle.
2. The running maximum is only moved (and O, l rescaled) when a tile's
   maximum exceeds it by more than 2^8 in the base-2 exponent; weights stay
   <= 2^8, so fp32 sums cannot overflow, and since the same maximum divides
   out at the end the result equals the exact softmax up to fp32 rounding.
   Emulated tile by tile in float32 on adversarial score sequences.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as OA

LOG2E = 1.0 / math.log(2.0)


def rne(x: np.ndarray, dtype) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(dtype).to(torch.float64).numpy()


def pv(p: np.ndarray, v: np.ndarray, dtype, two_terms: bool) -> np.ndarray:
    """p [n] (fp32 weights), v [n, d] already 16-bit values -> p.V as the tensor cores see it."""
    hi = rne(p, dtype)
    out = hi @ v
    if two_terms:
        out = out + rne(np.asarray(p, np.float64) - hi, dtype) @ v
    return out


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_one_rounding_of_p_misses_the_gate_and_two_terms_meet_it(dtype):
    rng = np.random.default_rng(11)
    worst_one, worst_two = 0.0, 0.0
    for _ in range(400):
        n, d = int(rng.integers(2, 5)), 64
        q = rne(rng.standard_normal(d), dtype)
        k = rne(rng.standard_normal((n, d)), dtype)
        v = rne(3.0 * rng.standard_normal((n, d)), dtype)
        ref = OA.contiguous_attention(q, k, v, d ** -0.5)
        s = (k @ q) * d ** -0.5
        p = np.exp(s - s.max()).astype(np.float32)
        l = float(p.astype(np.float64).sum())
        worst_one = max(worst_one, float(np.abs(pv(p, v, dtype, False) / l - ref).max()))
        worst_two = max(worst_two, float(np.abs(pv(p, v, dtype, True) / l - ref).max()))
    if dtype == torch.bfloat16:
        assert worst_one > 2e-3          # a single bf16 rounding breaks the gate
    assert worst_two < 2e-4              # two terms keep ~16 bits of every weight


def lazy_softmax_fp32(scores: np.ndarray, v: np.ndarray, scale: float, tile: int = 64, threshold: float = 8.0):
    """The kernels' online softmax over key tiles, in float32."""
    f32 = np.float32
    m_use, l = f32(-np.inf), f32(0.0)
    o = np.zeros(v.shape[1], f32)
    s2 = f32(scale * LOG2E)
    for t0 in range(0, len(scores), tile):
        s = scores[t0:t0 + tile].astype(f32)
        mt = f32(s.max()) * s2
        if mt > m_use + f32(threshold):
            alpha = f32(np.exp2(m_use - mt)) if np.isfinite(m_use) else f32(0.0)
            m_use = mt
            l = l * alpha
            o = o * alpha
        p = np.exp2(s * s2 - m_use).astype(f32)
        with np.errstate(over="ignore"):
            assert np.all(p <= np.exp2(f32(threshold)) * f32(1.0001))   # weights never exceed 2^threshold
        l = f32(l + p.sum(dtype=f32))
        o = (o + p @ v[t0:t0 + tile].astype(f32)).astype(f32)
    return o / l


@pytest.mark.parametrize("pattern", ["rising", "falling", "spike_late", "flat", "sawtooth"])
def test_lazy_rescale_equals_the_softmax(pattern):
    rng = np.random.default_rng(hash(pattern) % 2 ** 32)
    n, d, scale = 64 * 40 + 17, 32, 0.125
    if pattern == "rising":            # the max grows on every tile, by less and more than 2^8
        scores = np.linspace(-50, 400, n) + rng.standard_normal(n)
    elif pattern == "falling":
        scores = np.linspace(400, -50, n) + rng.standard_normal(n)
    elif pattern == "spike_late":      # one huge score in the last tile
        scores = rng.standard_normal(n)
        scores[-3] = 900.0
    elif pattern == "flat":
        scores = np.full(n, 3.0)
    else:                              # rises by steps just under the threshold, then drops
        scores = (np.arange(n) // 64 % 7) * (7.9 / LOG2E) + rng.standard_normal(n) * 0.1
    v = rng.standard_normal((n, d))
    # `scores` are the scaled logits; the kernels see raw q.k = scores / scale.
    # The oracle gets them through q = e_0 and K rows carrying the raw values.
    raw = scores / scale
    k = np.zeros((n, d))
    k[:, 0] = raw
    q = np.zeros(d)
    q[0] = 1.0
    ref = OA.contiguous_attention(q, k, v, scale)
    got = lazy_softmax_fp32(raw.astype(np.float32), v.astype(np.float32), scale)
    assert np.all(np.isfinite(got))
    assert np.abs(got - ref).max() < 2e-5


def test_without_rescaling_fp32_overflows():
    """The rescale is needed at all: keeping the first tile's maximum, a score
    200 above it in a later tile overflows float32 (2^288)."""
    n, d = 128, 8
    scores = np.zeros(n, np.float32)
    scores[100] = 200.0
    v = np.ones((n, d), np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        got = lazy_softmax_fp32(scores, v, 1.0, threshold=1e9)   # never rescales after the first tile
    assert not np.all(np.isfinite(got))
    assert np.all(np.isfinite(lazy_softmax_fp32(scores, v, 1.0)))
