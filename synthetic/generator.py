"""Counter-based random streams and value packing for the synthetic inputs.

SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014) is used in its counter form: output i of the stream
with key ``seed`` mixes ``seed + (i + 1) * 0x9E3779B97F4A7C15`` through the
two xor-shift-multiply rounds of the published finaliser. Every tensor of a
workload draws from its own window of the counter space, so the draws do not
depend on the order in which tensors are made.

Normals come from the Box–Muller transform in float64 and are rounded to
float32; bf16 values are the float32 values rounded to nearest-even and kept
as raw uint16 bit patterns (numpy has no bf16 type).
"""

from __future__ import annotations

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)

# Each tensor of a workload reads counters [tag << 40, (tag << 40) + count).
STREAM_SHIFT = 40
_CHUNK = 1 << 22


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the SplitMix64 stream keyed by ``seed``."""
    if count < 0:
        raise ValueError("count must be non-negative")
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GAMMA
    z = (z ^ (z >> np.uint64(30))) * _MIX1
    z = (z ^ (z >> np.uint64(27))) * _MIX2
    return z ^ (z >> np.uint64(31))


def uniform01(seed: int, start: int, count: int, *, open_left: bool = False) -> np.ndarray:
    """53-bit uniforms in [0, 1), or in (0, 1] when ``open_left``."""
    z = splitmix64(seed, start, count) >> np.uint64(11)
    if open_left:
        z = z + np.uint64(1)
    return z.astype(np.float64) * (1.0 / 9007199254740992.0)


def standard_normal(seed: int, tag: int, count: int) -> np.ndarray:
    """``count`` N(0,1) float64 draws from stream ``tag`` (Box–Muller, pairs in order)."""
    out = np.empty(count, dtype=np.float64)
    base = tag << STREAM_SHIFT
    pairs_total = (count + 1) // 2
    done = 0
    while done < pairs_total:
        pairs = min(_CHUNK, pairs_total - done)
        z = splitmix64(seed, base + 2 * done, 2 * pairs)
        u1 = ((z[0::2] >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (1.0 / 9007199254740992.0)
        u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
        r = np.sqrt(-2.0 * np.log(u1))
        theta = (2.0 * np.pi) * u2
        lo = 2 * done
        hi = min(count, 2 * (done + pairs))
        block = np.empty(2 * pairs, dtype=np.float64)
        block[0::2] = r * np.cos(theta)
        block[1::2] = r * np.sin(theta)
        out[lo:hi] = block[: hi - lo]
        done += pairs
    return out


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bit patterns.

    Only finite inputs are expected here (the generator never makes NaN).
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))
    return (b >> np.uint64(16)).astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def permutation(seed: int, tag: int, n: int) -> np.ndarray:
    """A seeded permutation of ``range(n)``: the stable argsort of n stream draws."""
    keys = splitmix64(seed, tag << STREAM_SHIFT, n)
    return np.argsort(keys, kind="stable").astype(np.int64)


def zipf_bias(seed: int, tag: int, n: int, s: float) -> np.ndarray:
    """Per-expert logit bias whose softmax weights follow Zipf(s) over a seeded ranking.

    The expert at rank r (0-based) of a seeded permutation gets ``-s * ln(r + 1)``,
    i.e. the log of the Zipf mass ``(r + 1) ** -s`` up to a constant.
    """
    perm = permutation(seed, tag, n)
    bias = np.empty(n, dtype=np.float64)
    bias[perm] = -s * np.log(np.arange(1, n + 1, dtype=np.float64))
    return bias
