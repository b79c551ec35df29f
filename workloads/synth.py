"""Seeded synthetic input generators.

This module is shared by the tests, the bench and the oracle harness.  It holds
no attention arithmetic: it only draws numbers.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used as a counter-based stream: output i of
stream `s` is the SplitMix64 finaliser applied to s + (i + 1) * 0x9E3779B97F4A7C15.
Normals come from the Box-Muller transform in float64; bf16 values are the
float64 normals rounded to float32 (round-to-nearest-even) and then to bf16
(round-to-nearest-even on the bit pattern).  Tensors are returned as numpy
uint16 arrays holding bf16 bit patterns.
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser, vectorised (uint64 wrap-around arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_seed(seed: int, *tags: int) -> int:
    """Derive an independent 64-bit stream key from a base seed and integer tags."""
    s = np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    with np.errstate(over="ignore"):
        for t in tags:
            s = _mix(s ^ _mix(np.array([(t + 1) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64) * _GOLDEN))
    return int(s[0])


def u64(key: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs offset .. offset+n-1 of the counter stream `key` (uint64)."""
    idx = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(np.uint64(key) + idx * _GOLDEN)


def uniform01(key: int, n: int, offset: int = 0) -> np.ndarray:
    """Uniform doubles in [0, 1) with 53 random bits."""
    return (u64(key, n, offset) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_f64(key: int, n: int) -> np.ndarray:
    """n standard normals (Box-Muller, float64)."""
    out = np.empty(n, dtype=np.float64)
    pairs = (n + 1) // 2
    done = 0
    while done < pairs:
        m = min(_CHUNK, pairs - done)
        u = uniform01(key, 2 * m, 2 * done)
        u1 = 1.0 - u[0::2]            # (0, 1]
        u2 = u[1::2]
        r = np.sqrt(-2.0 * np.log(u1))
        t = 2.0 * np.pi * u2
        z = np.empty(2 * m, dtype=np.float64)
        z[0::2] = r * np.cos(t)
        z[1::2] = r * np.sin(t)
        lo = 2 * done
        hi = min(n, lo + 2 * m)
        out[lo:hi] = z[: hi - lo]
        done += m
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bf16 (RNE on the bit pattern); finite inputs only."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (b >> np.uint32(16)).astype(np.uint16)


def f64_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> IEEE fp16 (numpy's round-to-nearest-even) as uint16 bit patterns."""
    return np.ascontiguousarray(x).astype(np.float16).view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(key: int, shape) -> np.ndarray:
    """bf16 ~N(0,1) tensor of `shape`, as uint16 bit patterns, generated in chunks."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    step = 1 << 24
    for lo in range(0, n, step):
        hi = min(n, lo + step)
        # each chunk is its own sub-stream so chunks can be drawn independently
        out[lo:hi] = f64_to_bf16_bits(normal_f64(stream_seed(key, lo // step), hi - lo))
    return out.reshape(shape)


def normal_f32(key: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return normal_f64(key, n).astype(np.float32).reshape(shape)


def randint(key: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers uniform in [lo, hi] (inclusive), modulo reduction of 64-bit draws."""
    span = np.uint64(hi - lo + 1)
    return (u64(key, n) % span).astype(np.int64) + lo


def permutation(key: int, n: int) -> np.ndarray:
    """A seeded permutation of 0..n-1 (sort by random 64-bit keys)."""
    return np.argsort(u64(key, n), kind="stable").astype(np.int64)
