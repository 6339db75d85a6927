"""Counter-based random numbers for the synthetic SSD workloads.

Every random draw is a pure function of (seed, stream, flat index), so any
slice of a tensor can be regenerated on its own: the GPU tests and the bench
materialise whole tensors, while a check at full size regenerates only the
(batch, head) chains it samples.  Nothing here belongs to the scan itself.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used in counter mode: draw i of a stream with
key K is mix64(K + (i + 1) * 0x9E3779B97F4A7C15), which is the i-th output of
the sequential generator seeded with K.  Normals come from the Box-Muller
transform (Box and Muller, 1958) on consecutive pairs of uniforms.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_TWO_M53 = 2.0 ** -53

# Stream identifiers: one independent stream per synthetic quantity.
STREAM_X = 1
STREAM_B = 2
STREAM_C = 3
STREAM_DT_NOISE = 4
STREAM_DT_BIAS = 5
STREAM_A = 6
STREAM_D = 7
STREAM_HEAD_SCALE = 8
STREAM_OUTLIER = 9


def _mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    """Key of one stream: the first SplitMix64 output of seed*2^16 + stream."""
    base = np.array([(int(seed) << 16) + int(stream)], dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(base + _GOLDEN)[0]


def u64(key: np.uint64, idx: np.ndarray) -> np.ndarray:
    """Draw number `idx` (uint64 array) of the stream with key `key`."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + (idx + np.uint64(1)) * _GOLDEN)


def uniform(key: np.uint64, idx: np.ndarray) -> np.ndarray:
    """Uniform on the open interval (0, 1) in float64: (top 53 bits + 1/2) / 2^53."""
    z = u64(key, idx)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * _TWO_M53


def normal(key: np.uint64, idx: np.ndarray) -> np.ndarray:
    """Standard normal number `idx` of a stream, float64.

    Normals 2k and 2k+1 are the cosine and sine outputs of Box-Muller applied to
    uniforms 2k and 2k+1 of the same stream.
    """
    idx = np.asarray(idx, dtype=np.uint64)
    pair = idx >> np.uint64(1)
    u1 = uniform(key, pair * np.uint64(2))
    u2 = uniform(key, pair * np.uint64(2) + np.uint64(1))
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = (2.0 * math.pi) * u2
    odd = (idx & np.uint64(1)).astype(bool)
    return np.where(odd, rad * np.sin(ang), rad * np.cos(ang))


def normal_block(key: np.uint64, lo: int, hi: int) -> np.ndarray:
    """Normals [lo, hi) of a stream (lo and hi even), float64.

    Same values as `normal(key, arange(lo, hi))`, computing each Box-Muller pair once.
    """
    u = uniform(key, np.arange(lo, hi, dtype=np.uint64))
    u1, u2 = u[0::2], u[1::2]
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = (2.0 * math.pi) * u2
    out = np.empty(hi - lo, dtype=np.float64)
    out[0::2] = rad * np.cos(ang)
    out[1::2] = rad * np.sin(ang)
    return out


def parallel_blocks(count: int, work, block: int = 1 << 15) -> None:
    """Run work(lo, hi) over [0, count) in even-sized blocks on a thread pool.

    Blocks stay small so that temporaries are recycled by the allocator instead
    of being mapped afresh for every block.
    """
    nblk = (count + block - 1) // block
    if nblk <= 1:
        if count:
            work(0, count)
        return
    nthr = min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=nthr) as pool:
        list(pool.map(lambda i: work(i * block, min(count, (i + 1) * block)), range(nblk)))


def normal_range(key: np.uint64, count: int) -> np.ndarray:
    """Normals [0, count) of a stream as float32."""
    out = np.empty(count, dtype=np.float32)

    def work(lo, hi):
        e = hi + (hi & 1)
        out[lo:hi] = normal_block(key, lo, e)[: hi - lo]

    parallel_blocks(count, work)
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rnd = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    with np.errstate(over="ignore"):
        return ((u + rnd) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact float32 value of bfloat16 bit patterns."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
