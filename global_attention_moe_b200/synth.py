"""Seeded synthetic inputs for the MiMo-V2 attention forward.

This module is the only code that both the CUDA path's tests/bench and the
FP64 oracle consume.  It holds none of the attention arithmetic: it draws
numbers and rounds them to the storage types the layer takes (BF16 Q/K/V,
FP32 sink logits, int32 ``cu_seqlens``).

Generator (counter-based, so any slice can be regenerated on its own):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): for seed ``s`` and counter ``c`` the output is
  ``mix64(s + (c + 1) * 0x9E3779B97F4A7C15 mod 2**64)`` with the published
  finaliser (xor-shift 30, multiply 0xBF58476D1CE4E5B9, xor-shift 27,
  multiply 0x94D049BB133111EB, xor-shift 31).
* Stream ``k`` uses counters ``(k << 40) + i``.  Streams: 0 = sequence
  lengths, 1 = q, 2 = k, 3 = v, 4 = sink.
* Uniforms take the top 53 bits: ``u = (z >> 11) * 2**-53`` in [0, 1); the
  Box-Muller radius uses ``(z >> 11) + 1`` so that its uniform is in (0, 1].
* Normals: Box-Muller on counter pairs (2j, 2j+1): element 2j takes the
  cosine branch and element 2j+1 the sine branch.  Computed in float64,
  rounded to float32 (numpy, round-to-nearest-even), then to BF16 with
  round-to-nearest-even on the bit pattern.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
STREAM_LENGTHS, STREAM_Q, STREAM_K, STREAM_V, STREAM_SINK, STREAM_PAGES = 0, 1, 2, 3, 4, 5
_STREAM_SHIFT = 40
_CHUNK = 1 << 22


def splitmix64(seed: int, counters: np.ndarray) -> np.ndarray:
    """SplitMix64 outputs for the given uint64 counters (vectorised)."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (counters.astype(np.uint64) + np.uint64(1)) * GOLDEN_GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def splitmix64_scalar(seed: int, counter: int) -> int:
    """Pure-Python SplitMix64 (used to pin the vectorised version)."""
    mask = (1 << 64) - 1
    z = (seed + (counter + 1) * 0x9E3779B97F4A7C15) & mask
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & mask
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & mask
    return z ^ (z >> 31)


def _counters(stream: int, start: int, count: int) -> np.ndarray:
    base = np.uint64((stream << _STREAM_SHIFT) + start)
    return base + np.arange(count, dtype=np.uint64)


def uniforms(seed: int, stream: int, count: int, start: int = 0) -> np.ndarray:
    """``count`` float64 uniforms in [0, 1) from ``stream``."""
    z = splitmix64(seed, _counters(stream, start, count))
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _normals_chunk(seed: int, stream: int, first: int, count: int) -> np.ndarray:
    """float64 normals for elements [first, first+count) of ``stream``."""
    j0 = first // 2
    j1 = (first + count + 1) // 2
    npairs = j1 - j0
    z = splitmix64(seed, _counters(stream, 2 * j0, 2 * npairs)).reshape(npairs, 2)
    u1 = ((z[:, 0] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (z[:, 1] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    r = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    both = np.empty((npairs, 2), dtype=np.float64)
    both[:, 0] = r * np.cos(ang)
    both[:, 1] = r * np.sin(ang)
    flat = both.reshape(-1)
    off = first - 2 * j0
    return flat[off:off + count]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (round-to-nearest-even) and return the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of BF16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, stream: int, shape, threads: int | None = None) -> np.ndarray:
    """N(0,1) samples of ``shape`` rounded to BF16; returns uint16 bit patterns."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def work(i0):
        cnt = min(_CHUNK, n - i0)
        vals = _normals_chunk(seed, stream, i0, cnt).astype(np.float32)
        out[i0:i0 + cnt] = f32_to_bf16_bits(vals)

    starts = list(range(0, n, _CHUNK))
    if len(starts) <= 1:
        for s in starts:
            work(s)
    else:
        nt = threads or min(32, os.cpu_count() or 1)
        with ThreadPoolExecutor(max_workers=nt) as ex:
            list(ex.map(work, starts))
    return out.reshape(shape)


def normal_f32(seed: int, stream: int, count: int) -> np.ndarray:
    """N(0,1) samples rounded to float32."""
    return _normals_chunk(seed, stream, 0, count).astype(np.float32)


def seq_lengths(seed: int, num_seqs: int, lo: int, hi: int) -> np.ndarray:
    """Integer lengths uniform in [lo, hi] (inclusive) from the lengths stream."""
    u = uniforms(seed, STREAM_LENGTHS, num_seqs)
    return (lo + np.floor(u * (hi - lo + 1))).astype(np.int64)


def cu_seqlens_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=cu[1:])
    if cu[-1] >= 2 ** 31:
        raise ValueError("total tokens exceed int32")
    return cu.astype(np.int32)
