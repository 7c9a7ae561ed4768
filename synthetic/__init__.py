"""Seeded synthetic inputs shared by the CPU oracle, the GPU tests and the bench.

This module holds only random-number generation and the shapes of the
workloads; none of the quantization arithmetic lives here.  Every draw comes
from one counter-based generator, SplitMix64 (Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014), so the same
(seed, index) always yields the same value on any machine:

    z = (seed * 2^32 + index + 1) * 0x9E3779B97F4A7C15        (mod 2^64)
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
    z = (z ^ (z >> 27)) * 0x94D049BB133111EB
    z =  z ^ (z >> 31)

Uniforms take the top 53 bits; normals use the Box-Muller transform in FP64;
BF16 tensors are FP64 -> FP32 (round to nearest even) -> BF16 (round to nearest
even), kept as uint16 bit patterns.

Workload recipes (sizes from the grouped-MoE, dense-RHT, DSA-indexer and
QMoE workloads the pages describe):
  * fp8_single:   BF16 [512, 128] ~ N(0, 1)
  * dsa_indexer:  BF16 q_pe, q_nope [4096, 64, 64] ~ N(0, 1)
  * dense_nvfp4:  BF16 [8192, 4096] ~ N(0, 1), each entry x50 with p = 0.001
  * grouped_moe:  BF16 [16384, 7168] ~ N(0, 1), 32 sections of 128-row units
  * qmoe:         BF16 [32768, 4096] ~ N(0, 1); FP32 gate|up [32768, 2*2048]
                  ~ N(0, 2) (variance 2)
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """SplitMix64 outputs for indices start .. start+count-1 of stream `seed`."""
    base = np.uint64(((seed & 0xFFFFFFFF) << 32) & 0xFFFFFFFFFFFFFFFF)
    idx = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (base + idx + np.uint64(1)) * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _MIX1
        z = (z ^ (z >> np.uint64(27))) * _MIX2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform(seed: int, n: int, start: int = 0) -> np.ndarray:
    """FP64 uniforms in [0, 1) from the top 53 bits of each SplitMix64 word."""
    out = np.empty(n, dtype=np.float64)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        out[s:s + c] = (splitmix64(seed, start + s, c) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return out


def normal(seed: int, n: int, std: float = 1.0) -> np.ndarray:
    """FP64 N(0, std^2) samples by Box-Muller on consecutive uniform pairs."""
    out = np.empty(n, dtype=np.float64)
    for s in range(0, n, _CHUNK * 4):
        c = min(_CHUNK * 4, n - s)
        out[s:s + c] = _normal_range(seed, s, c, std)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite FP32 values to BF16 (nearest even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _chunked(n: int, fill) -> None:
    """Run fill(start, count) over even-aligned chunks on a few host threads."""
    starts = list(range(0, n, _CHUNK * 4))
    if len(starts) <= 1:
        for s in starts:
            fill(s, min(_CHUNK * 4, n - s))
        return
    workers = max(1, min(8, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(lambda s: fill(s, min(_CHUNK * 4, n - s)), starts))


def normal_bf16(seed: int, shape, std: float = 1.0) -> np.ndarray:
    """BF16 bit patterns (uint16) of N(0, std^2) samples with the given shape."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def fill(s, c):
        out[s:s + c] = f32_to_bf16_bits(_normal_range(seed, s, c, std).astype(np.float32))

    _chunked(n, fill)
    return out.reshape(shape)


def normal_f32(seed: int, shape, std: float = 1.0) -> np.ndarray:
    """FP32 N(0, std^2) samples (FP64 draws rounded to nearest even)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)

    def fill(s, c):
        out[s:s + c] = _normal_range(seed, s, c, std).astype(np.float32)

    _chunked(n, fill)
    return out.reshape(shape)


def _normal_range(seed: int, start: int, count: int, std: float) -> np.ndarray:
    """Elements start .. start+count-1 of the stream `normal(seed, ...)` (start even)."""
    assert start % 2 == 0
    pairs = (count + 1) // 2
    u = uniform(seed, 2 * pairs, start=start)
    r = np.sqrt(-2.0 * np.log1p(-u[0::2]))
    th = (2.0 * np.pi) * u[1::2]
    z = np.empty(2 * pairs, dtype=np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return z[:count] * std


def with_outliers_bf16(bits: np.ndarray, seed: int, p: float = 0.001, factor: float = 50.0) -> np.ndarray:
    """Multiply each entry by `factor` (in FP32, re-rounded to BF16) with probability p."""
    flat = bits.reshape(-1)
    pick = uniform(seed, flat.size) < p
    vals = bf16_bits_to_f32(flat[pick]) * np.float32(factor)
    out = flat.copy()
    out[pick] = f32_to_bf16_bits(vals)
    return out.reshape(bits.shape)


def sign_mask16(seed: int) -> int:
    """A seeded 16-bit sign mask: bit i set means sign_i = -1."""
    return int(splitmix64(seed, 0, 1)[0] >> np.uint64(48)) & 0xFFFF


def moe_splits(seed: int, total_rows: int = 16384, sections: int = 32, unit: int = 128) -> list[int]:
    """Rows per MoE section: all multiples of `unit`.

    Section 0 is empty and section 1 holds exactly one unit; the remaining
    units go to sections 2.. by a seeded multinomial with p ~ exp(N(0, 1)),
    so further sections may come out empty.
    """
    units = total_rows // unit
    assert units * unit == total_rows and sections >= 3 and units >= 1
    counts = [0] * sections
    counts[1] = 1
    w = np.exp(normal(seed, sections - 2))
    cdf = np.cumsum(w / w.sum())
    cdf[-1] = 1.0
    draws = uniform(seed + 7919, units - 1)
    picks = np.searchsorted(cdf, draws, side="right")
    for p in picks:
        counts[2 + int(p)] += 1
    return [c * unit for c in counts]


def random_splits(seed: int, total_units: int, sections: int, unit: int = 128) -> list[int]:
    """Uniform random split of total_units units over `sections` (may be empty)."""
    draws = uniform(seed, total_units)
    picks = np.minimum((draws * sections).astype(np.int64), sections - 1)
    counts = np.bincount(picks, minlength=sections)
    return [int(c) * unit for c in counts]


# Seeds per workload: 1000 + workload index.
SEEDS = {"fp8_single": 1000, "dsa_indexer": 1001, "dense_nvfp4": 1002, "grouped_moe": 1003, "qmoe": 1004}
