"""Seeded synthetic inputs for the hashed N-gram embedding layer.

This module is shared by the test/bench harness on both sides of the parity
check (the fp64 oracle and the CUDA path). It holds none of the layer's
arithmetic: no hashing, no gathering, no projection. It only draws numbers.

Every value is a pure function of (seed, tag, counter) through SplitMix64
(Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014): the i-th output of a SplitMix64 stream seeded with `base` is
mix(base + (i + 1) * GAMMA). The device filler in `synth/csrc/synth_fill.cu`
implements the same definition, so a table of tens of GB can be written on the
GPU while the oracle regenerates only the rows it touches on the host.

Table values follow the init rule "E ~ N(0, 0.02), W ~ N(0, 1/width)":
a normal variate is approximated by the Irwin-Hall sum of four uniform 16-bit
lanes of one 64-bit draw, centred, then multiplied by one fp32 constant
(a single IEEE multiply, identical on host and device), then rounded to
bf16 by round-to-nearest-even on the bit pattern.
"""
from __future__ import annotations

import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1

# Tensor tags: which stream a tensor's values come from.
TAG_E0 = 0
TAG_SUBTABLE0 = 1          # sub-table s uses TAG_SUBTABLE0 + s
TAG_W = 100
TAG_TOKENS = 200
TAG_LENGTHS = 300
TAG_ACCEPT = 400
TAG_PROMPT_LEN = 500

# Irwin-Hall(4) of 16-bit lanes: mean 4 * 32767.5, variance 4 * (65536^2 - 1) / 12.
IH_MEAN = 131070
IH_STD = math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(base: int, counters) -> np.ndarray:
    """Outputs number `counters` (0-based) of the SplitMix64 stream seeded with `base`."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(base & _MASK64) + (c + np.uint64(1)) * GAMMA
        return _mix(z)


def stream_base(seed: int, tag: int) -> int:
    """The per-tensor stream seed: output `tag` of the stream seeded with `seed`."""
    return int(splitmix64(seed, np.array([tag], dtype=np.uint64))[0])


def value_scale(std: float) -> np.float32:
    """fp32 multiplier that turns a centred Irwin-Hall(4) integer into std `std`."""
    return np.float32(std / IH_STD)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of fp32 values to bf16 bit patterns (no NaN inputs)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))
    return (b >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def table_values_f32(seed: int, tag: int, rows, width: int, std: float) -> np.ndarray:
    """fp32 values of rows `rows` (array of row ids) of a [*, width] table, shape [len(rows), width]."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1)
    cols = np.arange(width, dtype=np.uint64)
    with np.errstate(over="ignore"):
        counters = rows[:, None] * np.uint64(width) + cols[None, :]
    z = splitmix64(stream_base(seed, tag), counters)
    m = np.uint64(0xFFFF)
    s = ((z & m) + ((z >> np.uint64(16)) & m) + ((z >> np.uint64(32)) & m) + (z >> np.uint64(48)))
    centred = s.astype(np.int64) - IH_MEAN          # |centred| < 2^18: exact in fp32
    return centred.astype(np.float32) * value_scale(std)


def table_rows_bf16(seed: int, tag: int, rows, width: int, std: float) -> np.ndarray:
    """bf16 bit patterns (uint16) of the given rows, shape [len(rows), width]."""
    return f32_to_bf16_bits(table_values_f32(seed, tag, rows, width, std))


def table_bf16(seed: int, tag: int, num_rows: int, width: int, std: float) -> np.ndarray:
    return table_rows_bf16(seed, tag, np.arange(num_rows), width, std)


def table_f32(seed: int, tag: int, num_rows: int, width: int, std: float) -> np.ndarray:
    return table_values_f32(seed, tag, np.arange(num_rows), width, std)


def uniform01(seed: int, tag: int, n: int, offset: int = 0) -> np.ndarray:
    """n doubles in [0, 1) with 53 random bits each."""
    z = splitmix64(stream_base(seed, tag), np.arange(offset, offset + n, dtype=np.uint64))
    return (z >> np.uint64(11)).astype(np.float64) * (1.0 / (1 << 53))


def uniform_tokens(seed: int, n: int, V0: int, tag: int = TAG_TOKENS, offset: int = 0) -> np.ndarray:
    z = splitmix64(stream_base(seed, tag), np.arange(offset, offset + n, dtype=np.uint64))
    return (z % np.uint64(V0)).astype(np.int32)


_ZIPF_CACHE: dict = {}


def zipf_cdf(V0: int, alpha: float) -> np.ndarray:
    key = (V0, alpha)
    if key not in _ZIPF_CACHE:
        w = np.arange(1, V0 + 1, dtype=np.float64) ** (-alpha)
        c = np.cumsum(w)
        _ZIPF_CACHE[key] = c / c[-1]
    return _ZIPF_CACHE[key]


def zipf_tokens(seed: int, n: int, V0: int, alpha: float = 1.1, tag: int = TAG_TOKENS,
                offset: int = 0) -> np.ndarray:
    """Token ids with p(id = r - 1) proportional to r^-alpha, r = 1..V0 (truncated Zipf)."""
    u = uniform01(seed, tag, n, offset)
    ids = np.searchsorted(zipf_cdf(V0, alpha), u, side="right")
    return np.minimum(ids, V0 - 1).astype(np.int32)


def varlen_lengths(seed: int, num_seqs: int, total: int, lo: int, hi: int,
                   fixed: tuple = ()) -> np.ndarray:
    """num_seqs lengths summing to `total`: the `fixed` ones first, the rest uniform in
    [lo, hi], the last one set to the remainder (redrawn until it lands in [1, 2*hi])."""
    fixed = list(fixed)
    n_free = num_seqs - len(fixed) - 1
    attempt = 0
    while True:
        u = uniform01(seed, TAG_LENGTHS, n_free, offset=attempt * n_free)
        free = (lo + np.floor(u * (hi - lo + 1))).astype(np.int64)
        last = total - sum(fixed) - int(free.sum())
        if 1 <= last <= 2 * hi:
            return np.array(fixed + free.tolist() + [last], dtype=np.int32)
        attempt += 1


def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off.astype(np.int32)
