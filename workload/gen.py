"""Seeded, counter-based random inputs shared by the CUDA path and the CPU oracle.

This module holds no arithmetic of the decoding method itself: only random numbers,
their mapping to bf16 / fp32 values, permutations and Xavier-uniform weights.  Every
value is a pure function of (key, index), so any slice of any tensor can be regenerated
without generating the rest (the 77 GB cache of the 128K-context workload is filled on
the device by ``workload/csrc/gen.cu`` and re-derived here slice by slice).

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014).  The i-th output (0-based) of a stream with state ``key`` is
``mix64(key + (i + 1) * GAMMA)`` with the published gamma and finaliser constants.

bf16 N(0,1): the top 16 bits of an output index a 65536-entry table holding the bf16
(round-to-nearest-even) value of the standard normal quantile at the bin midpoint
(j + 0.5) / 65536.  The table is built here in fp64 and uploaded to the device, so the
device generator is bit-identical by construction.
"""
from __future__ import annotations

import functools
from enum import IntEnum

import numpy as np
from scipy.special import ndtri

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1
_CHUNK = 1 << 22


class Tag(IntEnum):
    """Stream identifiers: the first id mixed into every key."""
    K_CACHE = 1
    V_CACHE = 2
    Q = 3
    K_NEW = 4
    V_NEW = 5
    EMB = 6
    H_PREV0 = 7
    HEAD_W = 8
    SCHED = 9
    PAGES = 10
    RATE = 11
    CTX = 12
    GDN_C = 13
    GDN_V = 14
    GDN_ALPHA = 15
    GDN_BETA = 16
    GDN_TAPS = 17
    GDN_STATE0 = 18
    GDN_CONV0 = 19
    BB_W = 20        # synthetic backbone weights, ids (layer, tensor)
    BB_NORM = 21     # synthetic backbone norm weights, ids (layer, tensor)
    BB_EMBED = 22    # token embedding table (tied output projection)
    TOKEN0 = 23      # first token of each sequence


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _mix64_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def key(seed: int, *ids: int) -> int:
    """64-bit stream key for (seed, id0, id1, ...): a SplitMix64 chain over the ids."""
    k = _mix64_int(int(seed) + 0x9E3779B97F4A7C15)
    for i in ids:
        k = _mix64_int((k ^ ((int(i) + 1) * 0xBF58476D1CE4E5B9)) + 0x9E3779B97F4A7C15)
    return k


def raw_u64(k: int, n: int, start: int = 0) -> np.ndarray:
    """Outputs start .. start+n-1 of the SplitMix64 stream with state ``k``."""
    out = np.empty(n, dtype=np.uint64)
    kk = np.uint64(k & _MASK64)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        idx = np.arange(start + c0 + 1, start + c1 + 1, dtype=np.uint64)
        with np.errstate(over="ignore"):
            out[c0:c1] = mix64(kk + idx * GAMMA)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@functools.lru_cache(maxsize=8)
def normal_bf16_table(log2_scale: int = 0) -> np.ndarray:
    """65536 bf16 bit patterns: N(0,1) quantiles at the midpoints (j + 0.5) / 65536, times
    2^log2_scale (an exact power of two, so the scaled table is the unscaled one with its
    exponents shifted)."""
    p = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
    t = f32_to_bf16_bits((ndtri(p) * 2.0 ** log2_scale).astype(np.float32))
    t.setflags(write=False)
    return t


def normal_bf16(k: int, n: int, start: int = 0, log2_scale: int = 0) -> np.ndarray:
    """n bf16 N(0, 4^log2_scale) draws (uint16 bit patterns) from stream ``k``."""
    table = normal_bf16_table(log2_scale)
    out = np.empty(n, dtype=np.uint16)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        out[c0:c1] = table[(raw_u64(k, c1 - c0, start + c0) >> np.uint64(48)).astype(np.int64)]
    return out


def uniform_f64(k: int, n: int, start: int = 0) -> np.ndarray:
    """n uniforms in [0, 1) with 53 random bits each."""
    return (raw_u64(k, n, start) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_f32(k: int, n: int, start: int = 0) -> np.ndarray:
    """n fp32 N(0,1) draws (fp64 inverse CDF at the bin midpoint, rounded to fp32)."""
    u = ((raw_u64(k, n, start) >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    return ndtri(u).astype(np.float32)


def uniform_f32(k: int, n: int, lo: float, hi: float, start: int = 0) -> np.ndarray:
    return (lo + (hi - lo) * uniform_f64(k, n, start)).astype(np.float32)


def xavier_uniform(k: int, fan_out: int, fan_in: int) -> np.ndarray:
    """[fan_out, fan_in] fp32, U(-a, a) with a = sqrt(6 / (fan_in + fan_out))."""
    a = np.sqrt(6.0 / (fan_in + fan_out))
    u = uniform_f64(k, fan_out * fan_in)
    return (a * (2.0 * u - 1.0)).astype(np.float32).reshape(fan_out, fan_in)


def bernoulli(k: int, n: int, p) -> np.ndarray:
    """n int32 draws in {0, 1} with P(1) = p (p may be an array of length n)."""
    return (uniform_f64(k, n) < np.asarray(p, dtype=np.float64)).astype(np.int32)


def permutation(k: int, n: int) -> np.ndarray:
    """A seeded permutation of 0..n-1 (argsort of n random 64-bit keys)."""
    return np.argsort(raw_u64(k, n), kind="stable").astype(np.int32)
