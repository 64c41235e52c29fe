"""Seeded synthetic inputs for the BitLinear path (host side, numpy only).

This module draws random numbers and formats them as the path's input dtypes.
It holds none of the method's arithmetic (no masking, no quantisation, no
matmul), so both the CUDA path and the CPU oracle may consume what it makes.

Generator (stated so that anyone can re-implement it bit for bit):

* ``splitmix64``: counter ``i`` (0-based) of stream ``seed`` gives
  ``z = seed*2^32 + stream_salt + (i+1)*0x9E3779B97F4A7C15 (mod 2^64)`` passed
  through the splitmix64 finaliser
  ``z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31``.
* uniform in [0,1): ``(z >> 11) * 2^-53``; uniform in (0,1]: ``((z >> 11) + 1) * 2^-53``.
* normal: Box-Muller in fp64 on draws ``2j`` (u1, in (0,1]) and ``2j+1`` (u2):
  ``sqrt(-2 ln u1) * cos(2 pi u2)``.
* outliers: element ``j`` is multiplied by 20 when draw ``j`` of the outlier
  stream is below 0.01 (Bernoulli(0.01)), before rounding to bf16.
* casts: fp64 -> fp32 by IEEE round-to-nearest-even (numpy), fp32 -> bf16 by
  round-to-nearest-even on the bit pattern.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

# stream salts keep the normal stream and the outlier stream of one seed apart
SALT_NORMAL = 0x1
SALT_OUTLIER = 0x2


def splitmix64(seed: int, salt: int, start: int, count: int) -> np.ndarray:
    """Counters ``start .. start+count-1`` of stream (seed, salt) as uint64."""
    base = np.uint64(((seed << 32) + salt) & 0xFFFFFFFFFFFFFFFF)
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = base + i * _GOLDEN
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def uniform01(seed: int, salt: int, start: int, count: int) -> np.ndarray:
    z = splitmix64(seed, salt, start, count)
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _chunked(count: int, fill) -> np.ndarray:
    """Fill an fp64 array chunk by chunk; chunks are independent (counter-based
    streams), so they run on a thread pool without changing any value."""
    out = np.empty(count, dtype=np.float64)
    starts = list(range(0, count, _CHUNK))
    if len(starts) <= 1:
        for s in starts:
            fill(out, s, min(_CHUNK, count - s))
        return out
    with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
        list(ex.map(lambda s: fill(out, s, min(_CHUNK, count - s)), starts))
    return out


def normal_f64(seed: int, count: int, std: float = 1.0) -> np.ndarray:
    """``count`` iid N(0, std^2) samples in fp64 (std is the standard deviation)."""
    def fill(out, s, c):
        z = splitmix64(seed, SALT_NORMAL, 2 * s, 2 * c)
        u1 = ((z[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
        u2 = (z[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        out[s:s + c] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2) * std
    return _chunked(count, fill)


def outlier_factor(seed: int, count: int, p: float = 0.01, scale: float = 20.0) -> np.ndarray:
    """Per-element factor: ``scale`` with probability ``p``, else 1."""
    def fill(out, s, c):
        u = uniform01(seed, SALT_OUTLIER, s, c)
        out[s:s + c] = np.where(u < p, scale, 1.0)
    return _chunked(count, fill)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even. No NaN handling
    is needed: the generator never produces NaN or Inf."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def latent_weight(seed: int, n_out: int, k_in: int, std: float = 0.02) -> np.ndarray:
    """Latent fp32 weights [n_out, k_in] ~ N(0, std^2)."""
    return normal_f64(seed, n_out * k_in, std).astype(np.float32).reshape(n_out, k_in)


def activation_bf16(seed: int, t: int, k: int, std: float = 1.0, outliers: bool = True) -> np.ndarray:
    """bf16 bit patterns [t, k]: N(0, std^2), optionally with 1% of entries x20."""
    v = normal_f64(seed, t * k, std)
    if outliers:
        v *= outlier_factor(seed, t * k)
    return f32_to_bf16_bits(v.astype(np.float32)).reshape(t, k)


def config_seed(config_index: int, tensor_index: int) -> int:
    """Seed of tensor ``tensor_index`` of workload ``config_index`` (1-based);
    the first workload starts at seed 0."""
    return (config_index - 1) * 1000 + tensor_index
