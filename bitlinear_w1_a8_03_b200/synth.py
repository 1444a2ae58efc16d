"""Seeded synthetic inputs for the BitLinear W1.58·A8 matmul.

This module only draws numbers; it holds none of the method's arithmetic
(no absmean, no absmax, no rounding to codes).  The same arrays feed both the
CUDA path and the CPU oracle, so the two never see different inputs.

Generator (fully specified, so any language can reproduce it):

* SplitMix64 used as a counter-based generator.  A stream is named by a
  key ``4*seed + role`` (role 1 = weights, 2 = activations, 3 = outlier
  channel choice); its base is ``mix64(key)`` and its i-th 64-bit draw is
  ``mix64(base + (i + 1) * GAMMA)`` (mod 2^64), with
  ``GAMMA = 0x9E3779B97F4A7C15`` and the standard SplitMix64 finaliser
  ``mix64``.  Hashing the key keeps streams of nearby seeds unrelated.
* Uniforms: ``u = ((z >> 11) + 1) * 2**-53`` lies in (0, 1].
* Normals: Box-Muller on the pair of uniforms (draws 2j, 2j+1):
  ``r = sqrt(-2 ln u0)``, ``t = 2*pi*u1``; element 2j is ``r*cos t`` and
  element 2j+1 is ``r*sin t``, evaluated in float64, scaled by the standard
  deviation, then rounded to float32 (and to bfloat16, round-to-nearest-even,
  where a bf16 tensor is asked for).
* Outlier channels: ``max(1, round(0.001*K))`` input channels, the K
  positions with the smallest draws of the role-3 stream, are multiplied by 20
  in every token.  The pages describe a few activation dimensions that are far
  larger than the rest (BitNet 三值权重实战, chenxutan.com/d/5049.html, §6.2).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22  # draws per worker block


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


ROLE_WEIGHTS, ROLE_ACT, ROLE_OUTLIERS = 1, 2, 3


def stream_key(seed: int, role: int) -> int:
    return (4 * seed + role) & 0xFFFFFFFFFFFFFFFF


def raw64(key: int, start: int, count: int) -> np.ndarray:
    """Draws ``start .. start+count-1`` of the stream named ``key``, as uint64."""
    base = _mix64(np.array([key & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0]
    idx = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(base + idx * GAMMA)


def uniform01(key: int, start: int, count: int) -> np.ndarray:
    """Uniforms in (0, 1], float64."""
    z = raw64(key, start, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def _normal_block(key: int, pair0: int, npairs: int) -> np.ndarray:
    u = uniform01(key, 2 * pair0, 2 * npairs)
    r = np.sqrt(-2.0 * np.log(u[0::2]))
    t = (2.0 * math.pi) * u[1::2]
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out


def normal_f32(key: int, count: int, std: float = 1.0) -> np.ndarray:
    """``count`` N(0, std^2) samples of stream ``key``, rounded to float32."""
    out = np.empty(count, dtype=np.float32)
    npairs = (count + 1) // 2
    blocks = [(p, min(_CHUNK, npairs - p)) for p in range(0, npairs, _CHUNK)]

    def work(b):
        p, n = b
        v = _normal_block(key, p, n) * std
        lo = 2 * p
        hi = min(count, lo + 2 * n)
        out[lo:hi] = v[: hi - lo].astype(np.float32)

    if len(blocks) == 1:
        work(blocks[0])
    else:
        with ThreadPoolExecutor(max_workers=min(len(blocks), os.cpu_count() or 1)) as ex:
            list(ex.map(work, blocks))
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_channels(seed: int, K: int) -> np.ndarray:
    """Indices of the outlier input channels for ``seed`` (role-3 stream)."""
    n = max(1, int(round(0.001 * K)))
    keys = raw64(stream_key(seed, ROLE_OUTLIERS), 0, K)
    return np.sort(np.argsort(keys, kind="stable")[:n])


def weights(seed: int, N: int, K: int, std: float) -> np.ndarray:
    """Weight matrix ``[N][K]`` float32, i.i.d. N(0, std^2) (row = out feature)."""
    return normal_f32(stream_key(seed, ROLE_WEIGHTS), N * K, std).reshape(N, K)


def activations(seed: int, M: int, K: int, std: float = 1.0, outliers: bool = False) -> np.ndarray:
    """Activation matrix ``[M][K]`` float32 (row = token), optional x20 outlier channels."""
    x = normal_f32(stream_key(seed, ROLE_ACT), M * K, std).reshape(M, K)
    if outliers:
        x[:, outlier_channels(seed, K)] *= np.float32(20.0)
    return x
