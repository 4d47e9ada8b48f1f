"""Counter-based SplitMix64 + Box-Muller normal draws (numpy, vectorised)."""

from __future__ import annotations

import numpy as np

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def splitmix64(seed: int, count: int, offset: int = 0) -> np.ndarray:
    """Draws ``offset .. offset+count-1`` of the SplitMix64 stream seeded with ``seed``."""
    with np.errstate(over="ignore"):
        idx = np.arange(offset + 1, offset + count + 1, dtype=np.uint64)
        state = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * GOLDEN_GAMMA
        return _mix64(state)


def stream_seed(seed: int, name: str) -> int:
    """Derives an independent stream seed for tensor ``name`` from a run seed."""
    h = 0xCBF29CE484222325  # FNV-1a over the name, then one SplitMix64 draw
    for ch in name.encode():
        h ^= ch
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return int(splitmix64(seed ^ h, 1)[0])


def uniform01(seed: int, count: int) -> np.ndarray:
    """Uniform float64 draws in the open interval (0, 1)."""
    z = splitmix64(seed, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def _box_muller(seed: int, p0: int, p1: int, out: np.ndarray) -> None:
    """Pairs p0 .. p1-1 of the stream (uniform draws 2p, 2p+1) into out[2p0 : 2p1]."""
    z = splitmix64(seed, 2 * (p1 - p0), offset=2 * p0)
    u = ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    u1, u2 = u[0::2], u[1::2]
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    seg = out[2 * p0:2 * p1]
    seg[0::2] = rad * np.cos(ang)
    seg[1::2] = rad * np.sin(ang)


_BLOCK_PAIRS = 1 << 20  # a multiple of the SIMD width, so every draw is computed the same way


def normal(seed: int, count: int, std: float = 1.0) -> np.ndarray:
    """float64 N(0, std^2) draws by Box-Muller on consecutive uniform pairs.

    Large draws are split into blocks of pairs computed on a thread pool (numpy
    releases the GIL in its loops); each draw depends only on its index, so the
    result is the same for any split."""
    pairs = (count + 1) // 2
    out = np.empty(2 * pairs, dtype=np.float64)
    blocks = [(p, min(pairs, p + _BLOCK_PAIRS)) for p in range(0, pairs, _BLOCK_PAIRS)]
    if len(blocks) > 1:
        from concurrent.futures import ThreadPoolExecutor
        import os
        with ThreadPoolExecutor(max_workers=min(len(blocks), os.cpu_count() or 1)) as ex:
            list(ex.map(lambda b: _box_muller(seed, b[0], b[1], out), blocks))
    elif blocks:
        _box_muller(seed, 0, pairs, out)
    return out[:count] * std


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (b & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    r = np.where(nan, (b >> np.uint32(16)) | np.uint32(0x40), r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f32(seed: int, shape, std: float) -> np.ndarray:
    n = int(np.prod(shape))
    return normal(seed, n, std).astype(np.float32).reshape(shape)


def normal_bf16_bits(seed: int, shape, std: float) -> np.ndarray:
    return f32_to_bf16_bits(normal_f32(seed, shape, std)).reshape(shape)
