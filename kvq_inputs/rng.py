"""Counter-based random numbers (no method arithmetic).

Generator definition (fixed here, used by everything):
  mix(z)   = splitmix64 finaliser: z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
             z *= 0x94D049BB133111EB; z ^= z >> 31            (all mod 2^64)
  h(s, i)  = mix(s + (i + 1) * 0x9E3779B97F4A7C15)           (the i-th draw of stream s)
  U(s, i)  = (h(s, i) >> 11) * 2^-53                           (uniform in [0, 1))

Rotation signs: D_i = -1 if h(rot_seed, i) & 1 else +1, i < d (per-head rotation: head h takes
                i = h d .. h d + d - 1).
QJL matrix:     S[j, i] = fp32( sqrt(-2 ln(1 - U(s, 2k))) cos(2 pi U(s, 2k + 1)) ), k = j d + i.
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, idx: np.ndarray) -> np.ndarray:
    """h(seed, idx) for an array of counters (uint64 wrap-around arithmetic)."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (np.asarray(idx, dtype=np.uint64) + np.uint64(1)) * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform53(seed: int, idx: np.ndarray) -> np.ndarray:
    return (splitmix64(seed, idx) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def rotation_signs(rot_seed: int, d: int) -> np.ndarray:
    """+-1 diagonal of the randomized Hadamard rotation, int8 [d]."""
    bit = splitmix64(rot_seed, np.arange(d, dtype=np.uint64)) & np.uint64(1)
    return np.where(bit == 1, -1, 1).astype(np.int8)


def rotation_signs_per_head(rot_seed: int, heads: int, d: int) -> np.ndarray:
    """One +-1 diagonal per KV head, int8 [heads, d]: head h takes draws h*d .. h*d + d - 1 of the
    same stream (head 0's diagonal is rotation_signs(rot_seed, d))."""
    return rotation_signs(rot_seed, heads * d).reshape(heads, d)


def qjl_matrix(qjl_seed: int, m: int, d: int) -> np.ndarray:
    """i.i.d. N(0,1) sketch matrix rounded to fp32, float32 [m, d]."""
    k = np.arange(m * d, dtype=np.uint64)
    u1 = uniform53(qjl_seed, 2 * k)
    u2 = uniform53(qjl_seed, 2 * k + 1)
    g = np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)
    return g.astype(np.float32).reshape(m, d)
