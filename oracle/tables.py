"""Oracle tables: Gaussian Lloyd-Max quantizers, the Sylvester-Hadamard matrix, FP8/FP4 codecs.

Test infrastructure only (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import functools
import math

import numpy as np


# ---------------------------------------------------------------------------------------------
# Lloyd-Max scalar quantizer for N(0, 1)
# "TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant and OSCAR",
# stage one: after the random rotation the coordinates are close to Gaussian, so one
# precomputed optimal (Lloyd-Max) scalar quantizer serves every coordinate.
# ---------------------------------------------------------------------------------------------

def _phi(x: float) -> float:
    """Standard normal density."""
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _Phi(x: float) -> float:
    """Standard normal CDF, via erfc so that the tails keep their relative accuracy."""
    if x == -math.inf:
        return 0.0
    if x == math.inf:
        return 1.0
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def lloyd_max_gaussian(bits: int, init: str = "uniform", tol: float = 1e-15,
                       max_iter: int = 1_000_000):
    """Lloyd-Max quantizer for a standard normal source with 2**bits levels.

    Alternates the two optimality conditions until neither moves:
      * centroid condition: c_k = E[X | t_{k-1} <= X < t_k]
                                = (phi(t_{k-1}) - phi(t_k)) / (Phi(t_k) - Phi(t_{k-1}))
      * nearest-neighbour condition: t_k = (c_k + c_{k+1}) / 2
    with t_0 = -inf and t_L = +inf. ``init`` picks the starting centroids ("uniform" spreads
    them over [-2, 2], "quantile" puts them at the Gaussian quantiles), so that a test can show
    that two different starts reach the same table.

    The source density is even, so the optimal table is odd: c_k = -c_{L-1-k}. Each iteration
    averages the two halves to keep that exact in floating point, which puts the middle
    threshold at exactly 0 (fp64 round-off would otherwise leave it at +-1e-16).

    Returns (centroids, thresholds) as fp64 arrays, ascending; thresholds has 2**bits - 1
    interior entries.
    """
    levels = 1 << bits
    if init == "uniform":
        c = np.linspace(-2.0, 2.0, levels)
    elif init == "quantile":
        from statistics import NormalDist
        c = np.array([NormalDist().inv_cdf((k + 0.5) / levels) for k in range(levels)])
    else:
        raise ValueError(init)
    for _ in range(max_iter):
        t = np.concatenate(([-math.inf], 0.5 * (c[:-1] + c[1:]), [math.inf]))
        c_new = np.array([
            (_phi(t[k]) - _phi(t[k + 1])) / (_Phi(t[k + 1]) - _Phi(t[k]))
            for k in range(levels)
        ])
        c_new = 0.5 * (c_new - c_new[::-1])
        delta = float(np.max(np.abs(c_new - c)))
        c = c_new
        if delta < tol:
            break
    t = 0.5 * (c[:-1] + c[1:])
    return c, t


def lloyd_max_mse(centroids: np.ndarray) -> float:
    """Mean squared error of the Lloyd-Max quantizer on N(0,1): E[X^2] - sum_k c_k^2 P_k.

    Valid because the centroid condition holds (each c_k is the conditional mean of its cell).
    """
    c = np.asarray(centroids, dtype=np.float64)
    t = np.concatenate(([-math.inf], 0.5 * (c[:-1] + c[1:]), [math.inf]))
    p = np.array([_Phi(t[k + 1]) - _Phi(t[k]) for k in range(len(c))])
    return float(1.0 - np.sum(c * c * p))


def lloyd_max_tables_f32(bits: int):
    """The fp32 tables that both the oracle and the product quantize against.

    Centroids and thresholds (midpoints of adjacent centroids) are computed in fp64 and then
    rounded once to fp32. Returns (centroids_f32, thresholds_f32) as float32 arrays.
    """
    c, t = lloyd_max_gaussian(bits)
    return c.astype(np.float32), t.astype(np.float32)


# ---------------------------------------------------------------------------------------------
# Sylvester-Hadamard matrix (natural order): H[i, j] = (-1)^popcount(i & j)
# The random rotation of stage one is realised as R = H D / sqrt(d), D a seeded +-1 diagonal.
# ---------------------------------------------------------------------------------------------

@functools.lru_cache(maxsize=None)
def hadamard(d: int) -> np.ndarray:
    """Explicit d x d Sylvester-Hadamard matrix, entry (-1)^popcount(i & j), as fp64
    (read-only; cached)."""
    if d <= 0 or d & (d - 1):
        raise ValueError("d must be a power of two")
    i = np.arange(d)[:, None]
    j = np.arange(d)[None, :]
    x = i & j
    pop = np.zeros_like(x)
    while np.any(x):
        pop += x & 1
        x >>= 1
    H = np.where(pop % 2 == 0, 1.0, -1.0)
    H.setflags(write=False)
    return H


# ---------------------------------------------------------------------------------------------
# FP8 E4M3 ("fn" variant: bias 7, no infinities, 0x7F/0xFF are NaN, largest finite 448) and
# FP4 E2M1 (bias 1, values 0, 0.5, 1, 1.5, 2, 3, 4, 6).
# "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2", section "Numerics and
# hardware efficiency": the latent is stored as E2M1 with one scale per 16 channels.
# The scale format is E4M3 (one byte per 16 channels).
# ---------------------------------------------------------------------------------------------

def e4m3_decode(byte: int) -> float:
    """Value of one E4M3 byte per the OCP 8-bit floating point definition."""
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * (m / 8.0) * 2.0 ** (1 - 7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_decode(b) for b in range(256)], dtype=np.float64)

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_decode(nibble: int) -> float:
    """Value of one E2M1 nibble: bit 3 is the sign, bits 0-2 index the magnitude grid."""
    mag = E2M1_GRID[nibble & 0x7]
    return -mag if nibble & 0x8 else mag


def _round_to_grid_rne(mag: float, grid: np.ndarray) -> int:
    """Index of the grid value nearest to ``mag`` (>= 0), ties to the even index.

    ``grid`` is the ascending list of non-negative representable magnitudes of a format whose
    encodings, for non-negative values, are the indices themselves; the even index is the one
    with a zero mantissa LSB, which is what round-to-nearest-even means for such a format.
    Values above the largest grid value saturate to it (the "satfinite" behaviour).
    """
    if mag >= grid[-1]:
        return len(grid) - 1
    hi = int(np.searchsorted(grid, mag, side="left"))
    if grid[hi] == mag:
        return hi
    lo = hi - 1
    dlo = mag - grid[lo]
    dhi = grid[hi] - mag
    if dlo < dhi:
        return lo
    if dhi < dlo:
        return hi
    return lo if lo % 2 == 0 else hi


_E4M3_POS = np.array([e4m3_decode(b) for b in range(0x7F)], dtype=np.float64)  # 0 .. 448


def e4m3_encode_rn_satfinite(x: float) -> int:
    """Round an fp32 value to E4M3, nearest-even, saturating to +-448 (NaN never produced).

    The non-negative E4M3 encodings 0x00..0x7E are in ascending value order, so rounding the
    magnitude on that list of values and keeping the sign bit gives the encoding.
    """
    if math.isnan(x):
        raise ValueError("NaN input")
    code = _round_to_grid_rne(abs(x), _E4M3_POS)
    return code | (0x80 if (x < 0 or (x == 0 and math.copysign(1.0, x) < 0)) else 0)


def e2m1_encode_rn_satfinite(x: float) -> int:
    """Round an fp32 value to E2M1, nearest-even, saturating to +-6.

    A negative value that rounds to zero keeps its sign (nibble 0x8).
    """
    if math.isnan(x):
        raise ValueError("NaN input")
    code = _round_to_grid_rne(abs(x), E2M1_GRID)
    neg = x < 0 or (x == 0 and math.copysign(1.0, x) < 0)
    return code | (0x8 if neg else 0)
