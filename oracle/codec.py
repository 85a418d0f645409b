"""Oracle codec: rotation, Lloyd-Max coding, QJL residual sketch, bit packing, 1-bit and FP4.

Test infrastructure only (see ``oracle/__init__.py``). Everything is fp64 unless a step's
definition fixes another precision (the stored norms are fp16; the FP4 scale and division are
fp32 by the format's definition).

Notation: d = head_dim, m = number of QJL sketch rows, D = diag(signs), H = Sylvester-Hadamard,
R = H D / sqrt(d) (orthonormal), S = m x d Gaussian matrix (fp32 values used exactly).
"""
from __future__ import annotations

import math

import numpy as np

from .tables import (hadamard, e4m3_decode, e4m3_encode_rn_satfinite, e2m1_decode,
                     e2m1_encode_rn_satfinite)


# ---------------------------------------------------------------------------------------------
# Stage one: random rotation, normalisation, per-coordinate Lloyd-Max code.
# "TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant and OSCAR".
# ---------------------------------------------------------------------------------------------

def rotate(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = R x = H (D x) / sqrt(d), with the explicit Hadamard matrix (no fast transform)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    H = hadamard(d)
    return (x * signs.astype(np.float64)) @ H.T / math.sqrt(d)


def unrotate(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """x = R^T y = D (H y) / sqrt(d)."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    H = hadamard(d)
    return (y @ H.T) * signs.astype(np.float64) / math.sqrt(d)


def normalise(x: np.ndarray, y: np.ndarray):
    """n = ||x||_2 and u = sqrt(d) y / n, so that each u_j is close to N(0, 1).

    A zero vector gives n = 0 and u = 0 (its reconstruction is zero whatever the codes).
    """
    d = y.shape[-1]
    n = float(np.sqrt(np.sum(np.asarray(x, dtype=np.float64) ** 2)))
    if n == 0.0:
        return 0.0, np.zeros(d)
    return n, math.sqrt(d) * y / n


def lm_code(u: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """code_j = #{k : u_j >= t_k}: the index of the Lloyd-Max cell holding u_j.

    A value exactly on a threshold goes to the upper cell.
    """
    t = np.asarray(thresholds, dtype=np.float64)
    return np.sum(np.asarray(u, dtype=np.float64)[:, None] >= t[None, :], axis=1).astype(np.int64)


# ---------------------------------------------------------------------------------------------
# Stage two: 1-bit QJL sketch of the residual.
# Same page and section: a 1-bit quantized Johnson-Lindenstrauss transform of the residual,
# giving an unbiased estimate of the attention logit with no stored normalisation constant
# other than the residual norm.
# ---------------------------------------------------------------------------------------------

def qjl_sketch(rho: np.ndarray, S: np.ndarray):
    """Returns (z, proj): z_j = 1 if (S rho)_j >= 0 else 0 (bit form of sign with sign(0) = +),
    and the fp64 projections (S rho) themselves (used by tests to locate near-zero cases)."""
    proj = np.asarray(S, dtype=np.float64) @ np.asarray(rho, dtype=np.float64)
    return (proj >= 0).astype(np.int64), proj


# ---------------------------------------------------------------------------------------------
# Bit packing: plane p of a vector holds bit p of each coordinate's code; 32-bit word w of a
# plane holds coordinates 32w .. 32w+31, coordinate 32w+i in bit i. Sign sketch words use the
# same word/bit order with bit = 1 for a non-negative projection.
# ---------------------------------------------------------------------------------------------

def pack_planes(codes: np.ndarray, bits: int) -> np.ndarray:
    """codes [d] -> uint32 [bits, d/32]."""
    codes = np.asarray(codes, dtype=np.int64)
    d = codes.shape[0]
    out = np.zeros((bits, d // 32), dtype=np.uint64)
    for p in range(bits):
        for j in range(d):
            if (codes[j] >> p) & 1:
                out[p, j // 32] |= np.uint64(1) << np.uint64(j % 32)
    return out.astype(np.uint32)


def unpack_planes(planes: np.ndarray, bits: int, d: int) -> np.ndarray:
    """Inverse of pack_planes: uint32 [bits, d/32] -> codes [d]."""
    planes = np.asarray(planes, dtype=np.uint64)
    codes = np.zeros(d, dtype=np.int64)
    for p in range(bits):
        for j in range(d):
            if (int(planes[p, j // 32]) >> (j % 32)) & 1:
                codes[j] |= 1 << p
    return codes


def pack_bits(z: np.ndarray) -> np.ndarray:
    """bits [k] (0/1) -> uint32 [k/32], element 32w+i in bit i of word w."""
    return pack_planes(np.asarray(z, dtype=np.int64), 1)[0]


def unpack_bits(words: np.ndarray, k: int) -> np.ndarray:
    return unpack_planes(np.asarray(words, dtype=np.uint32)[None, :], 1, k)


def to_f16(x: float) -> float:
    """Round to IEEE binary16 (nearest-even), returned as an fp64 value."""
    return float(np.float16(x))


def quantize_rotated(u: np.ndarray, bits: int, centroids32: np.ndarray, thresholds32: np.ndarray,
                     S: np.ndarray | None):
    """Code an already rotated and normalised vector u (stages one and two without rotation).

    Returns a dict: codes [d], planes uint32 [bits, d/32], and when S is given also
    rho [d], gamma (fp64), gamma16, z [m], z_words uint32 [m/32], proj [m].
    """
    u = np.asarray(u, dtype=np.float64)
    codes = lm_code(u, thresholds32)
    out = {"codes": codes, "planes": pack_planes(codes, bits)}
    if S is not None:
        c = np.asarray(centroids32, dtype=np.float64)[codes]
        rho = u - c
        gamma = float(np.sqrt(np.sum(rho * rho)))
        z, proj = qjl_sketch(rho, S)
        out.update(rho=rho, gamma=gamma, gamma16=to_f16(gamma), z=z, z_words=pack_bits(z),
                   proj=proj)
    return out


def quantize_vector(x: np.ndarray, bits: int, signs: np.ndarray, centroids32: np.ndarray,
                    thresholds32: np.ndarray, S: np.ndarray | None):
    """Full per-vector quantizer: rotate, normalise, Lloyd-Max code, and (if S) QJL sketch.

    Returns the dict of ``quantize_rotated`` plus y (rotated), u, n, n16.
    """
    y = rotate(x, signs)
    n, u = normalise(x, y)
    out = quantize_rotated(u, bits, centroids32, thresholds32, S)
    out.update(y=y, u=u, n=n, n16=to_f16(n))
    return out


# ---------------------------------------------------------------------------------------------
# FP4 E2M1 latent codec with one E4M3 scale per 16 channels.
# "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2", section "Numerics and
# hardware efficiency", and "DeepSeek-V4.1-Flash cuts KV cache to 890 bytes per token", FP4
# bullet. Per group of 16 channels: s = E4M3(amax / 6) rounded to nearest-even with saturation,
# each channel coded as E2M1(x / s) (nearest-even, saturating to +-6), both divisions in IEEE
# fp32. A zero scale codes the whole group as zeros.
# ---------------------------------------------------------------------------------------------

FP4_GROUP = 16


def fp4_quantize(latent: np.ndarray):
    """latent [C] (fp32-representable values) -> (packed uint8 [C/2], scales uint8 [C/16]).

    Packed byte k holds channel 2k in its low nibble and channel 2k+1 in its high nibble.
    """
    x = np.asarray(latent, dtype=np.float32)
    C = x.shape[0]
    nib = np.zeros(C, dtype=np.int64)
    scales = np.zeros(C // FP4_GROUP, dtype=np.uint8)
    for g in range(C // FP4_GROUP):
        blk = x[g * FP4_GROUP:(g + 1) * FP4_GROUP]
        amax = np.float32(np.max(np.abs(blk)))
        sc = e4m3_encode_rn_satfinite(float(np.float32(amax) / np.float32(6.0)))
        scales[g] = sc
        s = np.float32(e4m3_decode(sc))
        if s == 0:
            continue
        for i in range(FP4_GROUP):
            nib[g * FP4_GROUP + i] = e2m1_encode_rn_satfinite(float(blk[i] / s))
    packed = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    return packed, scales


def fp4_dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """(packed uint8 [C/2], scales uint8 [C/16]) -> latent estimate [C] in fp64."""
    packed = np.asarray(packed, dtype=np.int64)
    C = packed.shape[0] * 2
    out = np.zeros(C)
    for j in range(C):
        nib = (packed[j // 2] >> (4 * (j % 2))) & 0xF
        out[j] = e4m3_decode(int(scales[j // FP4_GROUP])) * e2m1_decode(int(nib))
    return out


# ---- KIVI-style asymmetric integer codes ------------------------------------------------------
#
# "TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant and OSCAR": KIVI
# quantizes keys per channel (keys have fixed outlier channels across tokens) and values per token.
# The pages give neither the group size nor the rounding; the readings used here:
#   * asymmetric b-bit integers: for a group of numbers x, z = min x and s = (max x - min x)/(2^b - 1),
#     both rounded once to fp16 (round to nearest even, saturating at 65504); the code of x is
#     rint((x - z) / s) clipped to [0, 2^b - 1], with the subtraction and the IEEE division in fp32
#     and rint rounding ties to even; s = 0 codes every x as 0. The estimate is z + s * code;
#   * keys: one (s, z) per channel over a group of KIVI_KEY_GROUP consecutive tokens;
#   * values: one (s, z) per token over its head_dim channels;
#   * the tokens of a sequence's last, incomplete key group stay in bf16 (keys and values) until
#     the group is complete.

KIVI_KEY_GROUP = 128


def _f16_sat(x):
    x = np.asarray(x, dtype=np.float32)
    return np.clip(x, -65504.0, 65504.0).astype(np.float16)


def kivi_params(lo: np.ndarray, hi: np.ndarray, bits: int):
    """fp16 scale and zero of a group from its fp32 minimum and maximum."""
    lo = np.asarray(lo, dtype=np.float32)
    hi = np.asarray(hi, dtype=np.float32)
    s16 = _f16_sat((hi - lo) / np.float32((1 << bits) - 1))
    z16 = _f16_sat(lo)
    return s16, z16


def kivi_code(x: np.ndarray, s16: np.ndarray, z16: np.ndarray, bits: int) -> np.ndarray:
    """Codes of fp32 values x against (broadcast) fp16 scale and zero, fp32 arithmetic."""
    x = np.asarray(x, dtype=np.float32)
    s = np.asarray(s16, dtype=np.float32)
    z = np.asarray(z16, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint((x - z) / np.where(s > 0, s, np.float32(1.0)))
    q = np.where(s > 0, q, 0)
    return np.clip(q, 0, (1 << bits) - 1).astype(np.int64)


def kivi_quantize_keys(K: np.ndarray, bits: int = 2):
    """One key group: K [T, d] (fp32 values) -> codes [T, d], s16 [d], z16 [d] (per channel)."""
    K = np.asarray(K, dtype=np.float32)
    s16, z16 = kivi_params(K.min(axis=0), K.max(axis=0), bits)
    return kivi_code(K, s16[None, :], z16[None, :], bits), s16, z16


def kivi_quantize_values(V: np.ndarray, bits: int = 2):
    """Values V [T, d] (fp32 values) -> codes [T, d], s16 [T], z16 [T] (per token)."""
    V = np.asarray(V, dtype=np.float32)
    s16, z16 = kivi_params(V.min(axis=1), V.max(axis=1), bits)
    return kivi_code(V, s16[:, None], z16[:, None], bits), s16, z16


def kivi_dequantize(codes: np.ndarray, s16, z16) -> np.ndarray:
    """z + s * code in fp64 (s16, z16 broadcast against codes)."""
    return np.asarray(z16, dtype=np.float64) + np.asarray(s16, dtype=np.float64) * np.asarray(codes, dtype=np.float64)
