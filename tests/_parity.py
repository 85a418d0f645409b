"""Shared parity machinery for the GPU tests: run the oracle on the same inputs and compare.

The oracle quantises every vector itself. Where a floating-point result decides a stored
integer -- a coordinate within 1e-5 of a Lloyd-Max threshold, an fp16 norm that fp32 and fp64
round to neighbouring values, a sketch projection within the fp32 error bound of zero -- the
two sides may legitimately disagree; those cases (and only those) are checked to be
rounding-level and then resolved to the kernel's decision, so that attention is compared over
identical codes.
"""
import math

import numpy as np

from oracle import attention, codec, tables
from tests._cache_reader import side_fields, codes_from_planes, bits_from_words

BOUNDARY = 1e-5          # |u - t_k| below which a code may differ by one level
REL_TOL = 2e-3           # attention: ||out - ref||_inf / ||ref||_inf per (sequence, head)


def fp16_ulp(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def resolve_side(x, planes_g, sketch_g, n16_g, g16_g, bits, signs, S, stats):
    """Oracle fields of one side for vectors x [T, d] (fp64), resolved against the kernel's.

    Returns codes [T, d], n16 [T], gamma16 [T], z [T, m] (or None) for the oracle to use.
    """
    c32, t32 = tables.lloyd_max_tables_f32(bits)
    d = x.shape[1]
    y = codec.rotate(x, signs)
    n = np.sqrt(np.sum(x * x, axis=1))
    u = np.where(n[:, None] > 0, math.sqrt(d) * y / np.where(n > 0, n, 1)[:, None], 0.0)
    codes_o = codec.lm_code(u.reshape(-1), t32).reshape(u.shape)
    codes_g = codes_from_planes(planes_g)
    diff = codes_o != codes_g
    if diff.any():
        dist = np.min(np.abs(u[..., None] - t32.astype(np.float64)[None, None, :]), axis=-1)
        assert np.all(dist[diff] < BOUNDARY), f"code mismatch away from a threshold: {dist[diff].max()}"
        assert np.all(np.abs(codes_o - codes_g)[diff] == 1)
    stats["code_flips"] = stats.get("code_flips", 0) + int(diff.sum())
    stats["coords"] = stats.get("coords", 0) + diff.size
    codes = codes_g  # identical to the oracle's except the boundary cases just checked

    n16_o = n.astype(np.float16).astype(np.float64)
    dn = np.abs(n16_o - n16_g)
    assert np.all(dn <= fp16_ulp(n) * 1.0001), f"norm differs by more than one fp16 ulp: {dn.max()}"
    n16 = n16_g

    z, g16 = None, np.zeros(len(x))
    if sketch_g is not None:
        rho = u - c32.astype(np.float64)[codes]
        gamma = np.sqrt(np.sum(rho * rho, axis=1))
        g16_o = gamma.astype(np.float16).astype(np.float64)
        dg = np.abs(g16_o - g16_g)
        assert np.all(dg <= fp16_ulp(gamma) * 1.0001), f"residual norm off by > 1 ulp: {dg.max()}"
        g16 = g16_g
        Sd = np.asarray(S, dtype=np.float64)
        proj = rho @ Sd.T
        z_o = (proj >= 0).astype(np.int64)
        z_g = bits_from_words(sketch_g)
        # fp32 error bound of the kernel's projection: its u carries ~1e-6 relative error
        # (bounded by BOUNDARY) and the 128-term fp32 dot product adds n*eps*sum|S||rho|.
        tol = BOUNDARY * np.abs(Sd).sum(axis=1)[None, :] + 4 * 128 * 2.0 ** -24 * (np.abs(rho) @ np.abs(Sd).T)
        zd = z_o != z_g
        assert np.all(np.abs(proj[zd]) < tol[zd]), "sketch bit differs away from zero"
        stats["sketch_flips"] = stats.get("sketch_flips", 0) + int(zd.sum())
        stats["sketch_bits"] = stats.get("sketch_bits", 0) + zd.size
        z = z_g
    return codes, n16, g16, z


def pair_reference(w, arena, info, b, hk, T, K, V, q, signs, S, stats):
    """Oracle decode output [g, d] for one (sequence b, kv-head hk) over its first T tokens.

    K, V: [T, d] fp64 inputs of that pair; q: [g, d] fp64 query heads of the group.
    """
    pair = b * w.n_kv_heads + hk
    if np.ndim(signs) == 2:  # one rotation diagonal per kv-head
        signs = signs[hk]
    kp, ks, kn, kg = side_fields(arena, info, 0, pair, T)
    vp, vs, vn, vg = side_fields(arena, info, 1, pair, T)
    kq = S if ks is not None else None
    vq = S if vs is not None else None
    codes_k, n16k, g16k, zk = resolve_side(K, kp, ks, kn, kg, w.k_bits, signs, kq, stats)
    codes_v, n16v, g16v, zv = resolve_side(V, vp, vs, vn, vg, w.v_bits, signs, vq, stats)
    ck, _ = tables.lloyd_max_tables_f32(w.k_bits)
    cv, _ = tables.lloyd_max_tables_f32(w.v_bits)
    Kh = attention.dequantize_many(codes_k, n16k, ck, signs, g16k, zk, kq)
    Vh = attention.dequantize_many(codes_v, n16v, cv, signs, g16v, zv, vq)
    return attention.decode_attention(q, Kh, Vh, 1.0 / math.sqrt(w.head_dim))


MAX_FLIP_RATE = 1e-3     # rounding-level code / sign decisions allowed, per decision compared


def check_flip_rates(stats, where=""):
    """Bound how often the rounding-level exceptions above were taken: at most MAX_FLIP_RATE of
    the codes and of the sketch sign bits compared may differ from the oracle's decision."""
    print(f"{where}: code flips {stats.get('code_flips', 0)}/{stats.get('coords', 0)}, "
          f"sketch flips {stats.get('sketch_flips', 0)}/{stats.get('sketch_bits', 0)}")
    assert stats.get("code_flips", 0) <= MAX_FLIP_RATE * max(1, stats.get("coords", 0)), stats
    assert stats.get("sketch_flips", 0) <= MAX_FLIP_RATE * max(1, stats.get("sketch_bits", 0)), stats


def rel_err(out, ref):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return np.max(np.abs(out - ref), axis=-1) / np.max(np.abs(ref), axis=-1)
