"""Oracle dequantisation and decode attention.

Test infrastructure only (see ``oracle/__init__.py``).

The reference computation materialises every dequantised key and value in the ORIGINAL
(unrotated) domain and runs plain softmax attention on them in fp64 with a two-pass
max-subtracted softmax. A second, rotated-domain formulation (query rotated and sketched once,
logits from centroids plus the sketch correction, value sketch folded in after the weighted
sum) is kept separately so that tests can check that the two agree.
"""
from __future__ import annotations

import math

import numpy as np

from .codec import rotate, unrotate, unpack_planes, unpack_bits, fp4_dequantize


def qjl_constant(m: int) -> float:
    """sqrt(pi/2) / m: with s ~ N(0, I), E[<s, a> sign(<s, rho>)] = sqrt(2/pi) <a, rho>/||rho||,
    so sqrt(pi/2)/m * ||rho|| * sum_j (S a)_j sign((S rho)_j) is an unbiased estimate of
    <a, rho> ("TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant
    and OSCAR", stage two)."""
    return math.sqrt(math.pi / 2.0) / m


def dequantize_rotated(codes: np.ndarray, n16: float, centroids32: np.ndarray,
                       gamma16: float | None = None, z: np.ndarray | None = None,
                       S: np.ndarray | None = None) -> np.ndarray:
    """Rotated-domain estimate of one vector: (n/sqrt(d)) (c[code] + k gamma S^T z_pm).

    z_pm = 2 z - 1 in {-1, +1}; the sketch term is present only when z and S are given.
    """
    d = codes.shape[0]
    est = np.asarray(centroids32, dtype=np.float64)[codes].copy()
    if z is not None:
        Sd = np.asarray(S, dtype=np.float64)
        zpm = 2.0 * np.asarray(z, dtype=np.float64) - 1.0
        est += qjl_constant(Sd.shape[0]) * gamma16 * (Sd.T @ zpm)
    return (n16 / math.sqrt(d)) * est


def dequantize(codes, n16, centroids32, signs, gamma16=None, z=None, S=None) -> np.ndarray:
    """Original-domain estimate x_hat = R^T (rotated-domain estimate)."""
    return unrotate(dequantize_rotated(codes, n16, centroids32, gamma16, z, S), signs)


def dequantize_many(codes, n16, centroids32, signs, gamma16=None, z=None, S=None) -> np.ndarray:
    """``dequantize`` applied to every row: codes [T, d], n16 [T], gamma16 [T], z [T, m] (0/1)
    -> x_hat [T, d]. The same arithmetic, written over a token axis."""
    codes = np.asarray(codes, dtype=np.int64)
    d = codes.shape[1]
    est = np.asarray(centroids32, dtype=np.float64)[codes]
    if z is not None:
        Sd = np.asarray(S, dtype=np.float64)
        zpm = 2.0 * np.asarray(z, dtype=np.float64) - 1.0
        est = est + qjl_constant(Sd.shape[0]) * np.asarray(gamma16, dtype=np.float64)[:, None] * (zpm @ Sd)
    est = est * (np.asarray(n16, dtype=np.float64) / math.sqrt(d))[:, None]
    return unrotate(est, signs)


def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """out = sum_t p_t V_t with p = softmax(scale * K q); two-pass, max-subtracted, fp64.

    q [dq], K [T, dq], V [T, dv]. T = 0 is rejected (attention over nothing is undefined).
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        raise ValueError("empty context")
    logits = scale * (K @ np.asarray(q, dtype=np.float64))
    m = np.max(logits)
    w = np.exp(logits - m)
    return (w[:, None] * V).sum(axis=0) / w.sum()


def softmax_state(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Softmax state of attention over one part of a context, fp64: (m, l, o) with
    m = max_t l_t, l = sum_t exp(l_t - m), o = sum_t exp(l_t - m) V_t, l_t = scale <q, K_t>.
    A part with no tokens has the state (-inf, 0, 0)."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return -math.inf, 0.0, np.zeros(V.shape[1])
    logits = scale * (K @ np.asarray(q, dtype=np.float64))
    m = float(np.max(logits))
    w = np.exp(logits - m)
    return m, float(w.sum()), (w[:, None] * V).sum(axis=0)


def merge_softmax_states(states):
    """Softmax attention over the union of disjoint context parts from their states:
    out = sum_i exp(m_i - M) o_i / sum_i exp(m_i - M) l_i, M = max_i m_i (zeros if every part is
    empty)."""
    M = max(m for m, _, _ in states)
    if M == -math.inf:
        return np.zeros_like(states[0][2])
    num = sum(math.exp(m - M) * o for m, _, o in states if m != -math.inf)
    den = sum(math.exp(m - M) * l for m, l, _ in states if m != -math.inf)
    return num / den


def decode_attention(q_heads: np.ndarray, K_hat: np.ndarray, V_hat: np.ndarray,
                     scale: float) -> np.ndarray:
    """GQA decode for one (sequence, kv-head): every query head of the group attends to the same
    dequantised keys and values. q_heads [g, dq] -> out [g, dv]."""
    return np.stack([softmax_attention(qh, K_hat, V_hat, scale) for qh in q_heads])


def decode_attention_rotated(q_heads, codes_k, n16_k, gamma16_k, z_k, codes_v, n16_v,
                             gamma16_v, z_v, centroids_k, centroids_v, signs, S, scale):
    """Rotated-domain decode for one (sequence, kv-head), step by step:

      q_r = R q, s_q = S q_r                                  (once per query head)
      l_t = scale (n_t/sqrt d) [<q_r, c_t> + k gamma_t <s_q, z_t>]      (logits)
      p   = softmax(l)                                         (two-pass, fp64)
      o_r = sum_t p_t (n_t/sqrt d) c_t + S^T sum_t p_t (n_t/sqrt d) k gamma_t z_t
      out = R^T o_r

    z_k / z_v may be None (no sketch on that side). Arrays are per token: codes [T, d],
    n16 [T], gamma16 [T], z [T, m] (0/1).
    """
    d = codes_k.shape[1]
    T = codes_k.shape[0]
    Sd = None if S is None else np.asarray(S, dtype=np.float64)
    kappa = None if S is None else qjl_constant(Sd.shape[0])
    outs = []
    for q in q_heads:
        q_r = rotate(q, signs)
        s_q = None if Sd is None else Sd @ q_r
        logits = np.empty(T)
        for t in range(T):
            dot = float(np.dot(q_r, np.asarray(centroids_k, dtype=np.float64)[codes_k[t]]))
            if z_k is not None:
                dot += kappa * gamma16_k[t] * float(np.dot(s_q, 2.0 * z_k[t] - 1.0))
            logits[t] = scale * n16_k[t] / math.sqrt(d) * dot
        p = np.exp(logits - logits.max())
        p /= p.sum()
        o_r = np.zeros(d)
        acc_z = None if z_v is None else np.zeros(Sd.shape[0])
        for t in range(T):
            w = p[t] * n16_v[t] / math.sqrt(d)
            o_r += w * np.asarray(centroids_v, dtype=np.float64)[codes_v[t]]
            if z_v is not None:
                acc_z += w * kappa * gamma16_v[t] * (2.0 * z_v[t] - 1.0)
        if z_v is not None:
            o_r += Sd.T @ acc_z
        outs.append(unrotate(o_r, signs))
    return np.stack(outs)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to bfloat16 (round to nearest, ties to even), returned as fp64: the
    precision the full-precision window of a mixed-precision cache keeps its tokens in."""
    import torch
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def window_segments(T: int, sink: int, recent: int):
    """Token ranges of a mixed-precision cache of T tokens ("TurboQuant vs OSCAR vs EpiCache",
    section "Quantization frontiers: TurboQuant and OSCAR", OSCAR's mixed-precision paged memory:
    sink tokens and recent tokens stay in BF16, the history in between is quantized):
    sink = [0, min(T, sink)), history = [sink, max(sink, T - recent)), recent = [max(sink, T - recent), T)."""
    s_end = min(T, sink)
    r_begin = max(sink, T - recent) if T > sink else s_end
    return (0, s_end), (s_end, max(s_end, r_begin)), (max(s_end, r_begin), T)


def window_decode_attention(q_heads: np.ndarray, K: np.ndarray, V: np.ndarray, sink: int, recent: int,
                            K_hist_hat: np.ndarray, V_hist_hat: np.ndarray, scale: float) -> np.ndarray:
    """Decode over a mixed-precision cache: keys and values of the sink and recent tokens are the
    inputs rounded to bf16, those of the history tokens are their dequantised estimates
    (K_hist_hat / V_hist_hat, one row per history token in order); softmax attention over all of them.
    q_heads [g, d], K, V [T, d] (inputs) -> out [g, d]."""
    T = K.shape[0]
    (s0, s1), (h0, h1), (r0, r1) = window_segments(T, sink, recent)
    assert K_hist_hat.shape[0] == h1 - h0 and V_hist_hat.shape[0] == h1 - h0
    Keff = np.concatenate([bf16_round(K[s0:s1]), np.asarray(K_hist_hat, np.float64), bf16_round(K[r0:r1])])
    Veff = np.concatenate([bf16_round(V[s0:s1]), np.asarray(V_hist_hat, np.float64), bf16_round(V[r0:r1])])
    return decode_attention(q_heads, Keff, Veff, scale)


def fp4_dequantize_many(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """``fp4_dequantize`` applied to every row: packed uint8 [T, C/2], scales uint8 [T, C/16]
    -> [T, C], through the oracle's own E2M1/E4M3 decode tables."""
    from .tables import E4M3_TABLE, e2m1_decode
    e2m1 = np.array([e2m1_decode(n) for n in range(16)])
    packed = np.asarray(packed, dtype=np.int64)
    T, half = packed.shape
    nib = np.empty((T, 2 * half), dtype=np.int64)
    nib[:, 0::2] = packed & 0xF
    nib[:, 1::2] = packed >> 4
    sc = E4M3_TABLE[np.asarray(scales, dtype=np.int64)]
    return e2m1[nib] * np.repeat(sc, 16, axis=1)


def mla_decode_attention_many(q, latent_packed, latent_scales, k_rope, scale, heads=None):
    """``mla_decode_attention`` over a long context, for the query heads listed in ``heads``
    (default all): the same keys/values, dequantised once for all tokens."""
    lat = fp4_dequantize_many(latent_packed, latent_scales)
    K = np.concatenate([lat, np.asarray(k_rope, dtype=np.float64)], axis=1)
    q = np.asarray(q, dtype=np.float64)
    hs = range(q.shape[0]) if heads is None else heads
    return np.stack([softmax_attention(q[h], K, lat, scale) for h in hs])


def mla_decode_attention(q: np.ndarray, latent_packed: np.ndarray, latent_scales: np.ndarray,
                         k_rope: np.ndarray, scale: float) -> np.ndarray:
    """MLA-style decode with an absorbed query over an FP4 latent cache.

    "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2", section "CSA2": one latent
    vector per token is shared by every attention head. Keys are [latent_hat ; k_rope] and the
    values are latent_hat itself:
      l_{h,t} = scale (q_lat[h] . latent_hat_t + q_rope[h] . k_rope_t)
      out_h   = sum_t softmax_t(l_h) latent_hat_t
    q [Hq, C + R], latent_packed [T, C/2] uint8, latent_scales [T, C/16] uint8,
    k_rope [T, R]. Returns out [Hq, C].
    """
    T = latent_packed.shape[0]
    C = latent_packed.shape[1] * 2
    lat = np.stack([fp4_dequantize(latent_packed[t], latent_scales[t]) for t in range(T)])
    K = np.concatenate([lat, np.asarray(k_rope, dtype=np.float64)], axis=1)
    return np.stack([softmax_attention(qh, K, lat, scale) for qh in np.asarray(q, np.float64)])


def unpack_lm_cache_vector(planes, bits, d):
    """Convenience re-export for tests that read stored planes."""
    return unpack_planes(planes, bits, d)


def unpack_sketch(words, m):
    return unpack_bits(words, m)
