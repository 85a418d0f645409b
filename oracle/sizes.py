"""Oracle KV-size arithmetic.

Test infrastructure only (see ``oracle/__init__.py``).

"TurboQuant vs OSCAR vs EpiCache", section "KV-cache bottleneck": a bf16 cache holds, per
token, layers x kv_heads x head_dim x 2 tensors (K and V) x 2 bytes. The page's own example is
a 70B GQA model (80 layers, 8 KV heads, head_dim 128).
"""
from __future__ import annotations


def bf16_kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int) -> int:
    return layers * kv_heads * head_dim * 2 * 2


def lm_vector_bytes(head_dim: int, bits: int, qjl_dim: int) -> int:
    """Packed bytes of one quantised vector: bits planes of head_dim bits, an fp16 norm, and,
    with a sketch, qjl_dim sign bits plus an fp16 residual norm."""
    b = bits * head_dim // 8 + 2
    if qjl_dim:
        b += qjl_dim // 8 + 2
    return b


def fp4_token_bytes(latent_dim: int, rope_dim: int) -> int:
    """FP4 latent (two channels per byte) + one E4M3 scale byte per 16 channels + bf16 RoPE."""
    return latent_dim // 2 + latent_dim // 16 + 2 * rope_dim
