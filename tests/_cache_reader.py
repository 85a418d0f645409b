"""Read a packed kvq cache arena (copied to the host) by the layout include/kvq.h documents.

Test helper only: it unpacks bytes; it computes nothing of the method.
"""
import numpy as np

TILE = 32


def _tiles(arena: np.ndarray, region: int, pair: int, tiles: int, tile_bytes: int, n_tokens: int):
    nt = (n_tokens + TILE - 1) // TILE
    start = region + pair * tiles * tile_bytes
    return arena[start:start + nt * tile_bytes].reshape(nt, tile_bytes)


ORDER_BYTE_LANE, ORDER_TOKEN, ORDER_OCTET = 0, 1, 2


def _octet_to_token_major(raw: np.ndarray, nt: int, nplanes: int) -> np.ndarray:
    """Octet-ordered planes [nt, nplanes * 512] bytes -> token-major uint8 [nt, nplanes, 32, 16].

    Octet order: [4 octets][32 words]; word x = 8t + 2m + h, byte i of it is coordinate
    32m + 16h + 4t + i, bit j of that byte is token 8 * octet + j."""
    B = raw.reshape(nt, nplanes, 4, 32, 4)
    x = np.arange(32)
    coord = (32 * ((x // 2) % 4) + 16 * (x % 2) + 4 * (x // 8))[:, None] + np.arange(4)[None, :]
    bits = (B[..., None] >> np.arange(8, dtype=np.uint8)) & 1          # [nt, np, o, x, i, j]
    per_tok = np.zeros((nt, nplanes, 4, 8, 128), dtype=np.uint8)       # [nt, np, o, j, coord]
    per_tok[..., coord] = bits.transpose(0, 1, 2, 5, 3, 4)
    per_tok = per_tok.reshape(nt, nplanes, 32, 16, 8)                  # coordinate 8k + b
    return (per_tok << np.arange(8, dtype=np.uint8)).sum(axis=-1).astype(np.uint8)


def side_fields(arena: np.ndarray, info, side: int, pair: int, n_tokens: int, m: int = 128):
    """planes uint32 [T, bits, 4], sketch uint32 [T, m/32] (or None), n16, gamma16 float64 [T]
    for one (sequence, kv-head) pair index (b * Hkv + h) and its first n_tokens tokens."""
    tile_bytes = int(info[1 + side])
    tiles = int(info[3])
    region = int(info[4 + side])
    off_planes, off_sketch, off_norm, off_gamma, bits = (int(v) for v in info[6 + 5 * side: 11 + 5 * side])
    qjl = off_norm > off_sketch  # a side without a sketch has an empty sketch block
    tb = _tiles(arena, region, pair, tiles, tile_bytes, n_tokens)
    nt = tb.shape[0]
    # keys: token-major [bits][32 tokens][16 B] or octet order (info[16]); values: byte-lane-major
    # [bits][16][32 tokens]
    order = (int(info[16]) if len(info) > 16 else ORDER_TOKEN) if side == 0 else ORDER_BYTE_LANE
    raw = tb[:, off_planes:off_planes + bits * TILE * 16]
    if order == ORDER_OCTET:
        planes = np.ascontiguousarray(_octet_to_token_major(raw, nt, bits).transpose(0, 2, 1, 3))
    elif order == ORDER_TOKEN:
        planes = np.ascontiguousarray(raw.reshape(nt, bits, TILE, 16).transpose(0, 2, 1, 3))
    else:
        planes = np.ascontiguousarray(raw.reshape(nt, bits, 16, TILE).transpose(0, 3, 1, 2))
    planes = planes.reshape(nt * TILE, bits, 16).view(np.uint32)[:n_tokens]
    n16 = np.ascontiguousarray(tb[:, off_norm:off_norm + TILE * 2]).view(np.float16).reshape(-1)[:n_tokens]
    sketch, g16 = None, np.zeros(n_tokens)
    if qjl:
        raw = tb[:, off_sketch:off_sketch + TILE * m // 8]
        if order == ORDER_OCTET:
            sk = np.ascontiguousarray(_octet_to_token_major(raw, nt, 1)).reshape(nt * TILE, m // 8)
        elif order == ORDER_TOKEN:
            sk = np.ascontiguousarray(raw).reshape(nt * TILE, m // 8)
        else:
            sk = np.ascontiguousarray(raw.reshape(nt, m // 8, TILE).transpose(0, 2, 1)).reshape(nt * TILE, m // 8)
        sketch = sk.view(np.uint32)[:n_tokens]
        g16 = np.ascontiguousarray(tb[:, off_gamma:off_gamma + TILE * 2]).view(np.float16) \
            .reshape(-1)[:n_tokens].astype(np.float64)
    return planes, sketch, n16.astype(np.float64), g16


def codes_from_planes(planes: np.ndarray) -> np.ndarray:
    """[T, bits, 4] uint32 planes -> [T, 128] integer codes (coordinate 32w+i in bit i of word w)."""
    T, bits, W = planes.shape
    shifts = np.arange(32, dtype=np.uint32)
    codes = np.zeros((T, 32 * W), dtype=np.int64)
    for p in range(bits):
        b = (planes[:, p, :, None] >> shifts[None, None, :]) & np.uint32(1)
        codes |= b.reshape(T, 32 * W).astype(np.int64) << p
    return codes


def bits_from_words(words: np.ndarray) -> np.ndarray:
    """[T, W] uint32 -> [T, 32W] 0/1."""
    T, W = words.shape
    shifts = np.arange(32, dtype=np.uint32)
    return ((words[:, :, None] >> shifts[None, None, :]) & np.uint32(1)).reshape(T, 32 * W).astype(np.int64)


def fp4_fields(arena: np.ndarray, info, seq: int, n_tokens: int, latent=512, rope=64):
    """codes uint8 [T, latent/2], scales uint8 [T, latent/16], k_rope float64 [T, rope]."""
    tile_bytes, tiles, region = int(info[1]), int(info[3]), int(info[4])
    off_codes, off_scales, off_rope = int(info[6]), int(info[7]), int(info[8])
    tb = _tiles(arena, region, seq, tiles, tile_bytes, n_tokens)
    nt = tb.shape[0]
    codes = tb[:, off_codes:off_codes + TILE * latent // 2].reshape(nt * TILE, latent // 2)[:n_tokens]
    scales = tb[:, off_scales:off_scales + TILE * latent // 16].reshape(nt * TILE, latent // 16)[:n_tokens]
    raw = np.ascontiguousarray(tb[:, off_rope:off_rope + TILE * rope * 2]).view(np.uint16).reshape(nt * TILE, rope)
    kr = (raw.astype(np.uint32) << 16).view(np.float32)[:n_tokens].astype(np.float64)
    return codes, scales, kr
