"""The test-side arena reader against slow per-bit constructions of each plane order (the layout
include/kvq.h documents). Pure host code: no GPU, no library calls."""
import numpy as np

from tests._cache_reader import ORDER_OCTET, ORDER_TOKEN, side_fields, _octet_to_token_major

TILE = 32


def _octet_bytes_slow(tok: np.ndarray) -> np.ndarray:
    """Token-major plane bytes [32 tokens, 16] -> octet order, 512 bytes, one bit at a time."""
    out = np.zeros(512, dtype=np.uint8)
    for tk in range(32):
        o, j = divmod(tk, 8)
        for c in range(128):
            bit = (int(tok[tk, c // 8]) >> (c % 8)) & 1
            m, r = divmod(c, 32)
            h, r = divmod(r, 16)
            t, i = divmod(r, 4)
            x = 8 * t + 2 * m + h
            out[o * 128 + 4 * x + i] |= bit << j
    return out


def test_octet_order_round_trip():
    rng = np.random.default_rng(5)
    tok = rng.integers(0, 256, size=(3, 2, 32, 16), dtype=np.uint8)  # [tile, plane, token, byte]
    raw = np.stack([np.concatenate([_octet_bytes_slow(tok[n, p]) for p in range(2)]) for n in range(3)])
    np.testing.assert_array_equal(_octet_to_token_major(raw, 3, 2), tok)


def test_side_fields_reads_octet_keys():
    """A one-tile arena in octet order decodes to the token-major words it was built from."""
    rng = np.random.default_rng(6)
    bits = 2
    tok = rng.integers(0, 256, size=(bits, 32, 16), dtype=np.uint8)
    sk = rng.integers(0, 256, size=(32, 16), dtype=np.uint8)
    norms = rng.standard_normal(32).astype(np.float16)
    gam = rng.random(32).astype(np.float16)
    tile = np.concatenate([_octet_bytes_slow(tok[p]) for p in range(bits)] + [_octet_bytes_slow(sk)] +
                          [norms.view(np.uint8), gam.view(np.uint8)])
    tile_bytes = (tile.size + 15) // 16 * 16
    arena = np.zeros(tile_bytes, dtype=np.uint8)
    arena[:tile.size] = tile
    off_sketch = bits * 512
    info = np.zeros(18, dtype=np.int64)
    info[:11] = [TILE, tile_bytes, 0, 1, 0, 0, 0, off_sketch, off_sketch + 512, off_sketch + 576, bits]
    info[16] = ORDER_OCTET
    planes, sketch, n16, g16 = side_fields(arena, info, 0, 0, 32)
    np.testing.assert_array_equal(planes, np.ascontiguousarray(tok.transpose(1, 0, 2)).view(np.uint32))
    np.testing.assert_array_equal(sketch, sk.view(np.uint32))
    np.testing.assert_array_equal(n16, norms.astype(np.float64))
    np.testing.assert_array_equal(g16, gam.astype(np.float64))
    # the same tile in token order reads back identically
    tile_t = np.concatenate([tok.reshape(-1), sk.reshape(-1), norms.view(np.uint8), gam.view(np.uint8)])
    arena_t = np.zeros(tile_bytes, dtype=np.uint8)
    arena_t[:tile_t.size] = tile_t
    info[16] = ORDER_TOKEN
    planes_t, sketch_t, _, _ = side_fields(arena_t, info, 0, 0, 32)
    np.testing.assert_array_equal(planes_t, planes)
    np.testing.assert_array_equal(sketch_t, sketch)
