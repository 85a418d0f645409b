"""GPU parity of the KIVI-style codec ("TurboQuant vs OSCAR vs EpiCache", section "Quantization
frontiers: TurboQuant and OSCAR": keys per channel, values per token). Codes, scales and zeros are
bit-exact against the oracle (both sides take every rounding decision in fp32 and fp16 alike); the
incomplete last key group stays bf16; attention over [coded groups | bf16 tail] matches the oracle."""
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_seeded_b200 as kvq
from kvq_inputs import WORKLOADS, generate
from oracle import attention, codec
from tests._cache_reader import side_fields, codes_from_planes
from tests._parity import rel_err, REL_TOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvq.load()


def kivi_workload(name, batch, **over):
    w = WORKLOADS[name]
    return w.with_(batch=batch, k_mode="kivi", v_mode="kivi", k_bits=2, v_bits=2, qjl_dim=0, **over)


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check(w, cache, data, lens):
    torch.cuda.synchronize()
    out = f64(cache.decode(data["q"]))
    arena, info = cache.arena.cpu().numpy(), cache.layout()
    stats_off = None
    for b, T in enumerate(lens):
        H = T // 128 * 128
        for hk in range(w.n_kv_heads):
            pair = b * w.n_kv_heads + hk
            K = f64(data["k"][b, hk, :T]).astype(np.float32)
            V = f64(data["v"][b, hk, :T]).astype(np.float32)
            Kh = np.zeros((H, 128))
            Vh = np.zeros((H, 128))
            if H:
                kp, _, _, _ = side_fields(arena, info, 0, pair, H)
                vp, _, _, _ = side_fields(arena, info, 1, pair, H)
                kcodes, vcodes = codes_from_planes(kp), codes_from_planes(vp)
                vs, vz = value_stats(arena, info, pair, H)
                for g in range(H // 128):
                    c, s16, z16 = codec.kivi_quantize_keys(K[128 * g:128 * g + 128])
                    np.testing.assert_array_equal(kcodes[128 * g:128 * g + 128], c)
                    gs, gz = key_stats(cache, arena, pair, g)
                    np.testing.assert_array_equal(gs, s16)
                    np.testing.assert_array_equal(gz, z16)
                    Kh[128 * g:128 * g + 128] = codec.kivi_dequantize(c, s16[None], z16[None])
                c, s16, z16 = codec.kivi_quantize_values(V[:H])
                np.testing.assert_array_equal(vcodes, c)
                np.testing.assert_array_equal(vs, s16)
                np.testing.assert_array_equal(vz, z16)
                Vh = codec.kivi_dequantize(c, s16[:, None], z16[:, None])
            g = w.group
            if T == 0:
                assert np.all(out[b, hk * g:(hk + 1) * g] == 0)
                continue
            ref = attention.window_decode_attention(f64(data["q"][b, hk * g:(hk + 1) * g]), K.astype(np.float64),
                                                    V.astype(np.float64), 0, T - H, Kh, Vh, 1.0 / math.sqrt(128))
            err = rel_err(out[b, hk * g:(hk + 1) * g], ref)
            assert np.all(err <= REL_TOL), (b, hk, T, err.max())


def value_stats(arena, info, pair, n):
    tb, tiles, region = int(info[2]), int(info[3]), int(info[5])
    off_norm = int(info[13])
    s, z = [], []
    for t in range((n + 31) // 32):
        base = region + (pair * tiles + t) * tb
        s.append(arena[base + off_norm:base + off_norm + 64].view(np.float16))
        z.append(arena[base + off_norm + 64:base + off_norm + 128].view(np.float16))
    return np.concatenate(s)[:n], np.concatenate(z)[:n]


def key_stats(cache, arena, pair, g):
    # statistics region: after the window region, [pairs][groups][2][128] fp16
    info = cache.layout()
    groups = int(info[3]) // 4
    pairs = cache.batch * cache.cfg.n_kv_heads
    off = int(info[18]) + 2 * pairs * int(info[19]) * 128 * 2
    off = (off + 255) // 256 * 256 + (pair * groups + g) * 512
    st = arena[off:off + 512].view(np.float16)
    return st[:128], st[128:]


@pytest.mark.parametrize("kernel", ["mma", "tc", "cuda"])
@pytest.mark.parametrize("name,lens", [("llama8b", [1000, 128, 127, 0]), ("llama70b", [700, 300]), ("tiny", [1024]),
                                       ("llama8b", [4000, 2500, 129])])
def test_kivi_prefill(name, lens, kernel, monkeypatch):
    """The three KIVI decode kernels: the mma.sync instance (default), the tcgen05 one
    (KVQ_DECODE_KERNEL=tc) and the CUDA-core one (KVQ_DECODE_KERNEL=cuda); the longest case spans
    several splits per sequence."""
    if kernel != "mma":
        monkeypatch.setenv("KVQ_DECODE_KERNEL", kernel)
    w = kivi_workload(name, len(lens))
    data = generate(w, DEV, seqs=range(len(lens)), ctx=max(lens))
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), max(lens) + 128)
    for b, T in enumerate(lens):
        if T:
            cache.quantize(data["k"][b:b + 1, :, :T].contiguous(), data["v"][b:b + 1, :, :T].contiguous(), seq_ids=[b])
    check(w, cache, data, lens)
    cache.close()


def test_kivi_query_group_2():
    """The KIVI instance for query groups of 2 (16 query heads over 8 kv-heads)."""
    lens = [640, 200]
    w = kivi_workload("llama8b", len(lens), n_q_heads=16)
    data = generate(w, DEV, seqs=range(len(lens)), ctx=max(lens))
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), max(lens) + 128)
    for b, T in enumerate(lens):
        cache.quantize(data["k"][b:b + 1, :, :T].contiguous(), data["v"][b:b + 1, :, :T].contiguous(), seq_ids=[b])
    check(w, cache, data, lens)
    cache.close()


def test_kivi_appends_fill_groups_from_the_tail():
    """Token appends fill the bf16 tail until a group completes (coded from the tail), then appends
    of 100 and 300 tokens (groups coded from tail and input rows together)."""
    w = kivi_workload("llama8b", 2)
    T = 130 + 100 + 300
    data = generate(w, DEV, seqs=range(2), ctx=T)
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), 2, T + 128)
    pos = 0
    for step in [1] * 130 + [100, 300]:
        cache.quantize(data["k"][:, :, pos:pos + step].contiguous(), data["v"][:, :, pos:pos + step].contiguous())
        pos += step
        if pos in (127, 128, 129, 230):
            check(w, cache, data, [pos, pos])
    check(w, cache, data, [T, T])
    out1 = cache.decode(data["q"]).clone()
    # the fused step on KIVI caches is append then decode
    new = generate(w, DEV, seqs=range(2), step=0)
    out2 = cache.step(new["k"], new["v"], data["q"])
    torch.cuda.synchronize()
    assert torch.isfinite(out2).all() and not torch.equal(out1, out2)
    cache.close()
