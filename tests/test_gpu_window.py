"""GPU parity of the mixed-precision window ("TurboQuant vs OSCAR vs EpiCache", section
"Quantization frontiers: TurboQuant and OSCAR", OSCAR: sink and recent tokens stay BF16, the
history is quantized): the window's bf16 K and V are the inputs rounded to bf16, the history holds
the coded tokens of positions sink .. T - recent, and decode attention over the three segments
matches the oracle's window_decode_attention, for prefills, token-by-token appends that move tokens
out of the ring into the history, appends larger than the window, and the fused decode step."""
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_seeded_b200 as kvq
from kvq_inputs import WORKLOADS, generate
from kvq_inputs.workloads import rotation_and_sketch
from oracle import attention, tables
from tests._cache_reader import side_fields
from tests._parity import resolve_side, rel_err, REL_TOL, check_flip_rates

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvq.load()


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def window_bytes(arena, info, w, side, pair, slot):
    off = int(info[18]) + (side * w.batch * w.n_kv_heads + pair) * int(info[19]) * 128 * 2 + slot * 256
    return arena[off:off + 256].view(np.uint16)


def check(w, cache, data, lens, q, stats):
    torch.cuda.synchronize()
    out = f64(cache.decode(q))
    arena, info = cache.arena.cpu().numpy(), cache.layout()
    sink, recent = w.sink_tokens, w.recent_tokens
    assert int(info[20]) == sink and int(info[21]) == recent
    signs, S = rotation_and_sketch(w)
    ck, _ = tables.lloyd_max_tables_f32(w.k_bits)
    cv, _ = tables.lloyd_max_tables_f32(w.v_bits)
    for b, T in enumerate(lens):
        for hk in range(w.n_kv_heads):
            pair = b * w.n_kv_heads + hk
            K, V = f64(data["k"][b, hk, :T]), f64(data["v"][b, hk, :T])
            (s0, s1), (h0, h1), (r0, r1) = attention.window_segments(T, sink, recent)
            # window slots hold the bf16-rounded inputs
            for pos in list(range(s0, s1)) + list(range(r0, r1)):
                slot = pos if pos < sink else sink + (pos - sink) % recent
                for side, X in ((0, K), (1, V)):
                    want = torch.tensor(X[pos], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
                    np.testing.assert_array_equal(window_bytes(arena, info, w, side, pair, slot), want)
            nh = h1 - h0
            if nh:
                kp, ks, kn, kg = side_fields(arena, info, 0, pair, nh)
                vp, vs, vn, vg = side_fields(arena, info, 1, pair, nh)
                codes_k, n16k, g16k, zk = resolve_side(K[h0:h1], kp, ks, kn, kg, w.k_bits, signs, S if ks is not None else None, stats)
                codes_v, n16v, g16v, zv = resolve_side(V[h0:h1], vp, vs, vn, vg, w.v_bits, signs, S if vs is not None else None, stats)
                Kh = attention.dequantize_many(codes_k, n16k, ck, signs, g16k, zk, S if ks is not None else None)
                Vh = attention.dequantize_many(codes_v, n16v, cv, signs, g16v, zv, S if vs is not None else None)
            else:
                Kh = Vh = np.zeros((0, 128))
            g = w.group
            if T == 0:
                assert np.all(out[b, hk * g:(hk + 1) * g] == 0)
                continue
            ref = attention.window_decode_attention(f64(q[b, hk * g:(hk + 1) * g]), K, V, sink, recent, Kh, Vh,
                                                    1.0 / math.sqrt(128))
            err = rel_err(out[b, hk * g:(hk + 1) * g], ref)
            assert np.all(err <= REL_TOL), (b, hk, T, err.max())


@pytest.mark.parametrize("name,sink,recent,lens", [
    ("llama8b", 32, 64, [1000, 70, 20, 0]),
    ("llama8b", 0, 96, [500, 96]),
    ("llama8b", 64, 0, [400, 64]),
    ("llama70b", 64, 256, [2000, 300]),
    ("onebit", 16, 48, [700, 5]),
])
def test_window_prefill(name, sink, recent, lens):
    w = WORKLOADS[name].with_(batch=len(lens), sink_tokens=sink, recent_tokens=recent)
    data = generate(w, DEV, seqs=range(len(lens)), ctx=max(max(lens), 1))
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), max(lens) + 64)
    for b, T in enumerate(lens):
        if T:
            cache.quantize(data["k"][b:b + 1, :, :T].contiguous(), data["v"][b:b + 1, :, :T].contiguous(), seq_ids=[b])
    stats = {}
    check(w, cache, data, lens, data["q"], stats)
    check_flip_rates(stats, name)
    cache.close()


@pytest.mark.parametrize("first", [[10, 10], [10, 20], [32, 32]])
def test_window_batched_prefill_after_a_short_start(first):
    """A batched append after each sequence already holds a few tokens inside the sink: with equal
    lengths the history is coded from the input rows after the sink (whole tiles), with unequal
    lengths token by token; both against the oracle."""
    w = WORKLOADS["llama8b"].with_(batch=2, sink_tokens=32, recent_tokens=64)
    n_more = 700
    T = [first[0] + n_more, first[1] + n_more]
    data = generate(w, DEV, seqs=range(2), ctx=max(T))
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), 2, max(T) + 64)
    for b in range(2):
        cache.quantize(data["k"][b:b + 1, :, :first[b]].contiguous(), data["v"][b:b + 1, :, :first[b]].contiguous(),
                       seq_ids=[b])
    k_more = torch.stack([data["k"][b, :, first[b]:first[b] + n_more] for b in range(2)]).contiguous()
    v_more = torch.stack([data["v"][b, :, first[b]:first[b] + n_more] for b in range(2)]).contiguous()
    cache.quantize(k_more, v_more)
    stats = {}
    check(w, cache, data, T, data["q"], stats)
    check_flip_rates(stats, "window batched prefill")
    cache.close()


def test_window_appends_move_tokens_through_the_ring():
    """Token-by-token appends (each evicting one ring token into the history), then appends of 40
    and of 150 tokens (more than the window holds: some go straight to the history)."""
    w = WORKLOADS["llama8b"].with_(batch=2, sink_tokens=32, recent_tokens=64)
    T = 32 + 64 + 20 + 40 + 150
    data = generate(w, DEV, seqs=range(2), ctx=T)
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), 2, T + 64)
    stats = {}
    pos = 0
    for step in [1] * (32 + 64 + 20) + [40, 150]:
        cache.quantize(data["k"][:, :, pos:pos + step].contiguous(), data["v"][:, :, pos:pos + step].contiguous())
        pos += step
        if pos in (50, 96, 97, 116, 156):
            check(w, cache, data, [pos, pos], data["q"], stats)
    check(w, cache, data, [T, T], data["q"], stats)
    check_flip_rates(stats, "window appends")
    cache.close()


def test_window_decode_step_equals_append_then_decode():
    w = WORKLOADS["llama70b"].with_(batch=3, sink_tokens=64, recent_tokens=256)
    data = generate(w, DEV, seqs=range(3), ctx=600)
    a, b = kvq.KvqCache(kvq.cfg_for_workload(w), 3, 704), kvq.KvqCache(kvq.cfg_for_workload(w), 3, 704)
    for c in (a, b):
        c.quantize(data["k"][:, :, :500].contiguous(), data["v"][:, :, :500].contiguous())
    for t in range(500, 505):
        kn, vn = data["k"][:, :, t:t + 1].contiguous(), data["v"][:, :, t:t + 1].contiguous()
        o1 = a.step(kn, vn, data["q"]).clone()
        b.quantize(kn, vn)
        o2 = b.decode(data["q"])
        torch.cuda.synchronize()
        assert torch.equal(o1, o2)
    check(w, a, data, [505] * 3, data["q"], {})
    a.close()
    b.close()


@pytest.mark.parametrize("name,over,sink,recent,lens,kernel", [
    ("tiny", {}, 8, 40, [300], "mma"),                                   # query group 1
    ("llama8b", {"n_q_heads": 16}, 16, 48, [400, 33], "mma"),           # query group 2
    ("llama8b", {}, 512, 512, [1500, 1024, 600], "mma"),                # the largest window: 16 parts
    ("llama8b", {}, 64, 256, [900, 200], "tc"),                         # window kernel beside the tcgen05 kernels
    ("llama8b", {}, 64, 256, [900, 200], "ws"),
    ("llama8b", {"k_bits": 1, "v_mode": "lm", "v_bits": 1}, 32, 64, [600, 50], "mma"),  # beside the CUDA-core kernel
])
def test_window_decode_paths(name, over, sink, recent, lens, kernel, monkeypatch):
    """The window parts on every decode path: as extra CTAs of the mma.sync split kernel (query
    groups 1, 2, 4; 16 parts), and as their own kernel beside the tcgen05 split kernels (lockstep
    and warp-specialised) and beside the CUDA-core kernel (a code combination without a tensor-core
    instance)."""
    if kernel != "mma":
        monkeypatch.setenv("KVQ_DECODE_KERNEL", kernel)
    w = WORKLOADS[name].with_(batch=len(lens), sink_tokens=sink, recent_tokens=recent, **over)
    data = generate(w, DEV, seqs=range(len(lens)), ctx=max(lens))
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), max(lens) + 64)
    for b, T in enumerate(lens):
        cache.quantize(data["k"][b:b + 1, :, :T].contiguous(), data["v"][b:b + 1, :, :T].contiguous(), seq_ids=[b])
    stats = {}
    check(w, cache, data, lens, data["q"], stats)
    check_flip_rates(stats, name)
    cache.close()
