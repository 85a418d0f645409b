"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded inputs.

Covers bit-exact packing on shared rotated fp32 inputs, end-to-end codes with the 1e-5
boundary rule, attention within 2e-3 relative over identical codes for every workload shape
(small contexts with ragged tails, then sampled pairs at full size), FP4 codes bit-exact, and
the edge cases: one token, empty sequences, token-by-token appends, capacity overflow.
"""
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_seeded_b200 as kvq
from kvq_inputs import WORKLOADS, generate
from kvq_inputs.workloads import rotation_and_sketch
from oracle import codec, tables, attention
from tests._cache_reader import fp4_fields, side_fields
from tests._parity import pair_reference, rel_err, REL_TOL, BOUNDARY, check_flip_rates

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvq.load()


def new_cache(w, batch, capacity):
    signs, S = rotation_and_sketch(w)
    return kvq.KvqCache(kvq.cfg_for_workload(w), batch, capacity, signs, S), signs, S


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_same_token_fields(c1, c2, w, lens):
    """Two caches hold the same codes, sign words and norms for every stored token (bytes past a
    sequence's last token are whatever the arena held and are not compared)."""
    A, B = c1.arena.cpu().numpy(), c2.arena.cpu().numpy()
    i1, i2 = c1.layout(), c2.layout()
    for b, L in enumerate(lens):
        for hk in range(w.n_kv_heads):
            for side in (0, 1):
                f1 = side_fields(A, i1, side, b * w.n_kv_heads + hk, L)
                f2 = side_fields(B, i2, side, b * w.n_kv_heads + hk, L)
                for x, y in zip(f1, f2):
                    if x is not None:
                        np.testing.assert_array_equal(x, y)


# ---------------------------------------------------------------- packing on shared u

@pytest.mark.parametrize("bits,qjl", [(2, True), (3, True), (1, False), (3, False)])
def test_debug_quantize_rotated_bit_exact(bits, qjl):
    w = WORKLOADS["tiny"].with_(k_bits=bits, v_bits=bits, k_mode="lm_qjl" if qjl else "lm",
                                v_mode="lm_qjl" if qjl else "lm")
    cache, signs, S = new_cache(w, 1, 32)
    c32, t32 = tables.lloyd_max_tables_f32(bits)
    rng = np.random.default_rng(bits)
    u = rng.standard_normal((300, 128)).astype(np.float32)
    u[0, :len(t32)] = t32                       # exactly on thresholds: upper cell
    u[1, :len(t32)] = np.nextafter(t32, -np.inf)  # just below
    u[2] = 0.0
    ut = torch.tensor(u, device=DEV)
    planes, sketch, gamma = kvq.kvq_debug_quantize_rotated(cache.handle, ut, bits, qjl)
    torch.cuda.synchronize()
    planes = planes.cpu().numpy().view(np.uint32)
    flips = 0
    for i in range(u.shape[0]):
        r = codec.quantize_rotated(u[i].astype(np.float64), bits, c32, t32, S if qjl else None)
        np.testing.assert_array_equal(planes[i], r["planes"])
        if qjl:
            zg = sketch[i].cpu().numpy().view(np.uint32)
            mism = np.nonzero(codec.unpack_bits(zg, 128) != r["z"])[0]
            tol = 4 * 128 * 2.0 ** -24 * (np.abs(S.astype(np.float64)) @ np.abs(r["rho"]))
            assert np.all(np.abs(r["proj"][mism]) < tol[mism])
            flips += len(mism)
            g = float(gamma[i:i + 1].cpu().numpy().view(np.float16)[0])
            assert abs(g - r["gamma16"]) <= 2.0 ** (math.floor(math.log2(max(r["gamma"], 2 ** -14))) - 10)
    print(f"sign bits differing inside the fp32 bound: {flips} of {u.shape[0] * 128}")
    assert flips <= 1e-3 * u.shape[0] * 128
    cache.close()


# ---------------------------------------------------------------- decode parity, small contexts

def run_small(name, batch, lens, seed_appends=1, w=None):
    """Quantize lens[b] tokens into sequence b (in `seed_appends` calls), decode, compare every
    (sequence, kv-head) with the oracle."""
    w = w if w is not None else WORKLOADS[name]
    T = max(lens)
    data = generate(w, DEV, seqs=range(batch), ctx=T)
    cache, signs, S = new_cache(w, batch, T + 40)
    # append per sequence, in chunks, to exercise positions inside tiles
    for b in range(batch):
        L = lens[b]
        cuts = np.linspace(0, L, seed_appends + 1).astype(int)
        for a, e in zip(cuts[:-1], cuts[1:]):
            if e > a:
                cache.quantize(data["k"][b:b + 1, :, a:e].contiguous(), data["v"][b:b + 1, :, a:e].contiguous(),
                               seq_ids=[b])
    assert list(cache.lengths()) == list(lens)
    out = f64(cache.decode(data["q"]))
    torch.cuda.synchronize()
    arena = cache.arena.cpu().numpy()
    info = cache.layout()
    stats = {}
    for b in range(batch):
        for hk in range(w.n_kv_heads):
            g = w.group
            if lens[b] == 0:
                assert np.all(out[b, hk * g:(hk + 1) * g] == 0)
                continue
            ref = pair_reference(w, arena, info, b, hk, lens[b], f64(data["k"][b, hk, :lens[b]]),
                                 f64(data["v"][b, hk, :lens[b]]), f64(data["q"][b, hk * g:(hk + 1) * g]),
                                 signs, S, stats)
            err = rel_err(out[b, hk * g:(hk + 1) * g], ref)
            assert np.all(err <= REL_TOL), (b, hk, err.max())
    cache.close()
    check_flip_rates(stats, w.name)
    return stats


def test_tiny_full():
    w = WORKLOADS["tiny"]
    stats = run_small("tiny", 1, [w.ctx])
    assert stats["code_flips"] <= 1e-3 * stats["coords"]


def test_tiny_token_by_token_and_ragged():
    run_small("tiny", 1, [77], seed_appends=77)


def test_cuda_core_code_combination():
    """1-bit keys with a sketch and 1-bit values without: a combination the tensor-core kernel has
    no instance for, decoded by the CUDA-core kernel (token-ordered keys)."""
    w = WORKLOADS["tiny"].with_(k_bits=1, v_bits=1, k_mode="lm_qjl", v_mode="lm", n_q_heads=4, n_kv_heads=1)
    run_small("tiny", 2, [300, 65], seed_appends=2, w=w)


@pytest.mark.parametrize("lens", [[1000, 333, 1, 0], [32, 31, 64, 65]])
def test_llama8b_small_ragged(lens):
    run_small("llama8b", len(lens), lens, seed_appends=3)


def test_llama70b_small():
    run_small("llama70b", 2, [700, 129], seed_appends=2)


def test_onebit_small():
    run_small("onebit", 3, [500, 1, 257])


def test_single_token_equals_dequantised_value():
    """ctx = 1: softmax weight 1, so every head's output is that token's dequantised value."""
    run_small("llama8b", 1, [1])


# ---------------------------------------------------------------- full-size, sampled pairs

@pytest.mark.parametrize("name", ["llama8b", "llama70b", "onebit"])
def test_full_size_sampled_pairs(name):
    w = WORKLOADS[name]
    torch.cuda.empty_cache()
    cache, signs, S = new_cache(w, w.batch, w.ctx)
    # generate and append in slices of sequences to bound memory
    step = max(1, w.batch // 8)
    q_all = []
    sampled = [(0, 0), (w.batch - 1, w.n_kv_heads - 1), (w.batch // 2, w.n_kv_heads // 2)]
    keep = {}
    for b0 in range(0, w.batch, step):
        seqs = list(range(b0, min(w.batch, b0 + step)))
        data = generate(w, DEV, seqs=seqs)
        cache.quantize(data["k"], data["v"], seq_ids=seqs)
        q_all.append(data["q"])
        for (b, hk) in sampled:
            if b in seqs:
                keep[(b, hk)] = (f64(data["k"][b - b0, hk]), f64(data["v"][b - b0, hk]))
        del data
    q = torch.cat(q_all)
    out = f64(cache.decode(q))
    torch.cuda.synchronize()
    arena = cache.arena.cpu().numpy()
    info = cache.layout()
    stats = {}
    for (b, hk) in sampled:
        g = w.group
        K, V = keep[(b, hk)]
        ref = pair_reference(w, arena, info, b, hk, w.ctx, K, V, f64(q[b, hk * g:(hk + 1) * g]), signs, S, stats)
        err = rel_err(out[b, hk * g:(hk + 1) * g], ref)
        assert np.all(err <= REL_TOL), (name, b, hk, err.max())
    assert np.all(np.isfinite(out))
    check_flip_rates(stats, name)
    cache.close()


# ---------------------------------------------------------------- FP4 latent cache

def fp4_check(ctx, heads_checked=None, batch=1, lens=None, n_q_heads=None):
    w = WORKLOADS["mla_fp4"]
    if n_q_heads is not None:
        w = w.with_(n_q_heads=n_q_heads)
    lens = lens or [ctx] * batch
    data = generate(w, DEV, seqs=range(batch), ctx=max(lens))
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), batch, max(lens) + 32)
    for b in range(batch):
        if lens[b]:
            cache.quantize(data["latent"][b:b + 1, :lens[b]].contiguous(), data["rope"][b:b + 1, :lens[b]].contiguous(),
                           seq_ids=[b])
    out = f64(cache.decode(data["q"]))
    torch.cuda.synchronize()
    arena = cache.arena.cpu().numpy()
    info = cache.layout()
    for b in range(batch):
        if lens[b] == 0:
            assert np.all(out[b] == 0)
            continue
        codes, scales, kr = fp4_fields(arena, info, b, lens[b])
        lat = f64(data["latent"][b, :lens[b]]).astype(np.float32)
        # codes: bit-exact against the oracle's own encoding, on sampled tokens
        idx = np.unique(np.concatenate([np.arange(min(64, lens[b])), np.linspace(0, lens[b] - 1, 64).astype(int)]))
        for t in idx:
            pk, sc = codec.fp4_quantize(lat[t])
            np.testing.assert_array_equal(codes[t], pk)
            np.testing.assert_array_equal(scales[t], sc)
        np.testing.assert_array_equal(kr, f64(data["rope"][b, :lens[b]]))
        heads = heads_checked or list(range(w.n_q_heads))
        ref = attention.mla_decode_attention_many(f64(data["q"][b]), codes, scales, kr,
                                                  1.0 / math.sqrt(w.latent_dim + w.rope_dim), heads)
        err = rel_err(out[b, heads], ref)
        assert np.all(err <= REL_TOL), err.max()
    cache.close()


def test_fp4_small_ragged():
    fp4_check(0, batch=3, lens=[1000, 0, 33])


def test_fp4_few_tiles_per_cta():
    """A context whose split plan gives every CTA a few 64-token tiles, the last one ragged: the
    tcgen05 kernel's first, middle and last iterations (S of the next tile issued after O^T of
    the current one) on every CTA."""
    fp4_check(0, batch=1, lens=[3 * 147 * 64 + 33])


def test_fp4_sixteen_heads_ragged():
    """16 query heads decode on the mma.sync kernel (the tcgen05 kernel is for 64 heads)."""
    fp4_check(0, batch=2, lens=[700, 65], n_q_heads=16)


def test_fp4_full_context_sampled_heads():
    fp4_check(WORKLOADS["mla_fp4"].ctx, heads_checked=[0, 21, 63])


# ---------------------------------------------------------------- launch accounting

def test_launch_counts_per_call():
    """quantize: one kernel; decode: query prep + split decode + reduce on the tensor-core path
    (query groups of 8 as two pieces of 4 heads), split decode + reduce for FP4."""
    for name, per_decode in (("llama8b", 3), ("llama70b", 3), ("mla_fp4", 2)):
        w = WORKLOADS[name]
        data = generate(w, DEV, seqs=range(2), ctx=100)
        if w.k_mode == "fp4":
            cache = kvq.KvqCache(kvq.cfg_for_workload(w), 2, 128)
            a, b = data["latent"], data["rope"]
        else:
            cache, _, _ = new_cache(w, 2, 128)
            a, b = data["k"], data["v"]
        n0 = kvq.kvq_kernel_launches()
        cache.quantize(a, b)
        assert kvq.kvq_kernel_launches() - n0 == 1
        cache.decode(data["q"])
        assert kvq.kvq_kernel_launches() - n0 == 1 + per_decode, name
        torch.cuda.synchronize()
        cache.close()


# ---------------------------------------------------------------- fused decode step

@pytest.mark.parametrize("name", ["llama8b", "llama70b", "onebit", "mla_fp4"])
def test_decode_step_equals_append_then_decode(name):
    """kvq_decode_step (append one token, then attend, with the query prep overlapping the append)
    leaves the same cache and returns the same output as kvq_quantize followed by
    kvq_decode_attention."""
    w = WORKLOADS[name]
    fp4 = w.k_mode == "fp4"
    B = 3
    data = generate(w, DEV, seqs=range(B), ctx=200)
    new = generate(w, DEV, seqs=range(B), step=0)
    if fp4:
        a, v, na, nv = data["latent"], data["rope"], new["latent"], new["rope"]
        mk = lambda: kvq.KvqCache(kvq.cfg_for_workload(w), B, 256)
    else:
        a, v, na, nv = data["k"], data["v"], new["k"], new["v"]
        mk = lambda: new_cache(w, B, 256)[0]
    c1, c2 = mk(), mk()
    for c in (c1, c2):
        c.quantize(a[:, :, :150].contiguous() if not fp4 else a[:, :150].contiguous(),
                   v[:, :, :150].contiguous() if not fp4 else v[:, :150].contiguous())
    c1.quantize(na, nv)
    ref = c1.decode(data["q"])
    out = c2.step(na, nv, data["q"])
    torch.cuda.synchronize()
    assert list(c1.lengths()) == list(c2.lengths()) == [151] * B
    assert torch.equal(out, ref)
    # the written part of the caches is identical (tile tails past the lengths are never written)
    a1, a2, info = c1.arena.cpu().numpy(), c2.arena.cpu().numpy(), c1.layout()
    if fp4:
        for b in range(B):
            for f1, f2 in zip(fp4_fields(a1, info, b, 151), fp4_fields(a2, info, b, 151)):
                np.testing.assert_array_equal(f1, f2)
    else:
        for pair in range(B * w.n_kv_heads):
            for side in (0, 1):
                for f1, f2 in zip(side_fields(a1, info, side, pair, 151), side_fields(a2, info, side, pair, 151)):
                    if f1 is not None:
                        np.testing.assert_array_equal(f1[:151], f2[:151])
    c1.close()
    c2.close()


def test_decode_step_ragged_long():
    """Ragged lengths long enough that most splits issue their first key fills before waiting for
    the append: the fused step still equals append-then-decode, and matches the oracle."""
    w = WORKLOADS["llama8b"]
    B, lens = 3, [1000, 333, 700]
    T = max(lens)
    data = generate(w, DEV, seqs=range(B), ctx=T)
    new = generate(w, DEV, seqs=range(B), step=0)
    c1, signs, S = new_cache(w, B, T + 64)
    c2, _, _ = new_cache(w, B, T + 64)
    for c in (c1, c2):
        for b in range(B):
            c.quantize(data["k"][b:b + 1, :, :lens[b]].contiguous(), data["v"][b:b + 1, :, :lens[b]].contiguous(),
                       seq_ids=[b])
    c1.quantize(new["k"], new["v"])
    ref = c1.decode(data["q"])
    out = c2.step(new["k"], new["v"], data["q"])
    torch.cuda.synchronize()
    assert list(c2.lengths()) == [n + 1 for n in lens]
    assert torch.equal(out, ref)
    c1.close()
    c2.close()


@pytest.mark.parametrize("name,pinned", [("llama8b", True), ("llama70b", False), ("mla_fp4", True)])
def test_decode_step_host_equals_device_step(name, pinned):
    """kvq_decode_step_host (inputs and output in host memory, copies enqueued by the library)
    appends the same tokens and returns the same output as kvq_decode_step on device buffers."""
    w = WORKLOADS[name]
    fp4 = w.k_mode == "fp4"
    B = 3
    data = generate(w, DEV, seqs=range(B), ctx=256)
    mk = (lambda: kvq.KvqCache(kvq.cfg_for_workload(w), B, 256)) if fp4 else (lambda: new_cache(w, B, 256)[0])
    a, v = (data["latent"], data["rope"]) if fp4 else (data["k"], data["v"])
    c1, c2 = mk(), mk()
    for c in (c1, c2):
        c.quantize(a[:, :150].contiguous() if fp4 else a[:, :, :150].contiguous(),
                   v[:, :150].contiguous() if fp4 else v[:, :, :150].contiguous())
    host = lambda t: t.cpu().pin_memory() if pinned else t.cpu()
    # four steps enqueued back to back (inputs of step j + 1 cross while step j runs), then compared
    refs, outs, keep = [], [], []
    for step in range(4):
        new = generate(w, DEV, seqs=range(B), step=step)
        na, nv = (new["latent"], new["rope"]) if fp4 else (new["k"], new["v"])
        refs.append(c1.step(na, nv, data["q"]).clone())
        keep.append((host(na), host(nv), host(data["q"])))
    torch.cuda.synchronize()
    # odd steps hand the library an event to record after the output copy (the stream does not
    # wait for that copy); even steps let the stream wait for it
    events = [torch.cuda.Event() if step % 2 else None for step in range(4)]
    for step in range(4):
        outs.append(host(torch.empty(refs[0].shape, dtype=torch.float32)))
        c2.step_host(*keep[step], outs[step], out_event=events[step])
    events[3].synchronize()
    assert torch.equal(outs[3], refs[3].cpu()), (name, 3)
    torch.cuda.synchronize()
    for step in range(4):
        assert torch.equal(outs[step], refs[step].cpu()), (name, step)
    assert list(c1.lengths()) == list(c2.lengths()) == [154] * B
    # a step past the capacity is refused before anything is copied or appended
    full = mk()
    full.quantize(a[:, :256].contiguous() if fp4 else a[:, :, :256].contiguous(),
                  v[:, :256].contiguous() if fp4 else v[:, :, :256].contiguous())
    with pytest.raises(kvq.KvqError) as e:
        full.step_host(*keep[0], host(torch.empty(refs[0].shape, dtype=torch.float32)))
    assert e.value.status == 3  # KVQ_ERR_CAPACITY
    assert list(full.lengths()) == [256] * B
    for c in (c1, c2, full):
        c.close()


# ---------------------------------------------------------------- bounded waits

def test_bounded_wait_sets_status_and_returns():
    """Every wait of the tensor-core decode kernel is bounded. The test entry adds one wait on a
    barrier that nothing completes: each CTA gives up after ~1e5 cycles, sets the status bit and
    carries on, so the call returns, its output equals the plain call's, and the cache reports
    KVQ_STATUS_WAIT_TIMEOUT. No GPU fault is involved: the wait simply runs out."""
    w = WORKLOADS["llama8b"]
    data = generate(w, DEV, seqs=range(2), ctx=300)
    cache, _, _ = new_cache(w, 2, 320)
    cache.quantize(data["k"], data["v"])
    ref = cache.decode(data["q"])
    assert kvq.kvq_cache_status(cache.handle) == 0
    out = torch.empty_like(ref)
    kvq.kvq_debug_decode_unset_wait(cache.handle, data["q"], out, cache.workspace, 100000)
    assert kvq.kvq_cache_status(cache.handle) == kvq.KVQ_STATUS_WAIT_TIMEOUT
    assert torch.equal(out, ref)
    cache.close()
    # a code combination only the CUDA-core kernel decodes (1-bit keys with a sketch, 1-bit values
    # without): the test entry refuses and launches nothing
    w1 = WORKLOADS["tiny"].with_(k_bits=1, v_bits=1, k_mode="lm_qjl", v_mode="lm")
    d1 = generate(w1, DEV, seqs=range(1), ctx=64)
    c1, _, _ = new_cache(w1, 1, 64)
    c1.quantize(d1["k"], d1["v"])
    n0 = kvq.kvq_kernel_launches()
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_debug_decode_unset_wait(c1.handle, d1["q"], torch.empty(1, 1, 128, device=DEV),
                                        c1.workspace, 100000)
    assert e.value.status == 2 and kvq.kvq_kernel_launches() == n0
    assert kvq.kvq_cache_status(c1.handle) == 0
    c1.close()


# ---------------------------------------------------------------- errors

def test_capacity_overflow_writes_nothing():
    w = WORKLOADS["llama8b"]
    data = generate(w, DEV, seqs=range(2), ctx=80)
    cache, _, _ = new_cache(w, 2, 64)  # capacity is whole pairs of 32-token tiles: 64
    cache.quantize(data["k"][:, :, :20].contiguous(), data["v"][:, :, :20].contiguous())
    before = cache.arena.clone()
    with pytest.raises(kvq.KvqError) as e:
        cache.quantize(data["k"][:, :, 20:80].contiguous(), data["v"][:, :, 20:80].contiguous())
    assert e.value.status == 3
    torch.cuda.synchronize()
    assert torch.equal(before, cache.arena)
    assert list(cache.lengths()) == [20, 20]
    with pytest.raises(kvq.KvqError) as e:
        cache.quantize(data["k"][:1, :, :1].contiguous(), data["v"][:1, :, :1].contiguous(), seq_ids=[5])
    assert e.value.status == 1
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attention(cache.handle, data["q"], torch.empty(2, 32, 128, device=DEV), small)
    assert e.value.status == 5
    cache.close()


# ---------------------------------------------------------------- seeded draws inside the library

def test_seeded_cache_equals_cache_from_explicit_tables():
    """A cache given only the configuration's seeds draws the same rotation signs and sketch matrix
    as the seeded generator: both arenas are byte-identical after the same appends, and decode gives
    identical outputs."""
    w = WORKLOADS["llama8b"].with_(batch=2)
    data = generate(w, DEV, seqs=range(2), ctx=200)
    signs, S = rotation_and_sketch(w)
    explicit = kvq.KvqCache(kvq.cfg_for_workload(w), 2, 256, signs, S)
    seeded = kvq.KvqCache(kvq.cfg_for_workload(w), 2, 256)  # no arrays: drawn from cfg seeds
    for c in (explicit, seeded):
        c.quantize(data["k"], data["v"])
    a = explicit.decode(data["q"])
    b = seeded.decode(data["q"])
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert_same_token_fields(explicit, seeded, w, [200, 200])
    # the tables in the arenas (signs, S, S^T) are the same bytes
    info = explicit.layout()
    A, B = explicit.arena.cpu().numpy(), seeded.arena.cpu().numpy()
    np.testing.assert_array_equal(A[:int(info[4])][256:], B[:int(info[4])][256:])
    explicit.close()
    seeded.close()


def test_per_head_rotation_parity():
    """Every kv-head with its own rotation diagonal (drawn from the same seed stream): codes and
    attention against the oracle, which rotates each head with that head's diagonal."""
    w = WORKLOADS["llama8b"].with_(rot_per_head=True)
    signs, _ = rotation_and_sketch(w)
    assert signs.shape == (w.n_kv_heads, w.head_dim) and not np.all(signs[0] == signs[1])
    run_small("llama8b", 2, [300, 97], seed_appends=2, w=w)
    w70 = WORKLOADS["llama70b"].with_(rot_per_head=True)
    run_small("llama70b", 1, [260], w=w70)


# ---------------------------------------------------------------- prefill-rate quantize

@pytest.mark.parametrize("name", ["llama8b", "llama70b", "onebit"])
def test_tile_quantize_equals_token_by_token(name):
    """Appends of many tokens (whole tiles built in shared memory, 16-byte stores) store the same
    codes and norms as token-by-token appends (per-vector kernel, atomics), also for tiles a call
    only partly covers; sketch sign bits may differ only where the two fp32 summation orders
    disagree on a projection's sign, which the oracle parity bounds, here at most 1e-3 of them."""
    w = WORKLOADS[name].with_(batch=2)
    data = generate(w, DEV, seqs=range(2), ctx=150)
    tiles, tokens = new_cache(w, 2, 192)[0], new_cache(w, 2, 192)[0]
    # tile path: 37 tokens (a partial tile), then 113 more (starting inside that tile)
    for a, e in ((0, 37), (37, 150)):
        tiles.quantize(data["k"][:, :, a:e].contiguous(), data["v"][:, :, a:e].contiguous())
    for t in range(150):
        tokens.quantize(data["k"][:, :, t:t + 1].contiguous(), data["v"][:, :, t:t + 1].contiguous())
    torch.cuda.synchronize()
    A, B = tiles.arena.cpu().numpy(), tokens.arena.cpu().numpy()
    info = tiles.layout()
    assert list(tiles.lengths()) == list(tokens.lengths()) == [150, 150]
    flips = bits = 0
    for pair in range(2 * w.n_kv_heads):
        for side in (0, 1):
            pa, sa, na, ga = side_fields(A, info, side, pair, 150)
            pb, sb, nb, gb = side_fields(B, info, side, pair, 150)
            np.testing.assert_array_equal(pa, pb)
            np.testing.assert_array_equal(na, nb)
            if sa is not None:
                np.testing.assert_array_equal(ga, gb)
                d = np.unpackbits(np.bitwise_xor(sa, sb).view(np.uint8))
                flips += int(d.sum())
                bits += d.size
    assert flips <= 1e-3 * max(bits, 1), (flips, bits)
    tiles.close()
    tokens.close()


# ---------------------------------------------------------------- the two LM decode kernels

@pytest.mark.parametrize("kernel", ["tc", "ws"])
@pytest.mark.parametrize("name,lens", [("llama8b", [700, 65]), ("llama70b", [1000, 129]), ("onebit", [300, 1])])
def test_tcgen05_kernel_parity(name, lens, kernel, monkeypatch):
    """The tcgen05 decode kernels (chosen with KVQ_DECODE_KERNEL=tc, the lockstep one, or =ws, the
    warp-specialised one, at cache creation) against the oracle, as the mma.sync kernel is by
    default."""
    monkeypatch.setenv("KVQ_DECODE_KERNEL", kernel)
    run_small(name, len(lens), lens, seed_appends=2)


@pytest.mark.parametrize("kernel", ["tc", "ws"])
@pytest.mark.parametrize("name", ["llama8b", "llama70b", "onebit"])
def test_tcgen05_and_mma_sync_kernels_agree(name, kernel, monkeypatch):
    """A tcgen05 kernel and the mma.sync kernel on the same cache contents: outputs within the
    attention tolerance of each other, over contexts that span several iterations with a ragged
    tail."""
    w = WORKLOADS[name].with_(batch=3)
    lens = [1500, 700, 64]
    data = generate(w, DEV, seqs=range(3), ctx=max(lens))
    monkeypatch.delenv("KVQ_DECODE_KERNEL", raising=False)
    c_mma = new_cache(w, 3, 1536)[0]
    monkeypatch.setenv("KVQ_DECODE_KERNEL", kernel)
    c_tc = new_cache(w, 3, 1536)[0]
    for c in (c_mma, c_tc):
        for b, L in enumerate(lens):
            c.quantize(data["k"][b:b + 1, :, :L].contiguous(), data["v"][b:b + 1, :, :L].contiguous(), seq_ids=[b])
    a = f64(c_mma.decode(data["q"]))
    t = f64(c_tc.decode(data["q"]))
    torch.cuda.synchronize()
    assert_same_token_fields(c_mma, c_tc, w, lens)
    err = rel_err(t.reshape(-1, t.shape[-1]), a.reshape(-1, a.shape[-1]))
    assert np.all(err <= REL_TOL), err.max()
    c_mma.close()
    c_tc.close()


# ---------------------------------------------------------------- instances and edge cases

def test_query_group_of_two():
    w = WORKLOADS["llama8b"].with_(n_q_heads=16)
    run_small("llama8b", 2, [900, 65], seed_appends=2, w=w)


@pytest.mark.parametrize("heads", [8, 32])
def test_fp4_mma_sync_head_counts(heads):
    """8 and 32 query heads decode on the mma.sync MLA kernel (64 on tcgen05, 16 tested above)."""
    fp4_check(0, batch=2, lens=[900, 33], n_q_heads=heads)


@pytest.mark.parametrize("kb,kq,vb,vq", [(2, True, 2, False), (3, True, 3, True), (2, False, 2, False),
                                         (3, False, 3, False)])
def test_other_code_combinations(kb, kq, vb, vq):
    w = WORKLOADS["llama8b"].with_(k_bits=kb, v_bits=vb, k_mode="lm_qjl" if kq else "lm",
                                   v_mode="lm_qjl" if vq else "lm", qjl_dim=128 if (kq or vq) else 0)
    run_small("llama8b", 2, [700, 100], seed_appends=2, w=w)
    w8 = WORKLOADS["llama70b"].with_(k_bits=kb, v_bits=vb, k_mode="lm_qjl" if kq else "lm",
                                     v_mode="lm_qjl" if vq else "lm", qjl_dim=128 if (kq or vq) else 0)
    run_small("llama70b", 1, [400], w=w8)


def test_zero_key_and_value_vectors():
    """A zero key (norm 0: no logit contribution, n = 0 stored) and a zero value, end to end."""
    w = WORKLOADS["llama8b"].with_(batch=2)
    T = 300
    data = generate(w, DEV, seqs=range(2), ctx=T)
    data["k"][0, 1, 7] = 0
    data["v"][0, 1, 9] = 0
    data["k"][1, :, 100] = 0
    data["v"][1, :, 100] = 0
    cache, signs, S = new_cache(w, 2, T + 32)
    cache.quantize(data["k"], data["v"])
    out = f64(cache.decode(data["q"]))
    torch.cuda.synchronize()
    arena, info = cache.arena.cpu().numpy(), cache.layout()
    stats = {}
    for b, hk in ((0, 1), (1, 3)):
        g = w.group
        ref = pair_reference(w, arena, info, b, hk, T, f64(data["k"][b, hk]), f64(data["v"][b, hk]),
                             f64(data["q"][b, hk * g:(hk + 1) * g]), signs, S, stats)
        assert np.all(rel_err(out[b, hk * g:(hk + 1) * g], ref) <= REL_TOL)
    _, _, kn, _ = side_fields(arena, info, 0, 0 * w.n_kv_heads + 1, T)
    assert kn[7] == 0
    cache.close()
