"""Context-parallel decode: shards of the context on several ranks, their softmax states exchanged
and merged.

CPU (gloo, world size 2): the exchange of bit_kv_cache_seeded_b200.context_parallel, fed with the
oracle's per-shard softmax states, gathers them in rank order and their merge equals the oracle's
attention over the whole context. GPU: caches holding disjoint shards of every sequence's tokens,
kvq_decode_partials on each and kvq_combine_partials over them, against one cache holding all the
tokens and against the oracle (FP4 latent and LM caches, an empty shard included)."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_kv_cache_seeded_b200.context_parallel import shard_range  # noqa: E402


def test_shard_ranges_cover_the_context_disjointly():
    for ctx in (0, 1, 7, 1024, 1 << 20):
        for world in (1, 2, 3, 8):
            rs = [shard_range(ctx, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == ctx
            assert all(a[1] == b[0] for a, b in zip(rs[:-1], rs[1:]))
            sizes = [e - b for b, e in rs]
            assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    rng = np.random.default_rng(44)
    B, H, T, dq, dv = 2, 3, 101, 24, 16
    return (rng.standard_normal((B, H, dq)), rng.standard_normal((B, T, dq)) * 2,
            rng.standard_normal((B, T, dv)), 0.4)


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from oracle import attention
    from bit_kv_cache_seeded_b200.context_parallel import exchange_states
    dist.init_process_group("gloo", rank=rank, world_size=world)
    Q, K, V, scale = _problem()
    B, H, _ = Q.shape
    a, e = shard_range(K.shape[1], rank, world)
    local = torch.zeros((B, H, 2 + V.shape[2]), dtype=torch.float64)
    for b in range(B):
        for h in range(H):
            m, l, o = attention.softmax_state(Q[b, h], K[b, a:e], V[b, a:e], scale)
            local[b, h, 0], local[b, h, 1] = m, l
            local[b, h, 2:] = torch.from_numpy(o)
    got = exchange_states(local)
    q.put((rank, got.numpy(), local.numpy()))
    dist.destroy_process_group()


def test_exchange_over_two_gloo_ranks_then_merge_equals_full_attention():
    from oracle import attention
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(60)
    assert [p.exitcode for p in procs] == [0, 0]
    locals_ = [r[2] for r in res]
    Q, K, V, scale = _problem()
    for rank, got, _ in res:
        np.testing.assert_array_equal(got[0], locals_[0])  # rank order
        np.testing.assert_array_equal(got[1], locals_[1])
        for b in range(Q.shape[0]):
            for h in range(Q.shape[1]):
                states = [(got[r, b, h, 0], got[r, b, h, 1], got[r, b, h, 2:]) for r in range(2)]
                merged = attention.merge_softmax_states(states)
                full = attention.softmax_attention(Q[b, h], K[b], V[b], scale)
                np.testing.assert_allclose(merged, full, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- GPU: shards on one device

def _shard_caches(kvq, w, data, lens, n_shards, lm):
    """n_shards caches, shard s holding tokens shard_range(lens[b], s, n) of sequence b."""
    caches = []
    for s in range(n_shards):
        if lm:
            from kvq_inputs.workloads import rotation_and_sketch
            signs, S = rotation_and_sketch(w)
            c = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), max(lens) + 64, signs, S)
        else:
            c = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), max(lens) + 64)
        for b, L in enumerate(lens):
            a, e = shard_range(L, s, n_shards)
            if e > a:
                if lm:
                    c.quantize(data["k"][b:b + 1, :, a:e].contiguous(), data["v"][b:b + 1, :, a:e].contiguous(), seq_ids=[b])
                else:
                    c.quantize(data["latent"][b:b + 1, a:e].contiguous(), data["rope"][b:b + 1, a:e].contiguous(), seq_ids=[b])
        caches.append(c)
    return caches


@pytest.mark.gpu
@pytest.mark.parametrize("name,lens,n_shards", [("mla_fp4", [3000, 40], 2), ("mla_fp4", [5000, 1], 3),
                                                 ("llama8b", [1200, 300], 2), ("llama70b", [900, 2], 3)])
def test_sharded_decode_equals_whole_cache(name, lens, n_shards):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_kv_cache_seeded_b200 as kvq
    from kvq_inputs import WORKLOADS, generate
    from oracle import attention
    from tests._parity import rel_err, REL_TOL
    from tests._cache_reader import fp4_fields
    kvq.load()
    lm = name != "mla_fp4"
    w = WORKLOADS[name].with_(batch=len(lens))
    data = generate(w, "cuda", seqs=range(len(lens)), ctx=max(lens))
    whole = _shard_caches(kvq, w, data, lens, 1, lm)[0]
    shards = _shard_caches(kvq, w, data, lens, n_shards, lm)
    ref = whole.decode(data["q"])
    parts = torch.stack([c.decode_partials(data["q"]) for c in shards])
    out = torch.empty_like(ref)
    kvq.kvq_combine_partials(parts, out)
    torch.cuda.synchronize()
    r = ref.double().cpu().numpy().reshape(-1, ref.shape[-1])
    o = out.double().cpu().numpy().reshape(-1, out.shape[-1])
    err = rel_err(o, r)
    assert np.all(err <= REL_TOL), err.max()
    # the shortest sequence has an empty shard when it holds fewer tokens than there are shards
    if not lm:  # FP4 against the oracle over the whole context, from the shards' own codes
        arena, info = whole.arena.cpu().numpy(), whole.layout()
        for b, L in enumerate(lens):
            codes, scales, kr = fp4_fields(arena, info, b, L)
            heads = [0, 31, 63]
            oref = attention.mla_decode_attention_many(data["q"][b].double().cpu().numpy(), codes, scales, kr,
                                                       1.0 / math.sqrt(w.latent_dim + w.rope_dim), heads)
            assert np.all(rel_err(out[b, heads].double().cpu().numpy(), oref) <= REL_TOL)
    for c in [whole, *shards]:
        c.close()
