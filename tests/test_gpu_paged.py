"""Paged caches: tiles in a pool of 64-token pages named by a caller-owned block table.

Shuffled pages give byte-identical tiles and identical decode outputs to the contiguous layout (same
codes, same arithmetic; only the addresses differ); sequences sharing a prefix's pages decode as if
each held its own copy; a block-table entry outside the pool sets the status bit instead of reaching
memory outside the arena."""
import numpy as np
import pytest
import torch

import bit_kv_cache_seeded_b200 as kvq
from kvq_inputs import WORKLOADS, generate
from kvq_inputs.workloads import rotation_and_sketch
from tests._cache_reader import side_fields

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvq.load()


def contiguous_info(info, side, ntiles):
    """Layout info of a buffer holding just one (sequence, kv-head)'s ntiles tiles of one side at 0."""
    i = np.array(info, copy=True)
    i[3] = ntiles
    i[4 + side] = 0
    return i


@pytest.mark.parametrize("kernel", ["mma", "tc", "ws"])
@pytest.mark.parametrize("name,lens", [("llama8b", [900, 64, 1]), ("llama70b", [700, 130]), ("onebit", [333, 64])])
def test_shuffled_pages_equal_contiguous(name, lens, kernel, monkeypatch):
    """On each LM decode kernel (mma.sync by default, tcgen05 with KVQ_DECODE_KERNEL=tc or ws), whose
    fills find a paged cache's tiles through the block table."""
    if kernel == "mma":
        monkeypatch.delenv("KVQ_DECODE_KERNEL", raising=False)
    else:
        monkeypatch.setenv("KVQ_DECODE_KERNEL", kernel)
    w = WORKLOADS[name].with_(batch=len(lens))
    pps = (max(lens) + 63) // 64 + 1
    n_pages = len(lens) * pps + 3
    rng = np.random.default_rng(7)
    perm = rng.permutation(n_pages)[:len(lens) * pps].reshape(len(lens), pps).astype(np.int32)
    table = torch.tensor(perm, device=DEV)
    signs, S = rotation_and_sketch(w)
    data = generate(w, DEV, seqs=range(len(lens)), ctx=max(lens))
    paged = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), 0, signs, S, block_table=table, n_pages=n_pages)
    flat = kvq.KvqCache(kvq.cfg_for_workload(w), len(lens), pps * 64, signs, S)
    for c in (paged, flat):
        for b, L in enumerate(lens):  # a prefill, then token appends into the same pages
            if L > 1:
                c.quantize(data["k"][b:b + 1, :, :L - 1].contiguous(), data["v"][b:b + 1, :, :L - 1].contiguous(), seq_ids=[b])
            c.quantize(data["k"][b:b + 1, :, L - 1:L].contiguous(), data["v"][b:b + 1, :, L - 1:L].contiguous(), seq_ids=[b])
    o1, o2 = paged.decode(data["q"]), flat.decode(data["q"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    # every stored token's fields are identical: its tile found through the block table in the pool,
    # at its contiguous place in the other cache (bytes past a sequence's last token not compared)
    ip, ic = paged.layout(), flat.layout()
    A, B = paged.arena.cpu().numpy(), flat.arena.cpu().numpy()
    tiles_per_seq = int(ic[3])
    for side in (0, 1):
        tb = int(ic[1 + side])
        for b, L in enumerate(lens):
            for h in range(w.n_kv_heads):
                ntiles = (L + 31) // 32
                flat_tiles = np.stack([B[int(ic[4 + side]) + ((b * w.n_kv_heads + h) * tiles_per_seq + t) * tb:][:tb]
                                       for t in range(ntiles)])
                paged_tiles = np.stack([A[int(ip[4 + side]) + ((int(perm[b, t // 2]) * w.n_kv_heads + h) * 2 + t % 2) * tb:][:tb]
                                        for t in range(ntiles)])
                fa = side_fields(paged_tiles.reshape(-1), contiguous_info(ic, side, ntiles), side, 0, L)
                fb = side_fields(flat_tiles.reshape(-1), contiguous_info(ic, side, ntiles), side, 0, L)
                for x, y in zip(fa, fb):
                    if x is not None:
                        np.testing.assert_array_equal(x, y)
    assert kvq.kvq_cache_status(paged.handle) == 0
    paged.close()
    flat.close()


def test_shared_prefix_pages():
    """Sequences 0 and 1 share the pages of a 256-token prefix; their outputs equal those of a cache
    where each holds its own copy."""
    w = WORKLOADS["llama8b"].with_(batch=2)
    signs, S = rotation_and_sketch(w)
    data = generate(w, DEV, seqs=range(2), ctx=600)
    data["k"][1, :, :256] = data["k"][0, :, :256]
    data["v"][1, :, :256] = data["v"][0, :, :256]
    pps = 10
    table = torch.tensor([[0, 1, 2, 3, 4, 5, 6, 7, 8, 9], [0, 1, 2, 3, 10, 11, 12, 13, 14, 15]], dtype=torch.int32, device=DEV)
    paged = kvq.KvqCache(kvq.cfg_for_workload(w), 2, 0, signs, S, block_table=table, n_pages=16)
    flat = kvq.KvqCache(kvq.cfg_for_workload(w), 2, pps * 64, signs, S)
    paged.quantize(data["k"][0:1].contiguous(), data["v"][0:1].contiguous(), seq_ids=[0])
    torch.cuda.synchronize()
    # sequence 1: its prefix pages already hold the tokens; append them again (identical bytes), then its own
    paged.quantize(data["k"][1:2].contiguous(), data["v"][1:2].contiguous(), seq_ids=[1])
    flat.quantize(data["k"].contiguous(), data["v"].contiguous())
    o1, o2 = paged.decode(data["q"]), flat.decode(data["q"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    paged.close()
    flat.close()


def test_block_table_entry_outside_the_pool_sets_status():
    w = WORKLOADS["llama8b"].with_(batch=1)
    signs, S = rotation_and_sketch(w)
    data = generate(w, DEV, seqs=range(1), ctx=200)
    table = torch.tensor([[0, 1, 99, 2]], dtype=torch.int32, device=DEV)  # page 2 of the sequence: not in the pool
    c = kvq.KvqCache(kvq.cfg_for_workload(w), 1, 0, signs, S, block_table=table, n_pages=4)
    c.quantize(data["k"].contiguous(), data["v"].contiguous())
    out = c.decode(data["q"])
    torch.cuda.synchronize()
    assert kvq.kvq_cache_status(c.handle) & 2
    assert torch.isfinite(out).all()
    c.close()
