"""The allocation-free decode entry point (kvq_decode_attention_static) against the regular one.

kvq_decode_attention_static exists for callers that cannot allocate device memory on the decode
path; it keeps its split partials in a fixed array inside the library. This test calls it twice
in a row through the C ABI and checks both results against kvq_decode_attention with a
caller-owned workspace, within the attention tolerance the parity tests use. It sits in a file of
its own, collected last, and passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_kv_cache_seeded_b200 as kvq
from kvq_inputs import WORKLOADS, generate
from kvq_inputs.workloads import rotation_and_sketch

REL_TOL = 2e-3

pytestmark = pytest.mark.gpu


def test_static_scratch_decode_matches_workspace_decode():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = kvq.load()
    w = WORKLOADS["llama8b"].with_(batch=3)
    data = generate(w, "cuda", seqs=range(3), ctx=700)
    signs, S = rotation_and_sketch(w)
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), 3, 720, signs, S)
    cache.quantize(data["k"][:, :, :690].contiguous(), data["v"][:, :, :690].contiguous())
    cache.quantize(data["k"][1:, :, 690:].contiguous(), data["v"][1:, :, 690:].contiguous(), seq_ids=[1, 2])
    ref = cache.decode(data["q"]).clone()
    outs = []
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        st = lib.kvq_decode_attention_static(cache.handle, ctypes.c_void_p(data["q"].data_ptr()), 1,
                                             ctypes.c_void_p(out.data_ptr()),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, kvq.kvq_status_str(st)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy().astype(np.float64))
    r = ref.cpu().numpy().astype(np.float64)
    for o in outs:
        err = np.max(np.abs(o - r), axis=-1) / np.max(np.abs(r), axis=-1)
        assert np.all(np.isfinite(o)) and np.all(err <= REL_TOL), err.max()
    cache.close()


def test_static_scratch_refuses_partials_beyond_its_size():
    """A cache whose split partials cannot fit the fixed array (batch 512, 64 query heads: 512 x 64 x
    (2 + 128) floats already at one split, about 17 MB) is refused with KVQ_ERR_WORKSPACE, and the
    output buffer is left untouched."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = kvq.load()
    w = WORKLOADS["llama70b"].with_(batch=512)
    signs, S = rotation_and_sketch(w)
    cache = kvq.KvqCache(kvq.cfg_for_workload(w), 512, 64, signs, S)
    q = torch.randn(512, 64, 128, device="cuda").to(torch.bfloat16)
    out = torch.full((512, 64, 128), 7.0, device="cuda")
    st = lib.kvq_decode_attention_static(cache.handle, ctypes.c_void_p(q.data_ptr()), 1,
                                         ctypes.c_void_p(out.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == 5, kvq.kvq_status_str(st)  # KVQ_ERR_WORKSPACE
    assert torch.all(out == 7.0)
    cache.close()
