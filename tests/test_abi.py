"""The C-ABI library builds, loads and exports every symbol include/kvq.h declares; host-only
entry points (tables, sizes, validation) behave as documented. No GPU needed."""
import os
import re

import numpy as np
import pytest

import bit_kv_cache_seeded_b200 as kvq
from bit_kv_cache_seeded_b200 import build
from oracle import tables, sizes
from kvq_inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kvq.load()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"\b(kvq_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(kvq.EXPORTS)


def test_lloyd_max_table_bit_equal_to_oracle(lib):
    for bits in (1, 2, 3):
        c, t = kvq.kvq_lloyd_max_table(bits)
        oc, ot = tables.lloyd_max_tables_f32(bits)
        assert c.tobytes() == oc.tobytes()
        assert t.tobytes() == ot.tobytes()


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_packed_bytes_match_oracle_sizes(lib, name):
    w = WORKLOADS[name]
    cfg = kvq.cfg_for_workload(w)
    got = kvq.kvq_packed_bytes_per_token(cfg)
    if w.k_mode == "fp4":
        want = sizes.fp4_token_bytes(w.latent_dim, w.rope_dim)
    else:
        want = (sizes.lm_vector_bytes(128, w.k_bits, 128 if w.k_mode == "lm_qjl" else 0)
                + sizes.lm_vector_bytes(128, w.v_bits, 128 if w.v_mode == "lm_qjl" else 0))
    assert got == want


def test_cache_bytes_scales_with_capacity(lib):
    cfg = kvq.cfg_for_workload(WORKLOADS["llama8b"])
    a = kvq.kvq_cache_bytes(cfg, 16, 8192)
    b = kvq.kvq_cache_bytes(cfg, 16, 8192 + 64)
    assert b - a == 16 * 8 * 104 * 64
    assert kvq.kvq_cache_bytes(cfg, 16, 8193) == b  # capacity rounds up to whole tile pairs


def test_validation_errors(lib):
    bad = kvq.make_cfg(head_dim=64)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_cache_bytes(bad, 1, 32)
    assert e.value.status == 2  # unsupported
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_cache_bytes(kvq.make_cfg(n_q_heads=3, n_kv_heads=2), 1, 32)
    assert e.value.status == 1
    with pytest.raises(kvq.KvqError):
        kvq.kvq_cache_bytes(kvq.make_cfg(k_bits=4), 1, 32)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_cache_bytes(kvq.make_cfg(k_mode="fp4"), 1, 32)  # fp4 on one side only
    with pytest.raises(kvq.KvqError):
        kvq.kvq_cache_bytes(kvq.make_cfg(), 0, 32)
    assert kvq.kvq_status_str(3) == "cache capacity exceeded"


def test_init_rejects_null_and_misaligned_before_any_launch(lib):
    import ctypes
    cfg = kvq.make_cfg()
    h = ctypes.c_void_p()
    signs = np.ones(128, dtype=np.int8)
    st = lib.kvq_cache_init(ctypes.byref(h), ctypes.byref(cfg), 1, 32, None, 1 << 20,
                            signs.ctypes.data_as(ctypes.c_void_p), None, None)
    assert st == 1
    st = lib.kvq_cache_init(ctypes.byref(h), ctypes.byref(cfg), 1, 32, ctypes.c_void_p(0x1010), 1 << 20,
                            signs.ctypes.data_as(ctypes.c_void_p), None, None)
    assert st == 4
    st = lib.kvq_cache_init(ctypes.byref(h), ctypes.byref(cfg), 1, 32, ctypes.c_void_p(0x10000), 16,
                            signs.ctypes.data_as(ctypes.c_void_p), None, None)
    assert st == 5
    bad_signs = np.zeros(128, dtype=np.int8)
    S = np.zeros((128, 128), dtype=np.float32)
    st = lib.kvq_cache_init(ctypes.byref(h), ctypes.byref(cfg), 1, 32, ctypes.c_void_p(0x10000), 1 << 20,
                            bad_signs.ctypes.data_as(ctypes.c_void_p), S.ctypes.data_as(ctypes.c_void_p), None)
    assert st == 1


def test_rejected_calls_launch_nothing(lib):
    """Validation failures return before any kernel is enqueued: the launch counter stays put."""
    n0 = kvq.kvq_kernel_launches()
    with pytest.raises(kvq.KvqError):
        kvq.kvq_cache_bytes(kvq.make_cfg(k_bits=4), 1, 32)
    import ctypes
    h = ctypes.c_void_p()
    signs = np.ones(128, dtype=np.int8)
    assert lib.kvq_cache_init(ctypes.byref(h), ctypes.byref(kvq.make_cfg()), 1, 32, None, 1 << 20,
                              signs.ctypes.data_as(ctypes.c_void_p), None, None) == 1
    assert kvq.kvq_kernel_launches() == n0


def test_step_host_checks_host_buffer_sizes(lib):
    """KvqCache.step_host refuses host tensors whose sizes do not match the cache's step layout
    (the library cannot see host buffer sizes) before anything reaches the library; the C entry
    refuses a null cache."""
    import torch
    cache = object.__new__(kvq.KvqCache)
    cache.batch, cache.cfg, cache.out_dim, cache.handle = 3, kvq.make_cfg(n_q_heads=32, n_kv_heads=8), 128, None
    K = torch.zeros(3, 8, 1, 128, dtype=torch.bfloat16)
    q = torch.zeros(3, 32, 128, dtype=torch.bfloat16)
    out = torch.zeros(3, 32, 128)
    n0 = kvq.kvq_kernel_launches()
    for bad in ((K[:2], K, q, out), (K, K, q[:, :16], out), (K, K.float(), q, out), (K, K, q, out[:1]),
                (K, K, q, out.double())):
        with pytest.raises(ValueError):
            cache.step_host(*bad)
    with pytest.raises(kvq.KvqError):  # sizes right: the library itself refuses the null cache
        cache.step_host(K, K, q, out)
    assert kvq.kvq_kernel_launches() == n0


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "kvq.h"
int main(void) {
  float c[8], t[7];
  size_t bytes = 0;
  kvq_cfg cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.head_dim = 128; cfg.n_q_heads = 32; cfg.n_kv_heads = 8; cfg.k_mode = KVQ_MODE_LM_QJL;
  cfg.v_mode = KVQ_MODE_LM_QJL; cfg.k_bits = 2; cfg.v_bits = 2; cfg.qjl_dim = 128;
  if (kvq_lloyd_max_table(2, c, t) != KVQ_OK) return 1;
  if (kvq_lloyd_max_table(4, c, t) != KVQ_ERR_INVALID_ARG) return 2;
  if (kvq_packed_bytes_per_token(&cfg, &bytes) != KVQ_OK) return 3;
  if (kvq_decode_step_host(NULL, NULL, NULL, NULL, KVQ_BF16, NULL, NULL, 0, NULL, 0, NULL, NULL) != KVQ_ERR_INVALID_ARG) return 4;
  /* the seeded draws a cache makes from cfg.rot_seed / cfg.qjl_seed when given no arrays */
  cfg.rot_seed = 0x5EED00A4ull; cfg.qjl_seed = 0x5EED005Bull;
  {
    static int8_t d[128];
    static float s[128 * 128];
    long sum = 0;
    double ssum = 0.0;
    int i;
    if (kvq_draw_rotation_signs(cfg.rot_seed, 128, d) != KVQ_OK) return 5;
    if (kvq_draw_qjl_matrix(cfg.qjl_seed, 128, 128, s) != KVQ_OK) return 6;
    if (kvq_draw_qjl_matrix(cfg.qjl_seed, 0, 128, s) != KVQ_ERR_INVALID_ARG) return 7;
    for (i = 0; i < 128; ++i) sum += (long)d[i] * (i + 1);
    for (i = 0; i < 128 * 128; ++i) ssum += (double)s[i] * (double)((i % 97) + 1);
    printf("%s|%zu|%.6f|%ld|%.17g|%.9g\n", kvq_status_str(KVQ_ERR_CAPACITY), bytes, c[3], sum, ssum, (double)s[12345]);
  }
  return 0;
}
"""


def test_plain_c_client_links_and_runs(lib, tmp_path):
    """A C99 program that includes kvq.h, links libkvq.so and calls its host-only entries: the
    boundary is usable without C++ or Python."""
    import subprocess
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(kvq.LIB_PATH)
    try:
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-L", libdir, "-lkvq", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       check=True, capture_output=True, text=True)
    except FileNotFoundError:
        pytest.skip("gcc not available")
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    name, nbytes, c3, dsum, ssum, s12345 = out.stdout.strip().split("|")
    from kvq_inputs import rotation_signs, qjl_matrix
    d = rotation_signs(0x5EED00A4, 128).astype(np.int64)
    S = qjl_matrix(0x5EED005B, 128, 128).astype(np.float64).reshape(-1)
    assert int(dsum) == int(np.sum(d * np.arange(1, 129)))
    assert np.float32(float(s12345)) == np.float32(S[12345])
    assert abs(float(ssum) - float(np.sum(S * ((np.arange(S.size) % 97) + 1)))) < 1e-6 * np.sum(np.abs(S)) * 97
    cfg = kvq.make_cfg(head_dim=128, n_q_heads=32, n_kv_heads=8, k_bits=2, v_bits=2, qjl_dim=128)
    assert name == kvq.kvq_status_str(3)
    assert int(nbytes) == kvq.kvq_packed_bytes_per_token(cfg)
    assert abs(float(c3) - float(kvq.kvq_lloyd_max_table(2)[0][3])) < 1e-6


def test_binding_refuses_host_tensors_and_wrong_shapes(lib):
    """The library reads device pointers with the extents the cache's configuration implies; the
    binding refuses host tensors at every device entry and KvqCache refuses shapes that do not
    match its configuration, before anything reaches the library."""
    import torch
    cache = object.__new__(kvq.KvqCache)
    cache.batch, cache.cfg, cache.out_dim, cache.handle = 2, kvq.make_cfg(n_q_heads=8, n_kv_heads=2), 128, None
    cache.workspace = torch.zeros(16, dtype=torch.uint8)
    K = torch.zeros(2, 2, 5, 128)
    q = torch.zeros(2, 8, 128)
    n0 = kvq.kvq_kernel_launches()
    bad_shapes = [lambda: cache.quantize(K, K[:, :1]), lambda: cache.quantize(torch.zeros(3, 2, 5, 128), torch.zeros(3, 2, 5, 128)),
                  lambda: cache.quantize(K[..., :64], K[..., :64]), lambda: cache.decode(q[:, :4]),
                  lambda: cache.decode(q, torch.zeros(2, 8, 64)), lambda: cache.step(K, K, q),
                  lambda: cache.step(K[:, :, :1], K[:, :, :1], q[:1])]
    for call in bad_shapes:
        with pytest.raises(ValueError, match="must be|more sequences"):
            call()
    host = [lambda: cache.quantize(K, K), lambda: cache.decode(q, torch.zeros(2, 8, 128)),
            lambda: cache.step(K[:, :, :1].contiguous(), K[:, :, :1].contiguous(), q, torch.zeros(2, 8, 128)),
            lambda: kvq.kvq_decode_attention_static(None, q, torch.zeros(2, 8, 128)),
            lambda: kvq.kvq_cache_init(kvq.make_cfg(), 1, 32, torch.zeros(16, dtype=torch.uint8))]
    for call in host:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
    assert kvq.kvq_kernel_launches() == n0


@pytest.mark.parametrize("seed", [0, 1, 0x5EED00A5, 0x5EED005A, 0xFFFFFFFFFFFFFFFF, 0x0123456789ABCDEF])
def test_seeded_draws_are_the_generator_bit_for_bit(lib, seed):
    """The library's host draws (what kvq_cache_init uses when it gets seeds and no arrays) equal
    the seeded generator's, bit for bit: rotation signs over several heads' worth of counters, and
    the Box-Muller sketch matrix."""
    from kvq_inputs import rotation_signs, qjl_matrix
    from kvq_inputs.rng import rotation_signs_per_head
    np.testing.assert_array_equal(kvq.kvq_draw_rotation_signs(seed, 1024), rotation_signs(seed, 1024))
    np.testing.assert_array_equal(kvq.kvq_draw_rotation_signs(seed, 8 * 128).reshape(8, 128),
                                  rotation_signs_per_head(seed, 8, 128))
    a = kvq.kvq_draw_qjl_matrix(seed, 128, 128)
    b = qjl_matrix(seed, 128, 128)
    np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32))


def test_cfg_struct_layout_matches_header(lib):
    """The ctypes mirror of kvq_cfg has the C layout: 12 int32-sized fields, two uint64 seeds, then the
    two window sizes."""
    import ctypes
    assert ctypes.sizeof(kvq.kvq_cfg) == 72
    assert kvq.kvq_cfg.rot_seed.offset == 48 and kvq.kvq_cfg.qjl_seed.offset == 56
    assert kvq.kvq_cfg.sink_tokens.offset == 64 and kvq.kvq_cfg.recent_tokens.offset == 68
    with pytest.raises(kvq.KvqError):  # window over 1024 tokens
        kvq.kvq_cache_bytes(kvq.make_cfg(sink_tokens=64, recent_tokens=1000), 1, 32)
    assert kvq.kvq_cache_bytes(kvq.make_cfg(sink_tokens=64, recent_tokens=256), 2, 64) > \
        kvq.kvq_cache_bytes(kvq.make_cfg(), 2, 64) + 2 * 2 * 320 * 128 * 2 - 1
    cfg = kvq.make_cfg(rot_per_head=2)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_cache_bytes(cfg, 1, 32)
    fp4 = kvq.make_cfg(head_dim=512, n_q_heads=64, k_mode="fp4", v_mode="fp4", k_bits=4, v_bits=4, qjl_dim=0,
                       latent_dim=512, rope_dim=64, rot_per_head=1)
    with pytest.raises(kvq.KvqError):
        kvq.kvq_cache_bytes(fp4, 1, 32)
