"""Python binding of the kvq C ABI (include/kvq.h): argument marshalling only.

Every step of the hot path -- rotation, Lloyd-Max coding, QJL sketch, packing, decode
attention, split reduce -- runs in the CUDA kernels of ``libkvq.so``. This module loads that
library (built in-tree by ``bit_kv_cache_seeded_b200.build``) and raises if it is missing or
if no CUDA device is present when a call needs one; there is no fallback path.

The C functions are exposed under their own names (``kvq_cache_bytes``, ``kvq_cache_init``,
``kvq_quantize``, ``kvq_workspace_bytes``, ``kvq_decode_attention``, ...), taking torch
tensors for device buffers. ``KvqCache`` bundles the arena, the host handle and the
workspace for convenience.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvq.so")

KVQ_OK = 0
STATUS_NAMES = {0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_UNSUPPORTED",
                3: "KVQ_ERR_CAPACITY", 4: "KVQ_ERR_ALIGNMENT", 5: "KVQ_ERR_WORKSPACE",
                6: "KVQ_ERR_CUDA"}
MODES = {"lm_qjl": 0, "lm": 1, "sign1": 2, "fp4": 3, "kivi": 4}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}

# Every symbol include/kvq.h declares.
EXPORTS = ("kvq_status_str", "kvq_cache_bytes", "kvq_packed_bytes_per_token", "kvq_cache_init",
           "kvq_quantize", "kvq_workspace_bytes", "kvq_decode_attention", "kvq_cache_lengths",
           "kvq_cache_layout", "kvq_lloyd_max_table", "kvq_cache_destroy",
           "kvq_debug_quantize_rotated", "kvq_decode_attention_static", "kvq_kernel_launches",
           "kvq_cache_status", "kvq_debug_decode_unset_wait", "kvq_debug_decode_timed", "kvq_decode_step",
           "kvq_step_staging_bytes", "kvq_decode_step_host", "kvq_draw_rotation_signs", "kvq_draw_qjl_matrix",
           "kvq_partial_floats", "kvq_decode_partials", "kvq_combine_partials",
           "kvq_cache_bytes_paged", "kvq_cache_init_paged")
KVQ_STATUS_WAIT_TIMEOUT = 1


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class kvq_cfg(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("k_mode", ctypes.c_int32),
                ("v_mode", ctypes.c_int32), ("k_bits", ctypes.c_int32),
                ("v_bits", ctypes.c_int32), ("qjl_dim", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("latent_dim", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("rot_per_head", ctypes.c_int32),
                ("rot_seed", ctypes.c_uint64), ("qjl_seed", ctypes.c_uint64),
                ("sink_tokens", ctypes.c_int32), ("recent_tokens", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libkvq.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise OSError(f"{LIB_PATH} not built: run `python -m bit_kv_cache_seeded_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p
    sig = {
        "kvq_status_str": ([I32], ctypes.c_char_p),
        "kvq_cache_bytes": ([P(kvq_cfg), I32, I32, P(SZ)], I32),
        "kvq_packed_bytes_per_token": ([P(kvq_cfg), P(SZ)], I32),
        "kvq_cache_init": ([P(VP), P(kvq_cfg), I32, I32, VP, SZ, VP, VP, VP], I32),
        "kvq_quantize": ([VP, VP, VP, I32, I32, VP, I32, VP], I32),
        "kvq_workspace_bytes": ([VP, P(SZ)], I32),
        "kvq_decode_attention": ([VP, VP, I32, VP, VP, SZ, VP], I32),
        "kvq_cache_lengths": ([VP, VP], I32),
        "kvq_cache_layout": ([VP, VP, I32], I32),
        "kvq_lloyd_max_table": ([I32, VP, VP], I32),
        "kvq_cache_destroy": ([VP], None),
        "kvq_debug_quantize_rotated": ([VP, VP, I32, VP, VP, VP, VP], I32),
        "kvq_decode_attention_static": ([VP, VP, I32, VP, VP], I32),
        "kvq_kernel_launches": ([], ctypes.c_uint64),
        "kvq_cache_status": ([VP, VP, VP], I32),
        "kvq_debug_decode_unset_wait": ([VP, VP, I32, VP, VP, SZ, ctypes.c_int64, VP], I32),
        "kvq_debug_decode_timed": ([VP, VP, I32, VP, VP, SZ, VP, VP], I32),
        "kvq_decode_step": ([VP, VP, VP, VP, I32, VP, VP, SZ, VP], I32),
        "kvq_step_staging_bytes": ([VP, I32, P(SZ)], I32),
        "kvq_decode_step_host": ([VP, VP, VP, VP, I32, VP, VP, SZ, VP, SZ, VP, VP], I32),
        "kvq_draw_rotation_signs": ([ctypes.c_uint64, I32, VP], I32),
        "kvq_draw_qjl_matrix": ([ctypes.c_uint64, I32, I32, VP], I32),
        "kvq_partial_floats": ([VP, P(I32)], I32),
        "kvq_cache_bytes_paged": ([P(kvq_cfg), I32, I32, P(SZ)], I32),
        "kvq_cache_init_paged": ([P(VP), P(kvq_cfg), I32, I32, I32, VP, VP, SZ, VP, VP, VP], I32),
        "kvq_decode_partials": ([VP, VP, I32, VP, VP, SZ, VP], I32),
        "kvq_combine_partials": ([VP, I32, I32, I32, I32, VP, VP], I32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != KVQ_OK:
        raise KvqError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _on_device(fn: str, **tensors):
    """Device entry points take device pointers: a host tensor would reach a kernel as an address
    it cannot read, so refuse it here."""
    for name, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise ValueError(f"{fn}: {name} must be a CUDA tensor")


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_cfg(head_dim=128, n_q_heads=1, n_kv_heads=1, k_mode="lm_qjl", v_mode="lm_qjl", k_bits=2,
             v_bits=2, qjl_dim=128, softmax_scale=0.0, latent_dim=0, rope_dim=0, rot_per_head=0,
             rot_seed=0, qjl_seed=0, sink_tokens=0, recent_tokens=0) -> kvq_cfg:
    return kvq_cfg(head_dim, n_q_heads, n_kv_heads, MODES[k_mode], MODES[v_mode], k_bits, v_bits,
                   qjl_dim, softmax_scale, latent_dim, rope_dim, int(rot_per_head), rot_seed, qjl_seed,
                   sink_tokens, recent_tokens)


def cfg_for_workload(w) -> kvq_cfg:
    """kvq_cfg of a kvq_inputs.Workload (its seeds included)."""
    if w.k_mode == "fp4":
        return make_cfg(head_dim=w.latent_dim, n_q_heads=w.n_q_heads, n_kv_heads=1, k_mode="fp4",
                        v_mode="fp4", k_bits=4, v_bits=4, qjl_dim=0, latent_dim=w.latent_dim,
                        rope_dim=w.rope_dim)
    return make_cfg(w.head_dim, w.n_q_heads, w.n_kv_heads, w.k_mode, w.v_mode, w.k_bits, w.v_bits,
                    w.qjl_dim, rot_per_head=int(getattr(w, "rot_per_head", False)), rot_seed=w.rot_seed,
                    qjl_seed=w.qjl_seed, sink_tokens=getattr(w, "sink_tokens", 0),
                    recent_tokens=getattr(w, "recent_tokens", 0))


def kvq_draw_rotation_signs(seed: int, n: int) -> np.ndarray:
    """The library's seeded +-1 draws (int8 [n]), as kvq_cache_init makes them from a seed."""
    out = np.zeros(n, dtype=np.int8)
    _check("kvq_draw_rotation_signs", load().kvq_draw_rotation_signs(seed, n, out.ctypes.data_as(ctypes.c_void_p)))
    return out


def kvq_draw_qjl_matrix(seed: int, m: int, d: int) -> np.ndarray:
    """The library's seeded Gaussian sketch matrix (float32 [m, d])."""
    out = np.zeros((m, d), dtype=np.float32)
    _check("kvq_draw_qjl_matrix", load().kvq_draw_qjl_matrix(seed, m, d, out.ctypes.data_as(ctypes.c_void_p)))
    return out


# ---------------------------------------------------------------- same-name wrappers

def kvq_status_str(status: int) -> str:
    return load().kvq_status_str(status).decode()


def kvq_cache_bytes(cfg: kvq_cfg, batch: int, capacity: int) -> int:
    out = ctypes.c_size_t()
    _check("kvq_cache_bytes", load().kvq_cache_bytes(ctypes.byref(cfg), batch, capacity, ctypes.byref(out)))
    return out.value


def kvq_packed_bytes_per_token(cfg: kvq_cfg) -> int:
    out = ctypes.c_size_t()
    _check("kvq_packed_bytes_per_token", load().kvq_packed_bytes_per_token(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def kvq_cache_init(cfg: kvq_cfg, batch: int, capacity: int, arena: torch.Tensor, rot_signs=None,
                   qjl_matrix=None, stream=None) -> ctypes.c_void_p:
    _on_device("kvq_cache_init", arena=arena)
    handle = ctypes.c_void_p()
    signs = None if rot_signs is None else np.ascontiguousarray(rot_signs, dtype=np.int8)
    S = None if qjl_matrix is None else np.ascontiguousarray(qjl_matrix, dtype=np.float32)
    st = load().kvq_cache_init(ctypes.byref(handle), ctypes.byref(cfg), batch, capacity, _ptr(arena),
                               arena.numel() * arena.element_size(),
                               None if signs is None else signs.ctypes.data_as(ctypes.c_void_p),
                               None if S is None else S.ctypes.data_as(ctypes.c_void_p), _stream(stream))
    _check("kvq_cache_init", st)
    return handle


def kvq_cache_bytes_paged(cfg: kvq_cfg, batch: int, n_pages: int) -> int:
    out = ctypes.c_size_t()
    _check("kvq_cache_bytes_paged", load().kvq_cache_bytes_paged(ctypes.byref(cfg), batch, n_pages, ctypes.byref(out)))
    return out.value


def kvq_cache_init_paged(cfg: kvq_cfg, batch: int, n_pages: int, block_table: torch.Tensor, arena: torch.Tensor,
                         rot_signs=None, qjl_matrix=None, stream=None) -> ctypes.c_void_p:
    """A paged cache: block_table int32 CUDA tensor [batch, pages_per_seq] (the caller keeps it)."""
    _on_device("kvq_cache_init_paged", arena=arena, block_table=block_table)
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != batch \
            or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 [batch, pages_per_seq] tensor")
    handle = ctypes.c_void_p()
    signs = None if rot_signs is None else np.ascontiguousarray(rot_signs, dtype=np.int8)
    S = None if qjl_matrix is None else np.ascontiguousarray(qjl_matrix, dtype=np.float32)
    st = load().kvq_cache_init_paged(ctypes.byref(handle), ctypes.byref(cfg), batch, block_table.shape[1], n_pages,
                                     _ptr(block_table), _ptr(arena), arena.numel() * arena.element_size(),
                                     None if signs is None else signs.ctypes.data_as(ctypes.c_void_p),
                                     None if S is None else S.ctypes.data_as(ctypes.c_void_p), _stream(stream))
    _check("kvq_cache_init_paged", st)
    return handle


def kvq_quantize(handle, K: torch.Tensor, V: torch.Tensor, seq_ids=None, stream=None):
    _on_device("kvq_quantize", K=K, V=V)
    if K.dtype not in DTYPES or V.dtype != K.dtype:
        raise TypeError("K and V must both be float32 or bfloat16")
    if not (K.is_contiguous() and V.is_contiguous()):
        raise ValueError("K and V must be contiguous")
    n_seq = K.shape[0]
    n_new = K.shape[-2]
    ids = None
    if seq_ids is not None:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        if ids.shape[0] != n_seq:
            raise ValueError("seq_ids length must match K.shape[0]")
    st = load().kvq_quantize(handle, _ptr(K), _ptr(V), DTYPES[K.dtype], n_new,
                             None if ids is None else ids.ctypes.data_as(ctypes.c_void_p), n_seq,
                             _stream(stream))
    _check("kvq_quantize", st)


def kvq_workspace_bytes(handle) -> int:
    out = ctypes.c_size_t()
    _check("kvq_workspace_bytes", load().kvq_workspace_bytes(handle, ctypes.byref(out)))
    return out.value


def kvq_decode_attention(handle, q: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                         stream=None):
    _on_device("kvq_decode_attention", q=q, out=out, workspace=workspace)
    if q.dtype not in DTYPES or out.dtype != torch.float32:
        raise TypeError("q must be float32/bfloat16 and out float32")
    if not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous")
    st = load().kvq_decode_attention(handle, _ptr(q), DTYPES[q.dtype], _ptr(out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check("kvq_decode_attention", st)


def kvq_partial_floats(handle) -> int:
    n = ctypes.c_int32(0)
    _check("kvq_partial_floats", load().kvq_partial_floats(handle, ctypes.byref(n)))
    return int(n.value)


def kvq_decode_partials(handle, q: torch.Tensor, partials: torch.Tensor, workspace: torch.Tensor, stream=None):
    """Softmax state of this cache's tokens: partials [batch, n_q_heads, 2 + dv] float32 (m, l, o)."""
    _on_device("kvq_decode_partials", q=q, partials=partials, workspace=workspace)
    if q.dtype not in DTYPES or partials.dtype != torch.float32:
        raise TypeError("q must be float32/bfloat16 and partials float32")
    if not (q.is_contiguous() and partials.is_contiguous()):
        raise ValueError("q and partials must be contiguous")
    st = load().kvq_decode_partials(handle, _ptr(q), DTYPES[q.dtype], _ptr(partials), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check("kvq_decode_partials", st)


def kvq_combine_partials(partials: torch.Tensor, out: torch.Tensor, stream=None):
    """Merge partials [n_parts, batch, n_q_heads, 2 + dv] into out [batch, n_q_heads, dv]."""
    _on_device("kvq_combine_partials", partials=partials, out=out)
    if partials.dtype != torch.float32 or out.dtype != torch.float32:
        raise TypeError("partials and out must be float32")
    if partials.dim() != 4 or out.dim() != 3 or tuple(partials.shape[1:3]) != tuple(out.shape[:2]) \
            or partials.shape[3] != out.shape[2] + 2:
        raise ValueError("partials must be [n_parts, batch, n_q_heads, 2 + dv] for out [batch, n_q_heads, dv]")
    if not (partials.is_contiguous() and out.is_contiguous()):
        raise ValueError("partials and out must be contiguous")
    n, B, H, S = partials.shape
    _check("kvq_combine_partials", load().kvq_combine_partials(_ptr(partials), n, B, H, S - 2, _ptr(out),
                                                               _stream(stream)))


def kvq_decode_step(handle, K: torch.Tensor, V: torch.Tensor, q: torch.Tensor, out: torch.Tensor,
                    workspace: torch.Tensor, stream=None):
    """Append one token per sequence (K, V [B, Hkv, 1, d]; FP4: latent, rope) and decode with q."""
    _on_device("kvq_decode_step", K=K, V=V, q=q, out=out, workspace=workspace)
    if K.dtype != V.dtype or K.dtype != q.dtype or q.dtype not in DTYPES or out.dtype != torch.float32:
        raise TypeError("K, V and q must share float32/bfloat16; out is float32")
    if not (K.is_contiguous() and V.is_contiguous() and q.is_contiguous() and out.is_contiguous()):
        raise ValueError("K, V, q and out must be contiguous")
    if K.shape[-2] != 1 or V.shape[-2] != 1:
        raise ValueError("a decode step appends exactly one token per sequence")
    st = load().kvq_decode_step(handle, _ptr(K), _ptr(V), _ptr(q), DTYPES[q.dtype], _ptr(out), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check("kvq_decode_step", st)


def kvq_step_staging_bytes(handle, dtype) -> int:
    n = ctypes.c_size_t(0)
    _check("kvq_step_staging_bytes", load().kvq_step_staging_bytes(handle, DTYPES[dtype], ctypes.byref(n)))
    return n.value


def kvq_decode_step_host(handle, K: torch.Tensor, V: torch.Tensor, q: torch.Tensor, dtype, out: torch.Tensor,
                         staging: torch.Tensor, workspace: torch.Tensor, stream=None, out_event=None):
    """kvq_decode_step from host memory: K, V, q and out are CPU tensors (pinned for asynchronous
    copies) holding the bytes of the layouts kvq_decode_step takes, inputs of type `dtype`. Without
    out_event, out is valid once the stream reaches the end of the call's work; with a
    torch.cuda.Event, the library records it after the output copy (on its own copy stream) and the
    stream does not wait: out is valid once the event has completed. The sizes are the caller's to
    get right (KvqCache.step_host checks them)."""
    for t in (K, V, q, out):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("kvq_decode_step_host takes contiguous host tensors")
    ev = None
    if out_event is not None:
        if out_event.cuda_event == 0:  # torch creates the event lazily, on its first record
            out_event.record()
        ev = ctypes.c_void_p(out_event.cuda_event)
    st = load().kvq_decode_step_host(handle, _ptr(K), _ptr(V), _ptr(q), DTYPES[dtype], _ptr(out), _ptr(staging),
                                     staging.numel() * staging.element_size(), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream), ev)
    _check("kvq_decode_step_host", st)
    return out


def kvq_decode_attention_static(handle, q: torch.Tensor, out: torch.Tensor, stream=None):
    """Decode attention without a workspace (partials in the library's fixed device array)."""
    _on_device("kvq_decode_attention_static", q=q, out=out)
    if q.dtype not in DTYPES or out.dtype != torch.float32:
        raise TypeError("q must be float32/bfloat16 and out float32")
    if not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous")
    st = load().kvq_decode_attention_static(handle, _ptr(q), DTYPES[q.dtype], _ptr(out), _stream(stream))
    _check("kvq_decode_attention_static", st)


def kvq_cache_status(handle, stream=None) -> int:
    """The cache's device status word (KVQ_STATUS_* bits); waits for the stream."""
    v = ctypes.c_int32(0)
    _check("kvq_cache_status", load().kvq_cache_status(handle, ctypes.byref(v), _stream(stream)))
    return int(v.value)


def kvq_debug_decode_unset_wait(handle, q: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                                wait_limit_cycles: int, stream=None):
    """Test entry: decode with one extra bounded wait on a barrier that nothing completes."""
    _on_device("kvq_debug_decode_unset_wait", q=q, out=out, workspace=workspace)
    if q.dtype not in DTYPES or out.dtype != torch.float32:
        raise TypeError("q must be float32/bfloat16 and out float32")
    if not (q.is_contiguous() and out.is_contiguous()):
        raise ValueError("q and out must be contiguous")
    st = load().kvq_debug_decode_unset_wait(handle, _ptr(q), DTYPES[q.dtype], _ptr(out), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(),
                                            int(wait_limit_cycles), _stream(stream))
    _check("kvq_debug_decode_unset_wait", st)


def kvq_debug_decode_timed(handle, q: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, events,
                           stream=None):
    """Decode recording 4 torch.cuda.Events: start, after prep, after the split kernel, after reduce."""
    _on_device("kvq_debug_decode_timed", q=q, out=out, workspace=workspace)
    if q.dtype not in DTYPES or out.dtype != torch.float32:
        raise TypeError("q must be float32/bfloat16 and out float32")
    if len(events) != 4:
        raise ValueError("four events")
    for e in events:
        if e.cuda_event == 0:  # torch creates the event lazily, on its first record
            e.record()
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    st = load().kvq_debug_decode_timed(handle, _ptr(q), DTYPES[q.dtype], _ptr(out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream), arr)
    _check("kvq_debug_decode_timed", st)


def kvq_cache_lengths(handle, batch: int) -> np.ndarray:
    lens = np.zeros(batch, dtype=np.int32)
    _check("kvq_cache_lengths", load().kvq_cache_lengths(handle, lens.ctypes.data_as(ctypes.c_void_p)))
    return lens


def kvq_cache_layout(handle) -> np.ndarray:
    info = np.zeros(24, dtype=np.int64)
    _check("kvq_cache_layout", load().kvq_cache_layout(handle, info.ctypes.data_as(ctypes.c_void_p), 24))
    return info


def kvq_lloyd_max_table(bits: int):
    c = np.zeros(1 << bits, dtype=np.float32)
    t = np.zeros((1 << bits) - 1, dtype=np.float32)
    _check("kvq_lloyd_max_table", load().kvq_lloyd_max_table(bits, c.ctypes.data_as(ctypes.c_void_p),
                                                             t.ctypes.data_as(ctypes.c_void_p)))
    return c, t


def kvq_cache_destroy(handle):
    if handle:
        load().kvq_cache_destroy(handle)


def kvq_kernel_launches() -> int:
    """Kernels the library has enqueued since it was loaded (all threads and devices)."""
    return int(load().kvq_kernel_launches())


def kvq_debug_quantize_rotated(handle, u: torch.Tensor, k_bits: int, qjl: bool, stream=None):
    _on_device("kvq_debug_quantize_rotated", u=u)
    n = u.shape[0]
    planes = torch.zeros((n, k_bits, 4), dtype=torch.int32, device=u.device)
    sketch = torch.zeros((n, 4), dtype=torch.int32, device=u.device) if qjl else None
    gamma = torch.zeros((n,), dtype=torch.int16, device=u.device) if qjl else None
    st = load().kvq_debug_quantize_rotated(handle, _ptr(u), n, _ptr(planes), _ptr(sketch), _ptr(gamma),
                                           _stream(stream))
    _check("kvq_debug_quantize_rotated", st)
    return planes, sketch, gamma


# ---------------------------------------------------------------- convenience object

class KvqCache:
    """A packed cache in a torch-allocated device arena, plus its decode workspace.

    With block_table (an int32 CUDA tensor [batch, pages_per_seq]) and n_pages, the cache is paged:
    its tiles live in a pool of n_pages pages of 64 tokens and the table names the page of each
    64-token page of a sequence; the caller owns the table and fills it before tokens reach a page."""

    def __init__(self, cfg: kvq_cfg, batch: int, capacity: int, rot_signs=None, qjl_matrix=None,
                 device="cuda", block_table=None, n_pages=0):
        if not torch.cuda.is_available():
            raise RuntimeError("kvq needs a CUDA device")
        self.cfg, self.batch = cfg, batch
        if block_table is None:
            nbytes = kvq_cache_bytes(cfg, batch, capacity)
            self.arena = torch.empty(nbytes, dtype=torch.uint8, device=device)
            self.handle = kvq_cache_init(cfg, batch, capacity, self.arena, rot_signs, qjl_matrix)
        else:
            self.block_table = block_table
            nbytes = kvq_cache_bytes_paged(cfg, batch, n_pages)
            self.arena = torch.empty(nbytes, dtype=torch.uint8, device=device)
            self.handle = kvq_cache_init_paged(cfg, batch, n_pages, block_table, self.arena, rot_signs, qjl_matrix)
        self.workspace = torch.empty(max(16, kvq_workspace_bytes(self.handle)), dtype=torch.uint8,
                                     device=device)
        self.out_dim = cfg.latent_dim if cfg.k_mode == MODES["fp4"] else cfg.head_dim

    # Shapes the library reads and writes; it cannot see tensor extents, so they are checked here.
    def _kv_shapes(self, n_seq: int, n_new: int):
        cfg = self.cfg
        if cfg.k_mode == MODES["fp4"]:
            return (n_seq, n_new, cfg.latent_dim), (n_seq, n_new, cfg.rope_dim)
        kv = (n_seq, cfg.n_kv_heads, n_new, cfg.head_dim)
        return kv, kv

    def _check_kv(self, fn, K, V, n_seq, n_new):
        if K.dim() < 2 or (tuple(K.shape), tuple(V.shape)) != self._kv_shapes(n_seq, n_new):
            raise ValueError(f"{fn}: K, V must be {self._kv_shapes(n_seq, n_new)}, got {tuple(K.shape)}, {tuple(V.shape)}")

    def _check_q_out(self, fn, q, out):
        cfg = self.cfg
        dq = cfg.latent_dim + cfg.rope_dim if cfg.k_mode == MODES["fp4"] else cfg.head_dim
        if tuple(q.shape) != (self.batch, cfg.n_q_heads, dq):
            raise ValueError(f"{fn}: q must be {(self.batch, cfg.n_q_heads, dq)}, got {tuple(q.shape)}")
        if out is not None and tuple(out.shape) != (self.batch, cfg.n_q_heads, self.out_dim):
            raise ValueError(f"{fn}: out must be {(self.batch, cfg.n_q_heads, self.out_dim)}")

    def quantize(self, K, V, seq_ids=None, stream=None):
        n_seq = K.shape[0] if K.dim() else 0
        if seq_ids is None and n_seq > self.batch:
            raise ValueError("quantize: more sequences than the cache holds")
        self._check_kv("quantize", K, V, n_seq, K.shape[-2] if K.dim() >= 2 else 0)
        kvq_quantize(self.handle, K, V, seq_ids, stream)

    def step(self, K, V, q, out=None, stream=None):
        """Append one token per sequence and decode (kvq_decode_step); returns out."""
        self._check_kv("step", K, V, self.batch, 1)
        self._check_q_out("step", q, out)
        if out is None:
            out = torch.empty((self.batch, self.cfg.n_q_heads, self.out_dim), dtype=torch.float32,
                              device=q.device)
        kvq_decode_step(self.handle, K, V, q, out, self.workspace, stream)
        return out

    def step_host(self, K, V, q, out=None, stream=None, out_event=None):
        """step() with host (CPU) inputs and output: one call enqueues the input copies, the step
        and the output copy; returns out (valid after the stream reaches it, or, with out_event,
        once that event has completed)."""
        if out is None:
            out = torch.empty((self.batch, self.cfg.n_q_heads, self.out_dim), dtype=torch.float32).pin_memory()
        # the library cannot see host buffer sizes: check them here
        B, Hq, cfg = self.batch, self.cfg.n_q_heads, self.cfg
        if cfg.k_mode == MODES["fp4"]:
            want = (B * cfg.latent_dim, B * cfg.rope_dim, B * Hq * (cfg.latent_dim + cfg.rope_dim))
        else:
            want = (B * cfg.n_kv_heads * cfg.head_dim,) * 2 + (B * Hq * cfg.head_dim,)
        if tuple(t.numel() for t in (K, V, q)) != want or K.dtype != q.dtype or V.dtype != q.dtype:
            raise ValueError(f"step_host: K, V, q must hold {want} elements of one dtype")
        if out.dtype != torch.float32 or out.numel() != B * Hq * self.out_dim:
            raise ValueError("step_host: out must be float32 [batch, n_q_heads, out_dim]")
        need = kvq_step_staging_bytes(self.handle, q.dtype)
        if getattr(self, "staging", None) is None or self.staging.numel() < need:
            self.staging = torch.empty(need, dtype=torch.uint8, device=self.workspace.device)
        return kvq_decode_step_host(self.handle, K, V, q, q.dtype, out, self.staging, self.workspace, stream,
                                    out_event)

    def decode(self, q, out=None, stream=None):
        self._check_q_out("decode", q, out)
        if out is None:
            out = torch.empty((self.batch, self.cfg.n_q_heads, self.out_dim), dtype=torch.float32,
                              device=q.device)
        kvq_decode_attention(self.handle, q, out, self.workspace, stream)
        return out

    def decode_partials(self, q, partials=None, stream=None):
        """Softmax state of this cache's tokens (kvq_decode_partials): [batch, n_q_heads, 2 + dv]."""
        self._check_q_out("decode_partials", q, None)
        n = kvq_partial_floats(self.handle)
        if partials is None:
            partials = torch.empty((self.batch, self.cfg.n_q_heads, n), dtype=torch.float32, device=q.device)
        if tuple(partials.shape) != (self.batch, self.cfg.n_q_heads, n):
            raise ValueError(f"decode_partials: partials must be {(self.batch, self.cfg.n_q_heads, n)}")
        kvq_decode_partials(self.handle, q, partials, self.workspace, stream)
        return partials

    def lengths(self):
        return kvq_cache_lengths(self.handle, self.batch)

    def layout(self):
        return kvq_cache_layout(self.handle)

    def close(self):
        if self.handle:
            kvq_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
