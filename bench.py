"""Decode-step benchmark for the packed few-bit KV cache on B200.

One step = one decode step of a GQA layer of the workload: append the new token of every
sequence (kvq_quantize, n_new = 1) and run decode attention over the whole packed cache
(kvq_decode_attention). Metric: KV tokens/s = sum over steps of (batch x context length)
divided by the device time; also the packed HBM GB/s of the decode call.

    python bench.py [--gpus N --steps K --warmup W --workload llama8b --impl ours|reference]

With N > 1 (torchrun), every rank runs its own full copy of the workload (independent
sequences, no collective on the data path: weak scaling); the time is the max over ranks.
The timed region rotates over several cache replicas whose total size exceeds the 126 MB L2,
so every step reads its cache from HBM. Inputs of all steps are resident in HBM before timing.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kvq_inputs import WORKLOADS, VARIANTS, generate  # noqa: E402
from kvq_inputs.workloads import rotation_and_sketch  # noqa: E402

L2_BYTES = 126 * 2 ** 20
METRIC = "quantized-KV decode attention: KV tokens/s and HBM GB/s vs ~8 TB/s peak"
UNIT = "KV tokens/s"


def workload_config(w, world):
    """The `config` object of both arms' JSON lines (identical for the same workload)."""
    fp4 = w.k_mode == "fp4"
    return {"workload": w.name, "batch": w.batch, "n_q_heads": w.n_q_heads,
            "n_kv_heads": 1 if fp4 else w.n_kv_heads,
            "head_dim": w.latent_dim if fp4 else w.head_dim, "ctx": w.ctx,
            "codec": f"K {w.k_mode}{w.k_bits} / V {w.v_mode}{w.v_bits}",
            "l2": "inputs larger than L2: cache replicas (> 2.5 x 126 MB in total) rotated per step",
            "parallelism": f"replicas{world}",
            **({"window": {"sink": w.sink_tokens, "recent": w.recent_tokens}} if (w.sink_tokens or w.recent_tokens) else {}),
            **({"paged": "64-token pages, shuffled pool"} if w.paged else {})}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="llama70b", choices=list(WORKLOADS) + list(VARIANTS),
                    help="headline workload (default: the largest single-GPU configuration, 1.98 GB per step)")
    ap.add_argument("--only", action="store_true", help="time the headline workload alone")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ctx", type=int, default=0,
                    help="context length override (smaller cases for profiling); default: the workload's")
    return ap.parse_args()


# The dominant (split decode) kernel of each workload.
KERNEL_NAMES = {
    "tiny": "decode_lm_mma<1, 2, 1, 2, 1>", "llama8b": "decode_lm_mma<4, 2, 1, 2, 1>",
    "llama70b": "decode_lm_mma<8, 3, 1, 3, 0>", "onebit": "decode_lm_mma<4, 1, 0, 1, 0>",
    "mla_fp4": "decode_mla_umma",
    "llama8b_kivi": "decode_lm_mma<4, 2, 0, 2, 0, kivi> (key-group splits + window parts)",
    "llama8b_window": "decode_lm_mma<4, 2, 1, 2, 1> (history splits + window parts)",
    "llama8b_paged": "decode_lm_mma<4, 2, 1, 2, 1> (paged)",
}
EXTRA_WORKLOADS = ("llama8b", "onebit", "mla_fp4", "llama70b", "llama8b_kivi", "llama8b_window", "llama8b_paged")


def workload(name):
    return WORKLOADS[name] if name in WORKLOADS else VARIANTS[name]


def coded_len(w, L):
    """Tokens of a sequence of length L that the split kernel reads (the coded history)."""
    if w.k_mode == "kivi":
        return L // 128 * 128
    if w.sink_tokens or w.recent_tokens:
        return max(0, L - w.sink_tokens - w.recent_tokens)
    return L


def window_len(w, L):
    """bf16 window tokens of a sequence of length L (sink + recent; KIVI: the incomplete group)."""
    if w.k_mode == "kivi":
        return L % 128
    if w.sink_tokens or w.recent_tokens:
        return min(L, w.sink_tokens) + (min(w.recent_tokens, L - w.sink_tokens) if L > w.sink_tokens else 0)
    return 0

# DRAM bytes (read + write) of one launch of the split decode kernel, and the load efficiency of its
# packed streams, from ncu captures (full size, or a smaller context scaled to the full launch by the
# tokens processed). A record only counts while the kernel's sources are the ones captured (their
# SHA-256 below); after any change the bench reports null until a new capture.
TRAFFIC = {
    "llama70b": {"dram_bytes": 2039258112, "captured": "ctx 8192, scaled x4 by the tokens processed",
        "lsu_global_sectors_per_request": 7.17,
        "sources_sha256": "dea02c0843e6721dbcef2a62c5c8e5d49bdfabf21868936614c2c7adb4ab0fe5"},
    "llama8b": {"dram_bytes": 112607232, "captured": "full size",
        "lsu_global_sectors_per_request": 6.73,
        "sources_sha256": "dea02c0843e6721dbcef2a62c5c8e5d49bdfabf21868936614c2c7adb4ab0fe5"},
    "onebit": {"dram_bytes": 1261775872, "captured": "ctx 4096, scaled x4 by the tokens processed",
        "lsu_global_sectors_per_request": 5.83,
        "sources_sha256": "dea02c0843e6721dbcef2a62c5c8e5d49bdfabf21868936614c2c7adb4ab0fe5"},
    "mla_fp4": {"dram_bytes": 444171776, "captured": "ctx 524288, scaled x2 by the tokens processed",
        "lsu_global_sectors_per_request": 19.23,
        "sources_sha256": "dea02c0843e6721dbcef2a62c5c8e5d49bdfabf21868936614c2c7adb4ab0fe5"},
    "llama8b_kivi": {"dram_bytes": 79039488, "captured": "full size",
        "lsu_global_sectors_per_request": 1.77,
        "sources_sha256": "dea02c0843e6721dbcef2a62c5c8e5d49bdfabf21868936614c2c7adb4ab0fe5"},
    "llama8b_window": {"dram_bytes": 130097920, "captured": "full size",
        "lsu_global_sectors_per_request": 5.57,
        "sources_sha256": "dea02c0843e6721dbcef2a62c5c8e5d49bdfabf21868936614c2c7adb4ab0fe5"},
    "llama8b_paged": {"dram_bytes": 112652544, "captured": "full size",
        "lsu_global_sectors_per_request": 6.67,
        "sources_sha256": "dea02c0843e6721dbcef2a62c5c8e5d49bdfabf21868936614c2c7adb4ab0fe5"},
}
TRAFFIC_SOURCES = tuple("bit_kv_cache_seeded_b200/csrc/" + f for f in (
    "kvq_decode_mma.cu", "kvq_async.cuh", "kvq_internal.h", "kvq_lm_common.cuh", "kvq_tiles.cuh", "kvq_window.cuh",
    "kvq_quantize_lm.cuh", "kvq_mla_umma.cu", "kvq_tcgen05.cuh"))


def kernel_sources_sha():
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_record(w):
    rec = TRAFFIC.get(w.name)
    if rec is None or rec["sources_sha256"] != kernel_sources_sha() or w.ctx != workload(w.name).ctx:
        return None
    return rec


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks during the timed region

class ClockSampler:
    """Polls NVML (read-only) for SM clock and throttle reasons while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                r = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                break
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() and args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _all_reduce(x: float, world: int, op) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, world: int) -> float:
    """Slowest rank's time: the job finishes when the last replica does."""
    import torch.distributed as dist
    return _all_reduce(x, world, dist.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(x: float, world: int) -> float:
    """Work done by all ranks together (each rank runs its own replica of the workload)."""
    import torch.distributed as dist
    return _all_reduce(x, world, dist.ReduceOp.SUM if world > 1 else None)


# ------------------------------------------------------------------ oracle (CPU) timing

def oracle_prepare(w, pairs, ctx, data=None):
    """Codes of ctx - 1 cached tokens for `pairs` (sequence 0, kv-head) pairs, prepared by the
    oracle itself (untimed: this is the prefill, not the decode step)."""
    from oracle import codec, tables
    signs, S = rotation_and_sketch(w)
    ck, tk = tables.lloyd_max_tables_f32(w.k_bits)
    cv, tv = tables.lloyd_max_tables_f32(w.v_bits)
    kS = S if w.k_mode == "lm_qjl" else None
    vS = S if w.v_mode == "lm_qjl" else None
    data = data or generate(w, "cpu", seqs=range(1), ctx=ctx)
    K = data["k"][0].double().numpy()
    V = data["v"][0].double().numpy()
    q = data["q"][0].double().numpy()
    prepared = []
    for hk in range(pairs):
        h = hk % w.n_kv_heads
        rk = [codec.quantize_vector(x, w.k_bits, signs, ck, tk, kS) for x in K[h, :ctx - 1]]
        rv = [codec.quantize_vector(x, w.v_bits, signs, cv, tv, vS) for x in V[h, :ctx - 1]]
        prepared.append((h, rk, rv, K[h, ctx - 1], V[h, ctx - 1], q[h * w.group:(h + 1) * w.group]))
    return dict(w=w, signs=signs, ck=ck, tk=tk, cv=cv, tv=tv, kS=kS, vS=vS, pairs=prepared, ctx=ctx)


def oracle_step(P):
    """One timed oracle decode step over the prepared pairs: quantize the new token, dequantize
    the cache, attend. Returns (seconds, KV tokens the step covers in the metric's unit)."""
    from oracle import attention, codec
    w, signs = P["w"], P["signs"]
    scale = 1.0 / math.sqrt(w.head_dim)
    t0 = time.perf_counter()
    for h, rk, rv, knew, vnew, qh in P["pairs"]:
        rk2 = rk + [codec.quantize_vector(knew, w.k_bits, signs, P["ck"], P["tk"], P["kS"])]
        rv2 = rv + [codec.quantize_vector(vnew, w.v_bits, signs, P["cv"], P["tv"], P["vS"])]
        Kh = attention.dequantize_many(np.stack([r["codes"] for r in rk2]), np.array([r["n16"] for r in rk2]),
                                       P["ck"], signs, np.array([r.get("gamma16", 0.0) for r in rk2]),
                                       np.stack([r["z"] for r in rk2]) if P["kS"] is not None else None, P["kS"])
        Vh = attention.dequantize_many(np.stack([r["codes"] for r in rv2]), np.array([r["n16"] for r in rv2]),
                                       P["cv"], signs, np.array([r.get("gamma16", 0.0) for r in rv2]),
                                       np.stack([r["z"] for r in rv2]) if P["vS"] is not None else None, P["vS"])
        attention.decode_attention(qh, Kh, Vh, scale)
    dt = time.perf_counter() - t0
    return dt, len(P["pairs"]) * P["ctx"] / w.n_kv_heads


FP4_SAMPLE_CTX = 4096  # tokens of the FP4 latent cache the oracle covers per step


def oracle_prepare_fp4(w, ctx):
    """FP4 latent cache of the first `ctx` tokens of sequence 0, coded by the oracle (untimed)."""
    from oracle import codec
    data = generate(w, "cpu", seqs=range(1), ctx=ctx)
    lat = data["latent"][0].float().numpy()
    coded = [codec.fp4_quantize(lat[t]) for t in range(ctx - 1)]
    return dict(w=w, packed=np.stack([c[0] for c in coded]), scales=np.stack([c[1] for c in coded]),
                new=lat[ctx - 1], rope=data["rope"][0].double().numpy(), q=data["q"][0].double().numpy(),
                ctx=ctx)


def oracle_step_fp4(P):
    """One oracle decode step over the sample: code the new token, dequantise, attend (all heads)."""
    from oracle import attention, codec
    w = P["w"]
    t0 = time.perf_counter()
    pk, sc = codec.fp4_quantize(P["new"])
    packed = np.concatenate([P["packed"], pk[None]])
    scales = np.concatenate([P["scales"], sc[None]])
    attention.mla_decode_attention_many(P["q"], packed, scales, P["rope"],
                                        1.0 / math.sqrt(w.latent_dim + w.rope_dim))
    return time.perf_counter() - t0, P["ctx"]


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def run_reference(args, world, rank):
    w = workload(args.workload)
    if args.ctx > 0:
        w = w.with_(ctx=args.ctx)
    metric, unit = METRIC, UNIT
    if rank != 0:
        return
    if w.k_mode == "fp4":
        P, step_fn = oracle_prepare_fp4(w, FP4_SAMPLE_CTX), oracle_step_fp4
        sample = f"sequence 0, first {FP4_SAMPLE_CTX} of {w.ctx} tokens, all {w.n_q_heads} heads, per step"
    else:
        pairs = 1
        P, step_fn = oracle_prepare(w, pairs, w.ctx), oracle_step
        sample = f"{pairs} (sequence, kv-head) pair of {w.batch * w.n_kv_heads} per step, ctx {w.ctx}"
    times = []
    for i in range(args.warmup + args.steps):
        dt, toks = step_fn(P)
        if i >= args.warmup:
            times.append(dt)
    per_step = sum(times) / len(times)
    value = toks / per_step
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": unit, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ------------------------------------------------------------------ our arm

def cpu_baseline(w, seconds):
    """The oracle, as it stands, on a bounded sample of workload w, scaled to KV tokens/s."""
    if w.k_mode == "fp4":
        P, step_fn = oracle_prepare_fp4(w, FP4_SAMPLE_CTX), oracle_step_fp4
        what = f"sequence 0, first {FP4_SAMPLE_CTX} of {w.ctx} tokens, all {w.n_q_heads} heads"
    else:
        pairs = 2
        P, step_fn = oracle_prepare(w, pairs, w.ctx), oracle_step
        what = f"{pairs} (sequence, kv-head) pairs at ctx {w.ctx} (of {w.batch * w.n_kv_heads} pairs per step)"
    tot, toks_tot, reps = 0.0, 0.0, 0
    while tot < seconds and reps < 200:
        dt, toks = step_fn(P)
        tot, toks_tot, reps = tot + dt, toks_tot + toks, reps + 1
    return {"value": toks_tot / tot, "unit": "KV tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{reps} repetitions of one decode step over {what}, fp64 numpy"}


def measure(kvq, w, args, world, dev):
    """One workload: device-resident timed steps, per-kernel times, end-to-end steps through the
    host-buffer call. Returns the fields of its JSON line (without cpu_baseline)."""
    stream = torch.cuda.current_stream()
    cfg = kvq.cfg_for_workload(w)
    per_tok = kvq.kvq_packed_bytes_per_token(cfg)
    heads_kv = 1 if w.k_mode == "fp4" else w.n_kv_heads
    bytes_prefix = w.batch * heads_kv * w.ctx * per_tok
    replicas = max(2, math.ceil(2.5 * L2_BYTES / max(bytes_prefix, 1)))
    n_steps = args.warmup + args.steps
    n_e2e = args.steps
    capacity = w.ctx + n_steps + n_e2e + 1

    # Prefix of ctx - 1 tokens in every replica (identical content), built in sequence slices. The
    # caches draw their rotation signs and sketch matrix from the configuration's seeds.
    def make_cache(r):
        if not w.paged:
            return kvq.KvqCache(cfg, w.batch, capacity, device=dev)
        pps = (capacity + 63) // 64  # pages of 64 tokens per sequence, shuffled over the pool
        perm = torch.randperm(w.batch * pps, generator=torch.Generator().manual_seed(r)).to(torch.int32)
        table = perm.reshape(w.batch, pps).to(dev)
        return kvq.KvqCache(cfg, w.batch, 0, device=dev, block_table=table, n_pages=w.batch * pps)
    caches = [make_cache(r) for r in range(replicas)]
    step_b = max(1, w.batch // 8)
    q = None
    a_name, b_name = ("latent", "rope") if w.k_mode == "fp4" else ("k", "v")
    q_ms = 0.0  # device time of the first replica's prefill appends (all sequences, ctx - 1 tokens)
    for b0 in range(0, w.batch, step_b):
        seqs = list(range(b0, min(w.batch, b0 + step_b)))
        d = generate(w, dev, seqs=seqs, ctx=w.ctx - 1)
        for ci, c in enumerate(caches):
            if ci == 0:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            c.quantize(d[a_name], d[b_name], seq_ids=seqs)
            if ci == 0:
                e1.record(stream)
                e1.synchronize()
                q_ms += e0.elapsed_time(e1)
        q = d["q"] if q is None else torch.cat([q, d["q"]])
        del d
    n_vec = w.batch * (w.ctx - 1) * (1 if w.k_mode == "fp4" else 2 * w.n_kv_heads)
    if w.k_mode != "fp4":  # vectors actually coded by the prefill (the window keeps the rest in bf16)
        n_vec = w.batch * coded_len(w, w.ctx - 1) * 2 * w.n_kv_heads
    # New tokens of every step, resident in HBM (the e2e steps draw theirs on the host).
    news = []
    for s in range(n_steps):
        d = generate(w, dev, step=s)
        news.append((d[a_name], d[b_name]))
    out = torch.empty((w.batch, w.n_q_heads, caches[0].out_dim), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    lens0 = int(caches[0].lengths()[0])
    caches_info = caches[0].layout()

    def step(i):
        # one decode step through the fused entry: append the new token of every sequence and
        # attend (kvq_decode_step = kvq_quantize + kvq_decode_attention, prep overlapping the append)
        c = caches[i % replicas]
        k_new, v_new = news[i % len(news)]
        c.step(k_new, v_new, q, out)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kv_tokens = 0
    launches0 = kvq.kvq_kernel_launches()
    # The timed steps run back to back, with no event between them (an event between two steps
    # would keep the next step's first kernel from overlapping the previous step's last one).
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        for j in range(args.steps):
            i = args.warmup + j
            step(i)
            kv_tokens += w.batch * (int(caches[i % replicas].lengths()[0]))
        end.record(stream)
        torch.cuda.synchronize()
    launches = kvq.kvq_kernel_launches() - launches0
    barrier(world)
    torch.cuda.synchronize()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    ms_per_step = elapsed_ms / args.steps
    value = sum_over_ranks(kv_tokens, world) / (elapsed_ms / 1e3)

    # Per-kernel device times: the same decode through the measurement entry, which records CUDA
    # events between its kernels (prep | split kernel | reduce), rotating over the replicas.
    n_k = min(max(args.steps, 10), 50)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_k)]
    torch.cuda.synchronize()
    for j in range(n_k):
        c = caches[j % replicas]
        kvq.kvq_debug_decode_timed(c.handle, q, out, c.workspace, kev[j])
    torch.cuda.synchronize()
    kern_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in kev) / n_k for i in range(3)]
    kern_ms = [max_over_ranks(x, world) for x in kern_ms]
    lens_k = sum(coded_len(w, int(caches[j % replicas].lengths()[0])) for j in range(n_k)) / n_k

    # End to end through the library's host-buffer call (kvq_decode_step_host): every step's new
    # keys, values and query start in pinned host memory and its output ends there. The library
    # copies the inputs in on its own stream (overlapping the previous step) and the output out on
    # another (overlapping the next step); each call records an event after its output copy, and
    # the closing event waits for the last ones, so the timed region spans every copy.
    host_news = []
    for s in range(n_e2e):
        k_new, v_new = news[s % len(news)]
        host_news.append((k_new.cpu().pin_memory(), v_new.cpu().pin_memory()))
    q_host = q.cpu().pin_memory()
    host_outs = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    out_events = [torch.cuda.Event() for _ in range(n_e2e)]
    for c in caches:  # one untimed call per cache: its staging buffer and copy streams now exist
        c.step_host(*host_news[0], q_host, host_outs[0])
    e2e_tokens = 0
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for j in range(n_e2e):
        c = caches[j % replicas]
        c.step_host(*host_news[j], q_host, host_outs[j % 2], out_event=out_events[j])
        e2e_tokens += w.batch * int(c.lengths()[0])
    for e in out_events[-2:]:
        stream.wait_event(e)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world)
    e2e_tokens = sum_over_ranks(e2e_tokens, world)
    e2e_value = e2e_tokens / (e2e_ms / 1e3) if e2e_ms > 0 else None
    h2d = sum(t.numel() * t.element_size() for t in (*host_news[0], q_host))
    d2h = host_outs[0].numel() * host_outs[0].element_size()

    peaks, peak_kind = measured_peaks()
    # bytes one decode call reads: packed history + bf16 K and V of the window
    bytes_step = w.batch * heads_kv * (coded_len(w, lens0 + 1) * per_tok + window_len(w, lens0 + 1) * 4 * w.head_dim)
    call_ms = sum(kern_ms)  # kvq_decode_attention alone, from the per-kernel events
    achieved_call = bytes_step / (call_ms / 1e3) / 1e9
    bytes_kernel = w.batch * heads_kv * lens_k * per_tok      # the split kernel's algorithmic bytes
    if w.k_mode == "kivi" or w.sink_tokens or w.recent_tokens:  # its extra CTAs read the bf16 window
        win_k = sum(window_len(w, int(caches[j % replicas].lengths()[0])) for j in range(n_k)) / n_k
        bytes_kernel += w.batch * heads_kv * win_k * 4 * w.head_dim
    if w.k_mode == "fp4":
        # 64 heads x (latent + rope) MACs for the logits and 64 x latent for the values, per token:
        # a dense contraction (146 GFLOP at 2^20 tokens), so the tensor roofline bounds it. The
        # kernel runs back to back for tens of ms: the sustained bf16 (= f16) figure applies.
        flops_kernel = 2.0 * w.batch * w.n_q_heads * (2 * w.latent_dim + w.rope_dim) * lens_k
        roof = {"bound": "tensor", "achieved": flops_kernel / (kern_ms[1] / 1e3) / 1e12,
                "peak": float(peaks["bf16_tflops_sustained"]), "unit": "TFLOP/s",
                "flops_per_launch": flops_kernel, "hbm_gbs_of_kernel": bytes_kernel / (kern_ms[1] / 1e3) / 1e9}
    else:
        roof = {"bound": "hbm", "achieved": bytes_kernel / (kern_ms[1] / 1e3) / 1e9,
                "peak": float(peaks["hbm_gbs"]), "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    tr = traffic_record(w)
    # load efficiency of the packed streams: the split kernels stage whole tile pairs with 1-D bulk
    # copies (TMA), so every copy moves full 16-byte-aligned, contiguous runs; its size follows from
    # the layout (FP4: the latent kernel loads 16-byte vectors into registers instead)
    info = caches_info
    if w.k_mode == "fp4":
        load_eff = {"path": "16-byte vector loads of whole tile rows", "bytes_per_request": 16}
    else:
        ktb, vtb = int(info[1]), int(info[2])
        nb = 128 if (w.v_mode == "lm_qjl") else 64
        load_eff = {"path": "1-D bulk copies (TMA) of whole tile pairs",
                    "bytes_per_copy": {"k_pair": 2 * ktb, "v_norms": nb, "v_pair": 2 * vtb},
                    "mean_bytes_per_copy": (2 * ktb + 2 * nb + 2 * vtb) / 4.0}
    line = {
        "value": value, "ms_per_step": ms_per_step,
        # the contractions' operand / accumulation types: exact int8 tensor-core products with int32
        # sums and fp32 softmax (LM), f16/bf16 tcgen05 products with fp32 accumulators (FP4 latent)
        "dtype": "f16/f32" if w.k_mode == "fp4" else "s8/s32/f32",
        "config": workload_config(w, world),
        "l2_detail": f"{replicas} cache replicas x {bytes_prefix / 1e6:.1f} MB rotated per step",
        "hbm_gbs": achieved_call, "frac_of_8tbs": achieved_call / 8000.0,
        "roofline": dict(roof, traffic=None if tr is None else tr["dram_bytes"], peak_kind=peak_kind,
                         kernel=KERNEL_NAMES[w.name],
                         bytes_per_launch=bytes_kernel, ms_per_launch=kern_ms[1],
                         load_efficiency=dict(load_eff, dram_over_algorithmic=None if tr is None else
                                              tr["dram_bytes"] / bytes_kernel,
                                              lsu_global_sectors_per_request=None if tr is None else
                                              tr["lsu_global_sectors_per_request"])),
        "decode_call": {"ms": call_ms, "bytes": bytes_step, "gbs": achieved_call,
                        "kernels_ms": {"prep": kern_ms[0], "split": kern_ms[1], "reduce": kern_ms[2]}},
        "e2e": {"value": e2e_value, "unit": "KV tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n_e2e,
                "path": "kvq_decode_step_host: pinned host inputs and output, library copy streams"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        # prefill-rate append (kvq_quantize with ctx - 1 tokens per sequence, in 8 calls of batch/8
        # sequences): vectors = K and V vectors of every kv-head (FP4: latent tokens)
        "quantize": {"vectors": n_vec, "ms": q_ms, "vectors_per_s": n_vec / (q_ms / 1e3) if q_ms > 0 else None,
                     "input_gbs": n_vec * (w.latent_dim + w.rope_dim if w.k_mode == "fp4" else w.head_dim) * 2
                     / (q_ms / 1e3) / 1e9 if q_ms > 0 else None},
    }
    for c in caches:
        c.close()
    del caches, news, host_news
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return line


def run_ours(args, world, rank, local):
    import bit_kv_cache_seeded_b200 as kvq
    kvq.load()
    dev = f"cuda:{local}"
    torch.cuda.set_device(dev)
    w = workload(args.workload)
    if args.ctx > 0:
        w = w.with_(ctx=args.ctx)
    head = measure(kvq, w, args, world, dev)
    line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "data": "synthetic"}
    line.update({k: v for k, v in head.items() if k not in ("value", "ms_per_step")})
    # the other full-size workloads, each with its own roofline and CPU baseline (one GPU only:
    # a scaling run times the headline workload alone)
    extra = [] if (world > 1 or args.ctx > 0 or args.only) else [n for n in EXTRA_WORKLOADS if n != w.name]
    if extra:
        line["workloads"] = {}
        for name in extra:
            line["workloads"][name] = measure(kvq, workload(name), args, world, dev)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, 10.0)
        for name in extra:
            if name in WORKLOADS:  # the variants' oracle is the same decode over another codec
                line["workloads"][name]["cpu_baseline"] = cpu_baseline(WORKLOADS[name], 3.0)
    if rank == 0:
        print(json.dumps(line))


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
