"""Multi-process plumbing of bench.py on CPU (gloo, world size 2): rendezvous, the max-over-ranks
time, the sum-over-ranks work, and the reference arm under torchrun printing exactly one line."""
import json
import os
import socket
import subprocess
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    args = types.SimpleNamespace(impl="reference")
    w, r, _ = bench.dist_setup(args)
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    bench.barrier(w)
    t = bench.max_over_ranks(1.5 + rank, w)      # each rank's own time
    n = bench.sum_over_ranks(1000.0 * (rank + 1), w)  # each rank's own work
    q.put((rank, t, n))
    dist.destroy_process_group()


def test_max_and_sum_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 2.5, 3000.0), (1, 2.5, 3000.0)]


def test_single_process_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.sum_over_ranks(7.0, 1) == 7.0


def test_reference_arm_under_torchrun_prints_one_line():
    """Rank 0 alone times the oracle and prints; rank 1 exits 0 without work."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    for _ in range(3):  # a free port can be taken between probing and binding: retry on that only
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
               "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.join(ROOT, "bench.py"),
               "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "0"]
        r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        if r.returncode == 0 or "ddress already in use" not in r.stderr:
            break
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["metric"].startswith("quantized-KV decode attention") and rec["value"] > 0
    assert rec["config"]["workload"] == "tiny" and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
