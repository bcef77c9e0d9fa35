"""The benchmark's multi-process path on CPU (gloo, world size 2): the
device time is the max over ranks, the throughput counts every rank's
tokens (weak scaling, one replica per rank), and only rank 0 runs the
reference (CPU oracle) arm."""
import os
import socket
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    total_ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
    mx = bench.reduce_max(total_ms, "cpu")
    value = bench.throughput(512, world, 20, mx)
    r, w, _ = bench.dist_env()
    args = types.SimpleNamespace(workload="tiny", ref_sample_tokens=1, warmup=3, steps=3)
    ran = None
    if rank != 0:
        import io
        import contextlib
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args)     # rank != 0: returns without work or output
        ran = buf.getvalue()
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, value, r, w, ran))


def test_two_ranks_max_time_and_weak_scaling_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, value, r, w, ran in out:
        assert r == rank and w == 2
        assert mx == 15.0                              # slowest rank's device time
        assert value == pytest.approx(512 * 2 * 20 / 0.015)  # all ranks' tokens / max time
    assert out[1][5] == ""                              # reference arm: rank 1 did nothing


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25, "cpu") == 3.25
    assert bench.throughput(8192, 1, 10, 33.0) == pytest.approx(8192 * 10 / 0.033)
