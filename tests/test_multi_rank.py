"""The N > 1 path of bench.py on CPU (gloo, world size 2).

The pass has no exchange step (every (batch, head) is independent), so N GPUs
run N independent replicas; the only cross-rank step is the timing: every
rank must see the max over ranks, and the whole-job value counts all
replicas' work against that max.
"""
import multiprocessing as mp
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r measured step / attention / pre-pass times
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)], dist, "cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_timings_are_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0] == results[1] == [2.0, 5.0, 0.5]


def test_replica_value_counts_all_ranks():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.replica_value(1, 1e12, 1.0) == pytest.approx(1000.0)
    assert bench.replica_value(8, 1e12, 2.0) == pytest.approx(4000.0)
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
