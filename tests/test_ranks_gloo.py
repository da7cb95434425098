"""Multi-process rank logic of bench.py on CPU (gloo, world size 2).

The layer shards into independent (sequence, head) problems, so multi-GPU
runs are replicas with no collective on the data path.  What does need more
than one process is the timing protocol: every rank enters the same
barriers, the reported time is the max over ranks, and the reference arm is
run by rank 0 only.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    m = bench.max_over_ranks(1.5 + rank, w)          # each rank's own step time
    args = type("A", (), {"steps": 1, "warmup": 0, "ref_tokens": 64})()
    ref = bench.bench_reference(args, w, r)
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((rank, m, ref is None))


def test_two_rank_timing_protocol():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [m for _, m, _ in res] == [2.5, 2.5]       # max over ranks on every rank
    assert [none for _, _, none in res] == [False, True]   # reference arm: rank 0 only
