"""The N > 1 host logic of bench.py on CPU: world_size 2 over gloo.

Each rank works on its own batch element (own input streams, no collective on
the data path); the only collective is the max over ranks of the device time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys

    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mx = bench.max_over_ranks(10.0 + rank * 5.0, world, "cpu")
        ids = bench.rank_tensor_ids(rank)
        out.put((rank, mx, ids))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_streams():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert [r[1] for r in results] == [15.0, 15.0]          # both ranks see the max
    ids = [set(r[2]) for r in results]
    assert not (ids[0] & ids[1])                              # disjoint input streams


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.rank_tensor_ids(0) == (0, 1, 2)
