"""The N > 1 host logic of bench.py on CPU: world_size 2 over gloo.

Head split (the default): each rank takes a contiguous head range of the one
problem, builds the static mask itself and computes its heads with no
collective on the data path; here each rank runs its slice of a tiny problem
through the oracle, and the gathered slices must reassemble into the
single-process result.  Batch split: each rank works on its own batch element
(own input streams).  In both, the only collective is the max over ranks of the
device time."""
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


def _split_worker(rank, world, port, out):
    import datetime
    import math
    import sys

    import numpy as np
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import oracle
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        c = dict(synth.CONFIGS["tiny_radial"], H=3)       # 3 heads over 2 ranks: 2 + 1
        n, d = c["f"] * c["s"], c["d"]
        q, k, v = bench.rank_inputs("tiny_radial", c, rank, world, "heads")
        h0, h1 = bench.head_range(rank, world, c["H"])
        spec = oracle.spec_from(c["masks"][0], c["f"], c["s"], c["grid"])
        hr = h1 - h0
        rows_bh, rows_q = np.repeat(np.arange(hr), n), np.tile(np.arange(n), hr)
        o, _, _ = oracle.default().attention_rows(q, k, v, spec, oracle.TOKEN_EXACT, 1 / math.sqrt(d), rows_bh,
                                                  rows_q)
        parts = [None] * world
        dist.all_gather_object(parts, (h0, h1, o.reshape(1, hr, n, d)))
        if rank == 0:
            out.put(parts)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_head_split_reassembles_the_single_process_result():
    import math

    import numpy as np

    import oracle
    import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    parts = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    c = dict(synth.CONFIGS["tiny_radial"], H=3)
    n, d = c["f"] * c["s"], c["d"]
    assert [(h0, h1) for h0, h1, _ in parts] == [(0, 2), (2, 3)]
    got = np.concatenate([o for _, _, o in parts], axis=1)
    Q, K, V = synth.qkv_bf16("tiny_radial", H=3)
    spec = oracle.spec_from(c["masks"][0], c["f"], c["s"], c["grid"])
    rows_bh, rows_q = np.repeat(np.arange(3), n), np.tile(np.arange(n), 3)
    want, _, _ = oracle.default().attention_rows(Q, K, V, spec, oracle.TOKEN_EXACT, 1 / math.sqrt(d), rows_bh,
                                                 rows_q)
    assert np.array_equal(got, want.reshape(1, 3, n, d))


@pytest.mark.parametrize("H", [1, 3, 24, 40])
def test_head_ranges_cover_every_head_once(H):
    import bench
    for world in range(1, min(H, 8) + 1):
        ranges = [bench.head_range(r, world, H) for r in range(world)]
        covered = [h for h0, h1 in ranges for h in range(h0, h1)]
        assert covered == list(range(H)), (H, world)
        sizes = [h1 - h0 for h0, h1 in ranges]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        bench.head_range(0, H + 1, H)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.rank_tensor_ids(0) == (0, 1, 2)
