"""The N > 1 path on CPU ranks (gloo, world size 2).

Sequences are independent and no step of decode attention exchanges data, so N GPUs run N
replicas with no collective on the data path; the only cross-rank step is bench.py's
max-over-ranks of the measured times.  This runs that step on two gloo ranks."""
import os
import socket

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r measured (1 + r) and (10 - r): every rank must end up with the slowest of each
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank], dist)
        q.put((rank, got, bench.aggregate(got[0], 1e6, world)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, agg in res:
        assert got == [2.0, 10.0]
        assert abs(agg - 2 * 1e6 / 2e-6 / 1e9) < 1e-9   # two replicas' bytes over the slowest time


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
