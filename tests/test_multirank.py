"""Multi-rank bookkeeping of bench.py on CPU: world size 2 over gloo.

The path shards by independent canvases (replicas, no data-path
collective); the only cross-rank step is the timing reduction: max of the
times, sum of the work."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                           timeout=__import__("datetime").timedelta(seconds=60))
    import bench
    times, work = bench.reduce_over_ranks([10.0 + rank, 3.0 * (rank + 1)], [48 * (rank + 1), rank, 5], world, "cpu")
    q.put((rank, times, work))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, times, work in res:
        assert times == [11.0, 6.0]          # max over ranks
        assert work == [144, 1, 10]          # sum over ranks


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_over_ranks([1.5, 2.5], [3, 4], 1, "cpu") == ([1.5, 2.5], [3, 4])
