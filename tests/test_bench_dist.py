"""The multi-process path of bench.py on CPU: two gloo ranks run the rank setup,
barrier and aggregation the benchmark uses for N GPU replicas (total tokens over
ranks / slowest rank's time)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "FT_BENCH_BACKEND": "gloo"})
    import bench
    import torch.distributed as dist
    r, w, lr = bench.dist_setup(world)
    bench.barrier()
    tokens, secs = bench.aggregate(100 * (r + 1), 0.5 + r, None)
    q.put((r, w, lr, tokens, secs))
    dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for r, (rank, world, local, tokens, secs) in enumerate(res):
        assert (rank, world, local) == (r, 2, r)
        assert tokens == 300.0 and secs == 1.5      # sum of tokens, max of times


def test_single_process_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(7, 2.5) == (7, 2.5)
