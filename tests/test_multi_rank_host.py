"""The N > 1 path of bench.py on CPU: two gloo ranks (one process each, as torchrun would
start them) set up the process group through bench.dist_setup and check the barrier and the
max / sum reductions behind the whole-job throughput of independent replicas (units summed
over ranks, time = the slowest rank)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    try:
        os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                          MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        import torch.distributed as dist

        import bench
        r, w, local = bench.dist_setup(world, backend="gloo")
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(w)
        mx = bench.max_over_ranks(1.5 + rank, w)
        sm = bench.sum_over_ranks(10.0 * (rank + 1), w)
        # rank r scored 1000 (r + 1) keys in (2 + r) ms: job = 3000 keys over the slowest 3 ms
        value, ms_max = bench.replica_throughput(1000.0 * (rank + 1), 2.0 + rank, w)
        bench.barrier(w)
        dist.destroy_process_group()
        q.put((rank, mx, sm, value, ms_max))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_reduce_like_the_bench():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for res in results:
        assert res[1] != "error", res
        _, mx, sm, value, ms_max = res
        assert mx == pytest.approx(2.5)
        assert sm == pytest.approx(30.0)
        assert ms_max == pytest.approx(3.0)
        assert value == pytest.approx(3000.0 / 3e-3)


def test_single_rank_reductions_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.0, 1) == 4.0
    assert bench.sum_over_ranks(4.0, 1) == 4.0
    value, ms = bench.replica_throughput(500.0, 2.0, 1)
    assert ms == 2.0 and value == pytest.approx(250000.0)
