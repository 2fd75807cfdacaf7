"""The multi-GPU path of bench.py (independent replicas, one process per GPU):
its process-group setup, barrier and whole-job aggregation -- the work of all
ranks over the slowest rank's time -- run as two gloo ranks on the CPU."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, _ = bench.dist_setup(world, backend="gloo")
    assert (w, r) == (world, rank)
    bench.barrier(w)
    # rank r processed (r+1)*100 units in (r+1)*10 ms
    value, ms_max = bench.replica_throughput((rank + 1) * 100.0, 10.0 * (rank + 1), w, 1.0)
    mx = bench.max_over_ranks(float(rank), w)
    sm = bench.sum_over_ranks(1.0, w)
    out.put((rank, value, ms_max, mx, sm))
    bench.barrier(w)
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_replica_aggregation_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms_max, mx, sm in results:
        assert ms_max == 20.0                       # slowest rank's time
        assert abs(value - 300.0 / 0.020) < 1e-6    # all ranks' work over that time
        assert mx == 1.0 and sm == 2.0


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    value, ms_max = bench.replica_throughput(500.0, 25.0, 1, 1e3)
    assert ms_max == 25.0 and abs(value - 500.0 / 0.025 / 1e3) < 1e-9
