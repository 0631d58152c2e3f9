"""The N > 1 bench path on CPU: two gloo ranks (replicas) agree on the max
elapsed time and the summed units, and only rank 0 prints.  CPU only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist("gloo")
    elapsed, units = bench.aggregate(dist, 10.0 + 5.0 * rank, 256.0)
    bench.barrier(dist)
    dist.destroy_process_group()
    q.put((rank, elapsed, units))


def test_two_rank_replica_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, elapsed, units in res:
        assert elapsed == 15.0          # max over ranks
        assert units == 512.0           # sum over the two replicas


def test_single_process_aggregation_is_identity():
    import bench
    assert bench.aggregate(None, 3.5, 7.0) == (3.5, 7.0)


def test_oracle_extrapolation_arithmetic():
    import bench
    W = bench.workload("full_b1")
    tps, step_s, block_s = bench.oracle_tokens_per_s(W, layer_s=2.0, head_row_s=0.1, steps_per_block=10)
    assert step_s == pytest.approx(30 * 2.0 + 256 * 0.1)
    assert block_s == pytest.approx(10 * step_s + 30 * 2.0)
    assert tps == pytest.approx(256 / block_s)
