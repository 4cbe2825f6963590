"""The benchmark's multi-rank host logic on CPU: two gloo ranks, the max
over ranks of the step time and the weak-scaling aggregate (every rank runs a
full batch; no data-path collective exists because images are independent)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist(world, "gloo")
    assert dist.is_initialized()
    r, w, lr = bench.dist_env()
    local_ms = [2.0, 5.0][rank]
    worst = bench.max_over_ranks(local_ms)
    bench.barrier()
    value = bench.weak_scaling_value(1e9, worst, w)
    q.put((r, w, worst, value))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for r, w, worst, value in out:
        assert w == 2 and worst == 5.0
        assert value == pytest.approx(2 * 1e9 / 5e-3 / 1e9)  # 400 GB/s


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.weak_scaling_value(2e9, 1.0, 1) == pytest.approx(2000.0)
