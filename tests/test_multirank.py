"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, max-over-ranks timing and the
whole-job value.  The path itself has no exchange step, so this is the only multi-rank logic."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 100.0 + 50.0 * rank  # rank 1 is the slowest
        mx = bench.reduce_max(my_ms, world, "cpu")
        results[rank] = (mx, bench.whole_job_value(10**9, 4, mx, world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(results)
    assert res[0][0] == res[1][0] == 150.0
    # 2 ranks x 1 GB x 4 steps in 0.15 s
    assert abs(res[0][1] - 2 * 4 / 0.15) < 1e-9


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.whole_job_value(2 * 10**9, 10, 1000.0, 1) == 20.0
