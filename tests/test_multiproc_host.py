"""The multi-process (one process per GPU) path of bench.py, exercised on the CPU with
two gloo ranks: the barrier, the max-over-ranks timing and the whole-job rate under
weak scaling (each rank its own batch, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    my_ms = [2.0, 5.0][rank]                       # rank 1 is the slow one
    ms = bench.max_over_ranks(world, my_ms)
    rate = bench.whole_job_rate(world, 1e12, ms)   # 1 TFLOP of work per rank
    result_q.put((rank, ms, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
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
    for rank, ms, rate in res:
        assert ms == pytest.approx(5.0)             # both ranks see the max
        assert rate == pytest.approx(2 * 1e12 / 5e-3)
