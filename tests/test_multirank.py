"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): the max-over-ranks
timing reduction and the whole-job aggregation used for --gpus N."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    r, w, local = bench.dist_info()
    t_total = 10.0 + 5.0 * rank            # rank 1 is the slowest
    tmax = bench.reduce_max(t_total, w, "cpu")
    bench.barrier(w)
    rate = bench.whole_job_rate(2.0e9, 4, w, tmax)
    q.put((r, w, local, tmax, rate))
    dist.destroy_process_group()


def test_two_ranks_take_max_and_count_all_work():
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
    for rank, (r, w, local, tmax, rate) in enumerate(res):
        assert (r, w, local) == (rank, 2, rank)
        assert tmax == 15.0
        assert rate == pytest.approx(2.0e9 * 4 * 2 / 15e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(1.0, 10, 1, 1000.0) == pytest.approx(10.0)
