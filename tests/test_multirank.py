"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks, each timing its own
replica, agree on the slowest rank's time and on the whole-job rates (weak scaling,
no collective on the data path)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
    ms = bench.reduce_max(local_ms, dist, torch.device("cpu"))
    gbs, tps = bench.weak_scaling_rates(1e9, 64, world, ms)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ms, gbs, tps))


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, gbs, tps in out:
        assert ms == pytest.approx(15.0)
        assert gbs == pytest.approx(2 * 1e9 / 15e-3 / 1e9)
        assert tps == pytest.approx(2 * 64 / 15e-3)


def test_single_process_is_the_identity():
    import bench
    assert bench.reduce_max(3.5, None, None) == 3.5
    gbs, tps = bench.weak_scaling_rates(2e9, 10, 1, 2.0)
    assert gbs == pytest.approx(1000.0) and tps == pytest.approx(5000.0)
