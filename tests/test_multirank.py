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


def test_launcher_starts_one_process_per_gpu_and_rank0_reports(tmp_path):
    """bench.py's launch command (torch.distributed.run, 127.0.0.1 rendezvous) starting
    two ranks of the rank plumbing (gloo): one JSON line, from rank 0, with the world
    size as n_gpus, the slowest rank's time and the work of both ranks."""
    import json
    import subprocess
    import sys
    import bench
    stub = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bench_rank_stub.py")
    cmd = bench.launch_command(["--gpus", "2", "--steps", "3", "--warmup", "3"], 2,
                               _free_port(), script=stub)
    assert cmd[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=2" in cmd and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    r = subprocess.run(["timeout", "-k", "30", "240", *cmd], capture_output=True, text=True,
                       env=env, cwd=str(tmp_path))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["n_gpus"] == 2 and res["rank"] == 0 and res["local_rank"] == 0
    assert res["ms_per_step"] == pytest.approx(15.0)
    assert res["value"] == pytest.approx(2 * 1e9 / 15e-3 / 1e9)


def test_main_relaunches_itself_when_not_under_a_launcher(monkeypatch):
    """--gpus N outside torch.distributed.run re-executes bench.py under it (N processes)
    and returns its exit code; a launched world that differs from --gpus is refused."""
    import subprocess
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    seen = {}

    def fake_call(cmd):
        seen["cmd"] = cmd
        return 7

    monkeypatch.setattr(subprocess, "call", fake_call)
    assert bench.main(["--gpus", "4", "--steps", "2", "--warmup", "3"]) == 7
    cmd = seen["cmd"]
    assert "--nproc-per-node=4" in cmd and cmd[-6:] == ["--gpus", "4", "--steps", "2",
                                                        "--warmup", "3"]
    assert cmd[cmd.index("--master-addr") + 4] == os.path.abspath(bench.__file__)
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse_args(["--gpus", "4"])
    with pytest.raises(SystemExit):
        bench.run_ranks(args, lambda *a: None, backend="gloo")
