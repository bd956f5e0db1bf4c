"""Host logic of the multi-GPU benchmark run, on CPU with two gloo ranks: the
slowest rank's time is what every rank reports, and the job's throughput is
all ranks' queries over that time (replicas, weak scaling)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = 1.0 + rank                      # rank 1 is the slower one
    m = bench.max_over_ranks(ms, world, device="cpu")
    out.put((rank, m, bench.job_throughput(256, m, world)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [m for _, m, _ in res] == [2.0, 2.0]
    assert res[0][2] == pytest.approx(2 * 256 / 2e-3)


def test_bench_gpus_two_starts_two_ranks():
    """`bench.py --gpus 2` run as a plain process starts two ranks itself (the
    reference arm runs on CPU: rank 0 prints the only line, with n_gpus 2)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--config", "1", "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=300, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2


def test_rank_count_must_equal_gpus(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        gpus = 2
    with pytest.raises(SystemExit):
        bench.dist_setup(A())
    with pytest.raises(SystemExit):
        bench.run_reference(A())


def test_relaunch_command_keeps_the_arguments():
    import bench
    cmd = bench.relaunch_command(["--gpus", "4", "--steps", "3"], 4, 29500)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]
