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


def test_reference_arm_on_non_zero_rank_does_nothing(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        config, batch, density, steps, warmup = 3, None, 0.38, 1, 1
    bench.run_reference(A())
    assert capsys.readouterr().out == ""
