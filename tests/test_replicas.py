"""The multi-GPU path of bench.py is replicas only: each rank times its own
copy of the layer step and the job's time is the max over ranks. Checked here
with world_size 2 over gloo on the CPU (no GPU)."""
import importlib.util
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        ms = b.job_ms(10.0 + 2.0 * rank, dist, "cpu")      # rank r timed 10 + 2 r ms
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(repr(ms))
    finally:
        dist.destroy_process_group()


def test_job_time_is_the_max_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [float(open(tmp_path / f"rank{r}.txt").read()) for r in range(world)]
    assert got == [12.0, 12.0]                               # every rank sees the slowest replica


def test_job_value_is_weak_scaling_over_the_job_time():
    b = _bench()
    assert b.job_ms(7.5) == 7.5                             # no process group: the local time
    one = b.job_value(1, 10**9, 10, 1000.0)                 # 10 GB in 1 s
    assert one == pytest.approx(10.0)
    assert b.job_value(2, 10**9, 10, 1000.0) == pytest.approx(2 * one)   # two replicas, same time
    assert b.job_value(2, 10**9, 10, 2000.0) == pytest.approx(one)       # the slow rank sets the time
