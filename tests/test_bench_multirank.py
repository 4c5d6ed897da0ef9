"""The multi-rank path of bench.py on CPU: two gloo ranks reduce their step
times to the slowest one, and the whole-job value counts every rank's work.
The reference arm prints nothing and does no work on ranks other than 0."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.reduce_max_ms(1.0 + rank, dist, torch.device("cpu"), world)
        out[rank] = (ms, bench.whole_job_value(2e9, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_sum_the_work():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == 2.0 and out[1][0] == 2.0          # slowest rank's time on both
    assert out[0][1] == pytest.approx(2 * 2e9 / 2e-3 / 1e12)  # both ranks' work over it


def test_reference_arm_is_silent_on_other_ranks(capsys, monkeypatch):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench

    class Args:
        steps, warmup, gpus = 1, 1, 2
        workload = bench.HEADLINE

    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""
