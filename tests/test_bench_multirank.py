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


@pytest.mark.parametrize("world", [2, 3, 8])
def test_expert_shards_partition_the_grouped_problems(oracle_mod, world):
    """Each rank's shard holds whole experts (renumbered from 0); together
    the shards hold every expert once, and each shard's oracle result equals
    the rows of the whole problem's result that belong to its experts."""
    import sys
    import numpy as np
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import dg_inputs as gi

    SENT = 0x7FC1
    # contiguous: uneven groups, an empty group, padding rows
    p = gi.contiguous_problem([100, 300, 0, 37, 128, 5, 260, 64], 144, 256, seed_a=91, seed_b=92)
    full = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"],
                                         np.full((p["M"], 144), SENT, np.uint16))[1]
    seen_rows = 0
    total_flop = 0.0
    lo = 0
    for r in range(world):
        q = bench.shard_experts(p, r, world)
        g0 = r * p["G"] // world
        assert q["G"] == (r + 1) * p["G"] // world - g0
        assert q["M"] % 128 == 0 and np.all(q["m_indices"] < q["G"])
        part = oracle_mod.grouped_contiguous(q["A"], q["sA"], q["B"], q["sB"], q["m_indices"],
                                             np.full((q["M"], 144), SENT, np.uint16))[1]
        assert np.array_equal(part, full[lo:lo + q["M"]])
        lo += q["M"]
        seen_rows += q["M"]
        total_flop += bench.workload_cost(q)[0]
    assert seen_rows == p["M"]
    assert total_flop == bench.workload_cost(p)[0]

    # masked: whole groups
    pm = gi.masked_problem(5, 200, 144, 256, masked_m=[0, 200, 77, 150, 3], seed_a=93, seed_b=94)
    fullm = oracle_mod.grouped_masked(pm["A"], pm["sA"], pm["B"], pm["sB"], pm["masked_m"],
                                      np.full((5, 200, 144), SENT, np.uint16))[1]
    got = []
    for r in range(world):
        q = bench.shard_experts(pm, r, world)
        if q["G"] == 0:
            continue  # more ranks than experts: this rank has none
        got.append(oracle_mod.grouped_masked(q["A"], q["sA"], q["B"], q["sB"], q["masked_m"],
                                             np.full((q["G"], 200, 144), SENT, np.uint16))[1])
    assert np.array_equal(np.concatenate(got), fullm)


@pytest.mark.parametrize("world", [2, 3])
def test_expert_shards_of_a_ue8m0_problem_keep_the_mode(oracle_mod, world):
    """`bench.py --scales ue8m0` shards grouped problems the same way: the
    shards keep the mode, and their (power-of-two) scales pack into UE8M0
    words and back unchanged."""
    import sys
    import numpy as np
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import dg_inputs as gi

    for p in (gi.contiguous_problem([100, 300, 37, 128], 144, 512, seed_a=95, seed_b=96, ue8m0=True),
              gi.masked_problem(4, 200, 144, 512, masked_m=[0, 200, 77, 3], seed_a=97, seed_b=98,
                                ue8m0=True)):
        p["ue8m0"] = True
        for r in range(world):
            q = bench.shard_experts(p, r, world)
            assert q["ue8m0"]
            if q["G"] == 0:
                continue
            for s in (q["sA"], q["sB"]):
                nkb = s.shape[-1]
                assert np.array_equal(oracle_mod.unpack_ue8m0(oracle_mod.pack_ue8m0(s), nkb), s)
