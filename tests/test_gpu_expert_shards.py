"""Expert-parallel shards of the grouped workloads, run through the library on
one GPU (the single-GPU half of the multi-GPU expert-parallel run).

bench.shard_experts gives rank r of `world` the experts
[r*G/world, (r+1)*G/world): for the contiguous layout their row segments
(each with the padding rows that follow it), for the masked layout whole
groups, with B, sB and the group metadata sliced and the indices renumbered
from 0.  Every shard of 2-, 4- and 8-way splits of a contiguous problem
shaped like the contiguous MoE workload (8 experts, K=2048; fewer rows and a
narrower N) and of a masked problem shaped like the masked MoE decode
workload (16 experts of at most 256 rows, K=7168; a narrower N) is run here
one after another, in both scale modes, and each shard's output must equal
its rows of the whole problem's oracle result: computed rows within the
parity tolerance, padding and masked rows bit for bit (sentinel pre-fill).
The masked layout is fed by expert-parallel decode (hada.io DeepGEMM
summary, section "Dense va Grouped GEMM")."""
import os
import sys

import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import SENTINEL, assert_close, bits

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402

WORLDS = (2, 4, 8)


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from moe_grouped_gemm_wt_b200 import build as b
    b.build()
    import moe_grouped_gemm_wt_b200 as m
    m.load_library()
    m.dg_set_num_sms(0)
    assert m.dg_get_device_status() == 0
    return m


def _run_shard(dg, q):
    """One shard through the library (the bench's own call path)."""
    dev = torch.device("cuda")
    d = bench.to_device(q, torch, dev, dg)
    d["D"].view(torch.int16).fill_(SENTINEL)
    bench.call(dg, q, d)
    st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    return bits(d["D"])


@pytest.fixture(scope="module", params=[False, True], ids=["fp32_scales", "ue8m0"])
def contiguous_case(request, oracle_mod):
    ue8m0 = request.param
    rows = [300, 512, 0, 128, 700, 64, 256, 200]   # 8 experts, ragged, one empty
    p = gi.contiguous_problem(rows, 512, 2048, seed_a=111, seed_b=112, ue8m0=ue8m0)
    p["kind"], p["ue8m0"] = "contiguous", ue8m0
    init = np.full((p["M"], p["N"]), SENTINEL, np.uint16)
    if ue8m0:
        _, ref = oracle_mod.grouped_contiguous_ue8m0(p["A"], oracle_mod.pack_ue8m0(p["sA"]), p["B"],
                                                     oracle_mod.pack_ue8m0(p["sB"]), p["m_indices"], init)
    else:
        _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"], init)
    return p, ref


@pytest.fixture(scope="module", params=[False, True], ids=["fp32_scales", "ue8m0"])
def masked_case(request, oracle_mod):
    ue8m0 = request.param
    mm = np.random.default_rng(113).integers(1, 257, 16).astype(np.int32)
    mm[5] = 0                                        # an expert with no tokens
    p = gi.masked_problem(16, 256, 384, 7168, masked_m=mm, seed_a=114, seed_b=115, ue8m0=ue8m0)
    p["kind"], p["ue8m0"] = "masked", ue8m0
    init = np.full((16, 256, 384), SENTINEL, np.uint16)
    if ue8m0:
        _, ref = oracle_mod.grouped_masked_ue8m0(p["A"], oracle_mod.pack_ue8m0(p["sA"]), p["B"],
                                                 oracle_mod.pack_ue8m0(p["sB"]), p["masked_m"], init)
    else:
        _, ref = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], p["masked_m"], init)
    return p, ref


@pytest.mark.parametrize("world", WORLDS)
def test_contiguous_shards_reassemble_the_whole_problem(dg, contiguous_case, world):
    p, ref = contiguous_case
    covered = np.zeros(p["M"], bool)
    for rank in range(world):
        q = bench.shard_experts(p, rank, world)
        if q["M"] == 0:
            continue
        lo, hi = q["row0"], q["row0"] + q["M"]
        assert not covered[lo:hi].any(), "shards overlap"
        covered[lo:hi] = True
        got = _run_shard(dg, q)
        want = ref[lo:hi]
        pad = q["m_indices"] < 0
        assert np.array_equal(got[pad], want[pad]), f"rank {rank}/{world}: padding rows written"
        assert_close(got[~pad], want[~pad], f"contiguous shard {rank}/{world}")
    # every non-padding row of the whole problem belongs to some shard
    assert covered[p["m_indices"] >= 0].all()


@pytest.mark.parametrize("world", WORLDS)
def test_masked_shards_reassemble_the_whole_problem(dg, masked_case, world):
    p, ref = masked_case
    seen = []
    for rank in range(world):
        q = bench.shard_experts(p, rank, world)
        g0, g1 = q["group0"], q["group0"] + q["G"]
        seen.extend(range(g0, g1))
        got = _run_shard(dg, q)
        want = ref[g0:g1]
        valid = np.arange(q["max_m"])[None, :] < q["masked_m"][:, None]
        assert np.array_equal(got[~valid], want[~valid]), f"rank {rank}/{world}: masked rows written"
        assert_close(got[valid], want[valid], f"masked shard {rank}/{world}")
    assert seen == list(range(p["G"]))
