"""Grouped GEMMs captured once in a CUDA graph and replayed with new group
metadata.

The grouped layouts read their group metadata (masked_m, m_indices) only on
the device.  That is what lets MoE decode run under CUDA graphs (hada.io
DeepGEMM summary, section "Dense va Grouped GEMM": the masked layout serves
decode under CUDA graphs, where the host does not know how many tokens each
expert received).  A graph captured after one direct call is replayed after
the caller has rewritten the activations and the metadata in place; every
replay must match the oracle for the metadata it saw, with the rows outside
the groups left untouched bit for bit."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import SENTINEL, assert_close, bits, dev_contiguous, dev_masked

pytestmark = pytest.mark.gpu


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


def _capture(call):
    call()  # the first call on the device (module, attributes, plan caches)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="global"):
        call()
    torch.cuda.synchronize()
    return graph


def test_masked_replay_with_new_masked_m(dg, oracle_mod):
    G, max_m, N, K = 8, 256, 2048, 1152
    counts = [np.array([1, 129, 256, 0, 64, 200, 128, 17], np.int32),
              np.array([256, 0, 3, 130, 77, 128, 255, 1], np.int32)]
    probs = [gi.masked_problem(G, max_m, N, K, masked_m=mm, seed_a=700 + i, seed_b=710)
             for i, mm in enumerate(counts)]
    A, sA, B, sB, D, m = dev_masked(probs[0])
    graph = _capture(lambda: dg.dg_fp8_grouped_gemm_masked(A, sA, B, sB, D, m, max_m))
    for p in probs:
        new_A, new_sA, _, _, _, new_m = dev_masked(p)  # same weights (same seed)
        for dst, src in ((A, new_A), (sA, new_sA), (m, new_m)):
            dst.copy_(src)
        D.view(torch.int16).fill_(SENTINEL)
        graph.replay()
        torch.cuda.synchronize()
        assert dg.dg_get_device_status() == 0
        got = bits(D)
        _, ref = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], p["masked_m"],
                                           np.full((G, max_m, N), SENTINEL, np.uint16))
        valid = np.arange(max_m)[None, :] < p["masked_m"][:, None]
        assert np.array_equal(got[~valid], ref[~valid])
        assert_close(got[valid], ref[valid], f"masked replay, masked_m={p['masked_m'].tolist()}")
    del graph


def test_contiguous_replay_with_new_m_indices(dg, oracle_mod):
    N, K = 2000, 1024
    # the same padded row count (1152) under two different expert loads
    probs = [gi.contiguous_problem(rows, N, K, seed_a=720 + i, seed_b=730)
             for i, rows in enumerate(([300, 0, 517, 128], [128, 640, 1, 250]))]
    assert probs[0]["M"] == probs[1]["M"]
    A, sA, B, sB, D, mi = dev_contiguous(probs[0])
    graph = _capture(lambda: dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi))
    for p in probs:
        new_A, new_sA, _, _, _, new_mi = dev_contiguous(p)  # same weights (same seed)
        for dst, src in ((A, new_A), (sA, new_sA), (mi, new_mi)):
            dst.copy_(src)
        D.view(torch.int16).fill_(SENTINEL)
        graph.replay()
        torch.cuda.synchronize()
        assert dg.dg_get_device_status() == 0
        got = bits(D)
        _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"],
                                               np.full((p["M"], N), SENTINEL, np.uint16))
        pad = p["m_indices"] < 0
        assert np.array_equal(got[pad], ref[pad])
        assert_close(got[~pad], ref[~pad], "contiguous replay")
    del graph
