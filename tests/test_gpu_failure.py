"""Failure detection on the GPU without faulting it.

Every pipeline wait in the kernels is bounded in time.  With the stall
injection hook on, CTA 0's producer never fills a stage -- its consumers wait
for a flag that nothing sets -- so, with a 20 ms limit, those waits run out:
the kernel must record DG_ERR_TIMEOUT (with the role that gave up) in the
device status word, drain its own copies and MMAs, free TMEM and return, and
the context must stay usable, so the next call is correct.  Covered for the
persistent one-CTA kernel, the K-split (cluster) kernel and the CTA-pair
kernel (where the first pair stalls, so either of its CTAs may report)."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import assert_close, bits, dev_dense

pytestmark = pytest.mark.gpu

DG_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from moe_grouped_gemm_wt_b200 import build as b
    b.build()
    import moe_grouped_gemm_wt_b200 as m
    m.load_library()
    m.dg_set_num_sms(0)
    m.dg_set_wait_timeout_ns(0)
    assert m.dg_get_device_status() == 0
    return m


@pytest.mark.parametrize("M,N,K,family,first_ctas", [
    (1024, 4096, 4096, 1, 1),   # persistent one-CTA tiles
    (128, 2112, 7168, 1, 1),    # K split over clusters
    (2048, 4096, 4096, 2, 2),   # 256-row tiles on CTA pairs
])
def test_wait_timeout_is_reported_and_the_context_survives(dg, oracle_mod, M, N, K, family, first_ctas):
    p = gi.dense_problem(M, N, K, seed_a=71, seed_b=72)
    A, sA, B, sB, D = dev_dense(p)
    dg.dg_set_tile_family(family)
    dg.dg_set_wait_timeout_ns(20_000_000)
    dg.dg_set_stall_injection(True)
    try:
        assert dg.dg_describe_config(0, M, N, K).split()[7] == f"pair={family - 1}"
        dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
        st, word = dg.dg_get_device_status_detail()
    finally:
        dg.dg_set_stall_injection(False)
        dg.dg_set_wait_timeout_ns(0)
        dg.dg_set_tile_family(0)
    assert st == DG_ERR_TIMEOUT, f"status {st}, word {word:#x}"
    assert word & 0xFF == DG_ERR_TIMEOUT
    assert (word >> 8) & 0xF in (2, 3)  # the MMA or promotion warps gave up
    assert word >> 20 < first_ctas        # in the stalled CTA (or pair)
    assert dg.dg_get_device_status() == DG_ERR_TIMEOUT  # read and cleared
    assert dg.dg_get_device_status() == 0

    # same buffers, default limit: the result is right
    dg.dg_set_tile_family(family)
    try:
        dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
    finally:
        dg.dg_set_tile_family(0)
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(bits(D), ref, f"after a timeout, {M}x{N}x{K}")
