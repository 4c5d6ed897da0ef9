"""GPU parity of the CTA-pair kernel (256-row tiles on two SMs, cta_group::2).

The tests restrict the planner to pair tiles (dg_set_tile_family) and cap
the SM count at 16 (8 pairs, so most problems take several waves), which runs
the pair kernel at sizes the oracle checks element by element: ragged
M (a pair whose second half is partly or wholly past M), ragged N (a
partial last tile, a 16-column remainder box), an odd number of K blocks (a two-block stage with one
block past K), several waves of tiles, contiguous groups whose 128-row blocks
pair up across groups and with padding, and masked groups whose valid rows
end in the first or the second half of a pair.  describe_config confirms the
path.  Placement and masking are bit-exact (sentinel pre-fill)."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import SENTINEL, assert_close, bits, dev_contiguous, dev_dense, dev_masked

pytestmark = pytest.mark.gpu

CAP_SMS = 16


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from moe_grouped_gemm_wt_b200 import build as b
    b.build()
    import moe_grouped_gemm_wt_b200 as m
    m.load_library()
    assert m.dg_get_device_status() == 0
    m.dg_set_num_sms(CAP_SMS)
    m.dg_set_tile_family(m.DG_TILES_PAIR)
    yield m
    m.dg_set_tile_family(m.DG_TILES_AUTO)
    m.dg_set_num_sms(0)


def _plan(dg, layout, M, N, K, G=1):
    return dict(kv.split("=") for kv in dg.dg_describe_config(layout, M, N, K, G).split())


@pytest.mark.parametrize("M,N,K", [
    (512, 1024, 1024),
    (1000, 1040, 896),    # ragged M and N, 7 K blocks
    (256, 4096, 512),     # one pair row, two waves over N
    (2048, 512, 2048),    # eight pair rows
    (130, 2048, 384),     # second half of the only pair row almost empty
])
def test_pair_dense_matches_oracle(dg, oracle_mod, M, N, K):
    plan = _plan(dg, 0, M, N, K)
    assert plan["pair"] == "1" and plan["BM"] == "256", plan
    p = gi.dense_problem(M, N, K, seed_a=3000 + M, seed_b=4000 + N)
    A, sA, B, sB, D = dev_dense(p)
    dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(bits(D), ref, f"pair dense {M}x{N}x{K}")


@pytest.mark.parametrize("rows,N,K", [
    ([384, 100, 300], 1024, 512),        # a pair split across groups, a padded block
    ([128, 128, 128, 128, 128, 256], 512, 384),  # every pair row spans two groups
    ([0, 640, 37], 1040, 256),           # an empty group, ragged N
])
def test_pair_contiguous_matches_oracle(dg, oracle_mod, rows, N, K):
    p = gi.contiguous_problem(rows, N, K, seed_a=61, seed_b=62)
    plan = _plan(dg, 1, p["M"], N, K, len(rows))
    assert plan["pair"] == "1", plan
    A, sA, B, sB, D, mi = dev_contiguous(p)
    dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi)
    assert dg.dg_get_device_status() == 0
    got = bits(D)
    init = np.full((p["M"], N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"], init)
    pad = p["m_indices"] < 0
    assert np.array_equal(got[pad], ref[pad])  # padding rows untouched, bit for bit
    assert_close(got[~pad], ref[~pad], f"pair contiguous {rows} N={N} K={K}")


@pytest.mark.parametrize("G,max_m,N,K,masked", [
    (4, 512, 1024, 384, [0, 100, 300, 512]),
    (3, 384, 512, 256, [384, 129, 1]),
    (2, 256, 2064, 128, [256, 255]),
])
def test_pair_masked_matches_oracle(dg, oracle_mod, G, max_m, N, K, masked):
    plan = _plan(dg, 2, max_m, N, K, G)
    assert plan["pair"] == "1", plan
    p = gi.masked_problem(G, max_m, N, K, masked_m=masked, seed_a=71, seed_b=72)
    A, sA, B, sB, D, mm = dev_masked(p)
    dg.dg_fp8_grouped_gemm_masked(A, sA, B, sB, D, mm)
    assert dg.dg_get_device_status() == 0
    got = bits(D)
    init = np.full((G, max_m, N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], p["masked_m"], init)
    valid = np.arange(max_m)[None, :] < np.asarray(masked)[:, None]
    assert np.array_equal(got[~valid], ref[~valid])  # rows past masked_m untouched
    assert_close(got[valid], ref[valid], f"pair masked G={G} max_m={max_m} N={N}")


def test_pair_deterministic_and_matches_one_cta_kernel(dg):
    M, N, K = 512, 1024, 1024
    p = gi.dense_problem(M, N, K, seed_a=81, seed_b=82)
    assert _plan(dg, 0, M, N, K)["pair"] == "1"
    A, sA, B, sB, D = dev_dense(p)
    dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
    first = bits(D)
    D.fill_(0)
    dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
    assert np.array_equal(first, bits(D))
    # the same problem on one-CTA tiles
    dg.dg_set_tile_family(dg.DG_TILES_ONE_CTA)
    try:
        assert _plan(dg, 0, M, N, K)["pair"] == "0"
        D.fill_(0)
        dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
        single = bits(D)
    finally:
        dg.dg_set_tile_family(dg.DG_TILES_PAIR)
    assert_close(first, single, "pair vs one-CTA kernel")
