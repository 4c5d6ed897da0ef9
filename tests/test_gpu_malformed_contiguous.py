"""Malformed contiguous-layout group data on the GPU, in both scale modes and
both tile families, against the oracle.

The segments of the contiguous layout are aligned to the 128-row M block
(hada.io DeepGEMM summary, section "Dense va Grouped GEMM"), so a block
belongs to the group of its first row.  A row is computed only when its
index equals that group; every other row stays untouched.  Input that breaks
the rule raises DG_ERR_BAD_GROUP_DATA in the device status word:
  * a mid-block change of group index,
  * a block whose first row is padding while later rows carry an index,
  * a block whose first-row index is out of range,
  * a row with an out-of-range index inside a valid block.
Each case checks the computed rows against the oracle (which follows the same
placement rule), the untouched rows bit for bit against the sentinel, and
the status word."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import SENTINEL, assert_close, bits, dev_contiguous

pytestmark = pytest.mark.gpu

BAD_GROUP = 6


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
    yield m
    m.dg_set_tile_family(m.DG_TILES_AUTO)


def _indices(case, M):
    idx = np.full(M, -1, np.int32)
    if case == "mid_block_change":
        idx[0:128] = 0
        idx[128:200] = 1
        idx[200:240] = 0        # differs from its block's first row (1)
        idx[256:M] = 1
    elif case == "padding_first_with_rows":
        idx[0:128] = 0
        idx[140:200] = 1        # block 1 starts with padding
        idx[256:M] = 1
    elif case == "out_of_range_row":
        idx[0:128] = 0
        idx[128:256] = 1
        idx[170] = 9            # index >= G inside a valid block
        idx[256:M] = 0
    else:  # "mixed": every kind at once, plus an out-of-range block
        idx[0:100] = 0
        idx[100:110] = 1
        idx[140:200] = 1
        idx[256:384] = 1
        idx[384:512] = 5
        idx[512:520] = 0
        idx[520] = 7
        idx[521:600] = 0
    return idx


CASES = ["mid_block_change", "padding_first_with_rows", "out_of_range_row", "mixed"]


@pytest.mark.parametrize("family", [1, 2], ids=["one_cta", "pair"])
@pytest.mark.parametrize("case", CASES)
def test_malformed_contiguous_fp32(dg, oracle_mod, family, case):
    N, K = 272, 384
    M = 5 * 128                  # 2.5 pair rows: the last pair has one half
    p = gi.contiguous_problem([256, 384], N, K, seed_a=91, seed_b=92)
    p["m_indices"] = _indices(case, M)
    dg.dg_set_tile_family(family)
    try:
        A, sA, B, sB, D, mi = dev_contiguous(p)
        dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi)
        st = dg.dg_get_device_status()
    finally:
        dg.dg_set_tile_family(dg.DG_TILES_AUTO)
    assert st == BAD_GROUP, dg.dg_status_string(st)
    got = bits(D)
    init = np.full((M, N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"], init)
    written = ref[:, 0] != SENTINEL
    assert written.any() and (~written).any()
    assert np.array_equal(got[~written], ref[~written]), "a row that must stay untouched was written"
    assert_close(got[written], ref[written], f"malformed contiguous ({case})")


@pytest.mark.parametrize("family", [1, 2], ids=["one_cta", "pair"])
@pytest.mark.parametrize("case", CASES)
def test_malformed_contiguous_ue8m0(dg, oracle_mod, family, case):
    N, K = 448, 640
    M = 5 * 128
    p = gi.contiguous_problem([256, 384], N, K, seed_a=93, seed_b=94, ue8m0=True)
    p["m_indices"] = _indices(case, M)
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sA = torch.from_numpy(gi.sa_to_kernel_layout(p["sA"])).to(dev)
    sB = torch.from_numpy(np.ascontiguousarray(p["sB"])).to(dev)
    sfa = dg.dg_transform_sf_ue8m0(sA, M, mn_major=True)
    sfb = dg.dg_transform_sf_ue8m0(sB, p["sB"].shape[-2], mn_major=False)
    assert dg.dg_get_device_status() == 0
    mi = torch.from_numpy(p["m_indices"]).to(dev)
    D = torch.full((M, N), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    dg.dg_set_tile_family(family)
    try:
        dg.dg_fp8_grouped_gemm_contiguous_ue8m0(A, sfa, B, sfb, D, mi)
        st = dg.dg_get_device_status()
    finally:
        dg.dg_set_tile_family(dg.DG_TILES_AUTO)
    assert st == BAD_GROUP, dg.dg_status_string(st)
    got = bits(D)
    init = np.full((M, N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_contiguous_ue8m0(p["A"], oracle_mod.pack_ue8m0(p["sA"]), p["B"],
                                                 oracle_mod.pack_ue8m0(p["sB"]), p["m_indices"], init)
    written = ref[:, 0] != SENTINEL
    assert written.any() and (~written).any()
    assert np.array_equal(got[~written], ref[~written]), "a row that must stay untouched was written"
    assert_close(got[written], ref[written], f"malformed contiguous ue8m0 ({case})")


def test_well_formed_padding_is_not_flagged(dg, oracle_mod):
    # padding at the tail of a segment and a whole padding block are legal
    N, K, M = 256, 256, 512
    p = gi.contiguous_problem([M // 2, M // 2], N, K, seed_a=95, seed_b=96)
    idx = np.full(M, -1, np.int32)
    idx[0:100] = 0
    idx[256:300] = 1
    p["m_indices"] = idx
    for family in (1, 2):
        dg.dg_set_tile_family(family)
        try:
            A, sA, B, sB, D, mi = dev_contiguous(p)
            dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi)
            st = dg.dg_get_device_status()
        finally:
            dg.dg_set_tile_family(dg.DG_TILES_AUTO)
        assert st == 0, dg.dg_status_string(st)
        got = bits(D)
        init = np.full((M, N), SENTINEL, np.uint16)
        _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], idx, init)
        assert np.array_equal(got[idx < 0], ref[idx < 0])
        assert_close(got[idx >= 0], ref[idx >= 0], f"well-formed padding (family {family})")
