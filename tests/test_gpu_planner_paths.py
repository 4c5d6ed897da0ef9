"""Every compiled tile path against the oracle, whole output, at mid size.

The benchmark workloads are too large for the oracle to check whole, so
their tile paths are also checked here on mid-size problems that run them on
the full GPU (several waves of tiles, no SM cap) with ragged M and N (partial
last row block and partial last column tile) and an odd number of K blocks
(a two-block pipeline stage with one block past K).  dg_set_block_n and
dg_set_tile_family force each path, and dg_describe_config confirms it:
  * fp32-scale one-CTA tiles of 112, 128, 224 and 256 columns (the 256-column
    tile in both depths: three stages on a short K range, four on a long one),
  * fp32-scale CTA-pair tiles of 160 and 192 columns,
  * the K-split decode tile (144 columns over a cluster),
  * the UE8M0 mode's one-CTA and pair tiles of 128, 160, 192 and 224 columns,
  * the grouped layouts on the tiles the benchmark's grouped workloads take.
Every output element is compared within the parity tolerance; rows the
grouped layouts must not write keep a sentinel, bit for bit."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import SENTINEL, assert_close, bits, dev_contiguous, dev_dense, dev_masked

pytestmark = pytest.mark.gpu

M_MID, N_MID, K_MID = 1000, 2000, 1152     # ragged against every tile; 9 K blocks


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
    m.dg_set_block_n(0)
    m.dg_set_tile_family(m.DG_TILES_AUTO)


class forced:
    """Pins the tile width and family for the duration of a with-block."""

    def __init__(self, dg, bn, family):
        self.dg, self.bn, self.family = dg, bn, family

    def __enter__(self):
        self.dg.dg_set_block_n(self.bn)
        self.dg.dg_set_tile_family(self.family)

    def __exit__(self, *exc):
        self.dg.dg_set_block_n(0)
        self.dg.dg_set_tile_family(self.dg.DG_TILES_AUTO)


def _plan(dg, layout, M, N, K, G=1):
    return dict(kv.split("=") for kv in dg.dg_describe_config(layout, M, N, K, G).split())


@pytest.fixture(scope="module")
def dense_mid(oracle_mod):
    p = gi.dense_problem(M_MID, N_MID, K_MID, seed_a=501, seed_b=502)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    return p, ref


@pytest.mark.parametrize("bn,family", [(112, 1), (128, 1), (224, 1), (256, 1), (160, 2), (192, 2)])
def test_dense_fp32_tile_path(dg, dense_mid, bn, family):
    p, ref = dense_mid
    with forced(dg, bn, family):
        plan = _plan(dg, 0, M_MID, N_MID, K_MID)
        assert plan["BN"] == str(bn) and plan["pair"] == str(family - 1) and plan["ksplit"] == "1", plan
        A, sA, B, sB, D = dev_dense(p)
        dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
        st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    assert_close(bits(D), ref, f"dense BN={bn} family={family}")


def test_dense_fp32_four_stage_tile(dg, oracle_mod):
    """128x256 tiles over a long K range (40 K blocks) take the four-stage
    ring, whose output goes through per-warp staging buffers; ragged M and N,
    several row blocks and column tiles, whole output against the oracle."""
    M, N, K = 600, 1040, 5120
    p = gi.dense_problem(M, N, K, seed_a=511, seed_b=512)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    with forced(dg, 256, 1):
        assert _plan(dg, 0, M_MID, N_MID, K_MID)["stages"] == "3"
        plan = _plan(dg, 0, M, N, K)
        assert (plan["BN"], plan["stages"], plan["ks"], plan["pair"], plan["ksplit"]) == ("256", "4", "1", "0", "1"), plan
        A, sA, B, sB, D = dev_dense(p)
        dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
        st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    assert_close(bits(D), ref, "dense BN=256 four stages")


def test_dense_k_split_path(dg, oracle_mod):
    M, N, K = 200, 2000, 4480                   # 14 x 2 tiles of 144 columns, 35 K blocks
    p = gi.dense_problem(M, N, K, seed_a=503, seed_b=504)
    with forced(dg, 144, 1):
        plan = _plan(dg, 0, M, N, K)
        assert plan["BN"] == "144" and int(plan["ksplit"]) > 1, plan
        A, sA, B, sB, D = dev_dense(p)
        dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
        st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(bits(D), ref, f"dense K split ksplit={plan['ksplit']}")


@pytest.fixture(scope="module")
def dense_mid_ue8m0(oracle_mod):
    p = gi.dense_problem(M_MID, N_MID, K_MID, seed_a=505, seed_b=506, ue8m0=True)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    return p, ref


def _pack(dg, p, rows):
    dev = torch.device("cuda")
    sA = torch.from_numpy(gi.sa_to_kernel_layout(p["sA"])).to(dev)
    sB = torch.from_numpy(np.ascontiguousarray(p["sB"])).to(dev)
    return (dg.dg_transform_sf_ue8m0(sA, rows, mn_major=True),
            dg.dg_transform_sf_ue8m0(sB, p["sB"].shape[-2], mn_major=False))


@pytest.mark.parametrize("family", [1, 2], ids=["one_cta", "pair"])
@pytest.mark.parametrize("bn", [128, 160, 192, 224])
def test_dense_ue8m0_tile_path(dg, dense_mid_ue8m0, bn, family):
    p, ref = dense_mid_ue8m0
    dev = torch.device("cuda")
    with forced(dg, bn, family):
        plan = _plan(dg, 3, M_MID, N_MID, K_MID)
        assert plan["BN"] == str(bn) and plan["pair"] == str(family - 1) and plan["ksplit"] == "1", plan
        sfa, sfb = _pack(dg, p, M_MID)
        A = torch.from_numpy(p["A"]).to(dev)
        B = torch.from_numpy(p["B"]).to(dev)
        D = torch.full((M_MID, N_MID), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
        dg.dg_fp8_gemm_nt_ue8m0(A, sfa, B, sfb, D)
        st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    assert_close(bits(D), ref, f"ue8m0 dense BN={bn} family={family}")


@pytest.mark.parametrize("bn,family", [(256, 1), (160, 2), (192, 2)])
def test_contiguous_tile_path(dg, oracle_mod, bn, family):
    rows, N, K = [900, 600, 0, 1300, 37], N_MID, 1024
    p = gi.contiguous_problem(rows, N, K, seed_a=507, seed_b=508)
    with forced(dg, bn, family):
        plan = _plan(dg, 1, p["M"], N, K, p["G"])
        assert plan["BN"] == str(bn) and plan["pair"] == str(family - 1), plan
        A, sA, B, sB, D, mi = dev_contiguous(p)
        dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi)
        st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    got = bits(D)
    init = np.full((p["M"], N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"], init)
    pad = p["m_indices"] < 0
    assert np.array_equal(got[pad], ref[pad])
    assert_close(got[~pad], ref[~pad], f"contiguous BN={bn} family={family}")


@pytest.mark.parametrize("bn", [128, 256])
def test_masked_tile_path(dg, oracle_mod, bn):
    G, max_m, N, K = 8, 256, N_MID, 1152
    mm = np.random.default_rng(509).integers(1, max_m + 1, G).astype(np.int32)
    p = gi.masked_problem(G, max_m, N, K, masked_m=mm, seed_a=510, seed_b=511)
    with forced(dg, bn, 1):
        plan = _plan(dg, 2, int(mm.mean()), N, K, G)
        assert plan["BN"] == str(bn) and plan["pair"] == "0", plan
        A, sA, B, sB, D, m = dev_masked(p)
        dg.dg_fp8_grouped_gemm_masked(A, sA, B, sB, D, m, int(mm.mean()))
        st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    got = bits(D)
    init = np.full((G, max_m, N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], p["masked_m"], init)
    valid = np.arange(max_m)[None, :] < mm[:, None]
    assert np.array_equal(got[~valid], ref[~valid])
    assert_close(got[valid], ref[valid], f"masked BN={bn}")



def test_grouped_four_stage_tile(dg, oracle_mod):
    """The four-stage 128x256 tile (a long K range, 40 K blocks) in both
    grouped layouts: its per-warp staged stores must leave every padding row
    of the contiguous layout and every masked row untouched, bit for bit,
    while partial row blocks and a ragged last column tile are written."""
    N, K = 1040, 5120
    pc = gi.contiguous_problem([300, 0, 517, 128], N, K, seed_a=530, seed_b=531)
    G, max_m = 4, 384
    mm = np.array([384, 1, 0, 250], dtype=np.int32)
    pm = gi.masked_problem(G, max_m, N, K, masked_m=mm, seed_a=532, seed_b=533)
    with forced(dg, 256, 1):
        plan = _plan(dg, 1, pc["M"], N, K, pc["G"])
        assert (plan["BN"], plan["stages"], plan["ks"], plan["pair"]) == ("256", "4", "1", "0"), plan
        A, sA, B, sB, D, mi = dev_contiguous(pc)
        dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi)
        plan = _plan(dg, 2, max_m, N, K, G)
        assert (plan["BN"], plan["stages"], plan["ks"], plan["pair"]) == ("256", "4", "1", "0"), plan
        Am, sAm, Bm, sBm, Dm, m = dev_masked(pm)
        dg.dg_fp8_grouped_gemm_masked(Am, sAm, Bm, sBm, Dm, m, max_m)
        st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    got = bits(D)
    _, ref = oracle_mod.grouped_contiguous(pc["A"], pc["sA"], pc["B"], pc["sB"], pc["m_indices"],
                                           np.full((pc["M"], N), SENTINEL, np.uint16))
    pad = pc["m_indices"] < 0
    assert pad.any()
    assert np.array_equal(got[pad], ref[pad])
    assert_close(got[~pad], ref[~pad], "contiguous, four-stage 128x256 tile")
    got = bits(Dm)
    _, ref = oracle_mod.grouped_masked(pm["A"], pm["sA"], pm["B"], pm["sB"], pm["masked_m"],
                                       np.full((G, max_m, N), SENTINEL, np.uint16))
    valid = np.arange(max_m)[None, :] < mm[:, None]
    assert np.array_equal(got[~valid], ref[~valid])
    assert_close(got[valid], ref[valid], "masked, four-stage 128x256 tile")

def test_masked_decode_tile_path(dg, oracle_mod):
    """The planner's own tile for decode-sized masked groups (no width or
    family pinned): 128 columns, three stages of two K blocks, a second
    producer warp for the B boxes, rows stored through per-warp buffers.  Whole output, with
    every group's masked rows checked bit for bit; K = 1152 leaves the last
    stage half outside K, and ragged masked_m values cover partial row
    blocks, a group of 128 + 1 rows and an empty group."""
    G, max_m, N, K = 8, 256, N_MID, 1152
    mm = np.array([1, 129, 256, 0, 64, 200, 128, 17], dtype=np.int32)
    p = gi.masked_problem(G, max_m, N, K, masked_m=mm, seed_a=520, seed_b=521)
    plan = _plan(dg, 2, max_m, N, K, G)
    assert (plan["BN"], plan["stages"], plan["ks"], plan["pair"]) == ("128", "3", "2", "0"), plan
    A, sA, B, sB, D, m = dev_masked(p)
    dg.dg_fp8_grouped_gemm_masked(A, sA, B, sB, D, m, 0)
    st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    got = bits(D)
    init = np.full((G, max_m, N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], p["masked_m"], init)
    valid = np.arange(max_m)[None, :] < mm[:, None]
    assert np.array_equal(got[~valid], ref[~valid])
    assert_close(got[valid], ref[valid], "masked decode tile")


@pytest.mark.parametrize("family,layout", [(2, "contiguous"), (1, "masked")])
def test_grouped_ue8m0_benchmark_tile_path(dg, oracle_mod, family, layout):
    """The UE8M0 tiles the grouped benchmark workloads take: 256 x 224 pairs
    for the contiguous layout, 128 x 128 one-CTA tiles for the masked one."""
    dev = torch.device("cuda")
    if layout == "contiguous":
        p = gi.contiguous_problem([900, 600, 0, 1300, 37], N_MID, 1024, seed_a=512, seed_b=513, ue8m0=True)
        bn = 224
    else:
        mm = np.random.default_rng(514).integers(1, 257, 8).astype(np.int32)
        p = gi.masked_problem(8, 256, N_MID, 1152, masked_m=mm, seed_a=515, seed_b=516, ue8m0=True)
        bn = 128
    rows = p["M"] if layout == "contiguous" else p["max_m"]
    with forced(dg, bn, family):
        sfa, sfb = _pack(dg, p, rows)
        A = torch.from_numpy(p["A"]).to(dev)
        B = torch.from_numpy(p["B"]).to(dev)
        if layout == "contiguous":
            plan = _plan(dg, 4, p["M"], N_MID, p["K"], p["G"])
            mi = torch.from_numpy(p["m_indices"]).to(dev)
            D = torch.full((p["M"], N_MID), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
            dg.dg_fp8_grouped_gemm_contiguous_ue8m0(A, sfa, B, sfb, D, mi)
        else:
            plan = _plan(dg, 5, int(mm.mean()), N_MID, p["K"], p["G"])
            m = torch.from_numpy(p["masked_m"]).to(dev)
            D = torch.full((8, 256, N_MID), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
            dg.dg_fp8_grouped_gemm_masked_ue8m0(A, sfa, B, sfb, D, m, int(mm.mean()))
        st = dg.dg_get_device_status()
    assert plan["BN"] == str(bn) and plan["pair"] == str(family - 1), plan
    assert st == 0, dg.dg_status_string(st)
    got = bits(D)
    if layout == "contiguous":
        init = np.full((p["M"], N_MID), SENTINEL, np.uint16)
        _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"], init)
        keep = p["m_indices"] < 0
    else:
        init = np.full((8, 256, N_MID), SENTINEL, np.uint16)
        _, ref = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], p["masked_m"], init)
        keep = ~(np.arange(256)[None, :] < mm[:, None])
    assert np.array_equal(got[keep], ref[keep])
    assert_close(got[~keep], ref[~keep], f"ue8m0 {layout} BN={bn}")
