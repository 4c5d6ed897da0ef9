"""GPU parity of the accumulate form D = C + A @ B^T (fp32 C and D) against
the oracle's gemm_nt_acc, on every path the dense planner can take: one-CTA
persistent tiles, the K split of decode shapes, and CTA-pair tiles (forced,
with a capped SM count); in place (C is D); and bit-exact on integer inputs
with an integer C."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import assert_close_f32

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
    m.dg_set_tile_family(m.DG_TILES_AUTO)
    assert m.dg_get_device_status() == 0
    return m


def _dev(p, c):
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev).view(torch.float8_e4m3fn)
    B = torch.from_numpy(p["B"]).to(dev).view(torch.float8_e4m3fn)
    sA = torch.from_numpy(gi.sa_to_kernel_layout(p["sA"])).to(dev)
    sB = torch.from_numpy(p["sB"]).to(dev)
    C = torch.from_numpy(c).to(dev)
    return A, sA, B, sB, C


def _plan(dg, M, N, K):
    return dict(kv.split("=") for kv in dg.dg_describe_config(0, M, N, K).split())


def _c(M, N, seed, scale=20.0):
    return (np.random.default_rng(seed).standard_normal((M, N)) * scale).astype(np.float32)


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512),      # one tile
    (77, 272, 384),       # ragged M and N
    (300, 2112, 640),     # several persistent tiles
    (128, 2112, 7168),    # decode shape: K split over a cluster
    (100, 4096, 3200),    # uneven K split
])
def test_acc_matches_oracle(dg, oracle_mod, M, N, K):
    p = gi.dense_problem(M, N, K, seed_a=5000 + M, seed_b=6000 + N)
    c = _c(M, N, 7)
    A, sA, B, sB, C = _dev(p, c)
    D = torch.full((M, N), float("nan"), device="cuda")
    dg.dg_fp8_gemm_nt_acc(A, sA, B, sB, C, D)
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.gemm_nt_acc(p["A"], p["sA"], p["B"], p["sB"], c, want_f64=False)
    assert_close_f32(D.cpu().numpy(), ref, f"acc {M}x{N}x{K} ({_plan(dg, M, N, K)['ksplit']}-way split)")


def test_acc_in_place(dg, oracle_mod):
    M, N, K = 256, 1024, 1024
    p = gi.dense_problem(M, N, K, seed_a=71, seed_b=72)
    c = _c(M, N, 8)
    A, sA, B, sB, C = _dev(p, c)
    dg.dg_fp8_gemm_nt_acc(A, sA, B, sB, C, C)  # D += A @ B^T
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.gemm_nt_acc(p["A"], p["sA"], p["B"], p["sB"], c, want_f64=False)
    assert_close_f32(C.cpu().numpy(), ref, "acc in place")


@pytest.mark.parametrize("M,N,K", [(512, 1024, 1024), (1000, 1040, 896)])
def test_acc_on_pair_tiles(dg, oracle_mod, M, N, K):
    dg.dg_set_num_sms(16)
    dg.dg_set_tile_family(dg.DG_TILES_PAIR)
    try:
        assert _plan(dg, M, N, K)["pair"] == "1"
        p = gi.dense_problem(M, N, K, seed_a=81 + M, seed_b=82 + N)
        c = _c(M, N, 9)
        A, sA, B, sB, C = _dev(p, c)
        D = torch.full((M, N), float("nan"), device="cuda")
        dg.dg_fp8_gemm_nt_acc(A, sA, B, sB, C, D)
        assert dg.dg_get_device_status() == 0
    finally:
        dg.dg_set_tile_family(dg.DG_TILES_AUTO)
        dg.dg_set_num_sms(0)
    _, ref = oracle_mod.gemm_nt_acc(p["A"], p["sA"], p["B"], p["sB"], c, want_f64=False)
    assert_close_f32(D.cpu().numpy(), ref, f"acc on pair tiles {M}x{N}x{K}")


def test_acc_integer_inputs_bit_exact(dg, oracle_mod):
    rng = np.random.default_rng(19)
    M, N, K = 256, 512, 1024
    ai = rng.integers(-4, 5, (M, K)).astype(np.float32)
    bi = rng.integers(-4, 5, (N, K)).astype(np.float32)
    to8 = lambda x: torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    p = dict(A=to8(ai), B=to8(bi), sA=np.ones((M, K // 128), np.float32),
             sB=np.ones((N // 128, K // 128), np.float32))
    c = rng.integers(-100000, 100001, (M, N)).astype(np.float32)
    A, sA, B, sB, C = _dev(p, c)
    D = torch.empty((M, N), device="cuda")
    dg.dg_fp8_gemm_nt_acc(A, sA, B, sB, C, D)
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.gemm_nt_acc(p["A"], p["sA"], p["B"], p["sB"], c, want_f64=False)
    assert np.array_equal(D.cpu().numpy(), ref)
