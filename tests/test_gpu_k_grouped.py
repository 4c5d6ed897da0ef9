"""GPU parity of the K-grouped TN GEMM (MoE weight gradients) against the
oracle's k_grouped_tn: uneven groups, an empty group, ragged M and N,
several tiles per group, bit-exact integer inputs, and malformed offsets
(flagged in the status word, the affected groups computed as empty)."""
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


def _run(dg, p, offsets=None):
    dev = torch.device("cuda")
    M, N, G = p["M"], p["N"], p["G"]
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sA = torch.from_numpy(gi.sa_to_kernel_layout(np.ascontiguousarray(p["sA"].T))).to(dev)
    sB = torch.from_numpy(p["sB"]).to(dev)
    off = torch.from_numpy(np.asarray(p["k_offsets"] if offsets is None else offsets, np.int32)).to(dev)
    D = torch.full((G, M, N), float("nan"), device=dev)
    dg.dg_fp8_k_grouped_gemm_tn_contiguous(A, sA, B, sB, D, off)
    return D


@pytest.mark.parametrize("ks,M,N", [
    ([256, 0, 128, 384], 208, 272),   # an empty group, ragged M and N
    ([1024, 512], 256, 512),          # several tiles per group
    ([128] * 6, 128, 2048),           # many small groups, wide N
])
def test_k_grouped_matches_oracle(dg, oracle_mod, ks, M, N):
    p = gi.k_grouped_problem(ks, M, N, seed_a=31 + M, seed_b=32 + N)
    D = _run(dg, p)
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.k_grouped_tn(p["A"], p["sA"], p["B"], p["sB"], p["k_offsets"], want_f64=False)
    got = D.cpu().numpy()
    for g, k in enumerate(ks):
        if k == 0:
            assert np.all(got[g] == 0.0)
        else:
            assert_close_f32(got[g], ref[g], f"k-grouped group {g} ({k} K rows) of {ks}, M={M} N={N}")


def test_k_grouped_integer_inputs_bit_exact(dg, oracle_mod):
    rng = np.random.default_rng(33)
    ks, M, N = [256, 384], 128, 256
    K = sum(ks)
    to8 = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    p = dict(A=to8(rng.integers(-4, 5, (K, M))), B=to8(rng.integers(-4, 5, (K, N))),
             sA=np.ones((K // 128, M), np.float32), sB=np.ones((K // 128, N), np.float32),
             k_offsets=np.array([0, 256, 640], np.int32), M=M, N=N, K=K, G=2)
    D = _run(dg, p)
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.k_grouped_tn(p["A"], p["sA"], p["B"], p["sB"], p["k_offsets"], want_f64=False)
    assert np.array_equal(D.cpu().numpy(), ref)


def test_k_grouped_bad_offsets_are_flagged_not_trapped(dg, oracle_mod):
    p = gi.k_grouped_problem([256, 256, 128], 128, 256, seed_a=35, seed_b=36)
    bad = [0, 100, 512, 640]          # groups 0 and 1 start or end off the 128-row grid
    D = _run(dg, p, offsets=bad)
    assert dg.dg_get_device_status() == 6
    assert dg.dg_get_device_status() == 0
    got = D.cpu().numpy()
    assert np.all(got[0] == 0.0) and np.all(got[1] == 0.0)
    _, ref = oracle_mod.k_grouped_tn(p["A"], p["sA"], p["B"], p["sB"], np.array([0, 512, 512, 640], np.int32),
                                     want_f64=False)
    assert_close_f32(got[2], ref[2], "the well-formed group next to bad ones")
