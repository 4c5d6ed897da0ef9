"""GPU parity: the CUDA library (called through its C ABI via the binding)
against the CPU oracle on the same seeded inputs.

Small and mid sizes are compared element by element over the whole output
(several tiles plus ragged tails); the full benchmark workloads are compared
on sampled outputs that the oracle computes one by one, in the same launch
configuration the benchmark times.  Placement and masking are bit-exact
(sentinel pre-fill)."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import SENTINEL, assert_close, bits, dev_contiguous, dev_dense, dev_masked

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


def _run_dense(dg, p):
    A, sA, B, sB, D = dev_dense(p)
    dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
    st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    return bits(D)


# ------------------------------------------------------------------- dense

@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512),      # the tiny benchmark shape
    (1, 16, 128),         # smallest legal problem
    (77, 48, 128),        # ragged M, one K block
    (200, 272, 384),      # ragged M and N (N spans 3 weight blocks)
    (256, 1024, 1024),
    (300, 2112, 640),
    (513, 7168, 256),     # wide N: 224/256-column tiles, ragged M tail
    # decode shapes: too few tiles to fill the GPU, so the K range of each
    # tile is split over a cluster; the splits' fp32 partials meet in an L2
    # workspace and each CTA sums its rows of them in split order
    (128, 1024, 4096),    # 8-way split
    (64, 2112, 7168),     # 8-way split
    (100, 4096, 3200),    # 25 K blocks: uneven 4-way split
    (64, 256, 4096),      # 16-way split: 8 rows of each tile per CTA
])
def test_dense_matches_oracle(dg, oracle_mod, M, N, K):
    p = gi.dense_problem(M, N, K, seed_a=1000 + M, seed_b=2000 + N)
    got = _run_dense(dg, p)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(got, ref, f"dense {M}x{N}x{K}")


def test_dense_integer_inputs_bit_exact(dg, oracle_mod):
    rng = np.random.default_rng(9)
    M, N, K = 256, 512, 1024
    ai = rng.integers(-4, 5, (M, K)).astype(np.float32)
    bi = rng.integers(-4, 5, (N, K)).astype(np.float32)
    to8 = lambda x: torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    p = dict(A=to8(ai), B=to8(bi), sA=np.ones((M, K // 128), np.float32),
             sB=np.ones((N // 128, K // 128), np.float32), M=M, N=N, K=K)
    got = _run_dense(dg, p)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert np.array_equal(got, ref)


def test_dense_identity_bit_exact(dg, oracle_mod):
    K = 128
    A = np.zeros((K, K), np.uint8)
    A[np.arange(K), np.arange(K)] = 0x38  # 1.0
    pb = gi.dense_problem(1, 320, K, seed_b=77)
    p = dict(A=A, B=pb["B"], sA=np.ones((K, 1), np.float32), sB=np.ones_like(pb["sB"]), M=K, N=320, K=K)
    got = _run_dense(dg, p)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert np.array_equal(got, ref)


def test_dense_zero_scales_give_zero(dg):
    p = gi.dense_problem(130, 256, 256, seed_a=5, seed_b=6)
    p["sA"] = np.zeros_like(p["sA"])
    got = _run_dense(dg, p)
    assert np.all(got == 0)


def test_dense_decode_full(dg, oracle_mod):
    """The decode-shaped benchmark problem, whole output."""
    p = gi.make_workload("dense_decode")
    got = _run_dense(dg, p)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(got, ref, "dense decode 128x2112x7168")


def _sample_rc(M, N, count, seed):
    rng = np.random.default_rng(seed)
    r = rng.integers(0, M, count)
    c = rng.integers(0, N, count)
    # always include the four corners and the last rows/cols (ragged tails)
    r = np.concatenate([r, [0, 0, M - 1, M - 1]])
    c = np.concatenate([c, [0, N - 1, 0, N - 1]])
    return r, c


@pytest.mark.slow
def test_dense_prefill_sampled(dg, oracle_mod):
    p = gi.make_workload("dense_prefill")
    got = _run_dense(dg, p)
    r, c = _sample_rc(p["M"], p["N"], 20000, 1)
    _, ref = oracle_mod.gemm_nt_sampled(p["A"], p["sA"], p["B"], p["sB"], r, c)
    assert_close(got[r, c], ref, "dense prefill (sampled)")
    assert not np.any(got == SENTINEL)


# -------------------------------------------------------------- contiguous

def _run_contiguous(dg, p):
    A, sA, B, sB, D, mi = dev_contiguous(p)
    dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi)
    st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    return bits(D)


@pytest.mark.parametrize("rows,N,K", [
    ([128, 256], 256, 256),
    ([100, 300, 0, 37], 336, 384),      # padding rows, an empty group, ragged N
    ([512] * 3, 7168, 256),
])
def test_contiguous_matches_oracle(dg, oracle_mod, rows, N, K):
    p = gi.contiguous_problem(rows, N, K, seed_a=11, seed_b=12)
    got = _run_contiguous(dg, p)
    init = np.full((p["M"], N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"], init)
    pad = p["m_indices"] < 0
    assert np.array_equal(got[pad], ref[pad])  # untouched, bit for bit
    assert_close(got[~pad], ref[~pad], f"contiguous {rows} N={N} K={K}")


@pytest.mark.slow
def test_contiguous_moe_sampled(dg, oracle_mod):
    p = gi.make_workload("contiguous_moe")
    got = _run_contiguous(dg, p)
    r, c = _sample_rc(p["M"], p["N"], 20000, 2)
    g = p["m_indices"][r]
    ref = np.empty(r.size, np.uint16)
    for gg in np.unique(g):
        sel = g == gg
        _, ref[sel] = oracle_mod.gemm_nt_sampled(p["A"], p["sA"], p["B"][gg], p["sB"][gg], r[sel], c[sel])
    assert_close(got[r, c], ref, "contiguous MoE (sampled)")
    assert not np.any(got == SENTINEL)


# ------------------------------------------------------------------ masked

def _run_masked(dg, p, expected_m=0):
    A, sA, B, sB, D, mm = dev_masked(p)
    dg.dg_fp8_grouped_gemm_masked(A, sA, B, sB, D, mm, expected_m)
    st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    return bits(D)


@pytest.mark.parametrize("G,max_m,N,K,masked", [
    (4, 256, 256, 256, [1, 128, 129, 256]),
    (3, 200, 336, 384, [0, 200, 77]),        # empty group, max_m not a multiple of 128
    (2, 64, 7168, 128, [64, 5]),
])
def test_masked_matches_oracle(dg, oracle_mod, G, max_m, N, K, masked):
    p = gi.masked_problem(G, max_m, N, K, masked_m=masked, seed_a=21, seed_b=22)
    got = _run_masked(dg, p)
    init = np.full((G, max_m, N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], p["masked_m"], init)
    valid = np.arange(max_m)[None, :] < np.asarray(masked)[:, None]
    assert np.array_equal(got[~valid], ref[~valid])  # untouched rows, bit for bit
    if valid.any():
        assert_close(got[valid], ref[valid], f"masked G={G} max_m={max_m} N={N}")


@pytest.mark.slow
def test_masked_moe_decode_sampled(dg, oracle_mod):
    p = gi.make_workload("masked_moe_decode")
    got = _run_masked(dg, p)
    G, max_m, N = p["G"], p["max_m"], p["N"]
    mm = p["masked_m"]
    valid = np.arange(max_m)[None, :] < mm[:, None]
    assert np.all(got[~valid] == SENTINEL)
    rng = np.random.default_rng(3)
    ref_all, got_all = [], []
    for g in range(G):
        r = rng.integers(0, mm[g], 1000)
        c = rng.integers(0, N, 1000)
        _, ref = oracle_mod.gemm_nt_sampled(p["A"][g], p["sA"][g], p["B"][g], p["sB"][g], r, c)
        ref_all.append(ref)
        got_all.append(got[g, r, c])
    assert_close(np.concatenate(got_all), np.concatenate(ref_all), "masked MoE decode (sampled)")


# ----------------------------------------------------------- device status

def test_bad_group_data_is_flagged_not_trapped(dg, oracle_mod):
    N, K = 256, 256
    p = gi.contiguous_problem([128, 128], N, K, seed_a=31, seed_b=32)
    p["m_indices"][128:256] = 7       # group index out of range: block skipped
    A, sA, B, sB, D, mi = dev_contiguous(p)
    dg.dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, mi)
    assert dg.dg_get_device_status() == 6
    assert dg.dg_get_device_status() == 0  # cleared
    got = bits(D)
    assert np.all(got[128:] == SENTINEL)
    _, ref = oracle_mod.gemm_nt(p["A"][:128], p["sA"][:128], p["B"][0], p["sB"][0], want_f64=False)
    assert_close(got[:128], ref, "valid block next to a bad one")

    pm = gi.masked_problem(2, 64, N, K, masked_m=[300, 3], seed_a=33, seed_b=34)
    A, sA, B, sB, D, mm = dev_masked(pm)
    dg.dg_fp8_grouped_gemm_masked(A, sA, B, sB, D, mm)
    assert dg.dg_get_device_status() == 6  # masked_m > max_m: clamped and flagged
    got = bits(D)
    _, ref = oracle_mod.gemm_nt(pm["A"][0], pm["sA"][0], pm["B"][0], pm["sB"][0], want_f64=False)
    assert_close(got[0], ref, "clamped group")


def test_num_sms_cap_gives_same_result(dg):
    p = gi.dense_problem(512, 1024, 512, seed_a=41, seed_b=42)
    full = _run_dense(dg, p)
    dg.dg_set_num_sms(7)
    try:
        assert dg.dg_get_num_sms() == 7
        capped = _run_dense(dg, p)
    finally:
        dg.dg_set_num_sms(0)
    assert np.array_equal(full, capped)


@pytest.mark.parametrize("M,N,K", [(384, 2112, 1024), (128, 2112, 7168)])
def test_repeated_calls_deterministic(dg, M, N, K):
    # the second shape takes the K-split path: its reduction order is fixed
    p = gi.dense_problem(M, N, K, seed_a=51, seed_b=52)
    a = _run_dense(dg, p)
    b = _run_dense(dg, p)
    assert np.array_equal(a, b)


def test_cpu_tensors_rejected(dg):
    p = gi.dense_problem(128, 256, 128)
    A = torch.from_numpy(p["A"])
    with pytest.raises(ValueError):
        dg.dg_fp8_gemm_nt(A, A, A, A, A)
