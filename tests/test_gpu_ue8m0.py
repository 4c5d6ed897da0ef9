"""GPU parity of the UE8M0 block-scaled mode against the oracle's UE8M0
variant (power-of-two scales, packed four to an int32; hada.io DeepGEMM
summary, section "Giao dien GEMM va rang buoc layout").

Inputs are quantised with power-of-two scales (the input recipe's ue8m0
option, whose rounding the CPU suite checks against the oracle), packed on
the GPU by dg_transform_sf_ue8m0 (checked word for word against the oracle's
packing) and multiplied by the block-scaled kernels, on one-CTA tiles and on
CTA-pair tiles (cta_group::2).  Shapes are chosen, with the SM count capped
at 16 for the small ones, so that every compiled tile width runs, with
ragged M and N, partial K-block groups (K/128 not a multiple of 4), several
waves of tiles, pairs whose halves belong to different groups, grouped
padding and masking.
Placement and masking are bit-exact (sentinel pre-fill)."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import SENTINEL, assert_close, bits

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
    m.dg_set_num_sms(0)
    assert m.dg_get_device_status() == 0
    yield m
    m.dg_set_num_sms(0)


def _plan(dg, layout, M, N, K, G=1):
    return dict(kv.split("=") for kv in dg.dg_describe_config(layout, M, N, K, G).split())


def _packed(dg, oracle_mod, sa_logical, sb_logical):
    """fp32 scales -> packed words on the GPU, checked against the oracle.
    sa_logical [..., rows, K/128], sb_logical [..., nbn, K/128]."""
    dev = torch.device("cuda")
    rows = sa_logical.shape[-2]
    sA = torch.from_numpy(gi.sa_to_kernel_layout(sa_logical)).to(dev)
    sfa = dg.dg_transform_sf_ue8m0(sA, rows, mn_major=True)
    sB = torch.from_numpy(np.ascontiguousarray(sb_logical)).to(dev)
    sfb = dg.dg_transform_sf_ue8m0(sB, sb_logical.shape[-2], mn_major=False)
    assert dg.dg_get_device_status() == 0
    want_a = oracle_mod.pack_ue8m0(sa_logical)          # [..., ng, rows]
    got_a = sfa.cpu().numpy()
    assert np.array_equal(got_a[..., :rows], want_a), "sfa packing differs from the oracle"
    assert np.all(got_a[..., rows:].view(np.uint32) == 0x7F7F7F7F)  # pad rows: scale 1
    assert np.array_equal(sfb.cpu().numpy(), oracle_mod.pack_ue8m0(sb_logical)), "sfb packing"
    return sfa, sfb


def _dense(dg, oracle_mod, p):
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sfa, sfb = _packed(dg, oracle_mod, p["sA"], p["sB"])
    D = torch.full((p["M"], p["N"]), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    dg.dg_fp8_gemm_nt_ue8m0(A, sfa, B, sfb, D)
    st = dg.dg_get_device_status()
    assert st == 0, dg.dg_status_string(st)
    return bits(D), (A, sfa, B, sfb, D)


@pytest.fixture(params=[1, 2], ids=["one_cta", "pair"])
def family(request, dg):
    """Runs a test on one tile family (dg_set_tile_family: 1 = one-CTA
    128-row tiles, 2 = CTA-pair 256-row tiles)."""
    dg.dg_set_tile_family(request.param)
    yield request.param
    dg.dg_set_tile_family(dg.DG_TILES_AUTO)


@pytest.mark.parametrize("M,N,K,bn", [
    (2048, 224, 512, "224"),   # 16 tiles of 224 on 16 SMs
    (2048, 192, 896, "192"),   # 7 K blocks: the last word holds 3
    (2048, 160, 384, "160"),
    (1024, 256, 128, "128"),   # a single K block
    (1000, 1040, 896, None),   # ragged M and N, several waves
    (130, 2064, 640, None),    # second m-block has 2 rows
    (384, 7168, 1152, None),   # wide N, 9 K blocks
])
def test_dense_ue8m0_matches_oracle(dg, oracle_mod, family, M, N, K, bn):
    dg.dg_set_num_sms(CAP_SMS)
    try:
        plan = _plan(dg, 3, M, N, K)
        assert plan["pair"] == ("1" if family == 2 else "0"), plan
        if bn is not None:
            assert plan["BN"] == bn, plan
        p = gi.dense_problem(M, N, K, seed_a=5000 + M, seed_b=6000 + N, ue8m0=True)
        got, _ = _dense(dg, oracle_mod, p)
    finally:
        dg.dg_set_num_sms(0)
    _, ref = oracle_mod.gemm_nt_ue8m0(p["A"], oracle_mod.pack_ue8m0(p["sA"]), p["B"],
                                      oracle_mod.pack_ue8m0(p["sB"]), want_f64=False)
    assert_close(got, ref, f"ue8m0 dense {M}x{N}x{K}")


def test_dense_ue8m0_integer_inputs_bit_exact(dg, oracle_mod, family):
    """Integer-valued codes with power-of-two scales: every partial and every
    scaled sum is exact in fp32, so the bf16 result equals the oracle's bit
    for bit."""
    rng = np.random.default_rng(13)
    M, N, K = 256, 448, 1024
    to8 = lambda v: torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    a8, b8 = to8(rng.integers(-6, 7, (M, K))), to8(rng.integers(-6, 7, (N, K)))
    sa = np.exp2(rng.integers(-4, 5, (M, K // 128))).astype(np.float32)
    sb = np.exp2(rng.integers(-4, 5, ((N + 127) // 128, K // 128))).astype(np.float32)
    p = dict(A=a8, B=b8, sA=sa, sB=sb, M=M, N=N, K=K)
    got, _ = _dense(dg, oracle_mod, p)
    _, ref = oracle_mod.gemm_nt_ue8m0(a8, oracle_mod.pack_ue8m0(sa), b8, oracle_mod.pack_ue8m0(sb),
                                      want_f64=False)
    assert np.array_equal(got, ref)


def test_ue8m0_and_fp32_modes_agree(dg, oracle_mod):
    """The same power-of-two-scaled inputs through both modes: the fp32-scale
    kernel (CUDA-core promotion) and the block-scaled one differ only in the
    order of fp32 additions."""
    from parity import dev_dense
    p = gi.dense_problem(512, 2112, 2048, seed_a=71, seed_b=72, ue8m0=True)
    got_bs, _ = _dense(dg, oracle_mod, p)
    A, sA, B, sB, D = dev_dense(p)
    dg.dg_fp8_gemm_nt(A, sA, B, sB, D)
    assert dg.dg_get_device_status() == 0
    assert_close(got_bs, bits(D), "ue8m0 vs fp32-scale mode")


def test_dense_ue8m0_deterministic(dg, oracle_mod, family):
    p = gi.dense_problem(384, 2112, 1024, seed_a=73, seed_b=74, ue8m0=True)
    a, _ = _dense(dg, oracle_mod, p)
    b, _ = _dense(dg, oracle_mod, p)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("M,N,K", [
    (64, 1024, 4096),     # 8 tiles, 4 K blocks per split
    (100, 4096, 3200),    # 25 K blocks: 7 per split, stages straddle K-block groups
    (200, 1024, 2048),    # two m-blocks, 16 K blocks: 2 or 4 per split
])
def test_dense_ue8m0_k_split(dg, oracle_mod, M, N, K):
    """Decode-shaped problems split each tile's K range over a cluster; the
    fp32 partials meet in the workspace and are summed in a fixed order."""
    plan = _plan(dg, 3, M, N, K)
    assert int(plan["ksplit"]) > 1, plan
    p = gi.dense_problem(M, N, K, seed_a=7000 + M, seed_b=8000 + N, ue8m0=True)
    got, _ = _dense(dg, oracle_mod, p)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(got, ref, f"ue8m0 split {M}x{N}x{K}")
    again, _ = _dense(dg, oracle_mod, p)
    assert np.array_equal(got, again)  # fixed reduction order


def test_dense_decode_ue8m0_full(dg, oracle_mod):
    """The decode-shaped benchmark problem (128 x 2112 x 7168), whole output."""
    p = gi.make_workload("dense_decode", ue8m0=True)
    got, _ = _dense(dg, oracle_mod, p)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(got, ref, "ue8m0 dense decode")


@pytest.mark.slow
def test_dense_prefill_ue8m0_sampled(dg, oracle_mod):
    p = gi.make_workload("dense_prefill", ue8m0=True)
    got, _ = _dense(dg, oracle_mod, p)
    rng = np.random.default_rng(2)
    r = np.concatenate([rng.integers(0, p["M"], 20000), [0, 0, p["M"] - 1, p["M"] - 1]])
    c = np.concatenate([rng.integers(0, p["N"], 20000), [0, p["N"] - 1, 0, p["N"] - 1]])
    _, ref = oracle_mod.gemm_nt_sampled(p["A"], p["sA"], p["B"], p["sB"], r, c)
    assert_close(got[r, c], ref, "ue8m0 dense prefill (sampled)")
    assert not np.any(got == SENTINEL)


# ---------------------------------------------------------------- grouped

@pytest.mark.parametrize("rows,N,K", [
    ([384, 100, 300], 1024, 512),     # padded blocks, ragged groups
    ([0, 640, 37], 1040, 256),        # an empty group, ragged N
    ([128] * 6, 224, 1152),           # many groups, 9 K blocks; every pair spans two groups
    ([256, 128, 384], 448, 640),      # pairs split across groups and padding
])
def test_contiguous_ue8m0_matches_oracle(dg, oracle_mod, family, rows, N, K):
    p = gi.contiguous_problem(rows, N, K, seed_a=81, seed_b=82, ue8m0=True)
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sfa, sfb = _packed(dg, oracle_mod, p["sA"], p["sB"])
    mi = torch.from_numpy(p["m_indices"]).to(dev)
    D = torch.full((p["M"], N), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    dg.dg_fp8_grouped_gemm_contiguous_ue8m0(A, sfa, B, sfb, D, mi)
    assert dg.dg_get_device_status() == 0
    got = bits(D)
    init = np.full((p["M"], N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_contiguous_ue8m0(p["A"], oracle_mod.pack_ue8m0(p["sA"]), p["B"],
                                                 oracle_mod.pack_ue8m0(p["sB"]), p["m_indices"], init)
    pad = p["m_indices"] < 0
    assert np.array_equal(got[pad], ref[pad])
    assert_close(got[~pad], ref[~pad], f"ue8m0 contiguous {rows} N={N} K={K}")


@pytest.mark.parametrize("G,max_m,N,K,masked", [
    (4, 512, 1024, 384, [0, 100, 300, 512]),
    (3, 200, 2064, 640, [200, 129, 1]),   # max_m not a multiple of 128
    (2, 256, 224, 128, [256, 255]),
])
def test_masked_ue8m0_matches_oracle(dg, oracle_mod, family, G, max_m, N, K, masked):
    p = gi.masked_problem(G, max_m, N, K, masked_m=masked, seed_a=91, seed_b=92, ue8m0=True)
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sfa, sfb = _packed(dg, oracle_mod, p["sA"], p["sB"])
    mm = torch.from_numpy(p["masked_m"]).to(dev)
    D = torch.full((G, max_m, N), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    dg.dg_fp8_grouped_gemm_masked_ue8m0(A, sfa, B, sfb, D, mm)
    assert dg.dg_get_device_status() == 0
    got = bits(D)
    init = np.full((G, max_m, N), SENTINEL, np.uint16)
    _, ref = oracle_mod.grouped_masked_ue8m0(p["A"], oracle_mod.pack_ue8m0(p["sA"]), p["B"],
                                             oracle_mod.pack_ue8m0(p["sB"]), p["masked_m"], init)
    valid = np.arange(max_m)[None, :] < np.asarray(masked)[:, None]
    assert np.array_equal(got[~valid], ref[~valid])
    assert_close(got[valid], ref[valid], f"ue8m0 masked G={G} max_m={max_m} N={N}")


@pytest.mark.slow
def test_masked_moe_decode_ue8m0_sampled(dg, oracle_mod):
    p = gi.make_workload("masked_moe_decode", ue8m0=True)
    G, max_m, N = p["G"], p["max_m"], p["N"]
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sfa, sfb = _packed(dg, oracle_mod, p["sA"], p["sB"])
    mm = torch.from_numpy(p["masked_m"]).to(dev)
    D = torch.full((G, max_m, N), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    dg.dg_fp8_grouped_gemm_masked_ue8m0(A, sfa, B, sfb, D, mm)
    assert dg.dg_get_device_status() == 0
    got = bits(D)
    valid = np.arange(max_m)[None, :] < p["masked_m"][:, None]
    assert np.all(got[~valid] == SENTINEL)
    rng = np.random.default_rng(4)
    refs, gots = [], []
    for g in range(G):
        r = rng.integers(0, p["masked_m"][g], 500)
        c = rng.integers(0, N, 500)
        _, ref = oracle_mod.gemm_nt_sampled(p["A"][g], p["sA"][g], p["B"][g], p["sB"][g], r, c)
        refs.append(ref)
        gots.append(got[g, r, c])
    assert_close(np.concatenate(gots), np.concatenate(refs), "ue8m0 masked MoE decode (sampled)")


@pytest.mark.slow
def test_contiguous_moe_ue8m0_sampled(dg, oracle_mod):
    """The contiguous MoE benchmark workload (8 experts x 4096 rows, N=7168,
    K=2048) in the launch configuration the benchmark times (the default
    plan: 256 x 224 pair tiles), on 20,004 sampled outputs, corners
    included; no output keeps the sentinel."""
    p = gi.make_workload("contiguous_moe", ue8m0=True)
    plan = _plan(dg, 4, p["M"], p["N"], p["K"], p["G"])
    dev = torch.device("cuda")
    A = torch.from_numpy(p["A"]).to(dev)
    B = torch.from_numpy(p["B"]).to(dev)
    sfa, sfb = _packed(dg, oracle_mod, p["sA"], p["sB"])
    mi = torch.from_numpy(p["m_indices"]).to(dev)
    D = torch.full((p["M"], p["N"]), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    dg.dg_fp8_grouped_gemm_contiguous_ue8m0(A, sfa, B, sfb, D, mi)
    assert dg.dg_get_device_status() == 0
    got = bits(D)
    assert not np.any(got == SENTINEL), plan
    rng = np.random.default_rng(5)
    r = np.concatenate([rng.integers(0, p["M"], 20000), [0, 0, p["M"] - 1, p["M"] - 1]])
    c = np.concatenate([rng.integers(0, p["N"], 20000), [0, p["N"] - 1, 0, p["N"] - 1]])
    g = p["m_indices"][r]
    ref = np.empty(r.size, np.uint16)
    for gg in np.unique(g):
        sel = g == gg
        _, ref[sel] = oracle_mod.gemm_nt_sampled(p["A"], p["sA"], p["B"][gg], p["sB"][gg], r[sel], c[sel])
    assert_close(got[r, c], ref, f"ue8m0 contiguous MoE (sampled), plan {plan}")


# ---------------------------------------------------------------- packing

def test_transform_flags_non_power_of_two(dg):
    dev = torch.device("cuda")
    s = np.ones((5, 8), np.float32)   # logical [rows][nkb]
    s[2, 5] = 3.0                     # not a power of two
    s[4, 0] = 0.0                     # zero is not a UE8M0 value
    sA = torch.from_numpy(gi.sa_to_kernel_layout(s)).to(dev)
    out = dg.dg_transform_sf_ue8m0(sA, 5, mn_major=True)
    assert dg.dg_get_device_status() == 8
    assert dg.dg_get_device_status() == 0  # cleared
    w = out.cpu().numpy().view(np.uint32)  # [2][8]
    assert (w[1, 2] >> 8) & 0xFF == 0xFF and (w[0, 4] & 0xFF) == 0xFF
    assert w[0, 0] == 0x7F7F7F7F and (w[1, 2] & 0xFF) == 0x7F


def test_transform_extreme_exponents(dg, oracle_mod):
    """Codes 0 (2^-127, an fp32 subnormal) through 254 (2^127) pack exactly."""
    dev = torch.device("cuda")
    e = np.arange(255).reshape(51, 5)
    s = np.exp2(e.astype(np.float64) - 127).astype(np.float32)
    out = dg.dg_transform_sf_ue8m0(torch.from_numpy(s).to(dev), 51, mn_major=False)
    assert dg.dg_get_device_status() == 0
    assert np.array_equal(out.cpu().numpy(), oracle_mod.pack_ue8m0(s))


# ------------------------------------------------------ bounded waits

@pytest.mark.parametrize("M,N,K,fam,first_ctas", [
    (1024, 4096, 4096, 1, 1),   # one-CTA tiles
    (2048, 4096, 4096, 2, 2),   # CTA pairs
])
def test_ue8m0_wait_timeout_is_reported_and_the_context_survives(dg, oracle_mod, M, N, K, fam, first_ctas):
    """With the stall injection hook the first CTA (or pair) never receives
    its operands: every wait of the block-scaled kernel is bounded, so it
    records DG_ERR_TIMEOUT, drains its scale copies, frees TMEM and returns,
    and the next call on the same buffers is correct."""
    p = gi.dense_problem(M, N, K, seed_a=75, seed_b=76, ue8m0=True)
    dg.dg_set_tile_family(fam)
    dg.dg_set_wait_timeout_ns(20_000_000)
    dg.dg_set_stall_injection(True)
    try:
        assert _plan(dg, 3, M, N, K)["pair"] == str(fam - 1)
        dev = torch.device("cuda")
        A = torch.from_numpy(p["A"]).to(dev)
        B = torch.from_numpy(p["B"]).to(dev)
        sfa, sfb = _packed(dg, oracle_mod, p["sA"], p["sB"])
        D = torch.full((M, N), SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
        dg.dg_fp8_gemm_nt_ue8m0(A, sfa, B, sfb, D)
        st, word = dg.dg_get_device_status_detail()
    finally:
        dg.dg_set_stall_injection(False)
        dg.dg_set_wait_timeout_ns(0)
    try:
        assert st == 5, f"status {st}, word {word:#x}"
        assert (word >> 8) & 0xF in (1, 2, 3)  # scale writers, MMA or epilogue
        assert word >> 20 < first_ctas          # in the stalled CTA (or pair)
        assert dg.dg_get_device_status() == 5   # read and cleared
        assert dg.dg_get_device_status() == 0
        dg.dg_fp8_gemm_nt_ue8m0(A, sfa, B, sfb, D)
        assert dg.dg_get_device_status() == 0
    finally:
        dg.dg_set_tile_family(dg.DG_TILES_AUTO)
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(bits(D), ref, f"ue8m0 after a timeout, {M}x{N}x{K}")
