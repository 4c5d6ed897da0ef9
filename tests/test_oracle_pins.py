"""Pins for the CPU oracle: every check compares it with something other than
itself -- torch's CPU casts, float64 matmul of the decoded inputs (a library
routine), closed forms, invariants and brute-force loops."""
import math

import numpy as np
import pytest
import torch

import dg_inputs as gi

BLOCK = 128


# ------------------------------------------------------------------ codecs

def test_e4m3_all_codes_match_torch(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle_mod.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2  # S.1111.111 for both signs
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros decode with their sign
    assert math.copysign(1.0, ours[0x80]) == -1.0


def test_e4m3_closed_form_points(oracle_mod):
    assert oracle_mod.e4m3_value(0x7E) == 448.0          # largest finite
    assert oracle_mod.e4m3_value(0x01) == 2.0 ** -9       # smallest subnormal
    assert oracle_mod.e4m3_value(0x08) == 2.0 ** -6       # smallest normal
    assert oracle_mod.e4m3_value(0x38) == 1.0
    assert oracle_mod.e4m3_value(0xB8) == -1.0


def _torch_bf16_bits(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x32.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_matches_torch_on_floats(oracle_mod):
    rng = np.random.default_rng(7)
    # random float32 values across many binades, plus exact bf16 ties
    x = (rng.standard_normal(200_000) * np.exp2(rng.integers(-140, 127, 200_000))).astype(np.float32)
    x = x[np.isfinite(x)]
    ties = (rng.integers(-(1 << 15), 1 << 15, 20_000).astype(np.int32) << 16) | 0x8000
    ties = ties.view(np.float32)
    ties = ties[np.isfinite(ties)]
    for arr in (x, ties):
        ours = oracle_mod.bf16_round(arr.astype(np.float64))
        ref = _torch_bf16_bits(arr)
        nanmask = np.isnan(arr)
        assert np.array_equal(ours[~nanmask], ref[~nanmask])


def test_bf16_rounds_doubles_once(oracle_mod):
    # 1 + 2^-8 is an exact tie between 1 and 1 + 2^-7 -> even (1.0).
    assert oracle_mod.bf16_from_double(1.0 + 2 ** -8) == 0x3F80
    # a hair above the tie must round up; a float-first path would lose it.
    assert oracle_mod.bf16_from_double(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81
    # 1 + 3*2^-8 is a tie between 1+2^-7 (odd) and 1+2^-6 (even) -> up.
    assert oracle_mod.bf16_from_double(1.0 + 3 * 2 ** -8) == 0x3F82
    # overflow: max bf16 = (2^8-1)*2^120; half an ulp above -> inf
    assert oracle_mod.bf16_from_double(255 * 2.0 ** 120) == 0x7F7F
    assert oracle_mod.bf16_from_double(255.5 * 2.0 ** 120) == 0x7F80
    assert oracle_mod.bf16_from_double(-255.5 * 2.0 ** 120) == 0xFF80
    # subnormals: quantum 2^-133
    assert oracle_mod.bf16_from_double(2.0 ** -133) == 0x0001
    assert oracle_mod.bf16_from_double(2.0 ** -134) == 0x0000          # tie -> even 0
    assert oracle_mod.bf16_from_double(1.5 * 2.0 ** -133) == 0x0002    # tie -> even 2
    assert oracle_mod.bf16_from_double(-0.0) == 0x8000
    assert oracle_mod.bf16_from_double(float("nan")) & 0x7FC0 == 0x7FC0


# ------------------------------------------------------------- contraction

def _dequant(codes, scales_rows, row_block):
    """codes [R][K] -> float64 values times their block scale (row_block=1 for
    1x128 scales indexed [r][kb], 128 for 128x128 scales indexed [r//128][kb])."""
    vals = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    R, K = vals.shape
    s = np.repeat(np.repeat(scales_rows.astype(np.float64), row_block, axis=0)[:R], BLOCK, axis=1)
    return vals * s


def test_unit_scales_equal_float64_matmul_exactly(oracle_mod):
    p = gi.dense_problem(80, 272, 512, seed_a=11, seed_b=12)
    sa = np.ones_like(p["sA"])
    sb = np.ones_like(p["sB"])
    d64, _ = oracle_mod.gemm_nt(p["A"], sa, p["B"], sb)
    a = _dequant(p["A"], sa, 1)
    b = _dequant(p["B"], sb, BLOCK)
    ref = torch.from_numpy(a) @ torch.from_numpy(b).T
    assert np.array_equal(d64, ref.numpy())


def test_scaled_equals_dequantised_float64_matmul(oracle_mod):
    # N spans three 128-row weight blocks (the last one partial), M is not a
    # multiple of 128, K has four scale blocks: wrong block indexing, a
    # transposed operand or a dropped block all show up here.
    p = gi.dense_problem(70, 336, 512, seed_a=21, seed_b=22)
    sa = p["sA"] * np.exp2(np.random.default_rng(3).integers(-3, 4, p["sA"].shape)).astype(np.float32)
    d64, d16 = oracle_mod.gemm_nt(p["A"], sa, p["B"], p["sB"])
    a = _dequant(p["A"], sa, 1)
    b = _dequant(p["B"], p["sB"], BLOCK)
    ref = a @ b.T
    bound = np.abs(a) @ np.abs(b).T
    assert np.all(np.abs(d64 - ref) <= 1e-12 * bound + 1e-300)
    # and the bf16 output is the one rounding of that value
    assert np.array_equal(d16, oracle_mod.bf16_round(d64))


def test_integer_inputs_exact(oracle_mod):
    rng = np.random.default_rng(5)
    M, N, K = 40, 160, 384
    ai = rng.integers(-4, 5, (M, K))
    bi = rng.integers(-4, 5, (N, K))
    a = torch.from_numpy(ai.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    b = torch.from_numpy(bi.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sa = np.ones((M, K // BLOCK), np.float32)
    sb = np.ones(((N + 127) // 128, K // BLOCK), np.float32)
    d64, d16 = oracle_mod.gemm_nt(a, sa, b, sb)
    exact = ai @ bi.T
    assert np.array_equal(d64, exact.astype(np.float64))
    # |exact| < 2^8 * ... fits in float32 exactly, so torch's cast is one rounding
    ref16 = _torch_bf16_bits(exact.astype(np.float32))
    assert np.array_equal(d16, ref16)


def test_identity_and_zero(oracle_mod):
    K = 128
    one = 0x38  # e4m3 code of 1.0
    A = np.zeros((K, K), np.uint8)
    A[np.arange(K), np.arange(K)] = one
    p = gi.dense_problem(1, 200, K, seed_b=31)
    sa = np.ones((K, 1), np.float32)
    sb = np.ones_like(p["sB"])
    _, d16 = oracle_mod.gemm_nt(A, sa, p["B"], sb)
    bt = torch.from_numpy(p["B"]).view(torch.float8_e4m3fn).to(torch.float32).T.contiguous()
    assert np.array_equal(d16, _torch_bf16_bits(bt.numpy()))
    Z = np.zeros((8, K), np.uint8)
    _, dz = oracle_mod.gemm_nt(Z, np.ones((8, 1), np.float32), p["B"], p["sB"])
    assert np.all(dz == 0)  # +0.0


def test_power_of_two_invariance(oracle_mod):
    p = gi.dense_problem(16, 256, 512, seed_a=41, seed_b=42)
    d64, _ = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"])
    for j in (-5, 3):
        d64j, _ = oracle_mod.gemm_nt(p["A"], p["sA"] * np.float32(2.0 ** j), p["B"], p["sB"])
        assert np.array_equal(d64j, d64 * 2.0 ** j)
    # a per-row scale change multiplies exactly that row
    sa = p["sA"].copy()
    sa[5] *= 4
    d64r, _ = oracle_mod.gemm_nt(p["A"], sa, p["B"], p["sB"])
    assert np.array_equal(d64r[5], d64[5] * 4)
    assert np.array_equal(np.delete(d64r, 5, 0), np.delete(d64, 5, 0))


def test_brute_force_tiny(oracle_mod):
    """Hand-rolled quadruple loop over decoded values (pure Python)."""
    M, N, K = 3, 136, 256  # N crosses a 128-row weight block boundary
    p = gi.dense_problem(M, N, K, seed_a=51, seed_b=52)
    dec = {c: float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float()) for c in range(256)}
    A, B, sA, sB = p["A"], p["B"], p["sA"], p["sB"]
    d64, _ = oracle_mod.gemm_nt(A, sA, B, sB)
    for m in range(M):
        for n in range(N):
            total = 0.0
            for kb in range(K // BLOCK):
                part = 0.0
                for k in range(kb * BLOCK, (kb + 1) * BLOCK):
                    part += dec[int(A[m, k])] * dec[int(B[n, k])]
                total += float(sA[m, kb]) * float(sB[n // BLOCK, kb]) * part
            assert abs(total - d64[m, n]) <= 1e-12 * (abs(total) + 1e-30) + 1e-300


def test_sampled_matches_full(oracle_mod):
    p = gi.dense_problem(130, 272, 256, seed_a=61, seed_b=62)
    d64, d16 = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"])
    rng = np.random.default_rng(0)
    r = rng.integers(0, 130, 500)
    c = rng.integers(0, 272, 500)
    s64, s16 = oracle_mod.gemm_nt_sampled(p["A"], p["sA"], p["B"], p["sB"], r, c)
    assert np.array_equal(s64, d64[r, c])
    assert np.array_equal(s16, d16[r, c])


# ------------------------------------------------------ D = C + A @ B.T

def test_acc_integer_inputs_and_integer_c_exact(oracle_mod):
    # integer-valued e4m3, unit scales and an integer C: every sum is an
    # integer below 2^24, so the float32 result is exact
    rng = np.random.default_rng(15)
    M, N, K = 36, 144, 384
    ai = rng.integers(-4, 5, (M, K))
    bi = rng.integers(-4, 5, (N, K))
    ci = rng.integers(-100000, 100001, (M, N))
    a = torch.from_numpy(ai.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    b = torch.from_numpy(bi.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sa = np.ones((M, K // BLOCK), np.float32)
    sb = np.ones(((N + 127) // 128, K // BLOCK), np.float32)
    d64, d32 = oracle_mod.gemm_nt_acc(a, sa, b, sb, ci.astype(np.float32))
    exact = ci + ai @ bi.T
    assert np.array_equal(d64, exact.astype(np.float64))
    assert np.array_equal(d32, exact.astype(np.float32))


def test_acc_zero_operand_returns_c(oracle_mod):
    # A = 0 (code 0x00): D = C bit for bit (C without negative zeros, which
    # -0 + +0 would turn positive), including subnormal and huge values
    rng = np.random.default_rng(16)
    M, N, K = 8, 32, 128
    c = (rng.standard_normal((M, N)) * np.exp2(rng.integers(-140, 120, (M, N)))).astype(np.float32)
    c[c == 0] = 1.0
    p = gi.dense_problem(M, N, K, seed_b=17)
    d64, d32 = oracle_mod.gemm_nt_acc(np.zeros((M, K), np.uint8), p["sA"], p["B"], p["sB"], c)
    assert np.array_equal(d32.view(np.uint32), c.view(np.uint32))


def test_acc_equals_c_plus_dequantised_matmul(oracle_mod):
    p = gi.dense_problem(50, 272, 384, seed_a=18, seed_b=19)
    c = np.random.default_rng(20).standard_normal((50, 272)).astype(np.float32) * 30
    d64, d32 = oracle_mod.gemm_nt_acc(p["A"], p["sA"], p["B"], p["sB"], c)
    a = _dequant(p["A"], p["sA"], 1)
    b = _dequant(p["B"], p["sB"], BLOCK)
    ref = c.astype(np.float64) + a @ b.T
    bound = np.abs(c.astype(np.float64)) + np.abs(a) @ np.abs(b).T
    assert np.all(np.abs(d64 - ref) <= 1e-12 * bound + 1e-300)
    # one rounding from double to float32 (numpy's conversion, to nearest even)
    assert np.array_equal(d32.view(np.uint32), d64.astype(np.float32).view(np.uint32))
    r = np.random.default_rng(0).integers(0, 50, 300)
    q = np.random.default_rng(1).integers(0, 272, 300)
    s64, s32 = oracle_mod.gemm_nt_acc_sampled(p["A"], p["sA"], p["B"], p["sB"], c, r, q)
    assert np.array_equal(s64, d64[r, q]) and np.array_equal(s32, d32[r, q])


# ------------------------------------------------ K-grouped TN (wgrad)

def test_k_grouped_equals_per_group_dequantised_matmul(oracle_mod):
    # uneven groups, an empty group, M and N not multiples of 128
    p = gi.k_grouped_problem([256, 0, 128, 384], 72, 144, seed_a=25, seed_b=26)
    d64, d32 = oracle_mod.k_grouped_tn(p["A"], p["sA"], p["B"], p["sB"], p["k_offsets"])
    vals = lambda c: torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    a = vals(p["A"]) * np.repeat(p["sA"].astype(np.float64), BLOCK, axis=0)  # [K][M]
    b = vals(p["B"]) * np.repeat(p["sB"].astype(np.float64), BLOCK, axis=0)  # [K][N]
    off = p["k_offsets"]
    for g in range(p["G"]):
        ag, bg = a[off[g]:off[g + 1]], b[off[g]:off[g + 1]]
        ref = ag.T @ bg
        bound = np.abs(ag).T @ np.abs(bg)
        assert np.all(np.abs(d64[g] - ref) <= 1e-12 * bound + 1e-300), g
    assert np.all(d64[1] == 0.0)  # the empty group
    assert np.array_equal(d32.view(np.uint32), d64.astype(np.float32).view(np.uint32))


def test_k_grouped_integer_inputs_exact(oracle_mod):
    rng = np.random.default_rng(27)
    ks, M, N = [128, 256], 40, 64
    K = sum(ks)
    ai, bi = rng.integers(-4, 5, (K, M)), rng.integers(-4, 5, (K, N))
    to8 = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    off = np.array([0, 128, 384], np.int32)
    _, d32 = oracle_mod.k_grouped_tn(to8(ai), np.ones((K // BLOCK, M), np.float32), to8(bi),
                                     np.ones((K // BLOCK, N), np.float32), off)
    assert np.array_equal(d32[0], (ai[:128].T @ bi[:128]).astype(np.float32))
    assert np.array_equal(d32[1], (ai[128:].T @ bi[128:]).astype(np.float32))


def test_k_grouped_rejects_bad_offsets(oracle_mod):
    p = gi.k_grouped_problem([128, 128], 16, 16)
    for bad in ([0, 100, 256], [0, 256, 128], [0, 128, 384]):
        with pytest.raises(ValueError):
            oracle_mod.k_grouped_tn(p["A"], p["sA"], p["B"], p["sB"], np.array(bad, np.int32))


# ----------------------------------------------------------------- grouped

SENTINEL = 0x7FC1  # a NaN pattern nobody computes


def test_contiguous_equals_per_group_dense(oracle_mod):
    N, K = 192, 256
    p = gi.contiguous_problem([100, 256, 0, 37], N, K, seed_a=71, seed_b=72)
    M = p["M"]
    assert oracle_mod.check_contiguous_alignment(p["m_indices"]) == -1
    init = np.full((M, N), SENTINEL, np.uint16)
    _, d16 = oracle_mod.grouped_contiguous(p["A"], p["sA"], p["B"], p["sB"], p["m_indices"], init)
    for g in range(p["G"]):
        rows = np.nonzero(p["m_indices"] == g)[0]
        if rows.size == 0:
            continue
        _, ref = oracle_mod.gemm_nt(p["A"][rows], p["sA"][rows], p["B"][g], p["sB"][g])
        assert np.array_equal(d16[rows], ref)
    pad = p["m_indices"] < 0
    assert pad.sum() == (128 - 100) + (128 - 37)
    assert np.all(d16[pad] == SENTINEL)


def test_contiguous_alignment_checker(oracle_mod):
    idx = np.array([0] * 128 + [1] * 127 + [2], np.int32)
    assert oracle_mod.check_contiguous_alignment(idx) == 255
    # padding after a segment is fine, a segment starting mid-block is not
    idx = np.array([0] * 100 + [-1] * 28 + [-1] * 10 + [1] * 118, np.int32)
    assert oracle_mod.check_contiguous_alignment(idx) == 138
    idx = np.array([0] * 100 + [-1] * 28 + [1] * 128, np.int32)
    assert oracle_mod.check_contiguous_alignment(idx) == -1


def test_contiguous_malformed_blocks_written_by_block_rule(oracle_mod):
    """Segments are aligned to the 128-row M block, so a block belongs to the
    group of its first row.  Hand-built blocks that break the rule: the rows
    listed below (and only they) are written, each equal to the dense GEMM
    of its group; every other row keeps the sentinel."""
    N, K, G = 144, 256, 2
    M = 5 * 128
    p = gi.contiguous_problem([M], N, K, seed_a=73, seed_b=74)
    rng = np.random.default_rng(75)
    B = np.stack([p["B"][0], rng.permutation(p["B"][0])])
    sB = np.stack([p["sB"][0], p["sB"][0] * 0.5])
    idx = np.full(M, -1, np.int32)
    idx[0:100] = 0        # block 0: group 0, then a mid-block change to group 1
    idx[100:110] = 1
    idx[140:200] = 1      # block 1: first row padding, later rows valid
    idx[256:384] = 1      # block 2: well formed
    idx[384:512] = 5      # block 3: group out of range
    idx[512:520] = 0      # block 4: group 0, then a row with an out-of-range index
    idx[520] = 7
    idx[521:600] = 0
    init = np.full((M, N), SENTINEL, np.uint16)
    _, d16 = oracle_mod.grouped_contiguous(p["A"], p["sA"], B, sB, idx, init)
    written = {0: list(range(0, 100)) + list(range(512, 520)) + list(range(521, 600)),
               1: list(range(256, 384))}
    for g, rows in written.items():
        rows = np.asarray(rows)
        _, ref = oracle_mod.gemm_nt(p["A"][rows], p["sA"][rows], B[g], sB[g])
        assert np.array_equal(d16[rows], ref), f"group {g}"
    untouched = np.setdiff1d(np.arange(M), np.concatenate([np.asarray(r) for r in written.values()]))
    assert untouched.size == M - 100 - 8 - 79 - 128
    assert np.all(d16[untouched] == SENTINEL)
    assert oracle_mod.check_contiguous_alignment(idx) == 100


def test_masked_equals_per_group_dense_and_leaves_rest(oracle_mod):
    G, max_m, N, K = 3, 160, 144, 256
    masked_m = np.array([1, 160, 0], np.int32)
    p = gi.masked_problem(G, max_m, N, K, masked_m=masked_m, seed_a=81, seed_b=82)
    init = np.full((G, max_m, N), SENTINEL, np.uint16)
    _, d16 = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], masked_m, init)
    for g in range(G):
        m = masked_m[g]
        if m:
            _, ref = oracle_mod.gemm_nt(p["A"][g, :m], p["sA"][g, :m], p["B"][g], p["sB"][g])
            assert np.array_equal(d16[g, :m], ref)
        assert np.all(d16[g, m:] == SENTINEL)


def test_masked_count_above_max_is_clamped(oracle_mod):
    G, max_m, N, K = 1, 8, 16, 128
    p = gi.masked_problem(G, max_m, N, K, masked_m=[50], seed_a=91, seed_b=92)
    init = np.full((G, max_m, N), SENTINEL, np.uint16)
    _, d16 = oracle_mod.grouped_masked(p["A"], p["sA"], p["B"], p["sB"], np.array([50], np.int32), init)
    _, ref = oracle_mod.gemm_nt(p["A"][0], p["sA"][0], p["B"][0], p["sB"][0])
    assert np.array_equal(d16[0], ref)


# -------------------------------------------------- fp32 promotion analysis

def test_fp32_promotion_emulation_matches_float32_recompute(oracle_mod):
    p = gi.dense_problem(8, 256, 512, seed_a=101, seed_b=102)
    r = np.repeat(np.arange(8), 256)
    c = np.tile(np.arange(256), 8)
    out = oracle_mod.fp32_promotion_sampled(p["A"], p["sA"], p["B"], p["sB"], r, c)
    a = torch.from_numpy(p["A"]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    b = torch.from_numpy(p["B"]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    acc = np.zeros(r.size, np.float32)
    for kb in range(512 // BLOCK):
        part = np.einsum("ik,ik->i", a[r, kb * 128:(kb + 1) * 128], b[c, kb * 128:(kb + 1) * 128]).astype(np.float32)
        s = (p["sA"][r, kb] * p["sB"][c // 128, kb]).astype(np.float32)
        acc = (part.astype(np.float64) * s.astype(np.float64) + acc.astype(np.float64)).astype(np.float32)
    assert np.array_equal(out, acc)


def test_generator_recipe():
    p = gi.dense_problem(4, 200, 256, seed_a=1, seed_b=2)
    x = gi.standard_normal(1, (4, 256))
    amax = np.abs(x.reshape(4, 2, 128)).max(-1)
    assert np.array_equal(p["sA"], (np.maximum(amax, np.float32(1e-4)) / np.float32(448)).astype(np.float32))
    # partial last weight block counts only its 72 real rows
    xb = gi.standard_normal(2, (200, 256))
    amax_b = np.abs(xb[128:].reshape(72, 2, 128)).max(axis=(0, 2))
    assert np.array_equal(p["sB"][1], (amax_b / np.float32(448)).astype(np.float32))
    dec = torch.from_numpy(p["A"]).view(torch.float8_e4m3fn).float().numpy()
    assert np.abs(dec).max() <= 448
