"""Pins of the oracle's UE8M0 block-scaled variant, each against something
other than the oracle itself.

UE8M0 (hada.io DeepGEMM summary, section "Giao dien GEMM va rang buoc
layout": the SM100 path takes its scaling factors as packed UE8M0, four to
an int) is an unsigned 8-bit biased exponent, value 2**(e-127), 255 = NaN.
The readings pinned here: byte j of word (g, r) is K block 4g+j, pad bytes
are 127, the packed array is [ceil(nkb/4)][rows]; a block's UE8M0 scale is
the smallest power of two >= amax/448.
"""
import math

import numpy as np
import pytest
import torch

import dg_inputs as gi


def test_value_of_every_code(oracle_mod):
    for e in range(255):
        assert oracle_mod.ue8m0_value(e) == 2.0 ** (e - 127)  # exact in Python floats
    assert math.isnan(oracle_mod.ue8m0_value(255))


def test_from_scale_round_trip_and_rejections(oracle_mod):
    for e in range(255):
        assert oracle_mod.ue8m0_from_scale(2.0 ** (e - 127)) == e
    for bad in [0.0, -1.0, -0.5, 3.0, 0.75, 1.0 + 2.0 ** -23, 2.0 ** -128, 2.0 ** 128,
                math.inf, -math.inf, math.nan]:
        assert oracle_mod.ue8m0_from_scale(bad) == -1, bad


def _ceil_pow2_by_search(x: float) -> float:
    # doubling / halving on exact powers of two; no frexp, no log2
    s = 1.0
    while s < x:
        s *= 2.0
    while s / 2.0 >= x:
        s /= 2.0
    return s


def test_ceil_pow2_against_search(oracle_mod):
    rng = np.random.default_rng(5)
    xs = list(np.exp2(rng.uniform(-100, 100, 3000)))
    for k in range(-60, 61, 7):
        p = 2.0 ** k
        xs += [p, math.nextafter(p, math.inf), math.nextafter(p, 0.0), 1.5 * p, 0.75 * p]
    for x in xs:
        assert oracle_mod.ue8m0_ceil_pow2(x) == _ceil_pow2_by_search(x), x


def test_pack_hand_worked_example(oracle_mod):
    # Row 0 scales per K block: 1, 2, 1/2, 8 | 32 ; row 1: 1/4, 1, 1, 1 | 1.
    # Codes (e = log2 s + 127): 0x7f 0x80 0x7e 0x82 | 0x84 ; 0x7d 0x7f 0x7f 0x7f | 0x7f,
    # byte j of a word = K block 4g + j, missing blocks of group 1 padded 0x7f.
    s = np.array([[1, 2, 0.5, 8, 32], [0.25, 1, 1, 1, 1]], np.float32)
    packed = oracle_mod.pack_ue8m0(s)
    assert packed.shape == (2, 2)
    want = np.array([[0x827E807F, 0x7F7F7F7D], [0x7F7F7F84, 0x7F7F7F7F]], dtype=np.uint32)
    assert np.array_equal(packed.view(np.uint32), want)
    assert np.array_equal(oracle_mod.unpack_ue8m0(packed, 5), s)


def test_pack_round_trip_random(oracle_mod):
    rng = np.random.default_rng(6)
    for rows, nkb in [(1, 1), (7, 4), (130, 9), (3, 56)]:
        s = np.exp2(rng.integers(-127, 128, (rows, nkb))).astype(np.float32)
        p = oracle_mod.pack_ue8m0(s)
        assert p.shape == ((nkb + 3) // 4, rows)
        assert np.array_equal(oracle_mod.unpack_ue8m0(p, nkb), s)
        # pad bytes of a partial last group are 127
        if nkb % 4:
            top = p[-1].view(np.uint32) >> np.uint32(8 * (nkb % 4))
            full = (1 << (8 * (4 - nkb % 4))) - 1
            assert np.all(top == (0x7F7F7F7F & full))


def test_pack_rejects_non_power_of_two(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.pack_ue8m0(np.array([[1.0, 3.0]], np.float32))


def test_inputs_ue8m0_rounding_matches_oracle_rule(oracle_mod):
    """The UE8M0 input recipe's scales follow the oracle's rounding rule, and
    the data is quantised with them: no block overflows, every block uses
    more than half of the e4m3 range, codes round to nearest."""
    x = gi.standard_normal(11, (64, 1024))
    x[3, :128] *= 1e-6     # a block near the amax floor
    x[5, 256:384] = 0.0    # an all-zero block
    codes, s = gi.quantize_1x128(x, ue8m0=True)
    amax = np.abs(x.reshape(64, 8, 128)).astype(np.float64).max(axis=-1)
    for (i, j), a in np.ndenumerate(amax):
        want = oracle_mod.ue8m0_ceil_pow2(max(a, 1e-4) / 448.0)
        assert s[i, j] == np.float32(want)
        assert oracle_mod.ue8m0_from_scale(float(s[i, j])) >= 0
    ratio = np.maximum(amax, 1e-4) / s.astype(np.float64)
    assert np.all(ratio <= 448.0) and np.all(ratio > 224.0)
    dec = oracle_mod.decode_e4m3(codes).reshape(64, 8, 128)
    y = x.reshape(64, 8, 128).astype(np.float64) / s[..., None].astype(np.float64)
    # e4m3 normals carry 3 mantissa bits: |y - q| <= 2^-4 |y| (half an ulp),
    # subnormals an absolute 2^-10
    assert np.all(np.abs(y - dec) <= np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10))


def test_inputs_ue8m0_weight_blocks(oracle_mod):
    x = gi.standard_normal(12, (300, 512))
    codes, s = gi.quantize_128x128(x, ue8m0=True)
    assert s.shape == (3, 4)
    for nb in range(3):
        blk = x[nb * 128:(nb + 1) * 128].reshape(-1, 4, 128)
        for kb in range(4):
            a = float(np.abs(blk[:, kb]).max())
            assert s[nb, kb] == np.float32(oracle_mod.ue8m0_ceil_pow2(max(a, 1e-4) / 448.0))


def test_gemm_with_packed_scales_integer_inputs_exact(oracle_mod):
    """Integer-valued codes with power-of-two scales: the block-scaled result
    is exact and equals an integer matmul times the scales."""
    rng = np.random.default_rng(9)
    M, N, K = 24, 160, 640
    ai, bi = rng.integers(-8, 9, (M, K)), rng.integers(-8, 9, (N, K))
    to8 = lambda v: torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    a8, b8 = to8(ai), to8(bi)
    sa = np.exp2(rng.integers(-6, 7, (M, K // 128))).astype(np.float32)
    sb = np.exp2(rng.integers(-6, 7, ((N + 127) // 128, K // 128))).astype(np.float32)
    d64, _ = oracle_mod.gemm_nt_ue8m0(a8, oracle_mod.pack_ue8m0(sa), b8, oracle_mod.pack_ue8m0(sb))
    want = np.zeros((M, N))
    for kb in range(K // 128):
        sl = slice(kb * 128, (kb + 1) * 128)
        part = (ai[:, sl] @ bi[:, sl].T).astype(np.float64)
        want += part * sa[:, kb][:, None] * np.repeat(sb[:, kb], 128)[:N][None, :]
    assert np.array_equal(d64, want)
