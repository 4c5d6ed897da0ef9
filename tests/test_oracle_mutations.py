"""Do the oracle's pins catch plausible mistakes?

Each case plants one mistake in a temporary copy of oracle/dg_oracle.c -- a
wrong weight-block index, a transposed operand stride, a dropped K block, a
lost accumulation, an exponent bias off by one, truncation instead of
round-to-nearest-even, a UE8M0 bias, rounding direction or byte order --
builds it with gcc, and checks that at least one of
the independent pins (torch's casts, float64 matmul of the dequantised
inputs) rejects it.  The committed oracle itself is never modified."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import dg_inputs as gi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dg_oracle.c")

MUTATIONS = {
    "weight-block index n%128 instead of n/128": (
        "            double v = dgo_element(A + (int64_t)m * K, sA + (int64_t)m * nkb,\n                                   B + (int64_t)n * K,\n                                   sB + (int64_t)(n / DGO_BLOCK) * nkb, K);",
        "            double v = dgo_element(A + (int64_t)m * K, sA + (int64_t)m * nkb,\n                                   B + (int64_t)n * K,\n                                   sB + (int64_t)(n % DGO_BLOCK) * nkb, K);"),
    "B row stride 1 instead of K (transposed operand)": (
        "            double v = dgo_element(A + (int64_t)m * K, sA + (int64_t)m * nkb,\n                                   B + (int64_t)n * K,\n",
        "            double v = dgo_element(A + (int64_t)m * K, sA + (int64_t)m * nkb,\n                                   B + (int64_t)n,\n"),
    "first K block dropped": (
        "    for (int kb = 0; kb < nkb; ++kb) {\n        double partial = 0.0;\n        for (int k = kb * DGO_BLOCK; k < (kb + 1) * DGO_BLOCK; ++k)\n            partial += g_lut[a_row[k]] * g_lut[b_row[k]];\n        double scale",
        "    for (int kb = 1; kb < nkb; ++kb) {\n        double partial = 0.0;\n        for (int k = kb * DGO_BLOCK; k < (kb + 1) * DGO_BLOCK; ++k)\n            partial += g_lut[a_row[k]] * g_lut[b_row[k]];\n        double scale"),
    "accumulation lost (acc = instead of acc +=)": (
        "        acc += scale * partial;",
        "        acc = scale * partial;"),
    "e4m3 exponent bias off by one": (
        "v = ldexp((double)(8 + m), e - 10);",
        "v = ldexp((double)(8 + m), e - 9);"),
    "bf16 truncation instead of round-to-nearest-even": (
        "double nq = nearbyint(r);",
        "double nq = floor(r);"),
    "K-grouped: B scale of the wrong column block": (
        "(double)sB[(int64_t)kb * N + n] * partial;",
        "(double)sB[(int64_t)kb * N + n / 2] * partial;"),
    "accumulator C dropped from D = C + A.B^T": (
        "            double v = (double)C[(int64_t)m * N + n] +\n                       dgo_element(",
        "            double v = 0.0 * (double)C[(int64_t)m * N + n] +\n                       dgo_element("),
    "UE8M0 exponent bias 128 instead of 127": (
        "    return ldexp(1.0, (int)e - 127);",
        "    return ldexp(1.0, (int)e - 128);"),
    "UE8M0 scale rounded down instead of up": (
        "    return m == 0.5 ? x : ldexp(1.0, ex);",
        "    return m == 0.5 ? x : ldexp(1.0, ex - 1);"),
    "contiguous: row's own index instead of its block's first-row index": (
        "        if (g < 0 || g >= G || g != m_indices[(m / DGO_BLOCK) * DGO_BLOCK])",
        "        if (g < 0 || g >= G)"),
    "UE8M0 packing byte order reversed": (
        "                word |= (uint32_t)code << (8 * j);",
        "                word |= (uint32_t)code << (8 * (3 - j));"),
}


def _build_variant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor must match the oracle source exactly once"
    mutated = tmp_path / "dg_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    lib_path = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           "-o", str(lib_path), str(mutated), "-lm"])
    lib = ctypes.CDLL(str(lib_path))
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.dgo_gemm_nt.argtypes = [P, P, P, P, I, I, I, P, P]
    lib.dgo_gemm_nt.restype = I
    lib.dgo_decode_e4m3.argtypes = [P, P, I64]
    lib.dgo_bf16_round.argtypes = [P, P, I64]
    lib.dgo_gemm_nt_acc.argtypes = [P, P, P, P, P, I, I, I, P, P]
    lib.dgo_gemm_nt_acc.restype = I
    lib.dgo_k_grouped_tn.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
    lib.dgo_k_grouped_tn.restype = I
    lib.dgo_ue8m0_value.restype = ctypes.c_double
    lib.dgo_ue8m0_value.argtypes = [ctypes.c_uint8]
    lib.dgo_ue8m0_ceil_pow2.restype = ctypes.c_double
    lib.dgo_ue8m0_ceil_pow2.argtypes = [ctypes.c_double]
    lib.dgo_pack_ue8m0.restype = I
    lib.dgo_pack_ue8m0.argtypes = [P, I, I, P]
    lib.dgo_grouped_contiguous.restype = I
    lib.dgo_grouped_contiguous.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
    return lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _pins_pass(lib) -> bool:
    """The independent pins of test_oracle_pins, run against `lib`."""
    # decode: all 256 codes vs torch
    codes = np.arange(256, dtype=np.uint8)
    dec = np.empty(256, np.float64)
    lib.dgo_decode_e4m3(_ptr(codes), _ptr(dec), 256)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    fin = ~np.isnan(ref)
    if not np.array_equal(dec[fin], ref[fin]):
        return False
    # bf16: torch's float32 -> bf16 on random floats
    x = np.random.default_rng(7).standard_normal(20000).astype(np.float32)
    out = np.empty(x.size, np.uint16)
    lib.dgo_bf16_round(_ptr(x.astype(np.float64)), _ptr(out), x.size)
    if not np.array_equal(out, torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)):
        return False
    # scaled contraction vs float64 matmul of the dequantised inputs
    p = gi.dense_problem(40, 336, 512, seed_a=21, seed_b=22)
    sa = np.ascontiguousarray(p["sA"])
    d64 = np.empty((40, 336), np.float64)
    d16 = np.empty((40, 336), np.uint16)
    lib.dgo_gemm_nt(_ptr(np.ascontiguousarray(p["A"])), _ptr(sa), _ptr(np.ascontiguousarray(p["B"])),
                    _ptr(np.ascontiguousarray(p["sB"])), 40, 336, 512, _ptr(d64), _ptr(d16))
    a = torch.from_numpy(p["A"]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    b = torch.from_numpy(p["B"]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    a = a * np.repeat(sa.astype(np.float64), 128, axis=1)
    b = b * np.repeat(np.repeat(p["sB"].astype(np.float64), 128, axis=0)[:336], 128, axis=1)
    bound = np.abs(a) @ np.abs(b).T
    if not np.all(np.abs(d64 - a @ b.T) <= 1e-12 * bound + 1e-300):
        return False
    # accumulate form: integer inputs and an integer C, exact
    rng = np.random.default_rng(8)
    ai, bi = rng.integers(-4, 5, (8, 256)), rng.integers(-4, 5, (128, 256))
    ci = rng.integers(-1000, 1001, (8, 128)).astype(np.float32)
    to8 = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    a8, b8 = np.ascontiguousarray(to8(ai)), np.ascontiguousarray(to8(bi))
    ones_a, ones_b = np.ones((8, 2), np.float32), np.ones((1, 2), np.float32)
    e64 = np.empty((8, 128), np.float64)
    e32 = np.empty((8, 128), np.float32)
    lib.dgo_gemm_nt_acc(_ptr(a8), _ptr(ones_a), _ptr(b8), _ptr(ones_b), _ptr(ci), 8, 128, 256,
                        _ptr(e64), _ptr(e32))
    if not np.array_equal(e64, (ci + ai @ bi.T).astype(np.float64)):
        return False
    # K-grouped: per-group float64 matmul of the dequantised slices
    pk = gi.k_grouped_problem([128, 256], 24, 48, seed_a=28, seed_b=29)
    off = pk["k_offsets"]
    k64 = np.empty((2, 24, 48), np.float64)
    k32 = np.empty((2, 24, 48), np.float32)
    lib.dgo_k_grouped_tn(_ptr(np.ascontiguousarray(pk["A"])), _ptr(np.ascontiguousarray(pk["sA"])),
                         _ptr(np.ascontiguousarray(pk["B"])), _ptr(np.ascontiguousarray(pk["sB"])),
                         _ptr(off), 2, 24, 48, 384, _ptr(k64), _ptr(k32))
    vals = lambda c: torch.from_numpy(np.ascontiguousarray(c)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ka = vals(pk["A"]) * np.repeat(pk["sA"].astype(np.float64), 128, axis=0)
    kb = vals(pk["B"]) * np.repeat(pk["sB"].astype(np.float64), 128, axis=0)
    for g in range(2):
        ref = ka[off[g]:off[g + 1]].T @ kb[off[g]:off[g + 1]]
        bound = np.abs(ka[off[g]:off[g + 1]]).T @ np.abs(kb[off[g]:off[g + 1]])
        if not np.all(np.abs(k64[g] - ref) <= 1e-12 * bound + 1e-300):
            return False
    # UE8M0: code values, the rounding rule against a doubling search, and
    # the hand-worked packing example
    if any(lib.dgo_ue8m0_value(e) != 2.0 ** (e - 127) for e in range(255)):
        return False
    for x in [3.0, 0.3, 1.0, 1e-9, 5e6, 2.0 ** -20 * 1.0000001]:
        s = 1.0
        while s < x:
            s *= 2.0
        while s / 2.0 >= x:
            s /= 2.0
        if lib.dgo_ue8m0_ceil_pow2(x) != s:
            return False
    sc = np.array([[1, 2, 0.5, 8, 32], [0.25, 1, 1, 1, 1]], np.float32)
    words = np.empty((2, 2), np.int32)
    if lib.dgo_pack_ue8m0(_ptr(sc), 2, 5, _ptr(words)) != 0:
        return False
    want = np.array([[0x827E807F, 0x7F7F7F7D], [0x7F7F7F84, 0x7F7F7F7F]], dtype=np.uint32)
    if not np.array_equal(words.view(np.uint32), want):
        return False
    # contiguous placement: a block belongs to the group of its first row;
    # hand-listed rows written (rows 0..99 and 256..383), all others untouched
    pc = gi.contiguous_problem([384], 32, 128, seed_a=31, seed_b=32)
    idx = np.full(384, -1, np.int32)
    idx[0:100], idx[100:110], idx[140:200], idx[256:384] = 0, 1, 1, 0
    b2 = np.ascontiguousarray(np.concatenate([pc["B"], pc["B"]]))
    sb2 = np.ascontiguousarray(np.concatenate([pc["sB"], pc["sB"]]))
    c16 = np.full((384, 32), 0x7FC1, np.uint16)
    if lib.dgo_grouped_contiguous(_ptr(np.ascontiguousarray(pc["A"])), _ptr(np.ascontiguousarray(pc["sA"])),
                                  _ptr(b2), _ptr(sb2), _ptr(idx), 384, 32, 128, 2, None, _ptr(c16)) != 0:
        return False
    written = np.zeros(384, bool)
    written[0:100] = written[256:384] = True
    if not (np.all(c16[~written] == 0x7FC1) and np.all(c16[written] != 0x7FC1)):
        return False
    return True


def test_unmutated_copy_passes(tmp_path):
    lib = _build_variant(tmp_path, "#define DGO_BLOCK 128", "#define DGO_BLOCK 128")
    assert _pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTATIONS[name]
    lib = _build_variant(tmp_path, old, new)
    assert not _pins_pass(lib), f"no pin caught: {name}"
