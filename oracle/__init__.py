"""CPU oracle for the fine-grained-scaled FP8 GEMM (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and this
package imports nothing from the product path.

The arithmetic lives in ``dg_oracle.c`` (plain C, OpenMP over output rows,
fp64 block sums, one double->bf16 rounding).  This module only compiles it
with gcc and marshals numpy arrays through ctypes.

Parity status of each function (what pins it is listed in the tests):
  e4m3_value / decode_e4m3      pinned: all 256 codes vs torch's e4m3fn cast
  bf16_from_double              pinned: torch float32->bf16 on exact floats,
                                closed-form ties, overflow and subnormals
  gemm_nt / gemm_nt_sampled     pinned: float64 matmul of decoded inputs
                                (exact with unit scales, 1e-12 with scales),
                                integer inputs, identity/zero, power-of-two
                                invariance, brute-force loops on tiny cases
  k_grouped_tn                  pinned: each group equals the float64 matmul
                                of its dequantised slices (1e-12), integer
                                inputs exact, empty groups give zeros
  gemm_nt_acc (+ _sampled)      pinned: integer inputs plus an integer C
                                (exact), C alone (A = 0), the closed form
                                C + float64 matmul, numpy's double->float32
  grouped_contiguous / masked   pinned: per-group dense results, placement,
                                untouched padding / masked rows, malformed
                                contiguous blocks written by hand-listed rows
  fp32_promotion_sampled        analysis aid (not a reference), pinned against
                                a float32 re-computation on small cases
  ue8m0_value / ue8m0_from_scale  pinned: every code vs Python's exact 2.0**k,
                                round trip of all 255 finite codes, rejection
                                of non-powers of two, zero, inf, NaN, range
  ue8m0_ceil_pow2               pinned: a doubling/halving search (no frexp)
                                on random and boundary values, exact powers
  pack_ue8m0 / unpack_ue8m0     pinned: a hand-worked example (byte j = K
                                block 4g+j, pad 127), round trip
  gemm_nt_ue8m0 (+ grouped)     the GEMM above on the unpacked scales
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.c")
_LIB = os.path.join(_HERE, "libdg_oracle.so")
_lib = None

BLOCK = 128


def build(force: bool = False) -> str:
    """Compile dg_oracle.c into libdg_oracle.so next to it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.dgo_e4m3_value.restype = ctypes.c_double
        lib.dgo_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.dgo_bf16_from_double.restype = ctypes.c_uint16
        lib.dgo_bf16_from_double.argtypes = [ctypes.c_double]
        lib.dgo_decode_e4m3.argtypes = [P, P, I64]
        lib.dgo_bf16_round.argtypes = [P, P, I64]
        lib.dgo_gemm_nt.restype = I
        lib.dgo_gemm_nt.argtypes = [P, P, P, P, I, I, I, P, P]
        lib.dgo_gemm_nt_acc.restype = I
        lib.dgo_gemm_nt_acc.argtypes = [P, P, P, P, P, I, I, I, P, P]
        lib.dgo_gemm_nt_acc_sampled.restype = I
        lib.dgo_gemm_nt_acc_sampled.argtypes = [P, P, P, P, P, I, I, I, P, P, I64, P, P]
        lib.dgo_ue8m0_value.restype = ctypes.c_double
        lib.dgo_ue8m0_value.argtypes = [ctypes.c_uint8]
        lib.dgo_ue8m0_from_scale.restype = I
        lib.dgo_ue8m0_from_scale.argtypes = [ctypes.c_double]
        lib.dgo_ue8m0_ceil_pow2.restype = ctypes.c_double
        lib.dgo_ue8m0_ceil_pow2.argtypes = [ctypes.c_double]
        lib.dgo_pack_ue8m0.restype = I
        lib.dgo_pack_ue8m0.argtypes = [P, I, I, P]
        lib.dgo_unpack_ue8m0.restype = I
        lib.dgo_unpack_ue8m0.argtypes = [P, I, I, P]
        lib.dgo_k_grouped_tn.restype = I
        lib.dgo_k_grouped_tn.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
        lib.dgo_gemm_nt_sampled.restype = I
        lib.dgo_gemm_nt_sampled.argtypes = [P, P, P, P, I, I, I, P, P, I64, P, P]
        lib.dgo_grouped_contiguous.restype = I
        lib.dgo_grouped_contiguous.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
        lib.dgo_check_contiguous_alignment.restype = I64
        lib.dgo_check_contiguous_alignment.argtypes = [P, I, I]
        lib.dgo_grouped_masked.restype = I
        lib.dgo_grouped_masked.argtypes = [P, P, P, P, P, I, I, I, I, P, P]
        lib.dgo_gemm_nt_fp32_promotion_sampled.restype = I
        lib.dgo_gemm_nt_fp32_promotion_sampled.argtypes = [P, P, P, P, I, I, I, P, P, I64, P]
        lib.dgo_num_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u8(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint8:
        a = a.view(np.uint8)
    return a


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return _load().dgo_num_threads()


def e4m3_value(code: int) -> float:
    return _load().dgo_e4m3_value(code)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    codes = _u8(codes)
    out = np.empty(codes.shape, dtype=np.float64)
    _load().dgo_decode_e4m3(_ptr(codes), _ptr(out), codes.size)
    return out


def bf16_from_double(x: float) -> int:
    return _load().dgo_bf16_from_double(float(x))


def bf16_round(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().dgo_bf16_round(_ptr(x), _ptr(out), x.size)
    return out


def gemm_nt(A, sA, B, sB, want_f64: bool = True):
    """Dense D = A @ B.T with 1x128 (sA: [M][K/128]) and 128x128
    (sB: [ceil(N/128)][K/128]) scales.  Returns (D64 or None, D16 bits)."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and sA.shape == (M, K // BLOCK)
    assert sB.shape == ((N + BLOCK - 1) // BLOCK, K // BLOCK)
    d64 = np.empty((M, N), dtype=np.float64) if want_f64 else None
    d16 = np.empty((M, N), dtype=np.uint16)
    rc = _load().dgo_gemm_nt(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N, K,
                             _ptr(d64), _ptr(d16))
    if rc:
        raise ValueError("dgo_gemm_nt: bad sizes")
    return d64, d16


def gemm_nt_sampled(A, sA, B, sB, rows, cols):
    """Dense result at the (rows[i], cols[i]) pairs: (f64 values, bf16 bits)."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    M, K = A.shape
    N = B.shape[0]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    assert rows.shape == cols.shape
    o64 = np.empty(rows.shape, dtype=np.float64)
    o16 = np.empty(rows.shape, dtype=np.uint16)
    rc = _load().dgo_gemm_nt_sampled(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N,
                                     K, _ptr(rows), _ptr(cols), rows.size,
                                     _ptr(o64), _ptr(o16))
    if rc:
        raise ValueError("dgo_gemm_nt_sampled: bad sizes or indices")
    return o64, o16


def gemm_nt_acc(A, sA, B, sB, C, want_f64: bool = True):
    """Dense D = C + A @ B.T with C, D float32 [M][N] (sum in double, one
    rounding to float32).  Returns (D64 or None, D32)."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    C = _f32(C)
    M, K = A.shape
    N = B.shape[0]
    assert B.shape[1] == K and sA.shape == (M, K // BLOCK) and C.shape == (M, N)
    assert sB.shape == ((N + BLOCK - 1) // BLOCK, K // BLOCK)
    d64 = np.empty((M, N), dtype=np.float64) if want_f64 else None
    d32 = np.empty((M, N), dtype=np.float32)
    rc = _load().dgo_gemm_nt_acc(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(C), M, N, K,
                                 _ptr(d64), _ptr(d32))
    if rc:
        raise ValueError("dgo_gemm_nt_acc: bad sizes")
    return d64, d32


def gemm_nt_acc_sampled(A, sA, B, sB, C, rows, cols):
    """gemm_nt_acc at the (rows[i], cols[i]) pairs: (f64 values, float32)."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    C = _f32(C)
    M, K = A.shape
    N = B.shape[0]
    assert C.shape == (M, N)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    o64 = np.empty(rows.shape, dtype=np.float64)
    o32 = np.empty(rows.shape, dtype=np.float32)
    rc = _load().dgo_gemm_nt_acc_sampled(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(C), M, N, K,
                                         _ptr(rows), _ptr(cols), rows.size, _ptr(o64), _ptr(o32))
    if rc:
        raise ValueError("dgo_gemm_nt_acc_sampled: bad sizes or indices")
    return o64, o32


def k_grouped_tn(A, sA, B, sB, k_offsets, want_f64: bool = True):
    """K-grouped TN GEMM: A [K][M], B [K][N] (MN-major), sA [K/128][M],
    sB [K/128][N], k_offsets [G+1].  Returns (D64 or None, D32), [G][M][N]."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    off = np.ascontiguousarray(k_offsets, dtype=np.int32)
    K, M = A.shape
    N = B.shape[1]
    G = off.size - 1
    assert B.shape[0] == K and sA.shape == (K // BLOCK, M) and sB.shape == (K // BLOCK, N)
    d64 = np.empty((G, M, N), dtype=np.float64) if want_f64 else None
    d32 = np.empty((G, M, N), dtype=np.float32)
    rc = _load().dgo_k_grouped_tn(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(off), G, M, N, K,
                                  _ptr(d64), _ptr(d32))
    if rc:
        raise ValueError("dgo_k_grouped_tn: bad sizes or offsets")
    return d64, d32


def fp32_promotion_sampled(A, sA, B, sB, rows, cols):
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    M, K = A.shape
    N = B.shape[0]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    out = np.empty(rows.shape, dtype=np.float32)
    rc = _load().dgo_gemm_nt_fp32_promotion_sampled(
        _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), M, N, K, _ptr(rows), _ptr(cols),
        rows.size, _ptr(out))
    if rc:
        raise ValueError("bad sizes")
    return out


def grouped_contiguous(A, sA, B, sB, m_indices, D16_init, want_f64=False):
    """Contiguous grouped GEMM.  D16_init ([M_total][N] uint16) is copied and
    only rows whose group index is valid and equals the index of the first
    row of their 128-row block are overwritten."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    m_indices = np.ascontiguousarray(m_indices, dtype=np.int32)
    M, K = A.shape
    G, N, _ = B.shape
    d16 = np.array(D16_init, dtype=np.uint16, copy=True, order="C")
    d64 = np.full((M, N), np.nan) if want_f64 else None
    rc = _load().dgo_grouped_contiguous(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB),
                                        _ptr(m_indices), M, N, K, G, _ptr(d64),
                                        _ptr(d16))
    if rc:
        raise ValueError("dgo_grouped_contiguous: bad sizes")
    return d64, d16


def check_contiguous_alignment(m_indices, align=BLOCK) -> int:
    m_indices = np.ascontiguousarray(m_indices, dtype=np.int32)
    return int(_load().dgo_check_contiguous_alignment(_ptr(m_indices),
                                                      m_indices.size, align))


def grouped_masked(A, sA, B, sB, masked_m, D16_init, want_f64=False):
    """Masked grouped GEMM.  A: [G][max_m][K]; rows at or beyond masked_m[g]
    keep the value they have in D16_init."""
    A, B, sA, sB = _u8(A), _u8(B), _f32(sA), _f32(sB)
    masked_m = np.ascontiguousarray(masked_m, dtype=np.int32)
    G, max_m, K = A.shape
    N = B.shape[1]
    d16 = np.array(D16_init, dtype=np.uint16, copy=True, order="C")
    d64 = np.full((G, max_m, N), np.nan) if want_f64 else None
    rc = _load().dgo_grouped_masked(_ptr(A), _ptr(sA), _ptr(B), _ptr(sB),
                                    _ptr(masked_m), G, max_m, N, K, _ptr(d64),
                                    _ptr(d16))
    if rc:
        raise ValueError("dgo_grouped_masked: bad sizes")
    return d64, d16


# ------------------------------------------------------------ UE8M0 scales

def ue8m0_value(code: int) -> float:
    """UE8M0 code -> 2**(code-127); 255 is NaN."""
    return _load().dgo_ue8m0_value(int(code))


def ue8m0_from_scale(s: float) -> int:
    """Exact code of a power-of-two scale in [2**-127, 2**127], else -1."""
    return _load().dgo_ue8m0_from_scale(float(s))


def ue8m0_ceil_pow2(x: float) -> float:
    """Smallest power of two >= x (finite x > 0): the UE8M0 scale of a block
    is ue8m0_ceil_pow2(amax / 448)."""
    return _load().dgo_ue8m0_ceil_pow2(float(x))


def pack_ue8m0(s):
    """s: [..., rows, nkb] fp32 powers of two -> [..., ceil(nkb/4), rows]
    int32, byte j of word (g, r) = code of K block 4g+j (127 past nkb)."""
    s = _f32(s)
    *lead, rows, nkb = s.shape
    ng = (nkb + 3) // 4
    flat = s.reshape(-1, rows, nkb)
    out = np.empty((flat.shape[0], ng, rows), dtype=np.int32)
    for i in range(flat.shape[0]):
        src = np.ascontiguousarray(flat[i])
        dst = np.empty((ng, rows), dtype=np.int32)
        if _load().dgo_pack_ue8m0(_ptr(src), rows, nkb, _ptr(dst)):
            raise ValueError("pack_ue8m0: a scale is not a power of two in UE8M0 range")
        out[i] = dst
    return out.reshape(*lead, ng, rows)


def unpack_ue8m0(packed, nkb: int):
    """Inverse of pack_ue8m0: [..., ceil(nkb/4), rows] -> [..., rows, nkb]."""
    packed = np.ascontiguousarray(packed, dtype=np.int32)
    *lead, ng, rows = packed.shape
    assert ng == (nkb + 3) // 4
    flat = packed.reshape(-1, ng, rows)
    out = np.empty((flat.shape[0], rows, nkb), dtype=np.float32)
    for i in range(flat.shape[0]):
        dst = np.empty((rows, nkb), dtype=np.float32)
        _load().dgo_unpack_ue8m0(_ptr(np.ascontiguousarray(flat[i])), rows, nkb, _ptr(dst))
        out[i] = dst
    return out.reshape(*lead, rows, nkb)


def gemm_nt_ue8m0(A, sfa, B, sfb, want_f64: bool = True):
    """Dense GEMM with packed UE8M0 scales: sfa [ceil(K/512)][M],
    sfb [ceil(K/512)][ceil(N/128)] (pack_ue8m0 of the logical scales)."""
    nkb = np.asarray(A).shape[-1] // BLOCK
    return gemm_nt(A, unpack_ue8m0(sfa, nkb), B, unpack_ue8m0(sfb, nkb), want_f64)


def grouped_contiguous_ue8m0(A, sfa, B, sfb, m_indices, D16_init, want_f64=False):
    """grouped_contiguous with packed UE8M0 scales: sfa [ceil(K/512)][M_total],
    sfb [G][ceil(K/512)][ceil(N/128)]."""
    nkb = np.asarray(A).shape[-1] // BLOCK
    return grouped_contiguous(A, unpack_ue8m0(sfa, nkb), B, unpack_ue8m0(sfb, nkb), m_indices,
                              D16_init, want_f64)


def grouped_masked_ue8m0(A, sfa, B, sfb, masked_m, D16_init, want_f64=False):
    """grouped_masked with packed UE8M0 scales: sfa [G][ceil(K/512)][max_m],
    sfb [G][ceil(K/512)][ceil(N/128)]."""
    nkb = np.asarray(A).shape[-1] // BLOCK
    return grouped_masked(A, unpack_ue8m0(sfa, nkb), B, unpack_ue8m0(sfb, nkb), masked_m,
                          D16_init, want_f64)
