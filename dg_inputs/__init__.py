"""Seeded synthetic inputs for the fine-grained-scaled FP8 GEMM.

This module is shared by the tests, the smoke check and the benchmark, and by
both sides of every parity check (the CPU oracle and the CUDA library).  It
holds the input recipe only -- random numbers, block amax scales and the cast
to e4m3 -- and none of the GEMM's arithmetic.

Recipe (the workloads the DeepGEMM pages benchmark are DeepSeek-V3/R1 layer
shapes; no dataset or weights are used, these synthetic tensors stand in):
  * x ~ N(0, 1) in float32 from numpy's PCG64 seeded per tensor
    (A: seed 1, B: seed 2, masked_m: seed 3 unless a test says otherwise);
  * one scale per 1x128 block of A's rows and per 128x128 block of B,
    scale = max(amax, 1e-4) / 448 in float32 (a partial last block of B's
    rows counts only its real rows);
  * codes = e4m3fn(clamp(x / scale, -448, 448)), cast by torch on the CPU
    (round to nearest even; the clamp makes the cast saturating);
  * UE8M0 inputs (``ue8m0=True``, the SM100 block-scaled mode: hada.io
    DeepGEMM summary, "Giao dien GEMM va rang buoc layout") take instead the
    smallest power of two scale >= max(amax, 1e-4) / 448, decided in float64,
    and quantise the data with it.
Fine-grained 1x128 / 128x128 scaling: "deepseek开源周第三天：DeepGEMM深度分析"
(pxiaoer.blog), FP8-training list.

Layouts returned here are the LOGICAL ones: sA [rows][K/128] and
sB [ceil(N/128)][K/128] (per group, groups outermost).  The CUDA library's
argument layout for sA is transposed (see ``sa_to_kernel_layout``).
"""
from __future__ import annotations

import numpy as np
import torch

BLOCK = 128
E4M3_MAX = 448.0
AMAX_FLOOR = 1e-4

SEED_A = 1
SEED_B = 2
SEED_MASK = 3


def standard_normal(seed: int, shape) -> np.ndarray:
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(
        shape, dtype=np.float32)


def _cast_e4m3(y: np.ndarray) -> np.ndarray:
    y = np.clip(y, -E4M3_MAX, E4M3_MAX)
    return torch.from_numpy(np.ascontiguousarray(y)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def _block_scale(amax: np.ndarray, ue8m0: bool) -> np.ndarray:
    """Scale of each block from its amax: amax/448 in float32, or with
    ue8m0 the smallest power of two >= amax/448 (in float64: x = f * 2**e
    with 0.5 <= f < 1 is itself a power of two iff f == 0.5)."""
    if not ue8m0:
        return (np.maximum(amax, np.float32(AMAX_FLOOR)) / np.float32(E4M3_MAX)).astype(np.float32)
    ratio = np.maximum(amax.astype(np.float64), AMAX_FLOOR) / E4M3_MAX
    frac, expo = np.frexp(ratio)
    return np.where(frac == 0.5, ratio, np.ldexp(1.0, expo)).astype(np.float32)


def quantize_1x128(x: np.ndarray, ue8m0: bool = False):
    """x: [..., K] float32 -> (codes uint8 [..., K], scales float32 [..., K/128])."""
    *lead, K = x.shape
    assert K % BLOCK == 0
    xb = x.reshape(*lead, K // BLOCK, BLOCK)
    amax = np.abs(xb).max(axis=-1)
    scale = _block_scale(amax, ue8m0)
    y = xb / scale[..., None]
    return _cast_e4m3(y).reshape(x.shape), scale


def quantize_128x128(x: np.ndarray, ue8m0: bool = False):
    """x: [N, K] float32 -> (codes uint8 [N, K], scales float32 [ceil(N/128), K/128])."""
    N, K = x.shape
    assert K % BLOCK == 0
    nbn = (N + BLOCK - 1) // BLOCK
    codes = np.empty((N, K), dtype=np.uint8)
    scales = np.empty((nbn, K // BLOCK), dtype=np.float32)
    for nb in range(nbn):
        rows = x[nb * BLOCK:(nb + 1) * BLOCK]
        r = rows.shape[0]
        xb = rows.reshape(r, K // BLOCK, BLOCK)
        amax = np.abs(xb).max(axis=(0, 2))
        s = _block_scale(amax, ue8m0)
        scales[nb] = s
        codes[nb * BLOCK:(nb + 1) * BLOCK] = _cast_e4m3(xb / s[None, :, None]).reshape(r, K)
    return codes, scales


def quantize_128x1(x: np.ndarray):
    """x: [K, C] float32 -> (codes uint8 [K, C], scales float32 [K/128, C]):
    one scale per 128 rows of K and per column (the granularity of the
    operands of the K-grouped weight-gradient GEMM, whose contraction runs
    along K)."""
    K, C = x.shape
    assert K % BLOCK == 0
    xb = x.reshape(K // BLOCK, BLOCK, C)
    amax = np.abs(xb).max(axis=1)
    scale = (np.maximum(amax, np.float32(AMAX_FLOOR)) / np.float32(E4M3_MAX)).astype(np.float32)
    return _cast_e4m3(xb / scale[:, None, :]).reshape(K, C), scale


def tma_aligned_size(x: int, elem_bytes: int = 4) -> int:
    """Round x up so that x * elem_bytes is a multiple of 16 bytes."""
    per = 16 // elem_bytes
    return (x + per - 1) // per * per


def sa_to_kernel_layout(sa_logical: np.ndarray) -> np.ndarray:
    """[..., rows, K/128] -> [..., K/128, rows_pad] (transposed, rows padded
    to a 16-byte multiple with zeros): the LHS-scale layout the library takes
    (hada.io DeepGEMM summary, "Giao dien GEMM va rang buoc layout": the LHS
    scale must be TMA-aligned and transposed)."""
    *lead, rows, nkb = sa_logical.shape
    rp = tma_aligned_size(rows, 4)
    out = np.zeros((*lead, nkb, rp), dtype=np.float32)
    out[..., :rows] = np.swapaxes(sa_logical, -1, -2)
    return out


# ----------------------------------------------------------- problem recipes

def dense_problem(M: int, N: int, K: int, seed_a: int = SEED_A, seed_b: int = SEED_B,
                  ue8m0: bool = False):
    a, sa = quantize_1x128(standard_normal(seed_a, (M, K)), ue8m0)
    b, sb = quantize_128x128(standard_normal(seed_b, (N, K)), ue8m0)
    return dict(kind="dense", A=a, sA=sa, B=b, sB=sb, M=M, N=N, K=K)


def grouped_weights(G: int, N: int, K: int, seed_b: int = SEED_B, ue8m0: bool = False):
    gen = np.random.Generator(np.random.PCG64(seed_b))
    nbn = (N + BLOCK - 1) // BLOCK
    B = np.empty((G, N, K), dtype=np.uint8)
    sB = np.empty((G, nbn, K // BLOCK), dtype=np.float32)
    for g in range(G):
        B[g], sB[g] = quantize_128x128(gen.standard_normal((N, K), dtype=np.float32), ue8m0)
    return B, sB


def k_grouped_problem(ks, M: int, N: int, seed_a: int = SEED_A, seed_b: int = SEED_B):
    """K-grouped layout (MoE weight gradient): group g owns ks[g] rows (a
    multiple of 128, possibly 0) of the shared K axis.  A [K][M] and B [K][N]
    are stored MN-major and scaled per 128 rows of K and per column."""
    assert all(k % BLOCK == 0 and k >= 0 for k in ks)
    K = int(sum(ks))
    k_offsets = np.concatenate([[0], np.cumsum(ks)]).astype(np.int32)
    a, sa = quantize_128x1(standard_normal(seed_a, (K, M)))
    b, sb = quantize_128x1(standard_normal(seed_b, (K, N)))
    return dict(kind="k_grouped", A=a, sA=sa, B=b, sB=sb, k_offsets=k_offsets,
                M=M, N=N, K=K, G=len(ks))


def contiguous_problem(rows_per_group, N: int, K: int, seed_a: int = SEED_A,
                       seed_b: int = SEED_B, pad_to: int = BLOCK, ue8m0: bool = False):
    """Contiguous grouped layout.  Group g's segment has rows_per_group[g]
    real rows, padded up to a multiple of ``pad_to`` with rows tagged -1."""
    G = len(rows_per_group)
    idx = []
    for g, r in enumerate(rows_per_group):
        padded = (r + pad_to - 1) // pad_to * pad_to
        idx += [g] * r + [-1] * (padded - r)
    m_indices = np.asarray(idx, dtype=np.int32)
    M = m_indices.size
    a, sa = quantize_1x128(standard_normal(seed_a, (M, K)), ue8m0)
    B, sB = grouped_weights(G, N, K, seed_b, ue8m0)
    return dict(kind="contiguous", A=a, sA=sa, B=B, sB=sB, m_indices=m_indices,
                M=M, N=N, K=K, G=G)


def masked_counts(G: int, max_m: int, seed: int = SEED_MASK, low: int = 1):
    return np.random.Generator(np.random.PCG64(seed)).integers(
        low, max_m + 1, size=G).astype(np.int32)


def masked_problem(G: int, max_m: int, N: int, K: int, masked_m=None,
                   seed_a: int = SEED_A, seed_b: int = SEED_B, seed_mask: int = SEED_MASK,
                   ue8m0: bool = False):
    if masked_m is None:
        masked_m = masked_counts(G, max_m, seed_mask)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    a, sa = quantize_1x128(standard_normal(seed_a, (G, max_m, K)), ue8m0)
    B, sB = grouped_weights(G, N, K, seed_b, ue8m0)
    return dict(kind="masked", A=a, sA=sa, B=B, sB=sB, masked_m=masked_m,
                G=G, max_m=max_m, N=N, K=K)


# The five benchmark workloads (DeepSeek-V3/R1-shaped, see module docstring).
WORKLOADS = {
    "dense_tiny": dict(kind="dense", M=128, N=256, K=512),
    "dense_decode": dict(kind="dense", M=128, N=2112, K=7168),
    "dense_prefill": dict(kind="dense", M=4096, N=7168, K=18432),
    "contiguous_moe": dict(kind="contiguous", G=8, rows=4096, N=7168, K=2048),
    "masked_moe_decode": dict(kind="masked", G=16, max_m=256, N=4096, K=7168),
}


def make_workload(name: str, ue8m0: bool = False):
    w = WORKLOADS[name]
    if w["kind"] == "dense":
        return dense_problem(w["M"], w["N"], w["K"], ue8m0=ue8m0)
    if w["kind"] == "contiguous":
        return contiguous_problem([w["rows"]] * w["G"], w["N"], w["K"], ue8m0=ue8m0)
    return masked_problem(w["G"], w["max_m"], w["N"], w["K"], ue8m0=ue8m0)
