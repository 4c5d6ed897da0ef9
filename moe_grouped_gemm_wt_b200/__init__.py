"""Python binding of the B200 fine-grained-scaled FP8 GEMM library.

Argument marshalling only: every step of the GEMM runs in the CUDA kernels of
``libdg_b200.so`` (see ``include/dg_b200.h`` for the C ABI).  The functions
keep the C names and take torch tensors that already live on the GPU; there is
no CPU path -- a CPU tensor, a missing library or a failed launch raises.

Layouts (row-major, packed):
  dense       A [M, K] e4m3, sA [K/128, M_pad] fp32, B [N, K] e4m3,
              sB [ceil(N/128), K/128] fp32, D [M, N] bf16
  contiguous  A [M_total, K], sA [K/128, M_total_pad], B [G, N, K],
              sB [G, ceil(N/128), K/128], D [M_total, N], m_indices [M_total] int32
  masked      A [G, max_m, K], sA [G, K/128, max_m_pad], B [G, N, K],
              sB [G, ceil(N/128), K/128], D [G, max_m, N], masked_m [G] int32
with X_pad = get_tma_aligned_size(X, 4) (the transposed, TMA-aligned LHS
scale layout of the DeepGEMM pages, hada.io summary, section "Giao dien GEMM
va rang buoc layout").

UE8M0 block-scaled mode (``*_ue8m0``): the same A, B, D and group metadata
with packed int32 scale words, four K blocks per word (ng = ceil(K/512)):
sfa [ng, M_pad] (masked: [G, ng, max_m_pad]) and sfb [G, ng, ceil(N/128)]
(dense: [1, ng, ceil(N/128)] or [ng, ceil(N/128)]); dg_transform_sf_ue8m0
packs them from the fp32 layouts above.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdg_b200.so")

DG_OK = 0
STATUS_NAMES = {
    0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_UNSUPPORTED", 3: "DG_ERR_ALIGNMENT",
    4: "DG_ERR_CUDA", 5: "DG_ERR_TIMEOUT", 6: "DG_ERR_BAD_GROUP_DATA",
    7: "DG_ERR_WORKSPACE_LIMIT", 8: "DG_ERR_BAD_SCALE",
}
LAYOUT_DENSE, LAYOUT_CONTIGUOUS, LAYOUT_MASKED = 0, 1, 2

# Every function the header declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGNATURES = {
    "dg_fp8_gemm_nt": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_gemm_nt_acc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_k_grouped_gemm_tn_contiguous": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "dg_fp8_gemm_nn": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_gemm_tn": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_gemm_tt": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_gemm_nt_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_grouped_gemm_contiguous": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "dg_fp8_grouped_gemm_masked": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "dg_fp8_gemm_nt_ue8m0": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_grouped_gemm_contiguous_ue8m0": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "dg_fp8_grouped_gemm_masked_ue8m0": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "dg_transform_sf_ue8m0": (_I, [_P, _P, _I, _I, _I, _I, _P]),
    "dg_get_mk_alignment_for_contiguous_layout": (_I, []),
    "dg_get_tma_aligned_size": (_I, [_I, _I]),
    "dg_set_num_sms": (_I, [_I]),
    "dg_get_num_sms": (_I, []),
    "dg_set_tile_family": (_I, [_I]),
    "dg_set_block_n": (_I, [_I]),
    "dg_set_timing_stamps": (_I, [_P]),
    "dg_get_tensor_map_encodes": (ctypes.c_ulonglong, []),
    "dg_get_device_allocations": (ctypes.c_ulonglong, []),
    "dg_set_wait_timeout_ns": (_I, [ctypes.c_uint64]),
    "dg_set_stall_injection": (_I, [_I]),
    "dg_get_device_status": (_I, [_P]),
    "dg_get_device_status_detail": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "dg_describe_config": (_I, [_I, _I, _I, _I, _I, ctypes.c_char_p, _I]),
    "dg_status_string": (ctypes.c_char_p, [_I]),
}

_lib = None


class DGError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


def load_library(path: str | None = None):
    """Loads libdg_b200.so (built by ``moe_grouped_gemm_wt_b200.build``)."""
    global _lib
    if _lib is None:
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(
                f"CUDA library {p} is missing: run `python -m moe_grouped_gemm_wt_b200.build` "
                "(there is no CPU fallback)")
        lib = ctypes.CDLL(p)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(fn: str, status: int):
    if status != DG_OK:
        raise DGError(fn, status)


def _stream_handle(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _dev(t: torch.Tensor, name: str, dtypes, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


_FP8 = (torch.float8_e4m3fn, torch.uint8)
_F32 = (torch.float32,)
_BF16 = (torch.bfloat16,)
_I32 = (torch.int32,)


def get_tma_aligned_size(x: int, elem_bytes: int = 4) -> int:
    return load_library().dg_get_tma_aligned_size(x, elem_bytes)


def get_mk_alignment_for_contiguous_layout() -> int:
    return load_library().dg_get_mk_alignment_for_contiguous_layout()


def dg_get_tma_aligned_size(x: int, elem_bytes: int) -> int:
    return get_tma_aligned_size(x, elem_bytes)


def dg_get_mk_alignment_for_contiguous_layout() -> int:
    return get_mk_alignment_for_contiguous_layout()


def dg_set_num_sms(n: int) -> None:
    _check("dg_set_num_sms", load_library().dg_set_num_sms(n))


def dg_get_num_sms() -> int:
    return load_library().dg_get_num_sms()


DG_TILES_AUTO, DG_TILES_ONE_CTA, DG_TILES_PAIR = 0, 1, 2


def dg_set_tile_family(family: int) -> None:
    """Restrict the planner to one tile family (DG_TILES_*); 0 = automatic."""
    _check("dg_set_tile_family", load_library().dg_set_tile_family(family))


def dg_set_block_n(n: int) -> None:
    """Pin the planner's tile width to a compiled BLOCK_N; 0 = automatic."""
    _check("dg_set_block_n", load_library().dg_set_block_n(n))


def dg_set_timing_stamps(stamps) -> None:
    """Record each launch's first-CTA start / last-CTA end (%globaltimer ns)
    into a CUDA int64 tensor of 2 elements (None turns it off)."""
    if stamps is None:
        _check("dg_set_timing_stamps", load_library().dg_set_timing_stamps(None))
        return
    ptr = _dev(stamps, "stamps", (torch.int64,), 1)
    if stamps.numel() != 2:
        raise ValueError("stamps must hold 2 elements")
    _check("dg_set_timing_stamps", load_library().dg_set_timing_stamps(ptr))


def dg_get_tensor_map_encodes() -> int:
    """Tensor maps encoded so far (cache misses of the library's map cache)."""
    return int(load_library().dg_get_tensor_map_encodes())


def dg_get_device_allocations() -> int:
    """Device allocations (cudaMalloc) the library has made so far."""
    return int(load_library().dg_get_device_allocations())


def dg_set_wait_timeout_ns(ns: int) -> None:
    _check("dg_set_wait_timeout_ns", load_library().dg_set_wait_timeout_ns(ns))


def dg_set_stall_injection(enable: bool) -> None:
    """Test hook: makes CTA 0 of every launch stall so its waits run out."""
    _check("dg_set_stall_injection", load_library().dg_set_stall_injection(1 if enable else 0))


def dg_get_device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status code."""
    return load_library().dg_get_device_status(_stream_handle(stream, None))


def dg_get_device_status_detail(stream=None):
    w = ctypes.c_uint32(0)
    st = load_library().dg_get_device_status_detail(_stream_handle(stream, None), ctypes.byref(w))
    return st, w.value


def dg_describe_config(layout: int, M: int, N: int, K: int, groups: int = 1) -> str:
    buf = ctypes.create_string_buffer(256)
    n = load_library().dg_describe_config(layout, M, N, K, groups, buf, 256)
    if n < 0:
        raise ValueError("bad arguments")
    return buf.value.decode()


def dg_status_string(status: int) -> str:
    return load_library().dg_status_string(status).decode()


def _dense_args(A, sA, B, sB, D):
    pa = _dev(A, "A", _FP8, 2)
    M, K = A.shape
    N = B.shape[0] if B.dim() == 2 else -1
    pb = _dev(B, "B", _FP8, 2)
    if B.shape[1] != K:
        raise ValueError("B must be [N, K]")
    psa = _dev(sA, "sA", _F32, 2)
    if tuple(sA.shape) != (K // 128, get_tma_aligned_size(M, 4)):
        raise ValueError(f"sA must be [K/128, M_pad] = {(K // 128, get_tma_aligned_size(M, 4))}")
    psb = _dev(sB, "sB", _F32, 2)
    if tuple(sB.shape) != ((N + 127) // 128, K // 128):
        raise ValueError("sB must be [ceil(N/128), K/128]")
    pd = _dev(D, "D", _BF16, 2)
    if tuple(D.shape) != (M, N):
        raise ValueError("D must be [M, N]")
    return pa, psa, pb, psb, pd, M, N, K


def dg_fp8_gemm_nt_noalloc(A, sA, B, sB, D, stream=None) -> None:
    """Dense GEMM that allocates no device memory (for callers that cannot
    call cudaMalloc while they run: code under CUDA-graph capture, code whose
    framework owns all device memory in its own pool, latency-critical
    loops).  Its K-split partials live in a fixed 32 MiB array inside the
    library; problems that need more raise DGError(DG_ERR_WORKSPACE_LIMIT).
    Calls share that array, so calls that could overlap on the GPU must be
    serialised."""
    pa, psa, pb, psb, pd, M, N, K = _dense_args(A, sA, B, sB, D)
    st = load_library().dg_fp8_gemm_nt_noalloc(pa, psa, pb, psb, pd, M, N, K,
                                               _stream_handle(stream, A.device))
    _check("dg_fp8_gemm_nt_noalloc", st)


def dg_fp8_gemm_nt(A, sA, B, sB, D, stream=None) -> None:
    pa = _dev(A, "A", _FP8, 2)
    M, K = A.shape
    N = B.shape[0] if B.dim() == 2 else -1
    pb = _dev(B, "B", _FP8, 2)
    if B.shape[1] != K:
        raise ValueError("B must be [N, K]")
    psa = _dev(sA, "sA", _F32, 2)
    if tuple(sA.shape) != (K // 128, get_tma_aligned_size(M, 4)):
        raise ValueError(f"sA must be [K/128, M_pad] = {(K // 128, get_tma_aligned_size(M, 4))}")
    psb = _dev(sB, "sB", _F32, 2)
    if tuple(sB.shape) != ((N + 127) // 128, K // 128):
        raise ValueError("sB must be [ceil(N/128), K/128]")
    pd = _dev(D, "D", _BF16, 2)
    if tuple(D.shape) != (M, N):
        raise ValueError("D must be [M, N]")
    st = load_library().dg_fp8_gemm_nt(pa, psa, pb, psb, pd, M, N, K, _stream_handle(stream, A.device))
    _check("dg_fp8_gemm_nt", st)


def _dense_layout(name, a_t, b_n, A, sA, B, sB, D, stream):
    pa = _dev(A, "A", _FP8, 2)
    pb = _dev(B, "B", _FP8, 2)
    if a_t:
        K, M = A.shape
    else:
        M, K = A.shape
    N = B.shape[1] if b_n else B.shape[0]
    if (B.shape[0] if b_n else B.shape[1]) != K:
        raise ValueError(f"{name}: B must be {'[K, N]' if b_n else '[N, K]'} with K = {K}")
    psa = _dev(sA, "sA", _F32, 2)
    if tuple(sA.shape) != (K // 128, get_tma_aligned_size(M, 4)):
        raise ValueError(f"sA must be [K/128, M_pad] = {(K // 128, get_tma_aligned_size(M, 4))}")
    psb = _dev(sB, "sB", _F32, 2)
    if tuple(sB.shape) != ((N + 127) // 128, K // 128):
        raise ValueError("sB must be [ceil(N/128), K/128]")
    pd = _dev(D, "D", _BF16, 2)
    if tuple(D.shape) != (M, N):
        raise ValueError("D must be [M, N]")
    st = getattr(load_library(), name)(pa, psa, pb, psb, pd, M, N, K, _stream_handle(stream, A.device))
    _check(name, st)


def dg_fp8_gemm_nn(A, sA, B, sB, D, stream=None) -> None:
    """D = A @ B with A [M, K] and B [K, N] (N-major)."""
    _dense_layout("dg_fp8_gemm_nn", False, True, A, sA, B, sB, D, stream)


def dg_fp8_gemm_tn(A, sA, B, sB, D, stream=None) -> None:
    """D = A^T @ B with A stored [K, M] (M-major) and B [K, N] (N-major)."""
    _dense_layout("dg_fp8_gemm_tn", True, True, A, sA, B, sB, D, stream)


def dg_fp8_gemm_tt(A, sA, B, sB, D, stream=None) -> None:
    """D = A^T @ B^T with A stored [K, M] (M-major) and B stored [N, K]."""
    _dense_layout("dg_fp8_gemm_tt", True, False, A, sA, B, sB, D, stream)


def dg_fp8_k_grouped_gemm_tn_contiguous(A, sA, B, sB, D, k_offsets, stream=None) -> None:
    """D[g] = A[K rows of g]^T @ B[K rows of g]: A [K, M], B [K, N] (MN-major),
    sA [K/128, M_pad], sB [K/128, N], D [G, M, N] float32, k_offsets [G+1]
    int32 on the device."""
    pa = _dev(A, "A", _FP8, 2)
    K, M = A.shape
    pb = _dev(B, "B", _FP8, 2)
    if B.shape[0] != K:
        raise ValueError("B must be [K, N]")
    N = B.shape[1]
    psa = _dev(sA, "sA", _F32, 2)
    if tuple(sA.shape) != (K // 128, get_tma_aligned_size(M, 4)):
        raise ValueError(f"sA must be [K/128, M_pad] = {(K // 128, get_tma_aligned_size(M, 4))}")
    psb = _dev(sB, "sB", _F32, 2)
    if tuple(sB.shape) != (K // 128, N):
        raise ValueError("sB must be [K/128, N]")
    po = _dev(k_offsets, "k_offsets", (torch.int32,), 1)
    G = k_offsets.shape[0] - 1
    pd = _dev(D, "D", _F32, 3)
    if tuple(D.shape) != (G, M, N):
        raise ValueError("D must be [G, M, N]")
    st = load_library().dg_fp8_k_grouped_gemm_tn_contiguous(pa, psa, pb, psb, pd, po, M, N, K, G,
                                                            _stream_handle(stream, A.device))
    _check("dg_fp8_k_grouped_gemm_tn_contiguous", st)


def dg_fp8_gemm_nt_acc(A, sA, B, sB, C, D, stream=None) -> None:
    """D = C + A @ B^T with float32 C and D of shape [M, N] (C may be D)."""
    pa = _dev(A, "A", _FP8, 2)
    M, K = A.shape
    N = B.shape[0] if B.dim() == 2 else -1
    pb = _dev(B, "B", _FP8, 2)
    if B.shape[1] != K:
        raise ValueError("B must be [N, K]")
    psa = _dev(sA, "sA", _F32, 2)
    if tuple(sA.shape) != (K // 128, get_tma_aligned_size(M, 4)):
        raise ValueError(f"sA must be [K/128, M_pad] = {(K // 128, get_tma_aligned_size(M, 4))}")
    psb = _dev(sB, "sB", _F32, 2)
    if tuple(sB.shape) != ((N + 127) // 128, K // 128):
        raise ValueError("sB must be [ceil(N/128), K/128]")
    pc = _dev(C, "C", _F32, 2)
    pd = _dev(D, "D", _F32, 2)
    if tuple(C.shape) != (M, N) or tuple(D.shape) != (M, N):
        raise ValueError("C and D must be [M, N]")
    st = load_library().dg_fp8_gemm_nt_acc(pa, psa, pb, psb, pc, pd, M, N, K,
                                           _stream_handle(stream, A.device))
    _check("dg_fp8_gemm_nt_acc", st)


def dg_fp8_grouped_gemm_contiguous(A, sA, B, sB, D, m_indices, stream=None) -> None:
    pa = _dev(A, "A", _FP8, 2)
    M, K = A.shape
    pb = _dev(B, "B", _FP8, 3)
    G, N, Kb = B.shape
    if Kb != K:
        raise ValueError("B must be [G, N, K]")
    psa = _dev(sA, "sA", _F32, 2)
    if tuple(sA.shape) != (K // 128, get_tma_aligned_size(M, 4)):
        raise ValueError("sA must be [K/128, M_pad]")
    psb = _dev(sB, "sB", _F32, 3)
    if tuple(sB.shape) != (G, (N + 127) // 128, K // 128):
        raise ValueError("sB must be [G, ceil(N/128), K/128]")
    pd = _dev(D, "D", _BF16, 2)
    if tuple(D.shape) != (M, N):
        raise ValueError("D must be [M_total, N]")
    pm = _dev(m_indices, "m_indices", _I32, 1)
    if m_indices.shape[0] != M:
        raise ValueError("m_indices must be [M_total]")
    st = load_library().dg_fp8_grouped_gemm_contiguous(pa, psa, pb, psb, pd, pm, M, N, K, G,
                                                       _stream_handle(stream, A.device))
    _check("dg_fp8_grouped_gemm_contiguous", st)


def dg_fp8_grouped_gemm_masked(A, sA, B, sB, D, masked_m, expected_m: int = 0, stream=None) -> None:
    pa = _dev(A, "A", _FP8, 3)
    G, max_m, K = A.shape
    pb = _dev(B, "B", _FP8, 3)
    if B.shape[0] != G or B.shape[2] != K:
        raise ValueError("B must be [G, N, K]")
    N = B.shape[1]
    psa = _dev(sA, "sA", _F32, 3)
    if tuple(sA.shape) != (G, K // 128, get_tma_aligned_size(max_m, 4)):
        raise ValueError("sA must be [G, K/128, max_m_pad]")
    psb = _dev(sB, "sB", _F32, 3)
    if tuple(sB.shape) != (G, (N + 127) // 128, K // 128):
        raise ValueError("sB must be [G, ceil(N/128), K/128]")
    pd = _dev(D, "D", _BF16, 3)
    if tuple(D.shape) != (G, max_m, N):
        raise ValueError("D must be [G, max_m, N]")
    pm = _dev(masked_m, "masked_m", _I32, 1)
    if masked_m.shape[0] != G:
        raise ValueError("masked_m must be [G]")
    st = load_library().dg_fp8_grouped_gemm_masked(pa, psa, pb, psb, pd, pm, G, max_m, N, K,
                                                   expected_m, _stream_handle(stream, A.device))
    _check("dg_fp8_grouped_gemm_masked", st)


# ------------------------------------------------------- UE8M0 block-scaled

def _ng(K: int) -> int:
    return (K // 128 + 3) // 4


def dg_transform_sf_ue8m0(sf, rows: int, mn_major: bool = True, out=None, stream=None):
    """Packs fp32 power-of-two scales into UE8M0 words (four K blocks per
    int32).  mn_major: sf [..., K/128, rows_pad] (the LHS layout, rows_pad =
    get_tma_aligned_size(rows, 4)) -> out [..., ceil(K/512), rows_pad]; else
    sf [..., rows, K/128] (the weight layout) -> out [..., ceil(K/512), rows].
    Returns out (allocated when None).  A scale that is not a power of two is
    packed as NaN and flagged DG_ERR_BAD_SCALE in the device status word."""
    if not isinstance(sf, torch.Tensor) or not sf.is_cuda or sf.dtype != torch.float32:
        raise ValueError("sf must be a float32 CUDA tensor")
    if not sf.is_contiguous() or sf.dim() < 2:
        raise ValueError("sf must be contiguous with at least 2 dims")
    batch = 1
    for d in sf.shape[:-2]:
        batch *= d
    if mn_major:
        nkb, ld = sf.shape[-2], sf.shape[-1]
        if ld != get_tma_aligned_size(rows, 4):
            raise ValueError(f"sf must be [..., K/128, {get_tma_aligned_size(rows, 4)}]")
    else:
        if sf.shape[-2] != rows:
            raise ValueError(f"sf must be [..., {rows}, K/128]")
        nkb, ld = sf.shape[-1], rows
    K = nkb * 128
    out_shape = (*sf.shape[:-2], _ng(K), ld)
    if out is None:
        out = torch.empty(out_shape, dtype=torch.int32, device=sf.device)
    po = _dev(out, "out", _I32, len(out_shape))
    if tuple(out.shape) != tuple(out_shape):
        raise ValueError(f"out must be {out_shape}")
    st = load_library().dg_transform_sf_ue8m0(sf.data_ptr(), po, rows, K, batch, 1 if mn_major else 0,
                                              _stream_handle(stream, sf.device))
    _check("dg_transform_sf_ue8m0", st)
    return out


def dg_fp8_gemm_nt_ue8m0(A, sfa, B, sfb, D, stream=None) -> None:
    """Dense NT GEMM in the UE8M0 block-scaled mode: sfa [ng, M_pad],
    sfb [ng, ceil(N/128)] (or [1, ng, ceil(N/128)]) packed int32."""
    pa = _dev(A, "A", _FP8, 2)
    M, K = A.shape
    pb = _dev(B, "B", _FP8, 2)
    if B.shape[1] != K:
        raise ValueError("B must be [N, K]")
    N = B.shape[0]
    psa = _dev(sfa, "sfa", _I32, 2)
    if tuple(sfa.shape) != (_ng(K), get_tma_aligned_size(M, 4)):
        raise ValueError(f"sfa must be [ceil(K/512), M_pad] = {(_ng(K), get_tma_aligned_size(M, 4))}")
    if isinstance(sfb, torch.Tensor) and sfb.dim() == 3 and sfb.shape[0] == 1:
        sfb = sfb[0]  # a one-group weight-scale array
    psb = _dev(sfb, "sfb", _I32, 2)
    if tuple(sfb.shape) != (_ng(K), (N + 127) // 128):
        raise ValueError("sfb must be [ceil(K/512), ceil(N/128)]")
    pd = _dev(D, "D", _BF16, 2)
    if tuple(D.shape) != (M, N):
        raise ValueError("D must be [M, N]")
    st = load_library().dg_fp8_gemm_nt_ue8m0(pa, psa, pb, psb, pd, M, N, K, _stream_handle(stream, A.device))
    _check("dg_fp8_gemm_nt_ue8m0", st)


def dg_fp8_grouped_gemm_contiguous_ue8m0(A, sfa, B, sfb, D, m_indices, stream=None) -> None:
    """Contiguous grouped GEMM in the UE8M0 mode: sfa [ng, M_total_pad],
    sfb [G, ng, ceil(N/128)]."""
    pa = _dev(A, "A", _FP8, 2)
    M, K = A.shape
    pb = _dev(B, "B", _FP8, 3)
    G, N, Kb = B.shape
    if Kb != K:
        raise ValueError("B must be [G, N, K]")
    psa = _dev(sfa, "sfa", _I32, 2)
    if tuple(sfa.shape) != (_ng(K), get_tma_aligned_size(M, 4)):
        raise ValueError("sfa must be [ceil(K/512), M_pad]")
    psb = _dev(sfb, "sfb", _I32, 3)
    if tuple(sfb.shape) != (G, _ng(K), (N + 127) // 128):
        raise ValueError("sfb must be [G, ceil(K/512), ceil(N/128)]")
    pd = _dev(D, "D", _BF16, 2)
    if tuple(D.shape) != (M, N):
        raise ValueError("D must be [M_total, N]")
    pm = _dev(m_indices, "m_indices", _I32, 1)
    if m_indices.shape[0] != M:
        raise ValueError("m_indices must be [M_total]")
    st = load_library().dg_fp8_grouped_gemm_contiguous_ue8m0(pa, psa, pb, psb, pd, pm, M, N, K, G,
                                                             _stream_handle(stream, A.device))
    _check("dg_fp8_grouped_gemm_contiguous_ue8m0", st)


def dg_fp8_grouped_gemm_masked_ue8m0(A, sfa, B, sfb, D, masked_m, expected_m: int = 0,
                                     stream=None) -> None:
    """Masked grouped GEMM in the UE8M0 mode: sfa [G, ng, max_m_pad],
    sfb [G, ng, ceil(N/128)]."""
    pa = _dev(A, "A", _FP8, 3)
    G, max_m, K = A.shape
    pb = _dev(B, "B", _FP8, 3)
    if B.shape[0] != G or B.shape[2] != K:
        raise ValueError("B must be [G, N, K]")
    N = B.shape[1]
    psa = _dev(sfa, "sfa", _I32, 3)
    if tuple(sfa.shape) != (G, _ng(K), get_tma_aligned_size(max_m, 4)):
        raise ValueError("sfa must be [G, ceil(K/512), max_m_pad]")
    psb = _dev(sfb, "sfb", _I32, 3)
    if tuple(sfb.shape) != (G, _ng(K), (N + 127) // 128):
        raise ValueError("sfb must be [G, ceil(K/512), ceil(N/128)]")
    pd = _dev(D, "D", _BF16, 3)
    if tuple(D.shape) != (G, max_m, N):
        raise ValueError("D must be [G, max_m, N]")
    pm = _dev(masked_m, "masked_m", _I32, 1)
    if masked_m.shape[0] != G:
        raise ValueError("masked_m must be [G]")
    st = load_library().dg_fp8_grouped_gemm_masked_ue8m0(pa, psa, pb, psb, pd, pm, G, max_m, N, K,
                                                         expected_m, _stream_handle(stream, A.device))
    _check("dg_fp8_grouped_gemm_masked_ue8m0", st)
