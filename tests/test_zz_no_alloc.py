"""The dense GEMM entry point that allocates no device memory.

Some callers cannot let a library allocate device memory behind their back:
frameworks that hand out all device memory from their own caching pool (an
outside cudaMalloc can fail once the pool has taken the memory, or fragment
it), and latency-critical loops in which the device-wide synchronisation that
cudaMalloc or cudaFree may cause is not acceptable.  dg_fp8_gemm_nt_noalloc
serves them by keeping its K-split partials in a fixed array inside the
library.  This file checks, through the C ABI, that its results match both
the CPU oracle and dg_fp8_gemm_nt (within the parity tolerance of the other
tests) on calls in a row -- each later call finds the previous call's
partials still in the shared array -- that its calls make no device
allocation (the library's own count of cudaMalloc calls does not move), and
that a call captured in a CUDA graph replays correctly.

It sits in a file pytest collects last, so a run that stops at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import ctypes

import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import assert_close, bits, dev_dense

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


@pytest.mark.parametrize("M,N,K", [
    (128, 2112, 7168),   # the decode benchmark shape
    (64, 1024, 2048),
    (300, 2112, 1152),   # three row blocks, 9 K blocks (split 2 ways: 5 + 4)
    (1024, 2112, 896),   # 120 tiles: the scratch bounds the split
    (2048, 2112, 1152),  # 240 tiles: only an unsplit pass (S = 1) fits the scratch
])
def test_noalloc_matches_oracle_and_default_entry_point(dg, oracle_mod, M, N, K):
    p = gi.dense_problem(M, N, K, seed_a=300 + M, seed_b=400 + N)
    _, oracle_ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    A, sA, B, sB, D_ref = dev_dense(p)
    dg.dg_fp8_gemm_nt(A, sA, B, sB, D_ref)
    assert dg.dg_get_device_status() == 0
    ref = bits(D_ref)
    assert_close(ref, oracle_ref, f"dg_fp8_gemm_nt vs oracle, {M}x{N}x{K}")

    outs = [torch.empty_like(D_ref) for _ in range(3)]
    # the library counts every cudaMalloc it makes (an allocation freed
    # again within one call is counted too); none of these calls may add one
    allocs_before = dg.dg_get_device_allocations()
    for out in outs:
        dg.dg_fp8_gemm_nt_noalloc(A, sA, B, sB, out)
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    assert dg.dg_get_device_allocations() == allocs_before, "the no-allocation entry point allocated"

    for i, out in enumerate(outs):
        got = bits(out)
        assert_close(got, oracle_ref, f"no-alloc call {i + 1} vs oracle, {M}x{N}x{K}")
        assert_close(got, ref, f"no-alloc call {i + 1} vs dg_fp8_gemm_nt, {M}x{N}x{K}")



@pytest.mark.parametrize("M,N,K", [(128, 2112, 7168), (300, 2112, 1152)])
def test_noalloc_under_cuda_graph_capture(dg, oracle_mod, M, N, K):
    """The use the entry point is made for: after one direct call on the
    device, a call captured in a CUDA graph (global capture mode, in which an
    allocation or a synchronising call would end the capture with an error)
    replays to the same bits as the direct call, and, once the captured
    input tensors are overwritten in place with another problem, to the
    oracle's result for that problem."""
    p = gi.dense_problem(M, N, K, seed_a=600 + M, seed_b=700 + N)
    A, sA, B, sB, D = dev_dense(p)
    dg.dg_fp8_gemm_nt_noalloc(A, sA, B, sB, D)  # the first call on the device
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    direct = bits(D).copy()

    allocs_before = dg.dg_get_device_allocations()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="global"):
        dg.dg_fp8_gemm_nt_noalloc(A, sA, B, sB, D)
    D.view(torch.int16).fill_(0)
    graph.replay()
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    assert np.array_equal(bits(D), direct), "the replayed call differs from the direct call"

    q = gi.dense_problem(M, N, K, seed_a=800 + M, seed_b=900 + N)
    _, oracle_ref = oracle_mod.gemm_nt(q["A"], q["sA"], q["B"], q["sB"], want_f64=False)
    for dst, src in zip((A, sA, B, sB), dev_dense(q)[:4]):
        dst.copy_(src)
    graph.replay()
    torch.cuda.synchronize()
    assert dg.dg_get_device_status() == 0
    assert dg.dg_get_device_allocations() == allocs_before, "capture or replay allocated"
    assert_close(bits(D), oracle_ref, f"replayed no-alloc call vs oracle, {M}x{N}x{K}")
    del graph

def test_noalloc_rejects_problems_beyond_its_scratch(dg):
    # 4096 x 7168 needs 32 x 50 tiles x 73,728 bytes = 118 MB of partials even
    # unsplit: more than the fixed 32 MiB, so nothing is launched.
    lib = dg.load_library()
    M, N, K = 4096, 7168, 256
    dev = torch.device("cuda")
    A = torch.zeros((M, K), dtype=torch.uint8, device=dev)
    B = torch.zeros((N, K), dtype=torch.uint8, device=dev)
    sA = torch.zeros((K // 128, M), dtype=torch.float32, device=dev)
    sB = torch.zeros(((N + 127) // 128, K // 128), dtype=torch.float32, device=dev)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    st = lib.dg_fp8_gemm_nt_noalloc(A.data_ptr(), sA.data_ptr(), B.data_ptr(), sB.data_ptr(),
                                    D.data_ptr(), M, N, K, None)
    assert st == 7 and lib.dg_status_string(st) == b"DG_ERR_WORKSPACE_LIMIT"
    with pytest.raises(dg.DGError):
        dg.dg_fp8_gemm_nt_noalloc(A, sA, B, sB, D)
    assert dg.dg_get_device_status() == 0
