"""GPU parity of the NN, TN and TT operand layouts of the dense GEMM.  The
inputs come from the NT generator; the GPU gets A transposed ([K][M],
M-major) for the t layouts of A and B transposed ([K][N], N-major) for the n
layouts of B, and the oracle gets the NT form of the same values.  Shapes
cover one tile, ragged M and N (partial and wholly out-of-range 128-column
boxes of an N-major B), several tiles, an odd number of K blocks, and the
decode shape (a K split for an M-major A)."""
import numpy as np
import pytest
import torch

import dg_inputs as gi
from parity import assert_close, bits

pytestmark = pytest.mark.gpu

LAYOUTS = {"nn": (False, True), "tn": (True, True), "tt": (True, False)}


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


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("M,N,K", [
    (128, 256, 512),
    (208, 272, 384),      # ragged M and N
    (512, 1040, 896),     # several tiles, 7 K blocks
    (128, 2112, 7168),    # decode shape
])
def test_layout_matches_oracle(dg, oracle_mod, layout, M, N, K):
    a_t, b_n = LAYOUTS[layout]
    p = gi.dense_problem(M, N, K, seed_a=7000 + M, seed_b=8000 + N)
    dev = torch.device("cuda")
    A = torch.from_numpy(np.ascontiguousarray(p["A"].T if a_t else p["A"])).to(dev)
    B = torch.from_numpy(np.ascontiguousarray(p["B"].T if b_n else p["B"])).to(dev)
    sA = torch.from_numpy(gi.sa_to_kernel_layout(p["sA"])).to(dev)
    sB = torch.from_numpy(p["sB"]).to(dev)
    D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
    getattr(dg, f"dg_fp8_gemm_{layout}")(A, sA, B, sB, D)
    assert dg.dg_get_device_status() == 0
    _, ref = oracle_mod.gemm_nt(p["A"], p["sA"], p["B"], p["sB"], want_f64=False)
    assert_close(bits(D), ref, f"{layout} {M}x{N}x{K}")


def test_layouts_agree_bit_for_bit_on_integer_inputs(dg, oracle_mod):
    rng = np.random.default_rng(23)
    M, N, K = 256, 512, 1024
    ai = rng.integers(-4, 5, (M, K)).astype(np.float32)
    bi = rng.integers(-4, 5, (N, K)).astype(np.float32)
    to8 = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn).view(torch.uint8)
    dev = torch.device("cuda")
    sA = torch.ones((K // 128, M), device=dev)
    sB = torch.ones((N // 128, K // 128), device=dev)
    _, ref = oracle_mod.gemm_nt(to8(ai).numpy(), np.ones((M, K // 128), np.float32), to8(bi).numpy(),
                                np.ones((N // 128, K // 128), np.float32), want_f64=False)
    for layout, (a_t, b_n) in LAYOUTS.items():
        A = to8(ai.T if a_t else ai).to(dev)
        B = to8(bi.T if b_n else bi).to(dev)
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        getattr(dg, f"dg_fp8_gemm_{layout}")(A, sA, B, sB, D)
        assert dg.dg_get_device_status() == 0
        assert np.array_equal(bits(D), ref), layout
