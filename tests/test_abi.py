"""CPU-side checks of the C-ABI library: it loads, exports every function the
header declares, and its host logic (validation, alignment helpers, status
names, tile choice) behaves as documented -- no GPU compute is called."""
import ctypes
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from moe_grouped_gemm_wt_b200 import build as b
    b.build()
    import moe_grouped_gemm_wt_b200 as dg
    return dg.load_library()


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert "dg_fp8_gemm_nt" in names and len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_binding_covers_header():
    import moe_grouped_gemm_wt_b200 as dg
    for n in _declared_functions():
        assert n in dg._SIGNATURES, n
        assert callable(getattr(dg, n)), n


def test_host_helpers(lib):
    assert lib.dg_get_mk_alignment_for_contiguous_layout() == 128
    assert lib.dg_get_tma_aligned_size(1, 4) == 4
    assert lib.dg_get_tma_aligned_size(130, 4) == 132
    assert lib.dg_get_tma_aligned_size(17, 1) == 32
    assert lib.dg_get_tma_aligned_size(5, 3) == -1
    assert lib.dg_get_tma_aligned_size(-1, 4) == -1
    assert lib.dg_status_string(0) == b"DG_OK"
    assert lib.dg_status_string(5) == b"DG_ERR_TIMEOUT"
    assert lib.dg_set_num_sms(-1) == 1
    assert lib.dg_set_wait_timeout_ns(0) == 0


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first


@pytest.mark.parametrize("M,N,K,expect", [
    (128, 256, 500, 2),    # K not a multiple of 128
    (128, 250, 512, 2),    # N not a multiple of 16
    (-1, 256, 512, 1),
    (128, 0, 512, 1),
])
def test_dense_validation(lib, M, N, K, expect):
    st = lib.dg_fp8_gemm_nt(FAKE, FAKE, FAKE, FAKE, FAKE, M, N, K, None)
    assert st == expect


def test_null_and_alignment(lib):
    assert lib.dg_fp8_gemm_nt(None, FAKE, FAKE, FAKE, FAKE, 128, 256, 512, None) == 1
    odd = ctypes.c_void_p(0x10008)
    assert lib.dg_fp8_gemm_nt(odd, FAKE, FAKE, FAKE, FAKE, 128, 256, 512, None) == 3
    # contiguous: M_total must be a multiple of the 128-row alignment
    assert lib.dg_fp8_grouped_gemm_contiguous(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 200, 256, 512, 2, None) == 2
    assert lib.dg_fp8_grouped_gemm_contiguous(FAKE, FAKE, FAKE, FAKE, FAKE, None, 256, 256, 512, 2, None) == 1
    # masked: bad counts
    assert lib.dg_fp8_grouped_gemm_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 256, 512, 0, None) == 1
    assert lib.dg_fp8_grouped_gemm_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, -1, 256, 512, 0, None) == 1
    # empty problems are no-ops
    assert lib.dg_fp8_gemm_nt(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 512, None) == 0
    # other layouts: an M-major A needs M % 16 == 0; the usual shape rules
    assert lib.dg_fp8_gemm_tn(FAKE, FAKE, FAKE, FAKE, FAKE, 200, 256, 512, None) == 2
    assert lib.dg_fp8_gemm_tt(FAKE, FAKE, FAKE, FAKE, FAKE, 200, 256, 512, None) == 2
    assert lib.dg_fp8_gemm_nn(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 250, 512, None) == 2
    assert lib.dg_fp8_gemm_nn(None, FAKE, FAKE, FAKE, FAKE, 128, 256, 512, None) == 1
    # K-grouped TN: sizes, alignment, group count
    kg = lib.dg_fp8_k_grouped_gemm_tn_contiguous
    assert kg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 512, 0, None) == 1
    assert kg(FAKE, FAKE, FAKE, FAKE, FAKE, None, 128, 256, 512, 2, None) == 1
    assert kg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 120, 256, 512, 2, None) == 2
    assert kg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 500, 2, None) == 2
    assert kg(FAKE, FAKE, FAKE, odd, FAKE, FAKE, 128, 256, 512, 2, None) == 3
    assert kg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 512, 2, None) == 0
    # accumulate form: C is required and 16-byte aligned; same shape rules
    assert lib.dg_fp8_gemm_nt_acc(FAKE, FAKE, FAKE, FAKE, None, FAKE, 128, 256, 512, None) == 1
    assert lib.dg_fp8_gemm_nt_acc(FAKE, FAKE, FAKE, FAKE, odd, FAKE, 128, 256, 512, None) == 3
    assert lib.dg_fp8_gemm_nt_acc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 250, 512, None) == 2
    assert lib.dg_fp8_gemm_nt_acc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 512, None) == 0


def test_ue8m0_validation(lib):
    odd = ctypes.c_void_p(0x10008)
    odd4 = ctypes.c_void_p(0x10004)
    nt = lib.dg_fp8_gemm_nt_ue8m0
    assert nt(None, FAKE, FAKE, FAKE, FAKE, 128, 256, 512, None) == 1
    assert nt(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 250, 512, None) == 2
    assert nt(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 500, None) == 2
    assert nt(FAKE, odd4, FAKE, FAKE, FAKE, 128, 256, 512, None) == 3  # sfa: 16-byte aligned
    assert nt(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 512, None) == 0
    assert nt(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 256, 512, None) == 1
    cg = lib.dg_fp8_grouped_gemm_contiguous_ue8m0
    assert cg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 200, 256, 512, 2, None) == 2
    assert cg(FAKE, FAKE, FAKE, FAKE, FAKE, None, 256, 256, 512, 2, None) == 1
    assert cg(FAKE, FAKE, odd, FAKE, FAKE, FAKE, 256, 256, 512, 2, None) == 3
    assert cg(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 512, 2, None) == 0
    mk = lib.dg_fp8_grouped_gemm_masked_ue8m0
    assert mk(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 256, 256, 512, 0, None) == 1
    assert mk(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, -1, 256, 512, 0, None) == 1
    assert mk(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 256, 256, 512, -1, None) == 1
    assert mk(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0, 256, 512, 0, None) == 0
    tr = lib.dg_transform_sf_ue8m0
    assert tr(None, FAKE, 128, 512, 1, 1, None) == 1
    assert tr(FAKE, FAKE, 128, 500, 1, 1, None) == 2
    assert tr(FAKE, FAKE, 128, 512, 0, 1, None) == 1
    assert tr(FAKE, FAKE, 128, 512, 1, 2, None) == 1
    assert tr(FAKE, FAKE, 0, 512, 1, 0, None) == 0
    assert lib.dg_status_string(8) == b"DG_ERR_BAD_SCALE"


def test_ue8m0_describe_config(lib):
    buf = ctypes.create_string_buffer(256)
    for layout in (3, 4, 5):
        assert lib.dg_describe_config(layout, 4096, 7168, 7168, 4, buf, 256) > 0
        desc = dict(kv.split("=") for kv in buf.value.decode().split())
        assert desc["ue8m0"] == "1" and desc["ksplit"] == "1"
        assert int(desc["BN"]) in (128, 160, 192, 224)
    # prefill shape: 16 pair rows x 32 column tiles of 224 fill 74 SM pairs
    # in 7 waves (98.8% of the last wave used)
    lib.dg_describe_config(3, 4096, 7168, 18432, 1, buf, 256)
    desc = dict(kv.split("=") for kv in buf.value.decode().split())
    assert (desc["BN"], desc["BM"], desc["pair"]) == ("224", "256", "1")
    # decode shape: too few pair tiles to fill the pairs, one-CTA tiles
    lib.dg_describe_config(3, 128, 2112, 7168, 1, buf, 256)
    assert dict(kv.split("=") for kv in buf.value.decode().split())["pair"] == "0"
    assert lib.dg_describe_config(7, 128, 256, 512, 1, buf, 256) == -1


def test_ue8m0_planner_under_an_sm_cap(lib):
    """The UE8M0 planner (host only): with 16 SMs, 16 one-CTA 128x224 tiles or
    8 pair tiles of 256x224 fill the GPU in one wave, and the pair family
    (half the B traffic per SM) wins; the masked layout takes the one-CTA
    128-column tile; a forced family is honoured."""
    buf = ctypes.create_string_buffer(256)
    desc = lambda *a: (lib.dg_describe_config(*a, buf, 256), dict(kv.split("=") for kv in buf.value.decode().split()))[1]
    assert lib.dg_set_num_sms(16) == 0
    try:
        d = desc(3, 2048, 224, 512, 1)
        assert (d["BN"], d["pair"], d["BM"]) == ("224", "1", "256"), d
        d = desc(5, 100, 4096, 7168, 16)
        assert (d["BN"], d["pair"], d["stages"]) == ("128", "0", "3"), d
        assert lib.dg_set_tile_family(1) == 0  # one-CTA tiles only
        d = desc(3, 2048, 224, 512, 1)
        assert (d["BN"], d["pair"]) == ("224", "0"), d
    finally:
        lib.dg_set_tile_family(0)
        lib.dg_set_num_sms(0)


def test_masked_decode_tile_choice(lib):
    """The fp32-scale masked planner (host only): decode-sized groups (max_m
    at most two 128-row blocks) take the 128-column tile of three two-K-block
    stages; larger groups go through the general cost model; a pinned tile
    width is honoured."""
    buf = ctypes.create_string_buffer(256)
    desc = lambda *a: (lib.dg_describe_config(*a, buf, 256), dict(kv.split("=") for kv in buf.value.decode().split()))[1]
    assert lib.dg_set_num_sms(148) == 0
    try:
        for max_m in (1, 128, 200, 256):
            d = desc(2, max_m, 4096, 7168, 16)
            assert (d["BN"], d["stages"], d["ks"], d["pair"]) == ("128", "3", "2", "0"), (max_m, d)
        d = desc(2, 1024, 4096, 7168, 16)
        assert (d["stages"], d["ks"]) != ("3", "2") or d["BN"] != "128", d
        assert lib.dg_set_block_n(256) == 0
        d = desc(2, 256, 4096, 7168, 16)
        assert d["BN"] == "256", d
    finally:
        lib.dg_set_block_n(0)
        lib.dg_set_num_sms(0)


def test_two_depths_of_the_256_column_tile(lib):
    """The fp32-scale planner (host only) with the tile width pinned to 256
    and one-CTA tiles: a short K range (16 K blocks, the contiguous MoE
    shape) takes three stages with staged TMA stores, a long one (56 or 144
    K blocks) four stages with per-warp stores."""
    buf = ctypes.create_string_buffer(256)
    desc = lambda *a: (lib.dg_describe_config(*a, buf, 256), dict(kv.split("=") for kv in buf.value.decode().split()))[1]
    assert lib.dg_set_num_sms(148) == 0
    try:
        assert lib.dg_set_block_n(256) == 0
        assert lib.dg_set_tile_family(1) == 0
        d = desc(1, 32768, 7168, 2048, 8)
        assert (d["BN"], d["stages"], d["ks"], d["pair"]) == ("256", "3", "1", "0"), d
        for K in (7168, 18432):
            d = desc(0, 4096, 7168, K, 1)
            assert (d["BN"], d["stages"], d["ks"], d["pair"]) == ("256", "4", "1", "0"), (K, d)
    finally:
        lib.dg_set_block_n(0)
        lib.dg_set_tile_family(0)
        lib.dg_set_num_sms(0)


def test_noalloc_split_choice_under_an_sm_cap(lib):
    """The split count of dg_fp8_gemm_nt_noalloc (host only, dg_describe_config
    layout 6): every split gets the same number (at least two) of K blocks,
    a cluster never has more CTAs than the SM cap allows, and the partials
    fit the fixed 32 MiB scratch (ksplit=0: the problem is refused)."""
    buf = ctypes.create_string_buffer(256)

    def split(M, N, K):
        assert lib.dg_describe_config(6, M, N, K, 1, buf, 256) > 0
        d = dict(kv.split("=") for kv in buf.value.decode().split())
        assert d["noalloc"] == "1" and d["BN"] == "144"
        return int(d["ksplit"])

    def even(S, K):
        nkb = K // 128
        kbps = -(-nkb // S)
        return S == 1 or (kbps >= 2 and -(-nkb // kbps) == S)

    try:
        for cap in (0, 7, 3, 2):
            assert lib.dg_set_num_sms(cap) == 0
            for M, N, K in [(128, 2112, 7168), (300, 2112, 1152), (2048, 2112, 256), (64, 1024, 2048),
                            (1024, 2112, 7168), (128, 256, 1152)]:
                S = split(M, N, K)
                tiles = -(-M // 128) * -(-N // 144)
                assert S >= 1 and even(S, K), (cap, M, N, K, S)
                assert cap == 0 or S <= cap, (cap, S)
                assert tiles * S * 144 * 128 * 4 <= 32 << 20
        # 9 K blocks never split 4 ways (3 + 3 + 3 + 0 would leave a split empty)
        assert lib.dg_set_num_sms(0) == 0
        assert split(4096, 2112, 1152) == 0          # 480 tiles: too large even unsplit
        assert split(1024, 2112, 1152) == 2
        assert split(128, 2112, 7168) == 8            # the dense planner's own split
        assert lib.dg_set_num_sms(7) == 0
        assert split(128, 2112, 7168) == 4
    finally:
        lib.dg_set_num_sms(0)


def test_sm_fill_example_from_pages(lib):
    """The unaligned-block-size example of the DeepGEMM article (lqnn.cn,
    section 非对齐块大小): M=256, N=7168 on 132 SMs -- 128x128 tiles occupy
    112 SMs, 128x112 tiles occupy 128, so BLOCK_N=112 is the better choice."""
    ex = json.load(open(os.path.join(ROOT, "tests", "golden", "sm_fill_example.json")))
    assert lib.dg_set_num_sms(ex["num_sms"]) == 0
    try:
        buf = ctypes.create_string_buffer(256)
        lib.dg_describe_config(0, ex["M"], ex["N"], 7168, 1, buf, 256)
        desc = dict(kv.split("=") for kv in buf.value.decode().split())
        assert int(desc["BN"]) == ex["chosen_block_n"]
        m_blocks = ex["M"] // 128
        for bn, used in ex["sms_used_by_block_n"].items():
            tiles = m_blocks * ((ex["N"] + int(bn) - 1) // int(bn))
            assert min(tiles, ex["num_sms"]) == used
    finally:
        lib.dg_set_num_sms(0)
