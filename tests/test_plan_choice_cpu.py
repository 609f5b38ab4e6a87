"""The kernel choice (family, tile width, K split, split tail, grid) on the host, without a GPU,
through gemm_epi_plan_preview: the rules a plan follows for the workloads the library is measured
on and at the boundaries between the rules.  The GPU suite checks that a real plan makes the same
choice (test_gpu_parity.py::test_preview_matches_plans)."""
import pytest

SMS = 148   # a B200


@pytest.fixture(scope="module")
def g():
    from activation_epilogue_tcgen05_b200 import build, gemm_epi
    build.build()
    return gemm_epi


def pv(g, m, n, k, dtype="bf16", epilogue="bias", axis="row", layout="kn", sms=SMS, **kw):
    return g.plan_preview(m, n, k, dtype, epilogue, axis, layout, num_sms=sms, **kw)


# ------------------------------------------------------------------ the measured workloads
def test_headline_relu_aux_bias_4096(g):
    p = pv(g, 4096, 4096, 4096, "bf16", "relu_aux_bias")
    # 256 tiles of 256 x 256 on 74 pairs: 3 whole waves, the 34 tiles of the last one in two parts
    assert (p["kernel"], p["block_m"], p["block_n"], p["cluster"]) == (g.KERNEL_TC2, 256, 256, 2)
    assert (p["tiles"], p["grid"], p["sk_tiles"], p["sk_split"]) == (256, 148, 34, 2)
    # ring stages of two 128-byte k-atoms (64 KB per CTA): three of them
    assert p["threads"] == 320 and (p["stages"], p["block_k"]) == (3, 128)


def test_small_gemm_bias_1024x512x2048(g):
    p = pv(g, 1024, 512, 2048, "f16", "bias")
    # 32 tiles of 128 x 128, fewer than the SMs: every tile in four k-parts on 128 CTAs
    assert (p["kernel"], p["block_n"], p["tiles"]) == (g.KERNEL_TC1, 128, 32)
    assert (p["sk_tiles"], p["sk_split"], p["grid"]) == (32, 4, 128)


def test_linear_gelu_batch16_splitk(g):
    p = pv(g, 16, 4096, 4096, "f16", "gelu_bias", "col", "nk")
    # swapped roles: 32 weight tiles of 128 rows, K split over clusters of 4 CTAs
    assert (p["kernel"], p["block_m"], p["split_k"], p["cluster"], p["grid"]) == (g.KERNEL_SPLITK, 16, 4, 4, 128)


def test_linear_gelu_batch16_splitk_grid_form(g, monkeypatch):
    monkeypatch.setenv("GEMM_EPI_SK_GRID", "1")
    p = pv(g, 16, 4096, 4096, "f16", "gelu_bias", "col", "nk")
    # every SM takes an equal range of the 2048 (tile, k-block) units (13 or 14), so a tile is
    # cut into 5 or 6 pieces
    assert (p["kernel"], p["block_m"], p["cluster"], p["grid"]) == (g.KERNEL_SPLITK, 16, 1, 148)
    assert p["split_k"] == 5 and p["stages"] == 11


def test_splitk_grid_follows_split_k_and_max_ctas(g, monkeypatch):
    monkeypatch.setenv("GEMM_EPI_SK_GRID", "1")
    # split_k caps the k-parts per tile: the grid is tiles x split_k
    p = pv(g, 16, 4096, 4096, "f16", "gelu_bias", "col", "nk", split_k=2)
    assert (p["grid"], p["split_k"]) == (64, 2)
    # one part per tile: whole tiles, no reduction
    assert pv(g, 16, 4096, 4096, "f16", "gelu_bias", "col", "nk", split_k=1)["grid"] == 32
    # fewer units than SMs: one CTA per (tile, k-block) unit
    q = pv(g, 8, 256, 256, "bf16", "bias", "col", "kn")
    assert q["kernel"] == g.KERNEL_SPLITK and q["grid"] == 2 * 4
    assert pv(g, 16, 4096, 4096, "f16", "bias", "col", "nk", max_ctas=100)["grid"] == 100


def test_large_relu_bias_wide_tiles(g):
    p = pv(g, 65536, 8192, 16384, "bf16", "relu_bias")
    assert (p["kernel"], p["block_n"], p["tiles"], p["grid"]) == (g.KERNEL_TC2, 512, 4096, 148)
    assert p["sk_tiles"] == 0       # 4096 tiles on 74 pairs: under 2 % lost to the last wave


def test_fp8_gelu_bias(g):
    p = pv(g, 8192, 14336, 4096, "e4m3", "gelu_bias", "col", "kn")
    assert (p["kernel"], p["block_n"], p["block_k"], p["tiles"]) == (g.KERNEL_TC2, 256, 256, 1792)
    assert (p["sk_tiles"], p["sk_split"]) == (16, 2)


# ------------------------------------------------------------------ family boundaries
@pytest.mark.parametrize("m,kernel", [(1, "splitk"), (16, "splitk"), (32, "splitk"), (33, "splitk"),
                                      (64, "splitk"), (65, "tc1"), (128, "tc1"), (256, "tc1")])
def test_batch_boundary(g, m, kernel):
    p = pv(g, m, 4096, 4096, "f16", "gelu_bias", "col", "nk")
    assert p["kernel"] == {"splitk": g.KERNEL_SPLITK, "tc1": g.KERNEL_TC1}[kernel]


@pytest.mark.parametrize("m,nm", [(1, 16), (16, 16), (17, 32), (32, 32), (33, 64), (64, 64)])
def test_splitk_batch_tile(g, m, nm):
    assert pv(g, m, 4096, 4096, "f16", "gelu_bias", "col", "nk")["block_m"] == nm


def test_pairs_need_a_tile_per_pair(g):
    # 256 x 256 tiles: 73 of them leave a pair idle (single CTAs), 74 fill every pair
    assert pv(g, 256 * 73, 256, 1024)["kernel"] == g.KERNEL_TC1
    assert pv(g, 256 * 74, 256, 1024)["kernel"] == g.KERNEL_TC2


def test_backward_and_transposed_a_never_take_splitk(g):
    assert pv(g, 16, 4096, 4096, "bf16", "drelu", "row", "kn")["kernel"] != g.KERNEL_SPLITK
    assert pv(g, 16, 4096, 4096, "bf16", "bias", "row", "kn", a_layout="km")["kernel"] != g.KERNEL_SPLITK


# ------------------------------------------------------------------ tile width
def test_wide_tiles_only_for_many_waves_of_light_16bit_work(g):
    big = (8192, 8192, 4096)             # 512 tiles of 256 x 512: 6.9 waves of pairs
    assert pv(g, *big, "bf16", "relu_bias")["block_n"] == 512
    assert pv(g, *big, "f16", "relu_aux_bias")["block_n"] == 512
    assert pv(g, *big, "bf16", "gelu_bias")["block_n"] == 256     # heavy epilogue
    assert pv(g, *big, "bf16", "tanh_bias")["block_n"] == 256
    assert pv(g, *big, "e4m3", "bias")["block_n"] == 256         # short fp8 mainloop
    assert pv(g, *big, "bf16", "drelu")["block_n"] == 256        # backward
    assert pv(g, 4096, 4096, 4096, "bf16", "bias")["block_n"] == 256   # 1.7 waves of wide tiles
    assert pv(g, 8192, 4096, 4096, "bf16", "bias")["block_n"] == 256   # 3.5 waves


def test_ring_stage_atoms(g):
    # two k-atoms per stage where one atom is at most 32 KB per CTA, one where it is 48 KB
    big = pv(g, 8192, 8192, 4096, "bf16", "relu_bias")                       # pair 256 x 512
    assert (big["block_n"], big["block_k"], big["stages"]) == (512, 64, 4)
    tc1 = pv(g, 4096, 4096, 4096, "bf16", "bias", kernel="tc1", block_n=256)   # single 128 x 256
    assert (tc1["block_k"], tc1["stages"]) == (64, 4)
    small = pv(g, 1024, 512, 2048, "f16", "bias")                             # single 128 x 128
    assert (small["block_k"], small["stages"]) == (128, 3)
    narrow = pv(g, 4096, 4096, 4096, "bf16", "bias", kernel="tc2", block_n=128)  # pair 256 x 128
    assert (narrow["block_k"], narrow["stages"]) == (128, 4)


def test_e4m3_pairs_with_b_kn_take_256(g):
    p = pv(g, 512, 256, 1024, "e4m3", "bias", "row", "kn", kernel="tc2")
    assert p["block_n"] == 256


def test_explicit_tile_width_is_kept(g):
    assert pv(g, 4096, 4096, 4096, "bf16", "bias", kernel="tc2", block_n=512)["block_n"] == 512
    assert pv(g, 4096, 4096, 4096, "bf16", "bias", kernel="tc1", block_n=128)["block_n"] == 128


# ------------------------------------------------------------------ split tail
def test_split_tail_parts(g):
    # fewer tiles than units: up to four parts of at least 8 k-blocks
    assert pv(g, 1024, 512, 4096, "f16", "bias")["sk_split"] == 4        # 64 k-blocks
    assert pv(g, 1024, 512, 1024, "f16", "bias")["sk_split"] == 2        # 16 k-blocks
    assert pv(g, 1024, 512, 256, "f16", "bias")["sk_tiles"] == 0         # 4 k-blocks: not worth it
    # 64 tiles on 148 SMs: only two parts fit
    assert pv(g, 256, 4096, 4096, "f16", "gelu_bias", "col", "nk")["sk_split"] == 2
    # behind whole waves: two parts for the last wave's tiles
    p = pv(g, 4096, 4096, 4096, "bf16", "relu_aux_bias", kernel="tc1", block_n=256)
    assert (p["tiles"], p["sk_tiles"], p["sk_split"]) == (512, 512 % 148, 2)


def test_split_tail_options(g):
    assert pv(g, 4096, 4096, 4096, "bf16", "bias", stream_k="off")["sk_tiles"] == 0
    assert pv(g, 4096, 4096, 4096, "bf16", "bias", split_k=3)["sk_split"] == 2   # 74 // 34 = 2 fit
    p = pv(g, 1024, 512, 4096, "f16", "bias", split_k=2)
    assert p["sk_split"] == 2 and p["grid"] == 64


@pytest.mark.parametrize("k,stages", [(192, 2), (320, 3), (448, 4)])
def test_split_k_capped_at_ring_stages(g, k, stages):
    # 4 tiles of 128 x 128 (fewer than the SMs); k is an odd number of 128-byte k-atoms, and the
    # single-CTA 128-wide tile holds two atoms per ring stage, so k makes ceil(atoms / 2) stages.
    # A split_k above that is lowered to the stage count: a part is whole stages.
    p = pv(g, 256, 256, k, "bf16", "bias", kernel="tc1", block_n=128, stream_k="on", split_k=8)
    assert p["block_k"] == 128 and p["tiles"] == 4
    assert (p["sk_tiles"], p["sk_split"]) == (4, stages)
    assert p["grid"] == 4 * stages


def test_units_follow_the_sm_count(g):
    # a smaller part (or max_ctas) changes the waves, not the rules
    p = pv(g, 4096, 4096, 4096, "bf16", "relu_aux_bias", sms=100)
    assert p["kernel"] == g.KERNEL_TC2 and p["grid"] == 100
    assert (p["sk_tiles"], p["sk_split"]) == (256 % 50, 2)          # 6 tiles left on 50 pairs
    # 132 SMs: the last wave's 58 tiles on 66 pairs cannot be cut in two, so no split tail
    assert pv(g, 4096, 4096, 4096, "bf16", "relu_aux_bias", sms=132)["sk_tiles"] == 0
    q = pv(g, 4096, 4096, 4096, "bf16", "relu_aux_bias", max_ctas=64)
    assert q["grid"] == 64 and q["sk_tiles"] == 0                   # 256 tiles on 32 pairs: 8 waves


# ------------------------------------------------------------------ argument checks
def test_preview_checks_arguments_like_a_plan(g):
    def status(**kw):
        with pytest.raises(g.GemmEpiError) as e:
            pv(g, **kw)
        return e.value.status
    assert status(m=0, n=128, k=128) == g.ERR_ARG
    assert status(m=128, n=128, k=100, dtype="f16") == g.ERR_ALIGN        # 200-byte rows
    assert status(m=128, n=128, k=128, dtype="e4m3", epilogue="tanh_bias", out_e4m3=True) == g.ERR_UNSUPPORTED
    assert status(m=200, n=128, k=128, kernel="splitk") == g.ERR_UNSUPPORTED   # m > 128
    assert status(m=128, n=128, k=128, sms=1) == g.ERR_ARG
    assert status(m=128, n=128, k=128, sms=4096) == g.ERR_ARG


# ------------------------------------------------------------------ tile raster from the L2 budget
def test_raster_from_l2_budget(g):
    # 4096^3 bf16, 256 x 256 pair tiles: A and B are 32 MB each; A resident, one column walk
    p = pv(g, 4096, 4096, 4096, "bf16", "relu_aux_bias")
    assert (p["group_m"], p["group_n"]) == (16, 0)
    # FP8 8192 x 14336 x 4096: A 32 MB < B 56 MB: A resident over all 32 tile-rows
    p = pv(g, 8192, 14336, 4096, "e4m3", "gelu_bias", "col", "kn")
    assert (p["group_m"], p["group_n"]) == (32, 0)
    # B the smaller and within the budget (16 MB against A's 64 MB): row walk, B resident
    p = pv(g, 8192, 2048, 4096, "bf16", "bias")
    assert (p["group_m"], p["group_n"]) == (0, p["tiles"] // 32)
    # neither fits (65536 x 8192 x 16384: A 2 GB, B 256 MB): groups of 8 tile-rows
    p = pv(g, 65536, 8192, 16384, "bf16", "relu_bias")
    assert (p["group_m"], p["group_n"]) == (8, 0)
    # the small-m kernel has no raster
    p = pv(g, 16, 4096, 4096, "f16", "gelu_bias", "col", "nk")
    assert (p["group_m"], p["group_n"]) == (0, 0)


# clusters that can all be resident at once: at most 4 CTAs a cluster and 128 CTAs a launch, or
# 8 clusters of 8 (measured split sizes, m = 16, k = 4096)
@pytest.mark.parametrize("n,split,grid", [(512, 8, 32), (1024, 8, 64), (2048, 4, 64), (3072, 4, 96),
                                          (4096, 4, 128), (5120, 3, 120), (6144, 2, 96), (8192, 2, 128),
                                          (12288, 1, 96), (14336, 1, 112)])
def test_splitk_cluster_residency(g, n, split, grid):
    p = pv(g, 16, n, 4096, "f16", "gelu_bias", "col", "nk")
    assert p["kernel"] == g.KERNEL_SPLITK
    assert (p["split_k"], p["cluster"], p["grid"]) == (split, split, grid)


def test_splitk_m64_split_limit(g):
    # NM = 64: splits up to 4
    p = pv(g, 64, 1024, 4096, "f16", "gelu_bias", "col", "nk")
    assert (p["kernel"], p["block_m"], p["split_k"], p["grid"]) == (g.KERNEL_SPLITK, 64, 4, 32)
