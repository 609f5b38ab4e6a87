"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small shapes that span several tiles plus ragged edges in m, n and k are
compared element by element for every dtype x epilogue x bias axis x B layout
and every kernel family; the five named workloads are checked at full size
(element by element where the oracle is fast enough, on seeded sampled
positions otherwise, plus invariants that hold at any size).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, aux_padding_bits, unpack_aux, band, tolerance
from parity import (alloc_outputs, check_against_oracle, compare, device_inputs, gpu_run,
                    make_plan, oracle_full, sampled_oracle, sigmas, unfused_extra)

from activation_epilogue_tcgen05_b200 import gemm_epi as g
from activation_epilogue_tcgen05_b200.workloads import (TORCH_DTYPE, WORKLOADS, Workload,
                                                        make_problem, sample_positions, storage)

pytestmark = pytest.mark.gpu

DTYPES = ["f16", "bf16", "e4m3"]
EPILOGUES = ["none", "bias", "relu_bias", "relu_aux_bias", "gelu_bias", "tanh_bias", "relu",
             "relu_aux", "gelu", "tanh"]


def small(dtype, epilogue, axis, layout, m=200, n=272, seed=1):
    k = 336 if dtype == "e4m3" else 328          # ragged last k-block
    return Workload(f"small_{dtype}_{epilogue}", m, n, k, dtype, epilogue, axis, layout, seed=seed)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip("needs sm_100")
    from activation_epilogue_tcgen05_b200 import build
    build.build()
    oracle.build()


# ------------------------------------------------------------------ persistent TC kernels
@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("axis", ["row", "col"])
@pytest.mark.parametrize("epilogue", EPILOGUES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("kernel,block_n", [("tc1", 128), ("tc1", 256), ("tc2", 256), ("tc2", 128), ("tc2", 512)])
def test_small_all_variants(kernel, block_n, dtype, epilogue, axis, layout):
    if kernel == "tc2" and block_n == 128 and dtype == "e4m3" and layout == "kn":
        pytest.skip("not instantiated: a 64-column e4m3 half-tile is narrower than one 128-byte box")
    wl = small(dtype, epilogue, axis, layout)
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel=kernel, block_n=block_n)
    assert info["kernel"] == g.KERNEL[kernel] and info["block_n"] == block_n
    assert worst <= 1.0


@pytest.mark.parametrize("kernel", ["tc1", "tc2"])
@pytest.mark.parametrize("dtype", DTYPES)
def test_persistent_many_tiles_per_cta(kernel, dtype):
    """Few CTAs, many tiles each: accumulator double-buffer and ring phases wrap many times."""
    k = 1024 if dtype == "e4m3" else 1000
    wl = Workload("persist", 600, 528, k, dtype, "relu_aux_bias", "col", "kn", seed=2)
    prob = make_problem(wl)
    # e4m3 with B stored (k, n) has no 128-wide pair tile (half a tile is narrower than one
    # 128-byte box), so the pair uses 256-wide tiles there
    bn = 256 if (kernel == "tc2" and dtype == "e4m3") else 128
    worst, info = check_against_oracle(wl, prob, kernel=kernel, block_n=bn, max_ctas=4)
    assert info["grid"] <= 4 and info["tiles"] >= 4
    assert worst <= 1.0


@pytest.mark.parametrize("kernel", ["tc1", "tc2"])
@pytest.mark.parametrize("m,n,k", [(1, 16, 16), (7, 24, 40), (129, 136, 72), (257, 264, 64)])
def test_tiny_and_edge_shapes(kernel, m, n, k):
    wl = Workload("edge", m, n, k, "bf16", "relu_aux_bias", "row", "kn", seed=3)
    prob = make_problem(wl)
    worst, _ = check_against_oracle(wl, prob, kernel=kernel)
    assert worst <= 1.0


@pytest.mark.parametrize("kernel", ["tc1", "tc2", "splitk"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("epilogue", ["bias", "relu_aux_bias", "none"])
def test_integer_inputs_bit_exact(kernel, dtype, epilogue):
    """Integer operands in {-2..2}: fp32 sums are exact, so D must equal RNE(oracle) bit for bit."""
    m = 48 if kernel == "splitk" else 300
    wl = Workload("int", m, 264, 200, dtype, epilogue, "row", "kn", seed=4, dist_a=("int", 2),
                  dist_b=("int", 2), dist_bias=("int", 2))
    prob = make_problem(wl)
    D, words, _ = gpu_run(wl, prob, kernel=kernel)
    ref, pre, mask = oracle_full(wl, prob)
    want = torch.from_numpy(ref).to(TORCH_DTYPE[dtype])
    assert torch.equal(D.view(torch.int16), want.view(torch.int16))
    if epilogue == "relu_aux_bias":
        np.testing.assert_array_equal(unpack_aux(words, wl.m, wl.n), mask)


# ------------------------------------------------------------------ activation accuracy
@pytest.mark.parametrize("epilogue", ["gelu", "tanh"])
@pytest.mark.parametrize("kernel", ["tc1", "splitk"])
def test_activation_dense_grid(epilogue, kernel):
    """act(A . I): every bf16 value in [-10, 10] through the kernel's activation.

    The product with an identity B is exact, so the only errors are the
    activation's and the final bf16 rounding: |gpu - ref| <= 2^-8 |ref| + 1e-6."""
    vals = torch.arange(-10.0, 10.0, 2.0 ** -7, dtype=torch.float64).to(torch.bfloat16).unique()
    n = 128
    m = (vals.numel() + n - 1) // n
    if kernel == "splitk":
        m = 64
        vals = vals[: m * n]
    grid = torch.zeros(m * n, dtype=torch.bfloat16)
    grid[: vals.numel()] = vals
    A = grid.view(m, n)
    eye = torch.eye(n, dtype=torch.bfloat16)
    D = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    with g.Plan(m, n, n, "bf16", epilogue, "row", "kn", kernel=kernel) as plan:
        plan.run(A.cuda(), eye.cuda(), None, D)
        plan.check()
    ref, _, _ = oracle.gemm_epi(storage(A), storage(eye), None, dtype="bf16", epilogue=epilogue)
    err = np.abs(D.double().cpu().numpy() - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6
    assert (err <= bound).all(), f"max excess {float((err - bound).max())}"


# ------------------------------------------------------------------ epilogue scaling factor
@pytest.mark.parametrize("kernel", ["tc1", "tc2", "splitk"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_alpha_scaling_16bit(kernel, dtype):
    """alpha = s_A*s_B multiplies the product of 16-bit operands when scales are set."""
    from dataclasses import replace as dc_replace
    m = 32 if kernel == "splitk" else 264
    wl = Workload("alpha", m, 272, 328, dtype, "gelu_bias", "col", "kn", seed=17)
    prob = dc_replace(make_problem(wl), scale_a=0.75, scale_b=-2.5)
    worst, _ = check_against_oracle(wl, prob, kernel=kernel)
    assert worst <= 1.0
    # both scale pointers NULL again: alpha back to 1
    A, B, bias = device_inputs(prob)
    D, _ = alloc_outputs(wl)
    plan = make_plan(wl, prob, kernel=kernel)
    g.gemm_epi_set_scales(plan.handle, None, None)
    plan.run(A, B, bias, D, None)
    plan.check()
    plan.close()
    ref, pre, mask = oracle_full(wl, dc_replace(prob, scale_a=1.0, scale_b=1.0))
    compare(wl, D.cpu(), None, ref, pre, mask, *sigmas(dc_replace(prob, scale_a=1.0, scale_b=1.0)))


# ------------------------------------------------------------------ stream-K tail
@pytest.mark.parametrize("kernel,max_ctas,m,n,parts", [
    ("tc1", 4, 600, 528, 2),    # 25 tiles on 4 CTAs: the last tile in two parts
    ("tc1", 8, 600, 528, 3),    # 25 tiles on 8 CTAs: the last tile in three parts
    ("tc1", 16, 256, 256, 4),   # fewer tiles than CTAs: every tile in four parts
    ("tc2", 12, 600, 528, 2),   # pairs: 3 x 5 tiles on 6 pairs
    ("tc2", 8, 256, 256, 2),    # pairs, fewer tiles than pairs (2 tiles on 4 pairs)
    ("tc2", 16, 256, 256, 4),   # pairs, fewer tiles than pairs, every tile in four parts
    ("tc2", 8, 600, 1104, 2),   # 512-wide pair tiles (block_n 512): 3 x 3 tiles on 4 pairs
])
@pytest.mark.parametrize("dtype,epilogue,axis,layout", [
    ("bf16", "relu_aux_bias", "row", "kn"), ("f16", "gelu_bias", "col", "nk"),
    ("e4m3", "bias", "col", "kn"), ("bf16", "none", "row", "nk"),
])
def test_stream_k(kernel, max_ctas, m, n, parts, dtype, epilogue, axis, layout):
    k = 1024 if dtype == "e4m3" else 1000
    wl = Workload("sk_tail", m, n, k, dtype, epilogue, axis, layout, seed=12)
    prob = make_problem(wl)
    bn = 256 if (kernel == "tc2" and dtype == "e4m3") else 128
    if n == 1104:
        bn = 512
    worst, info = check_against_oracle(wl, prob, kernel=kernel, block_n=bn, max_ctas=max_ctas,
                                       stream_k="on", split_k=parts)
    assert info["sk_tiles"] > 0 and info["sk_split"] == parts
    assert worst <= 1.0


@pytest.mark.parametrize("kernel", ["tc1", "tc2"])
def test_auto_split_depth_for_few_tiles(kernel):
    """Fewer tiles than units and a long k: the automatic plan cuts every tile into four
    parts; behind whole waves it keeps two."""
    wl = Workload("sk_auto", 256, 1024, 4096, "f16", "gelu_bias", "col", "nk", seed=15,
                  dist_b=("uniform", 1 / 64), dist_bias=("uniform", 1 / 64))
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel=kernel)
    assert info["sk_tiles"] > 0 and info["sk_split"] == 4
    assert worst <= 1.0
    big = g.Plan(4096, 4096, 4096, "bf16", "relu_aux_bias", "row", "kn", kernel=kernel, block_n=256)
    assert big.info["sk_tiles"] > 0 and big.info["sk_split"] == 2
    big.close()


@pytest.mark.parametrize("shape", [
    (4096, 4096, 4096, "bf16", "relu_aux_bias", "row", "kn", {}),
    (1024, 512, 2048, "f16", "bias", "row", "kn", {}),
    (16, 4096, 4096, "f16", "gelu_bias", "col", "nk", {}),
    (33, 4096, 4096, "f16", "gelu_bias", "col", "nk", {}),
    (65536, 8192, 16384, "bf16", "relu_bias", "row", "kn", {}),
    (8192, 14336, 4096, "e4m3", "gelu_bias", "col", "kn", {}),
    (4096, 4096, 4096, "bf16", "drelu_bgrad", "col", "kn", {}),
    (600, 528, 1000, "bf16", "relu_aux_bias", "row", "kn", {"max_ctas": 12, "kernel": "tc2"}),
    (256, 1024, 4096, "f16", "gelu_bias", "col", "nk", {"kernel": "tc1"}),
])
def test_preview_matches_plans(shape):
    """The host-only preview makes the choice a real plan makes on this device."""
    m, n, k, dt, epi, axis, layout, kw = shape
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    with g.Plan(m, n, k, dt, epi, axis, layout, **kw) as plan:
        assert g.plan_preview(m, n, k, dt, epi, axis, layout, num_sms=sms, **kw) == plan.info


def test_wide_tiles_chosen_for_many_waves():
    """4096 x 16384: 512 tiles of 256 x 512 for 74 pairs, so the plan takes 512-wide tiles;
    checked on seeded sampled positions (and element-exact mask outside the band)."""
    wl = Workload("wide", 4096, 16384, 256, "bf16", "relu_aux_bias", "row", "kn",
                  ("normal", 1.0 / 16), ("normal", 1.0 / 16), ("normal", 1.0), seed=52)
    prob = make_problem(wl)
    D, words, info = gpu_run(wl, prob)
    assert info["kernel"] == g.KERNEL_TC2 and info["block_n"] == 512
    rows, cols = sample_positions(wl.m, wl.n, 96, 96, seed=52, tile_n=512)
    ref, pre, mask = sampled_oracle(wl, prob, rows, cols)
    compare(wl, D, words, ref, pre, mask, *sigmas(prob), rows=rows, cols=cols)


@pytest.mark.parametrize("kernel", ["tc1", "tc2"])
def test_stream_k_deterministic_and_unfused(kernel):
    wl = Workload("sk_det", 600, 528, 1000, "bf16", "relu_aux_bias", "row", "kn", seed=13)
    prob = make_problem(wl)
    inputs = device_inputs(prob)
    opts = dict(kernel=kernel, block_n=128, max_ctas=6 if kernel == "tc1" else 12, stream_k="on")
    D1, w1, info = gpu_run(wl, prob, inputs=inputs, **opts)
    D2, w2, _ = gpu_run(wl, prob, inputs=inputs, **opts)
    assert info["sk_tiles"] > 0
    assert torch.equal(D1.view(torch.int16), D2.view(torch.int16))
    np.testing.assert_array_equal(w1, w2)
    Du, wu, _ = gpu_run(wl, prob, inputs=inputs, fused=False, **opts)
    ref, pre, mask = oracle_full(wl, prob)
    compare(wl, Du, wu, ref, pre, mask, *sigmas(prob), extra=unfused_extra(wl, prob, pre))


def test_stream_k_repeated_runs_on_one_plan():
    """Many runs of one plan: each launch must leave the partial-tile flags cleared."""
    wl = Workload("sk_rep", 384, 400, 512, "f16", "relu_bias", "col", "kn", seed=14)
    prob = make_problem(wl)
    A, B, bias = device_inputs(prob)
    D, _ = alloc_outputs(wl)
    plan = make_plan(wl, prob, kernel="tc1", block_n=128, max_ctas=5, stream_k="on")
    assert plan.info["sk_tiles"] > 0
    ref, pre, mask = oracle_full(wl, prob)
    sa, sb = sigmas(prob)
    for _ in range(20):
        D.fill_(float("nan"))
        plan.run(A, B, bias, D, None)
    plan.check()
    plan.close()
    compare(wl, D.cpu(), None, ref, pre, mask, sa, sb)


# ------------------------------------------------------------------ small-m split-K kernel
@pytest.mark.parametrize("layout", ["nk", "kn"])
@pytest.mark.parametrize("axis", ["col", "row"])
@pytest.mark.parametrize("epilogue", EPILOGUES)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("m", [16, 40, 100])
def test_splitk_variants(m, dtype, epilogue, axis, layout):
    k = 1024 if dtype == "e4m3" else 1000
    wl = Workload("sk", m, 400, k, dtype, epilogue, axis, layout, seed=5)
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel="splitk")
    assert info["kernel"] == g.KERNEL_SPLITK
    assert worst <= 1.0


@pytest.mark.parametrize("split", [1, 2, 3, 8])
def test_splitk_grid_parts_per_tile(split, monkeypatch):
    """The grid-wide split-K form (GEMM_EPI_SK_GRID=1) with split_k parts per tile (1 = whole
    tiles, no reduction)."""
    monkeypatch.setenv("GEMM_EPI_SK_GRID", "1")
    wl = Workload("sk_split", 16, 512, 2048, "f16", "gelu_bias", "col", "nk", seed=6,
                  dist_b=("uniform", 1 / 64), dist_bias=("uniform", 1 / 64))
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel="splitk", split_k=split)
    assert info["split_k"] == split and info["grid"] == 4 * split and info["cluster"] == 1
    assert worst <= 1.0


@pytest.mark.parametrize("ctas", [1, 3, 5, 7, 37, 100])
@pytest.mark.parametrize("epilogue", ["relu_aux_bias", "gelu_bias"])
def test_splitk_grid_uneven_ranges(ctas, epilogue, monkeypatch):
    """Grid-wide form: ranges of units that cut tiles at arbitrary k-blocks, and (few CTAs)
    ranges that span several whole and partial tiles: every piece's partial is added once."""
    monkeypatch.setenv("GEMM_EPI_SK_GRID", "1")
    wl = Workload("sk_ranges", 24, 656, 1000, "bf16", epilogue, "col", "kn", seed=16)
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel="splitk", max_ctas=ctas)
    assert info["grid"] == min(ctas, 6 * 16)          # 6 tiles x 16 k-blocks of units
    assert worst <= 1.0


@pytest.mark.parametrize("split", [1, 2, 3, 8])
def test_splitk_cluster_sizes(split):
    """The cluster form (partials reduced through distributed shared memory, no workspace),
    the default for small m and what the allocation-free entry point runs."""
    wl = Workload("sk_cluster", 16, 512, 2048, "f16", "gelu_bias", "col", "nk", seed=6,
                  dist_b=("uniform", 1 / 64), dist_bias=("uniform", 1 / 64))
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel="splitk", split_k=split)
    assert info["split_k"] == split and info["cluster"] == split
    assert worst <= 1.0


@pytest.mark.parametrize("m", [1, 16, 29, 64])
@pytest.mark.parametrize("dtype,epilogue,axis,layout", [
    ("f16", "gelu_bias", "col", "nk"), ("bf16", "relu_aux_bias", "row", "kn"),
    ("bf16", "bias", "col", "nk"), ("e4m3", "relu_bias", "row", "kn"), ("f16", "tanh_bias", "row", "kn")])
def test_splitk_one_cta_clusters(m, dtype, epilogue, axis, layout):
    """split_k = 1: each CTA holds its tile's whole sum and every epilogue warp finishes its own
    32 columns straight from its accumulator registers (no exchange), over ragged n, batch tiles
    of 16 / 32 / 64 rows and rows past m."""
    wl = Workload("sk_one", m, 1008, 1000 if dtype != "e4m3" else 1024, dtype, epilogue, axis, layout, seed=71)
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel="splitk", split_k=1)
    assert info["split_k"] == 1 and info["cluster"] == 1 and info["grid"] == 8
    assert worst <= 1.0


@pytest.mark.parametrize("kernel,block_n", [("tc1", 128), ("tc1", 256), ("tc2", 256), ("tc2", 512)])
@pytest.mark.parametrize("dtype,b_layout,a_layout", [("bf16", "kn", "mk"), ("f16", "nk", "mk"), ("bf16", "kn", "km"),
                                                     ("e4m3", "kn", "mk"), ("e4m3", "nk", "km")])
def test_stage_wide_copies(kernel, block_n, dtype, b_layout, a_layout, monkeypatch):
    """GEMM_EPI_FUSED_COPIES=1: one 3-D / 4-D copy per operand and ring stage (k a multiple of the
    128-byte atom, n and m of 128-byte blocks), several tiles and an odd k-atom count so that the
    last stage's second atom lies past k."""
    if block_n == 512 and (dtype == "e4m3" or a_layout == "km"):
        pytest.skip("512-wide tiles: 16-bit operands, A stored (m, k)")
    if a_layout == "km" and block_n != 256:
        pytest.skip("A stored (k, m): 256-wide tiles")
    monkeypatch.setenv("GEMM_EPI_FUSED_COPIES", "1")
    k = 640 if dtype == "e4m3" else 320          # 5 k-atoms of 128 bytes
    wl = Workload("fused", 512, 640 if block_n == 512 else 384, k, dtype, "relu_aux_bias", "row", b_layout,
                  seed=26, a_layout=a_layout)
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, kernel=kernel, block_n=block_n)
    assert info["block_n"] == block_n
    assert worst <= 1.0


# ------------------------------------------------------------------ fused vs unfused, determinism
@pytest.mark.parametrize("kernel", ["tc1", "tc2", "splitk"])
@pytest.mark.parametrize("epilogue", ["bias", "relu_bias", "relu_aux_bias", "gelu_bias", "tanh_bias",
                                      "relu", "relu_aux", "gelu", "tanh"])
def test_unfused_path_matches_oracle_and_fused(kernel, epilogue):
    m = 64 if kernel == "splitk" else 384
    wl = Workload("unf", m, 384, 512, "bf16", epilogue, "row", "kn", seed=7)
    prob = make_problem(wl)
    inputs = device_inputs(prob)
    Df, wf, _ = gpu_run(wl, prob, fused=True, inputs=inputs, kernel=kernel)
    Du, wu, _ = gpu_run(wl, prob, fused=False, inputs=inputs, kernel=kernel)
    ref, pre, mask = oracle_full(wl, prob)
    sa, sb = sigmas(prob)
    compare(wl, Df, wf, ref, pre, mask, sa, sb)
    # the unfused path rounds alpha*A.B to bf16 before the bias: one more rounding
    compare(wl, Du, wu, ref, pre, mask, sa, sb, extra=unfused_extra(wl, prob, pre))


@pytest.mark.parametrize("kernel", ["tc1", "tc2", "splitk"])
def test_run_to_run_bit_identical(kernel):
    m = 32 if kernel == "splitk" else 512
    wl = Workload("det", m, 512, 768, "bf16", "relu_aux_bias", "col", "kn", seed=8)
    prob = make_problem(wl)
    inputs = device_inputs(prob)
    D1, w1, _ = gpu_run(wl, prob, inputs=inputs, kernel=kernel)
    D2, w2, _ = gpu_run(wl, prob, inputs=inputs, kernel=kernel)
    assert torch.equal(D1.view(torch.int16), D2.view(torch.int16))
    np.testing.assert_array_equal(w1, w2)


@pytest.mark.parametrize("kernel", ["tc1", "tc2", "splitk"])
def test_guard_regions_untouched(kernel):
    """D and aux live inside larger buffers; the bytes around them must not change."""
    m = 24 if kernel == "splitk" else 136
    wl = Workload("guard", m, 200, 136, "f16", "relu_aux_bias", "row", "kn", seed=9)
    prob = make_problem(wl)
    A, B, bias = device_inputs(prob)
    G = 4096                                              # guard elements (16-byte multiple)
    pattern = -12345
    Dbuf = torch.full((G + wl.m * wl.n + G,), pattern, dtype=torch.int16, device="cuda")
    D = Dbuf[G:G + wl.m * wl.n].view(torch.float16).view(wl.m, wl.n)
    words = wl.m * g.aux_pitch_words(wl.n)
    Abuf = torch.full((G + words + G,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    aux = Abuf[G:G + words]
    plan = make_plan(wl, prob, kernel=kernel)
    plan.run(A, B, bias, D, aux)
    plan.check()
    plan.close()
    torch.cuda.synchronize()
    assert (Dbuf[:G] == pattern).all() and (Dbuf[G + wl.m * wl.n:] == pattern).all()
    assert (Abuf[:G] == 0x5A5A5A5A).all() and (Abuf[G + words:] == 0x5A5A5A5A).all()
    ref, pre, mask = oracle_full(wl, prob)
    sa, sb = sigmas(prob)
    compare(wl, D.cpu(), aux.cpu().numpy().view(np.uint32), ref, pre, mask, sa, sb)


def test_non_default_stream():
    wl = Workload("stream", 256, 256, 256, "bf16", "gelu_bias", "col", "nk", seed=10)
    prob = make_problem(wl)
    A, B, bias = device_inputs(prob)
    D, _ = alloc_outputs(wl)
    s = torch.cuda.Stream()
    plan = make_plan(wl, prob)
    with torch.cuda.stream(s):
        plan.run(A, B, bias, D, None, stream=s)
    plan.check(stream=s)
    plan.close()
    ref, pre, mask = oracle_full(wl, prob)
    compare(wl, D.cpu(), None, ref, pre, mask, *sigmas(prob))


@pytest.mark.parametrize("kernel2", ["tc1", "tc2", "splitk"])
@pytest.mark.parametrize("graph", [False, True])
def test_dependent_launches_keep_stream_order(kernel2, graph):
    """Back-to-back launches on one stream, each allowed to start before the previous one
    ends (programmatic dependent launch): the consumer must read the producer's output
    (read after write) and the producer's next launch must not overwrite it before the
    consumer has read it (write after read).  Producer: H = GELU(X.W1 + b1); consumer:
    Y = A2.H (H as the (k, n) operand).  Expected values: the oracle chain (the oracle's
    H rounded to f16, fed to the oracle again)."""
    m1, n1, k1 = 512, 256, 1024
    m2 = 48 if kernel2 == "splitk" else 384
    wl1 = Workload("pdl_h", m1, n1, k1, "f16", "gelu_bias", "col", "kn", seed=40)
    wl1b = wl1.with_(seed=41)
    wl2 = Workload("pdl_y", m2, n1, m1, "f16", "none", "row", "kn", seed=42)
    p1, p1b, p2 = make_problem(wl1), make_problem(wl1b), make_problem(wl2)
    X, W1, b1 = device_inputs(p1)
    Xb, W1b, b1b = device_inputs(p1b)
    A2 = p2.A.cuda()
    H = torch.full((m1, n1), float("nan"), dtype=torch.float16, device="cuda")
    Y = torch.full((m2, n1), float("nan"), dtype=torch.float16, device="cuda")
    plan1 = make_plan(wl1, p1, kernel="tc1")
    plan2 = make_plan(wl2, p2, kernel=kernel2)
    s = torch.cuda.Stream()
    try:
        def chain():
            plan1.run(X, W1, b1, H, None, stream=s)          # producer
            plan2.run(A2, H, None, Y, None, stream=s)        # consumer of H
            plan1.run(Xb, W1b, b1b, H, None, stream=s)       # overwrites H after the read
        with torch.cuda.stream(s):
            chain()                                           # also encodes the tensor maps
            s.synchronize()
            if graph:
                g_ = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g_, stream=s):
                    chain()
                H.fill_(float("nan"))
                Y.fill_(float("nan"))
                s.synchronize()
                for _ in range(3):
                    g_.replay()
            else:
                for _ in range(3):
                    H.fill_(float("nan"))
                    Y.fill_(float("nan"))
                    chain()
        s.synchronize()
        plan1.check(stream=s)
        plan2.check(stream=s)
    finally:
        plan1.close()
        plan2.close()
    h_ref, _, _ = oracle_full(wl1, p1)
    hb_ref, hb_pre, hb_mask = oracle_full(wl1b, p1b)
    # the consumer saw the first producer's H
    h16 = torch.tensor(h_ref, dtype=torch.float64).to(torch.float16)
    y_ref, y_pre, y_mask = oracle.gemm_epi(storage(p2.A), storage(h16), None, dtype="f16", epilogue="none")
    sa = float(p2.A.double().std(unbiased=False))
    sb = float(h16.double().std(unbiased=False))
    compare(wl2, Y.cpu(), None, y_ref, y_pre, y_mask, sa, sb)
    # and H holds the second producer's result
    compare(wl1b, H.cpu(), None, hb_ref, hb_pre, hb_mask, *sigmas(p1b))


# ------------------------------------------------------------------ A stored transposed, (k, m)
@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("epilogue", ["none", "bias", "relu_aux_bias", "gelu_bias", "tanh"])
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("kernel", ["tc1", "tc2"])
def test_a_stored_transposed(kernel, dtype, epilogue, layout):
    k = 336 if dtype == "e4m3" else 328
    wl = Workload("at", 208, 272, k, dtype, epilogue, "col", layout, seed=50, a_layout="km")
    worst, info = check_against_oracle(wl, make_problem(wl), kernel=kernel)
    assert info["kernel"] == g.KERNEL[kernel] and info["block_n"] == 256
    assert worst <= 1.0


@pytest.mark.parametrize("m", [16, 520])
def test_a_stored_transposed_auto_split_tail_and_unfused(m):
    wl = Workload("at2", m, 528, 1000, "bf16", "relu_aux_bias", "row", "kn", seed=51, a_layout="km")
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob, stream_k="on", max_ctas=8)
    assert info["kernel"] in (g.KERNEL_TC1, g.KERNEL_TC2) and worst <= 1.0
    D, words, _ = gpu_run(wl, prob, fused=False)
    ref, pre, mask = oracle_full(wl, prob)
    compare(wl, D, words, ref, pre, mask, *sigmas(prob), extra=unfused_extra(wl, prob, pre))


def test_a_stored_transposed_refusals():
    def status(fn):
        with pytest.raises(g.GemmEpiError) as e:
            fn()
        return e.value.status

    assert status(lambda: g.Plan(256, 256, 256, "bf16", "bias", a_layout="km", block_n=128)) == g.ERR_UNSUPPORTED
    assert status(lambda: g.Plan(16, 256, 256, "bf16", "bias", a_layout="km", kernel="splitk")) == g.ERR_UNSUPPORTED
    assert status(lambda: g.Plan(256, 256, 256, "bf16", "drelu", a_layout="km")) == g.ERR_UNSUPPORTED
    assert status(lambda: g.Plan(256, 256, 256, "e4m3", "bias", a_layout="km", out_e4m3=True)) == g.ERR_UNSUPPORTED


# ------------------------------------------------------------------ errors and failure paths
def test_run_argument_errors():
    wl = Workload("err", 128, 128, 128, "bf16", "relu_aux_bias", "row", "kn")
    prob = make_problem(wl)
    A, B, bias = device_inputs(prob)
    D, aux = alloc_outputs(wl)
    plan = make_plan(wl, prob)
    L, h = g.lib(), plan.handle
    s = None
    p = lambda t: None if t is None else t.data_ptr()
    assert L.gemm_epi_run(h, None, p(B), p(bias), p(D), p(aux), s) == g.ERR_NULL
    assert L.gemm_epi_run(h, p(A), p(B), None, p(D), p(aux), s) == g.ERR_NULL
    assert L.gemm_epi_run(h, p(A), p(B), p(bias), p(D), None, s) == g.ERR_NULL
    assert L.gemm_epi_run(h, p(A) + 2, p(B), p(bias), p(D), p(aux), s) == g.ERR_ALIGN
    assert L.gemm_epi_run(h, p(A), p(B), p(bias) + 2, p(D), p(aux), s) == g.ERR_ALIGN
    assert L.gemm_epi_run(h, p(A), p(B), p(bias), p(D), p(aux) + 4, s) == g.ERR_ALIGN
    assert L.gemm_epi_set_scales(h, p(A), None) == g.ERR_NULL          # one scale only
    plan.close()
    assert L.gemm_epi_run(h, p(A), p(B), p(bias), p(D), p(aux), s) == g.ERR_ARG  # freed
    # e4m3 without scales
    wl8 = Workload("err8", 128, 128, 128, "e4m3", "bias", "row", "kn")
    plan8 = g.Plan(128, 128, 128, "e4m3", "bias", "row", "kn")
    p8 = make_problem(wl8)
    A8, B8, b8 = device_inputs(p8)
    D8, _ = alloc_outputs(wl8)
    assert L.gemm_epi_run(plan8.handle, p(A8), p(B8), p(b8), p(D8), None, s) == g.ERR_NULL
    plan8.close()


@pytest.mark.parametrize("kernel", ["tc1", "tc2"])
def test_bounded_wait_reports_timeout_and_context_survives(kernel):
    """A wait that can never complete (nothing publishes the accumulator) must end in about a
    second with GEMM_EPI_ERR_TIMEOUT, and the next normal run must work."""
    wl = Workload("stall", 256, 256, 256, "bf16", "bias", "row", "kn", seed=11)
    prob = make_problem(wl)
    A, B, bias = device_inputs(prob)
    D, _ = alloc_outputs(wl)
    plan = make_plan(wl, prob, kernel=kernel, inject_stall=1)
    plan.run(A, B, bias, D, None)
    with pytest.raises(g.GemmEpiError) as e:
        plan.check()
    assert e.value.status == g.ERR_TIMEOUT
    plan.check()                               # the status word was cleared
    plan.close()
    worst, _ = check_against_oracle(wl, prob, kernel=kernel)
    assert worst <= 1.0


# ------------------------------------------------------------------ the five named workloads
def _named(name):
    return WORKLOADS[name]


def test_workload_gemm_bias_f16_full():
    wl = _named("gemm_bias_f16_1024x512x2048")
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob)
    assert worst <= 1.0


def test_workload_linear_gelu_f16_full_splitk():
    wl = _named("linear_gelu_f16_16x4096x4096")
    prob = make_problem(wl)
    worst, info = check_against_oracle(wl, prob)
    assert info["kernel"] == g.KERNEL_SPLITK
    assert worst <= 1.0


def _properties_relu(D, words, wl):
    """Invariants at any size: D >= 0; mask bit => D >= 0; D > 0 => mask bit; zero padding."""
    d = D.float()
    assert (d >= 0).all()
    if words is not None:
        bits = torch.from_numpy(unpack_aux(words, wl.m, wl.n).astype(np.bool_))
        assert not (bits & (d < 0)).any()
        assert not ((d > 0) & ~bits).any()
        assert aux_padding_bits(words, wl.m, wl.n) == 0


def _sampled_check(wl, prob, D, words):
    rows, cols = sample_positions(wl.m, wl.n, 64, 64, seed=0)
    ref, pre, mask = sampled_oracle(wl, prob, rows, cols)
    sa, sb = sigmas(prob)
    d = D[torch.as_tensor(rows), torch.as_tensor(cols)].double().numpy()
    tol = tolerance(ref, wl.dtype, wl.k, sa, sb)
    bad = ~(np.abs(d - ref) <= tol)
    assert not bad.any(), f"{int(bad.sum())} sampled outputs outside tolerance"
    if words is not None:
        bits = unpack_aux(words, wl.m, wl.n)[rows, cols]
        exact = band(pre, wl.dtype, wl.k, sa, sb)
        assert not (exact & (bits != mask)).any()


def test_workload_relu_aux_bias_bf16_4096():
    wl = _named("relu_aux_bias_bf16_4096x4096x4096")
    prob = make_problem(wl)
    inputs = device_inputs(prob)
    D, words, info = gpu_run(wl, prob, inputs=inputs)
    _properties_relu(D, words, wl)
    _sampled_check(wl, prob, D, words)
    # the unfused baseline agrees with the fused result within the tolerance
    Du, wu, _ = gpu_run(wl, prob, inputs=inputs, fused=False)
    sa, sb = sigmas(prob)
    tol = TOL["bf16"][0] * D.double().abs() + TOL["bf16"][1] * np.sqrt(wl.k) * sa * sb
    # |A.B| <= |D| + |bias| where the ReLU passes; one bf16 ulp of it for the extra rounding
    bias_rows = prob.bias.double()[:, None]
    extra = 2.0 ** -7 * (D.double().abs() + bias_rows.abs())
    assert ((Du.double() - D.double()).abs() <= 2 * tol + extra).all()


@pytest.mark.slow
def test_workload_relu_aux_bias_bf16_4096_full_oracle():
    wl = _named("relu_aux_bias_bf16_4096x4096x4096")
    prob = make_problem(wl)
    worst, _ = check_against_oracle(wl, prob)
    assert worst <= 1.0


def test_workload_fp8_gelu_bias():
    wl = _named("fp8_gelu_bias_8192x14336x4096")
    prob = make_problem(wl)
    D, words, _ = gpu_run(wl, prob)
    _sampled_check(wl, prob, D, words)


@pytest.mark.slow
def test_workload_fp8_gelu_bias_full_oracle():
    """Every output of the 8192 x 14336 x 4096 e4m3 GELU_BIAS workload against the oracle.

    Rows of D are independent, so the oracle runs on blocks of 1024 rows of A (all of B and
    the per-column bias each time), which bounds the host memory its fp64 results take."""
    wl = _named("fp8_gelu_bias_8192x14336x4096")
    prob = make_problem(wl)
    D, words, info = gpu_run(wl, prob)
    assert info["kernel"] == g.KERNEL_TC2
    sa, sb = sigmas(prob)
    Bs, bias = storage(prob.B), storage(prob.bias)
    worst = 0.0
    for r0 in range(0, wl.m, 1024):
        r1 = min(wl.m, r0 + 1024)
        ref, pre, mask = oracle.gemm_epi(storage(prob.A[r0:r1].contiguous()), Bs, bias, dtype=wl.dtype,
                                         epilogue=wl.epilogue, bias_axis=wl.bias_axis, b_layout=wl.b_layout,
                                         scale_a=prob.scale_a, scale_b=prob.scale_b)
        worst = max(worst, compare(wl.with_(m=r1 - r0), D[r0:r1], None, ref, pre, mask, sa, sb))
    assert worst <= 1.0


def test_workload_large_relu_bias_sampled():
    wl = _named("relu_bias_bf16_65536x8192x16384")
    prob = make_problem(wl, device="cuda")
    D, words, _ = gpu_run(wl, prob, inputs=(prob.A, prob.B, prob.bias))
    _properties_relu(D, words, wl)
    _sampled_check(wl, prob, D, words)
    del prob
    torch.cuda.empty_cache()
