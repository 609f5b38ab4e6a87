"""Pins for the fp64 CPU oracle against facts that do not come from the oracle.

Each test checks the oracle against something fixed independently of it: a
hand-computed case (tests/golden/tiny_cases.json), a textbook value, a
library routine on a special case (numpy matmul, numpy/torch float
conversions), or an invariant of the definition.  Together they are chosen so
that a plausible slip anywhere in the oracle -- a dropped bias, a bias on the
wrong axis, a transposed operand, a sign error in GELU, a ">=" for ">" in the
mask, a wrong exponent bias in a decoder, a missing FP8 scale -- fails at least
one of them (tests/test_oracle_mutants.py plants such slips and checks that).
"""
import math

import numpy as np
import pytest
import torch

from helpers import load_golden, to_storage_values

from activation_epilogue_tcgen05_b200.workloads import Workload, make_problem, storage


# ----------------------------------------------------------------------------- golden cases
CASES = load_golden("tiny_cases.json")["cases"]


def _case_inputs(c):
    dt = c["dtype"]
    if "e4m3_codes" in c:
        a = np.array(c["e4m3_codes"]["a"], dtype=np.uint8)
        b = np.array(c["e4m3_codes"]["b"], dtype=np.uint8)
    else:
        a = to_storage_values(c["a"], dt)
        b = to_storage_values(c["b"], dt)
    bias = to_storage_values(c["bias"], "bf16" if dt == "e4m3" else dt)
    return a, b, bias


@pytest.mark.parametrize("c", CASES, ids=[c["id"] for c in CASES])
def test_golden_tiny_case(oracle_lib, c):
    a, b, bias = _case_inputs(c)
    D, pre, mask = oracle_lib.gemm_epi(
        a, b, bias, dtype=c["dtype"], epilogue=c["epilogue"], bias_axis=c["bias_axis"],
        b_layout=c["b_layout"], scale_a=c.get("scale_a", 1.0), scale_b=c.get("scale_b", 1.0))
    want = np.array(c["d"], dtype=np.float64)
    rtol = c.get("rtol", 0.0)
    np.testing.assert_allclose(D, want, rtol=rtol, atol=0.0)
    np.testing.assert_array_equal(mask, np.array(c["mask"], dtype=np.uint8))
    # the sampled variant agrees at every position
    rows, cols = np.meshgrid(np.arange(D.shape[0]), np.arange(D.shape[1]), indexing="ij")
    Ds, pres, masks = oracle_lib.gemm_epi_sampled(
        a, b, bias, rows.ravel(), cols.ravel(), dtype=c["dtype"], epilogue=c["epilogue"],
        bias_axis=c["bias_axis"], b_layout=c["b_layout"], scale_a=c.get("scale_a", 1.0),
        scale_b=c.get("scale_b", 1.0))
    np.testing.assert_array_equal(Ds, D.ravel())
    np.testing.assert_array_equal(masks, mask.ravel())


# ----------------------------------------------------------------------------- decoders
def test_decode_f16_every_code_matches_numpy(oracle_lib):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle_lib.decode(codes, "f16")
    want = codes.view(np.float16).astype(np.float64)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def test_decode_bf16_every_code_matches_torch(oracle_lib):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle_lib.decode(codes, "bf16")
    want = torch.from_numpy(codes.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def test_decode_e4m3_fixed_points(oracle_lib):
    d = lambda code: float(oracle_lib.decode(np.array([code], np.uint8), "e4m3")[0])
    assert d(0x38) == 1.0
    assert d(0x7E) == 448.0
    assert d(0x01) == 2.0 ** -9
    assert d(0x08) == 2.0 ** -6           # smallest normal
    assert d(0x07) == 7 * 2.0 ** -9       # largest subnormal
    assert d(0x00) == 0.0 and math.copysign(1.0, d(0x80)) == -1.0
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))
    for code in range(0x80):
        if code != 0x7F:
            assert d(code | 0x80) == -d(code)


def test_decode_e4m3_every_code_matches_torch(oracle_lib):
    codes = np.arange(256, dtype=np.uint16).astype(np.uint8)
    got = oracle_lib.decode(codes, "e4m3")
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert ok.sum() == 254
    np.testing.assert_array_equal(got[ok], want[ok])
    # round trip of every finite code through the value
    back = torch.from_numpy(got[ok]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(back[codes[ok] != 0x80], codes[ok][codes[ok] != 0x80])


# ----------------------------------------------------------------------------- GELU
def test_gelu_textbook_values(oracle_lib):
    # Phi from a standard normal table: Phi(1), Phi(2), Phi(3)
    assert oracle_lib.gelu(1.0) == pytest.approx(0.841344746068543, rel=1e-14)
    assert oracle_lib.gelu(-1.0) == pytest.approx(-0.158655253931457, rel=1e-13)
    assert oracle_lib.gelu(2.0) == pytest.approx(1.954499736103642, rel=1e-14)
    assert oracle_lib.gelu(3.0) == pytest.approx(3 * 0.998650101968370, rel=1e-14)
    assert oracle_lib.gelu(0.0) == 0.0


@pytest.mark.parametrize("x", [0.25, 0.5, 1.0, 1.7, 3.0, 6.0])
def test_gelu_odd_part_is_identity(oracle_lib, x):
    # x*Phi(x) - (-x)*Phi(-x) = x*(Phi(x) + Phi(-x)) = x
    assert oracle_lib.gelu(x) - oracle_lib.gelu(-x) == pytest.approx(x, rel=1e-15, abs=1e-15)


def test_gelu_limits(oracle_lib):
    assert oracle_lib.gelu(10.0) == pytest.approx(10.0, rel=1e-15)
    assert abs(oracle_lib.gelu(-10.0)) < 1e-20


# ----------------------------------------------------------------------------- vs numpy matmul
def _decoded(arr, dtype):
    if dtype == "f16":
        return arr.view(np.float16).astype(np.float64)
    t = torch.from_numpy(arr.view(np.int16 if dtype == "bf16" else np.uint8).copy())
    t = t.view(torch.bfloat16 if dtype == "bf16" else torch.float8_e4m3fn)
    return t.double().numpy()


@pytest.mark.parametrize("dtype", ["f16", "bf16", "e4m3"])
@pytest.mark.parametrize("b_layout", ["kn", "nk"])
@pytest.mark.parametrize("bias_axis", ["row", "col"])
def test_pre_activation_equals_numpy_matmul_plus_bias(oracle_lib, dtype, b_layout, bias_axis):
    wl = Workload("t", 37, 29, 53, dtype, "relu_aux_bias", bias_axis, b_layout, seed=3)
    p = make_problem(wl)
    A, B, bias = storage(p.A), storage(p.B), storage(p.bias)
    D, pre, mask = oracle_lib.gemm_epi(A, B, bias, dtype=dtype, epilogue="relu_aux_bias",
                                       bias_axis=bias_axis, b_layout=b_layout,
                                       scale_a=p.scale_a, scale_b=p.scale_b)
    a = _decoded(A, dtype)
    b = _decoded(B, dtype)
    if b_layout == "nk":
        b = b.T
    bias_v = _decoded(bias, "bf16" if dtype == "e4m3" else dtype)
    want = (p.scale_a * p.scale_b) * (a @ b)
    want = want + (bias_v[:, None] if bias_axis == "row" else bias_v[None, :])
    np.testing.assert_allclose(pre, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(mask, (want > 0).astype(np.uint8))
    np.testing.assert_array_equal(D, np.maximum(pre, 0.0))


def test_none_is_bare_product(oracle_lib):
    wl = Workload("t", 16, 24, 40, "f16", "none", "row", "kn", seed=4)
    p = make_problem(wl)
    A, B = storage(p.A), storage(p.B)
    D, pre, _ = oracle_lib.gemm_epi(A, B, storage(p.bias), dtype="f16", epilogue="none")
    np.testing.assert_allclose(D, _decoded(A, "f16") @ _decoded(B, "f16"), rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(D, pre)


# ----------------------------------------------------------------------------- invariants
@pytest.mark.parametrize("epilogue", ["bias", "relu_bias", "gelu_bias"])
def test_identity_b(oracle_lib, epilogue):
    """B = I (k = n): D = act(A + bias) elementwise."""
    m, k = 9, 12
    wl = Workload("t", m, k, k, "bf16", epilogue, "col", "kn", seed=5)
    p = make_problem(wl)
    A, bias = storage(p.A), storage(p.bias)
    eye = to_storage_values(np.eye(k).tolist(), "bf16")
    D, pre, _ = oracle_lib.gemm_epi(A, eye, bias, dtype="bf16", epilogue=epilogue,
                                    bias_axis="col")
    x = _decoded(A, "bf16") + _decoded(bias, "bf16")[None, :]
    np.testing.assert_array_equal(pre, x)
    if epilogue == "bias":
        np.testing.assert_array_equal(D, x)
    elif epilogue == "relu_bias":
        np.testing.assert_array_equal(D, np.maximum(x, 0))
    else:
        for v, dv in zip(x.ravel(), D.ravel()):
            assert dv == pytest.approx(0.5 * v * (1 + math.erf(v / math.sqrt(2))), rel=1e-15,
                                       abs=1e-300)


def test_zero_bias_equals_bias_free_product(oracle_lib):
    wl = Workload("t", 11, 13, 17, "f16", "relu_bias", "row", "kn", seed=6,
                  dist_bias=("zeros", 0))
    p = make_problem(wl)
    D, pre, _ = oracle_lib.gemm_epi(storage(p.A), storage(p.B), storage(p.bias), dtype="f16",
                                    epilogue="relu_bias")
    Dn, _, _ = oracle_lib.gemm_epi(storage(p.A), storage(p.B), None, dtype="f16",
                                   epilogue="none")
    np.testing.assert_array_equal(pre, Dn)
    np.testing.assert_array_equal(D, np.maximum(Dn, 0))


def test_relu_properties(oracle_lib):
    wl = Workload("t", 33, 47, 64, "bf16", "relu_bias", "row", "kn", seed=7)
    p = make_problem(wl)
    D, pre, mask = oracle_lib.gemm_epi(storage(p.A), storage(p.B), storage(p.bias),
                                       dtype="bf16", epilogue="relu_bias")
    assert (D >= 0).all()
    np.testing.assert_array_equal(D[pre > 0], pre[pre > 0])
    assert (D[pre <= 0] == 0).all()
    np.testing.assert_array_equal(mask, (pre > 0).astype(np.uint8))
    frac = mask.mean()
    assert 0.3 < frac < 0.7          # symmetric data: about half positive


def test_bias_axis_swap_is_transpose(oracle_lib):
    """ROW bias on (A, B) equals COL bias on (B^T, A^T), transposed."""
    m, n, k = 10, 14, 20
    wl = Workload("t", m, n, k, "f16", "gelu_bias", "row", "kn", seed=8)
    p = make_problem(wl)
    A, B, bias = storage(p.A), storage(p.B), storage(p.bias)
    D1, _, _ = oracle_lib.gemm_epi(A, B, bias, dtype="f16", epilogue="gelu_bias",
                                   bias_axis="row", b_layout="kn")
    # (B^T)(n,k) as the A operand; A^T (k,m) as a kn B operand
    D2, _, _ = oracle_lib.gemm_epi(np.ascontiguousarray(B.T), np.ascontiguousarray(A.T), bias,
                                   dtype="f16", epilogue="gelu_bias", bias_axis="col",
                                   b_layout="kn")
    np.testing.assert_allclose(D2.T, D1, rtol=1e-13, atol=1e-13)


def test_nk_layout_equals_kn(oracle_lib):
    wl = Workload("t", 7, 19, 23, "bf16", "relu_aux_bias", "col", "kn", seed=9)
    p = make_problem(wl)
    A, B, bias = storage(p.A), storage(p.B), storage(p.bias)
    D1, pre1, m1 = oracle_lib.gemm_epi(A, B, bias, dtype="bf16", epilogue="relu_aux_bias",
                                       bias_axis="col", b_layout="kn")
    D2, pre2, m2 = oracle_lib.gemm_epi(A, np.ascontiguousarray(B.T), bias, dtype="bf16",
                                       epilogue="relu_aux_bias", bias_axis="col",
                                       b_layout="nk")
    np.testing.assert_array_equal(pre1, pre2)
    np.testing.assert_array_equal(m1, m2)


def test_fp8_unit_scales_equal_16bit_path(oracle_lib):
    """e4m3 with s_A = s_B = 1 on integer values equals the fp16 path on the same values."""
    wl = Workload("t", 12, 20, 32, "e4m3", "relu_aux_bias", "col", "kn", seed=10,
                  dist_a=("int", 4), dist_b=("int", 4), dist_bias=("int", 8))
    p = make_problem(wl, int_scales=True)
    A8, B8, bias = storage(p.A), storage(p.B), storage(p.bias)
    D8, pre8, m8 = oracle_lib.gemm_epi(A8, B8, bias, dtype="e4m3", epilogue="relu_aux_bias",
                                       bias_axis="col", scale_a=1.0, scale_b=1.0)
    A16 = to_storage_values(p.A.double().tolist(), "bf16")
    B16 = to_storage_values(p.B.double().tolist(), "bf16")
    D16, pre16, m16 = oracle_lib.gemm_epi(A16, B16, bias, dtype="bf16",
                                          epilogue="relu_aux_bias", bias_axis="col")
    np.testing.assert_array_equal(pre8, pre16)
    np.testing.assert_array_equal(D8, D16)
    np.testing.assert_array_equal(m8, m16)
    # with scales s_A = 2, s_B = 0.5 (alpha = 1) nothing changes; with s_A = 2, s_B = 2
    # the product (but not the bias) is multiplied by 4
    D8b, pre8b, _ = oracle_lib.gemm_epi(A8, B8, bias, dtype="e4m3", epilogue="relu_aux_bias",
                                        bias_axis="col", scale_a=2.0, scale_b=0.5)
    np.testing.assert_array_equal(pre8b, pre8)
    Dn, _, _ = oracle_lib.gemm_epi(A8, B8, None, dtype="e4m3", epilogue="none")
    _, pre4, _ = oracle_lib.gemm_epi(A8, B8, bias, dtype="e4m3", epilogue="relu_aux_bias",
                                     bias_axis="col", scale_a=2.0, scale_b=2.0)
    np.testing.assert_array_equal(pre4 - 4 * Dn, pre8 - Dn)


def test_integer_inputs_exact(oracle_lib):
    """Integer operands in {-2..2}: every partial sum is an exact integer."""
    wl = Workload("t", 24, 40, 64, "f16", "bias", "row", "kn", seed=11, dist_a=("int", 2),
                  dist_b=("int", 2), dist_bias=("int", 2))
    p = make_problem(wl)
    D, _, _ = oracle_lib.gemm_epi(storage(p.A), storage(p.B), storage(p.bias), dtype="f16",
                                  epilogue="bias")
    want = (p.A.long() @ p.B.long() + p.bias.long()[:, None]).double().numpy()
    np.testing.assert_array_equal(D, want)


def test_sampled_matches_full(oracle_lib):
    wl = Workload("t", 40, 36, 50, "e4m3", "gelu_bias", "col", "nk", seed=12)
    p = make_problem(wl)
    A, B, bias = storage(p.A), storage(p.B), storage(p.bias)
    kw = dict(dtype="e4m3", epilogue="gelu_bias", bias_axis="col", b_layout="nk",
              scale_a=p.scale_a, scale_b=p.scale_b)
    D, pre, mask = oracle_lib.gemm_epi(A, B, bias, **kw)
    rng = np.random.default_rng(0)
    rows = rng.integers(0, 40, 200)
    cols = rng.integers(0, 36, 200)
    Ds, pres, masks = oracle_lib.gemm_epi_sampled(A, B, bias, rows, cols, **kw)
    np.testing.assert_allclose(Ds, D[rows, cols], rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(masks, mask[rows, cols])


def test_bad_arguments_rejected(oracle_lib):
    a = to_storage_values([[1.0]], "f16")
    with pytest.raises(ValueError):
        oracle_lib.gemm_epi(a, a, a, dtype="f32", epilogue="bias")
    with pytest.raises(ValueError):
        oracle_lib.gemm_epi(a, a, a, dtype="f16", epilogue="swish")
    with pytest.raises(RuntimeError):
        oracle_lib.gemm_epi(a, a, None, dtype="f16", epilogue="bias")
    with pytest.raises(RuntimeError):
        oracle_lib.gemm_epi_sampled(a, a, a, [1], [0], dtype="f16", epilogue="bias")


# ----------------------------------------------------------------------------- more epilogues
@pytest.mark.parametrize("x", [0.125, 0.5, 1.0, 2.0, 4.0])
def test_tanh_is_odd_and_bounded(oracle_lib, x):
    a = to_storage_values([[x], [-x]], "f16")
    one = to_storage_values([[1.0]], "f16")
    D, pre, mask = oracle_lib.gemm_epi(a, one, None, dtype="f16", epilogue="tanh")
    assert D[0, 0] == -D[1, 0]
    assert 0 < D[0, 0] < 1 and D[0, 0] < x
    assert D[0, 0] == pytest.approx((math.exp(2 * x) - 1) / (math.exp(2 * x) + 1), rel=1e-14)


@pytest.mark.parametrize("pair", [("relu", "relu_bias"), ("relu_aux", "relu_aux_bias"),
                                  ("gelu", "gelu_bias"), ("tanh", "tanh_bias")])
def test_bias_free_epilogue_equals_zero_bias(oracle_lib, pair):
    nobias, withbias = pair
    wl = Workload("t", 13, 21, 34, "bf16", withbias, "col", "kn", seed=15, dist_bias=("zeros", 0))
    p = make_problem(wl)
    A, B, zero = storage(p.A), storage(p.B), storage(p.bias)
    D0, pre0, m0 = oracle_lib.gemm_epi(A, B, zero, dtype="bf16", epilogue=withbias, bias_axis="col")
    # a non-zero bias must be ignored by the bias-free epilogue
    junk = to_storage_values(np.arange(21, dtype=np.float64).tolist(), "bf16")
    D1, pre1, m1 = oracle_lib.gemm_epi(A, B, junk, dtype="bf16", epilogue=nobias, bias_axis="col")
    np.testing.assert_array_equal(D0, D1)
    np.testing.assert_array_equal(pre0, pre1)
    np.testing.assert_array_equal(m0, m1)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_scaling_factor_applies_to_16bit_inputs(oracle_lib, dtype):
    """alpha = s_A*s_B multiplies the product (not the bias) for 16-bit inputs too."""
    wl = Workload("t", 9, 17, 24, dtype, "bias", "row", "kn", seed=16)
    p = make_problem(wl)
    A, B, bias = storage(p.A), storage(p.B), storage(p.bias)
    _, pre1, _ = oracle_lib.gemm_epi(A, B, bias, dtype=dtype, epilogue="bias")
    _, pre3, _ = oracle_lib.gemm_epi(A, B, bias, dtype=dtype, epilogue="bias", scale_a=1.5,
                                     scale_b=2.0)
    Dn, _, _ = oracle_lib.gemm_epi(A, B, None, dtype=dtype, epilogue="none")
    np.testing.assert_allclose(pre3 - pre1, 2.0 * Dn, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- backward epilogues
BWD = load_golden("tiny_cases.json")["cases_bwd"]


@pytest.mark.parametrize("c", BWD, ids=[c["id"] for c in BWD])
def test_golden_backward_case(oracle_lib, c):
    a = to_storage_values(c["a"], c["dtype"])
    b = to_storage_values(c["b"], c["dtype"])
    D, dbias = oracle_lib.gemm_epi_bwd(a, b, np.array(c["mask_in"], np.uint8), dtype=c["dtype"],
                                       epilogue=c["epilogue"], bias_axis=c["bias_axis"],
                                       b_layout=c["b_layout"], scale_a=c.get("scale_a", 1.0),
                                       scale_b=c.get("scale_b", 1.0))
    np.testing.assert_array_equal(D, np.array(c["d"], dtype=np.float64))
    if "dbias" in c:
        np.testing.assert_array_equal(dbias, np.array(c["dbias"], dtype=np.float64))


@pytest.mark.parametrize("axis", ["row", "col"])
@pytest.mark.parametrize("layout", ["kn", "nk"])
def test_backward_equals_masked_numpy_product(oracle_lib, axis, layout):
    wl = Workload("t", 23, 31, 40, "bf16", "relu_aux_bias", axis, layout, seed=18)
    p = make_problem(wl)
    A, B = storage(p.A), storage(p.B)
    # the forward pass's own mask
    _, _, mask = oracle_lib.gemm_epi(A, B, storage(p.bias), dtype="bf16", epilogue="relu_aux_bias",
                                     bias_axis=axis, b_layout=layout)
    D, dbias = oracle_lib.gemm_epi_bwd(A, B, mask, dtype="bf16", epilogue="drelu_bgrad",
                                       bias_axis=axis, b_layout=layout, scale_a=2.0, scale_b=0.75)
    a, b = _decoded(A, "bf16"), _decoded(B, "bf16")
    prod = 1.5 * (a @ (b if layout == "kn" else b.T))
    np.testing.assert_allclose(D, np.where(mask == 1, prod, 0.0), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dbias, D.sum(axis=1 if axis == "row" else 0), rtol=1e-12, atol=1e-12)


def test_backward_mask_extremes(oracle_lib):
    wl = Workload("t", 8, 16, 24, "f16", "none", "row", "kn", seed=19)
    p = make_problem(wl)
    A, B = storage(p.A), storage(p.B)
    Dn, _, _ = oracle_lib.gemm_epi(A, B, None, dtype="f16", epilogue="none")
    ones = np.ones((8, 16), np.uint8)
    D1, db1 = oracle_lib.gemm_epi_bwd(A, B, ones, dtype="f16", epilogue="drelu_bgrad")
    np.testing.assert_array_equal(D1, Dn)
    D0, db0 = oracle_lib.gemm_epi_bwd(A, B, 0 * ones, dtype="f16", epilogue="drelu_bgrad",
                                      bias_axis="col")
    assert (D0 == 0).all() and (db0 == 0).all()


# ----------------------------------------------------------------------------- encoders (MLP block)
def _all_finite_codes(dtype):
    if dtype == "e4m3":
        c = np.arange(256, dtype=np.uint32)
        return c[(c & 0x7F) != 0x7F]
    c = np.arange(65536, dtype=np.uint32)
    exp_all_ones = ((c >> 10) & 0x1F) == 0x1F if dtype == "f16" else ((c >> 7) & 0xFF) == 0xFF
    return c[~exp_all_ones]


@pytest.mark.parametrize("dtype", ["e4m3", "f16", "bf16"])
def test_encode_inverts_decode_on_every_finite_code(oracle_lib, dtype):
    codes = _all_finite_codes(dtype)
    store = codes.astype(np.uint8 if dtype == "e4m3" else np.uint16)
    vals = oracle_lib.decode(store, dtype)
    np.testing.assert_array_equal(oracle_lib.encode(vals, dtype), store)


@pytest.mark.parametrize("dtype", ["e4m3", "f16", "bf16"])
def test_encode_midpoints_tie_to_even_and_neighbours_round_to_nearest(oracle_lib, dtype):
    """Between every pair of neighbouring non-negative codes (e4m3: all of them; 16-bit:
    a seeded sample plus the subnormal/normal seam and the top of the range)."""
    top = {"e4m3": 0x7E, "f16": 0x7BFF, "bf16": 0x7F7F}[dtype]
    if dtype == "e4m3":
        lo = np.arange(0, top, dtype=np.int64)
    else:
        rng = np.random.default_rng(5)
        seam = {"f16": 0x0400, "bf16": 0x0080}[dtype]
        lo = np.unique(np.concatenate([rng.integers(0, top, 3000), [0, 1, seam - 1, seam, top - 1]]))
    st = np.uint8 if dtype == "e4m3" else np.uint16
    a = oracle_lib.decode(lo.astype(st), dtype)
    b = oracle_lib.decode((lo + 1).astype(st), dtype)
    mid = 0.5 * (a + b)
    even = np.where(lo % 2 == 0, lo, lo + 1)
    np.testing.assert_array_equal(oracle_lib.encode(mid, dtype), even.astype(st))
    np.testing.assert_array_equal(oracle_lib.encode(-mid, dtype),
                                  (even | (0x80 if dtype == "e4m3" else 0x8000)).astype(st))
    eps = (b - a) * 1e-3
    np.testing.assert_array_equal(oracle_lib.encode(mid - eps, dtype), lo.astype(st))
    np.testing.assert_array_equal(oracle_lib.encode(mid + eps, dtype), (lo + 1).astype(st))


def test_encode_f16_matches_numpy_rounding(oracle_lib):
    rng = np.random.default_rng(6)
    x = rng.standard_normal(20000) * np.exp2(rng.integers(-26, 16, 20000))
    x = x[np.abs(x) < 65504]
    np.testing.assert_array_equal(oracle_lib.encode(x, "f16"), x.astype(np.float16).view(np.uint16))


def test_encode_bf16_and_e4m3_match_torch_rounding(oracle_lib):
    """fp32 inputs (so the library casts round once): bf16 everywhere, e4m3 inside +-448."""
    gen = torch.Generator().manual_seed(7)
    x = torch.randn(20000, generator=gen) * torch.exp2(torch.randint(-20, 20, (20000,), generator=gen).float())
    bf = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle_lib.encode(x.double().numpy(), "bf16"), bf)
    y = (torch.rand(20000, generator=gen) * 2 - 1) * 448 * torch.exp2(-torch.randint(0, 14, (20000,), generator=gen).float())
    e = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle_lib.encode(y.double().numpy(), "e4m3"), e)


def test_encode_saturation_and_overflow(oracle_lib):
    np.testing.assert_array_equal(oracle_lib.encode([448.0, 464.0, 480.0, 1e6, -1e6, -449.0], "e4m3"),
                                  np.array([0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE], np.uint8))
    # fp16: the largest finite value is 65504 with spacing 32, so 65520 rounds to infinity
    np.testing.assert_array_equal(oracle_lib.encode([65504.0, 65519.0, 65520.0, -70000.0], "f16"),
                                  np.array([0x7BFF, 0x7BFF, 0x7C00, 0xFC00], np.uint16))
    np.testing.assert_array_equal(oracle_lib.encode([0.0, -0.0, -1e-9], "e4m3"),
                                  np.array([0x00, 0x80, 0x80], np.uint8))


def test_encode_applies_the_scale(oracle_lib):
    # 8.5 / 0.25 = 34 -> e4m3 spacing 4 in [32, 64): 34 is halfway between 32 (0x60) and 36 (0x61)
    np.testing.assert_array_equal(oracle_lib.encode([8.5, 8.0, -9.0], "e4m3", 0.25),
                                  np.array([0x60, 0x60, 0xE1], np.uint8))


MLP = load_golden("tiny_cases.json")["cases_mlp"]


@pytest.mark.parametrize("c", MLP, ids=[c["id"] for c in MLP])
def test_golden_mlp_case(oracle_lib, c):
    dt = c["dtype"]
    bdt = "bf16" if dt == "e4m3" else dt
    args = [to_storage_values(c["x"], dt), to_storage_values(c["w1"], dt), to_storage_values(c["b1"], bdt),
            to_storage_values(c["w2"], dt), to_storage_values(c["b2"], bdt)]
    Y, H, Hs, amax = oracle_lib.mlp(*args, dtype=dt, act=c["act"], w_layout=c["w_layout"],
                                    scale_x=c["scale_x"], scale_w1=c["scale_w1"], scale_h=c["scale_h"],
                                    scale_w2=c["scale_w2"])
    np.testing.assert_allclose(H, np.array(c["h"]), rtol=1e-15, atol=0)
    np.testing.assert_array_equal(Hs, np.array(c["h_codes"]))
    assert amax == pytest.approx(c["amax"], rel=1e-15, abs=0)
    np.testing.assert_array_equal(Y, np.array(c["y"]))


@pytest.mark.parametrize("c", MLP, ids=[c["id"] for c in MLP])
def test_golden_mlp_case_stepwise(oracle_lib, c):
    dt = c["dtype"]
    bdt = "bf16" if dt == "e4m3" else dt
    args = [to_storage_values(c["x"], dt), to_storage_values(c["w1"], dt), to_storage_values(c["b1"], bdt),
            to_storage_values(c["w2"], dt), to_storage_values(c["b2"], bdt)]
    Y, H, Hs, amax = oracle_lib.mlp(*args, dtype=dt, act=c["act"], w_layout=c["w_layout"],
                                    scale_x=c["scale_x"], scale_w1=c["scale_w1"], scale_h=c["scale_h"],
                                    scale_w2=c["scale_w2"], stepwise=True)
    np.testing.assert_array_equal(H, np.array(c["h_stepwise"]))
    np.testing.assert_array_equal(Hs, np.array(c["h_codes_stepwise"]))
    assert amax == c["amax_stepwise"]
    np.testing.assert_array_equal(Y, np.array(c["y_stepwise"]))


@pytest.mark.parametrize("layout", ["kn", "nk"])
def test_mlp_equals_two_numpy_products(oracle_lib, layout):
    """16-bit MLP: H from the GELU of the first product, rounded to fp16 by numpy, then the
    second product by numpy matmul (with exactly representable integer weights)."""
    rng = np.random.default_rng(8)
    m, d, f = 5, 16, 24
    X = rng.integers(-2, 3, (m, d)).astype(np.float16)
    W1 = rng.integers(-2, 3, (d, f)).astype(np.float16)
    b1 = (rng.integers(-4, 5, f) / 4).astype(np.float16)
    W2 = rng.integers(-2, 3, (f, d)).astype(np.float16)
    b2 = (rng.integers(-4, 5, d) / 4).astype(np.float16)
    w1s = W1 if layout == "kn" else np.ascontiguousarray(W1.T)
    w2s = W2 if layout == "kn" else np.ascontiguousarray(W2.T)
    v = lambda a: a.view(np.uint16)
    Y, H, Hs, amax = oracle_lib.mlp(v(X), v(w1s), v(b1), v(w2s), v(b2), dtype="f16", act="gelu_bias",
                                    w_layout=layout)
    p = X.astype(np.float64) @ W1.astype(np.float64) + b1.astype(np.float64)
    gelu = np.vectorize(lambda t: 0.5 * t * (1 + math.erf(t / math.sqrt(2))))
    np.testing.assert_allclose(H, gelu(p), rtol=1e-14, atol=1e-15)
    np.testing.assert_array_equal(Hs, H.astype(np.float16).view(np.uint16))
    assert amax == np.abs(H).max()
    want = Hs.view(np.float16).astype(np.float64) @ W2.astype(np.float64) + b2.astype(np.float64)
    np.testing.assert_allclose(Y, want, rtol=1e-14, atol=1e-14)


# ----------------------------------------------------------------------------- A stored transposed
@pytest.mark.parametrize("c", [c for c in CASES if c["dtype"] != "e4m3" or "e4m3_codes" not in c],
                         ids=[c["id"] for c in CASES if c["dtype"] != "e4m3" or "e4m3_codes" not in c])
def test_golden_cases_with_a_stored_transposed(oracle_lib, c):
    """Every hand-computed case again, with A handed over as its (k, m) transpose."""
    a, b, bias = _case_inputs(c)
    at = np.ascontiguousarray(a.reshape(len(c["a"]), -1).T)
    kw = dict(dtype=c["dtype"], epilogue=c["epilogue"], bias_axis=c["bias_axis"], b_layout=c["b_layout"],
              scale_a=c.get("scale_a", 1.0), scale_b=c.get("scale_b", 1.0))
    D, pre, mask = oracle_lib.gemm_epi(at, b, bias, a_layout="km", **kw)
    np.testing.assert_allclose(D, np.array(c["d"], dtype=np.float64), rtol=c.get("rtol", 0.0), atol=0.0)
    np.testing.assert_array_equal(mask, np.array(c["mask"], dtype=np.uint8))
    rows, cols = np.meshgrid(np.arange(D.shape[0]), np.arange(D.shape[1]), indexing="ij")
    Ds, _, _ = oracle_lib.gemm_epi_sampled(at, b, bias, rows.ravel(), cols.ravel(), a_layout="km", **kw)
    np.testing.assert_array_equal(Ds, D.ravel())


def test_a_transposed_non_square_matches_numpy(oracle_lib):
    """m != k, so a swapped index cannot go unnoticed: numpy's product of the decoded values."""
    rng = np.random.default_rng(9)
    m, k, n = 5, 7, 3
    a = rng.integers(-3, 4, (m, k)).astype(np.float16)
    b = rng.integers(-3, 4, (k, n)).astype(np.float16)
    at = np.ascontiguousarray(a.T).view(np.uint16)
    D, _, _ = oracle_lib.gemm_epi(at, b.view(np.uint16), None, dtype="f16", epilogue="none", a_layout="km")
    np.testing.assert_array_equal(D, a.astype(np.float64) @ b.astype(np.float64))
