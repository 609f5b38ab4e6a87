"""GPU parity of the FP8-output epilogue and the MLP block against the oracle.

FP8 output: D = e4m3(y / s_out), a quantised code decided in fp32 on the GPU
and in fp64 by the oracle.  The decision band is the 16-bit tolerance
(4e-3 |y| + 2e-3 sqrt(k) sigma_A sigma_B): the fp32 value y the GPU quantises
differs from the oracle's only by fp32 accumulation and rounding (the operands
are the same e4m3 codes), far inside that band, while the fp8 tolerance of the
D values (6e-2 |y| + ...) is as wide as an e4m3 code step and would decide
nothing.  The code is unique wherever the oracle's v = y / s_out lies farther
than t = band / s_out from a rounding boundary; there the GPU's code must equal
the oracle's, elsewhere it may be either neighbour.  One check covers both: the
GPU's decoded value lies between decode(encode(v - t)) and decode(encode(v + t))
(encode is monotonic).  amax must be within the band at the largest element.

MLP block: H (codes as above) and Y = s_H s_W2 H.W2 + b2 within the fp8 (or
16-bit) tolerance with sigma_H taken from the oracle's own stored H.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, tolerance
from parity import sigmas

from activation_epilogue_tcgen05_b200 import gemm_epi as g
from activation_epilogue_tcgen05_b200.workloads import TORCH_DTYPE, Workload, make_problem, storage

pytestmark = pytest.mark.gpu

# one unit in the last place, relative, of a 16-bit type (upper bound for normal values)
OUT_ULP = {"f16": 2.0 ** -10, "bf16": 2.0 ** -7}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs sm_100")
    from activation_epilogue_tcgen05_b200 import build
    build.build()
    oracle.build()


def _f32(x):
    return torch.tensor([x], dtype=torch.float32, device="cuda")


def check_codes(codes_gpu, y_ref, tol, scale, dtype):
    """Quantised outputs: inside [decode(encode(v - t)), decode(encode(v + t))]."""
    v = y_ref / scale
    t = tol / scale
    lo = oracle.decode(oracle.encode(v - t, dtype), dtype)
    hi = oracle.decode(oracle.encode(v + t, dtype), dtype)
    gv = oracle.decode(np.ascontiguousarray(codes_gpu), dtype)
    bad = ~((gv >= lo) & (gv <= hi))
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{int(bad.sum())} of {bad.size} codes outside the band; first {i}: gpu "
                             f"{gv[i]}, oracle {v[i]} +- {t[i]} -> [{lo[i]}, {hi[i]}]")
    # and the codes are the oracle's wherever the decision is unique
    unique = lo == hi
    assert (gv[unique] == lo[unique]).all()
    # fraction decided uniquely among values clear of zero (a zero's band straddles +-0)
    away = np.abs(v) > t
    return float(unique[away].mean()) if away.any() else 1.0


def run_qout(wl, prob, scale_out, **opts):
    A, B, bias = prob.A.cuda(), prob.B.cuda(), prob.bias.cuda()
    if wl.epilogue not in g.HAS_BIAS:
        bias = None
    D = torch.full((wl.m, wl.n), 0x7F, dtype=torch.uint8, device="cuda")     # 0x7F: the e4m3 NaN
    amax = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    with g.Plan(wl.m, wl.n, wl.k, wl.dtype, wl.epilogue, wl.bias_axis, wl.b_layout, out_e4m3=True,
                **opts) as plan:
        plan.set_scales(_f32(prob.scale_a), _f32(prob.scale_b))
        s_t = _f32(scale_out)
        plan.set_out_scale(s_t, amax)
        plan.run(A, B, bias, D, None)
        plan.check()
        info = plan.info
    torch.cuda.synchronize()
    return D.cpu().numpy(), float(amax.item()), info


def check_qout(wl, scale_factor=1.0, **opts):
    prob = make_problem(wl)
    ref, pre, _ = oracle.gemm_epi(storage(prob.A), storage(prob.B), storage(prob.bias), dtype="e4m3",
                                  epilogue=wl.epilogue, bias_axis=wl.bias_axis, b_layout=wl.b_layout,
                                  scale_a=prob.scale_a, scale_b=prob.scale_b)
    amax_ref = float(np.abs(ref).max())
    scale = float(np.float32(amax_ref / 448.0 * scale_factor))   # the fp32 value the GPU reads
    codes, amax, info = run_qout(wl, prob, scale, **opts)
    sa, sb = sigmas(prob)
    band = tolerance(ref, "bf16", wl.k, sa, sb)          # the decision band (module docstring)
    frac_unique = check_codes(codes, ref, band, scale, "e4m3")
    assert abs(amax - amax_ref) <= band.max(), (amax, amax_ref)
    return frac_unique, info


@pytest.mark.parametrize("split", [1, 3])
@pytest.mark.parametrize("epilogue", ["gelu_bias", "relu_bias"])
def test_fp8_out_splitk_cluster_forms(split, epilogue):
    """e4m3 output from the small-m kernel: one-CTA clusters (finished from registers) and
    clusters of 3 (partials exchanged), codes and amax against the oracle."""
    wl = Workload("q_sk", 24, 1008, 1024, "e4m3", epilogue, "col", "kn", seed=72)
    frac, info = check_qout(wl, kernel="splitk", split_k=split)
    assert info["kernel"] == g.KERNEL_SPLITK and info["cluster"] == split
    assert frac > 0.5          # most codes decided uniquely (as in the single-GEMM variants)


# ------------------------------------------------------------------ FP8 output, single GEMM
@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("axis", ["row", "col"])
@pytest.mark.parametrize("epilogue", ["none", "bias", "relu_bias", "gelu_bias", "relu", "gelu"])
@pytest.mark.parametrize("kernel,block_n", [("tc1", 128), ("tc1", 256), ("tc2", 256), ("tc2", 128)])
def test_fp8_out_all_variants(kernel, block_n, epilogue, axis, layout):
    if kernel == "tc2" and block_n == 128 and layout == "kn":
        pytest.skip("not instantiated: a 64-column e4m3 half-tile is narrower than one 128-byte box")
    if epilogue in ("none", "relu", "gelu") and axis == "col":
        pytest.skip("no bias: the axis plays no part")
    wl = Workload("q", 200, 272, 336, "e4m3", epilogue, axis, layout, seed=31)
    frac, info = check_qout(wl, kernel=kernel, block_n=block_n)
    assert info["kernel"] == g.KERNEL[kernel]
    # the band leaves a single code for most values away from zero: those are matched exactly
    assert frac > 0.5


@pytest.mark.parametrize("factor", [0.25, 4.0])
def test_fp8_out_saturation_and_small_codes(factor):
    """factor 0.25: a quarter of the range saturates at +-448; factor 4: codes crowd near 0
    (subnormals)."""
    wl = Workload("qsat", 256, 256, 512, "e4m3", "gelu_bias", "col", "kn", seed=32)
    check_qout(wl, scale_factor=factor)


@pytest.mark.parametrize("kernel,max_ctas", [("tc1", 4), ("tc2", 12)])
def test_fp8_out_stream_k(kernel, max_ctas):
    wl = Workload("qsk", 600, 528, 1024, "e4m3", "bias", "col", "kn", seed=33)
    _, info = check_qout(wl, kernel=kernel, block_n=256 if kernel == "tc2" else 128, max_ctas=max_ctas,
                         stream_k="on")
    assert info["sk_tiles"] > 0


def test_fp8_out_small_m_uses_splitk():
    wl = Workload("qsmall", 16, 512, 1024, "e4m3", "gelu_bias", "col", "nk", seed=34)
    _, info = check_qout(wl)
    assert info["kernel"] == g.KERNEL_SPLITK


@pytest.mark.parametrize("layout", ["nk", "kn"])
@pytest.mark.parametrize("axis", ["col", "row"])
@pytest.mark.parametrize("epilogue", ["none", "bias", "relu_bias", "gelu_bias"])
@pytest.mark.parametrize("m", [16, 40, 100])
def test_fp8_out_splitk_variants(m, epilogue, axis, layout):
    if epilogue == "none" and axis == "col":
        pytest.skip("no bias: the axis plays no part")
    wl = Workload("qsk2", m, 400, 1024, "e4m3", epilogue, axis, layout, seed=38)
    _, info = check_qout(wl, kernel="splitk")
    assert info["kernel"] == g.KERNEL_SPLITK


def test_fp8_out_argument_errors():
    def status(fn):
        with pytest.raises(g.GemmEpiError) as e:
            fn()
        return e.value.status

    assert status(lambda: g.Plan(256, 256, 256, "bf16", "bias", out_e4m3=True)) == g.ERR_UNSUPPORTED
    assert status(lambda: g.Plan(256, 256, 256, "e4m3", "relu_aux_bias", out_e4m3=True)) == g.ERR_UNSUPPORTED
    assert status(lambda: g.Plan(256, 256, 256, "e4m3", "tanh_bias", out_e4m3=True)) == g.ERR_UNSUPPORTED
    A = torch.zeros((256, 256), dtype=torch.uint8, device="cuda")
    D = torch.zeros((256, 256), dtype=torch.uint8, device="cuda")
    bias = torch.zeros((256,), dtype=torch.bfloat16, device="cuda")
    one = _f32(1.0)
    with g.Plan(256, 256, 256, "e4m3", "bias", out_e4m3=True) as p:
        p.set_scales(one, one)
        assert status(lambda: p.run(A, A, bias, D)) == g.ERR_NULL              # no output scale
        assert status(lambda: p.set_out_scale(None)) == g.ERR_NULL
        p.set_out_scale(one)                                                    # amax optional
        assert status(lambda: p.run(A, A, bias, D, fused=False)) == g.ERR_UNSUPPORTED
        p.run(A, A, bias, D)
        p.check()
    with g.Plan(256, 256, 256, "e4m3", "bias") as p:
        assert status(lambda: p.set_out_scale(one)) == g.ERR_ARG                # not an FP8-output plan
    torch.cuda.synchronize()


# ------------------------------------------------------------------ MLP block
def mlp_problem(m, d_model, d_ff, dtype, act, layout, seed):
    std = 1.0 if dtype == "e4m3" else 1.0 / 16
    up = Workload("mlp_up", m, d_ff, d_model, dtype, act, "col", layout, ("normal", 1.0), ("normal", std),
                  ("normal", 0.1), seed=seed)
    down = Workload("mlp_down", m, d_model, d_ff, dtype, "bias", "col", layout, ("normal", 1.0),
                    ("normal", std), ("normal", 0.1), seed=seed + 1)
    return up, make_problem(up), down, make_problem(down)


def run_mlp(m, d_model, d_ff, dtype, act, layout, seed, rows=None, fused=True):
    up, pu, down, pd = mlp_problem(m, d_model, d_ff, dtype, act, layout, seed)
    X, W1, b1, W2, b2 = storage(pu.A), storage(pu.B), storage(pu.bias), storage(pd.B), storage(pd.bias)
    # the oracle on all rows (or on the sampled rows: MLP rows are independent)
    Xo = X if rows is None else np.ascontiguousarray(X[rows])
    if dtype == "e4m3":
        _, H0, _, amax0 = oracle.mlp(Xo, W1, b1, W2, b2, dtype="e4m3", act=act, w_layout=layout,
                                     scale_x=pu.scale_a, scale_w1=pu.scale_b, scale_h=1.0, scale_w2=pd.scale_b,
                                     stepwise=not fused)
        s_h = (amax0 if rows is None else float(np.abs(H0).max())) / 448.0
        if rows is not None:
            s_h *= 1.5                 # leave headroom for rows the sample did not see
        s_h = float(np.float32(s_h))   # the fp32 value the GPU reads
    else:
        s_h = 1.0
    # the unfused sequence is checked against the oracle's stepwise reading (each product
    # rounded to the 16-bit type before its bias, H rounded before it is quantised)
    Y_ref, H_ref, Hs_ref, amax_ref = oracle.mlp(Xo, W1, b1, W2, b2, dtype=dtype, act=act, w_layout=layout,
                                                scale_x=pu.scale_a, scale_w1=pu.scale_b, scale_h=s_h,
                                                scale_w2=pd.scale_b, stepwise=not fused)
    h_t = torch.uint8 if dtype == "e4m3" else TORCH_DTYPE[dtype]
    H = torch.full((m, d_ff), 0x7F if dtype == "e4m3" else 0, dtype=h_t, device="cuda")
    Y = torch.full((m, d_model), float("nan"), dtype=TORCH_DTYPE[up.out_dtype], device="cuda")
    amax = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    with g.MlpPlan(m, d_model, d_ff, dtype, act, layout) as mp:
        if dtype == "e4m3":
            mp.set_scales(_f32(pu.scale_a), _f32(pu.scale_b), _f32(s_h), amax, _f32(pd.scale_b))
        Hw = torch.empty((m, d_ff), dtype=torch.bfloat16, device="cuda") if not fused else None
        mp.run(pu.A.cuda(), pu.B.cuda(), pu.bias.cuda(), pd.B.cuda(), pd.bias.cuda(), H, Y, fused=fused, H_wide=Hw)
        mp.check()
        info = mp.info
    torch.cuda.synchronize()
    Hc, Yc = H.cpu(), Y.cpu()
    if rows is not None:
        Hc, Yc = Hc[torch.as_tensor(rows)], Yc[torch.as_tensor(rows)]
    # H: quantised (e4m3) or rounded (16-bit) codes within the band of the oracle's H
    sa1, sb1 = sigmas(pu)
    tol_h = tolerance(H_ref, "bf16" if dtype == "e4m3" else dtype, d_model, sa1, sb1)   # decision band
    hband_lo = oracle.encode(H_ref / s_h - tol_h / s_h, dtype)
    hband_hi = oracle.encode(H_ref / s_h + tol_h / s_h, dtype)
    hcodes = Hc.numpy() if dtype == "e4m3" else Hc.view(torch.int16).numpy().view(np.uint16)
    check_codes(hcodes, H_ref, tol_h, s_h, dtype)
    if dtype == "e4m3" and rows is None:
        assert abs(float(amax.item()) - amax_ref) <= tol_h.max()
    # Y within the down-projection's tolerance, sigma_H from the oracle's stored H
    sh = float(oracle.decode(Hs_ref, dtype).std()) * s_h
    sw2 = float(pd.B.double().std(unbiased=False)) * pd.scale_b
    tol_y = tolerance(Y_ref, dtype, d_ff, sh, sw2)
    if not fused:
        # The unfused path rounds each product to the 16-bit type before its bias (one ulp of
        # |Y - b2| for the down-projection) and its H differs from the oracle's wherever the two
        # product roundings disagree.  Bounds from the oracle's values alone:
        out16 = "bf16" if dtype == "e4m3" else dtype
        ulp = OUT_ULP[out16]
        b2v = oracle.decode(storage(pd.bias), out16)
        tol_y = tol_y + ulp * np.abs(Y_ref - b2v[None, :])
        w2 = np.abs(oracle.decode(storage(pd.B), dtype)) * pd.scale_b
        w2 = w2 if layout == "kn" else w2.T
        if dtype == "e4m3":
            # an e4m3 code the decision band leaves open may land on either neighbour
            dec = lambda c: oracle.decode(c, "e4m3")
            step = (dec(hband_hi) - dec(hband_lo)) * s_h             # 0 where the code is unique
            tol_y = tol_y + step @ w2
        else:
            # a 16-bit H element may be off by up to two ulps (one from its product's rounding,
            # carried through the activation, one from its own rounding)
            tol_y = tol_y + 2 * ulp * (np.abs(H_ref) @ w2)
    y = Yc.double().numpy()
    bad = ~(np.abs(y - Y_ref) <= tol_y)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} Y outside tolerance; first {np.argwhere(bad)[:3]}"
    return info


@pytest.mark.parametrize("layout", ["kn", "nk"])
@pytest.mark.parametrize("act", ["gelu_bias", "relu_bias", "bias"])
@pytest.mark.parametrize("dtype", ["e4m3", "bf16", "f16"])
def test_mlp_block(dtype, act, layout):
    run_mlp(200, 256, 512, dtype, act, layout, seed=35)


@pytest.mark.parametrize("m", [48, 200])
@pytest.mark.parametrize("dtype", ["e4m3", "bf16"])
def test_mlp_block_unfused_baseline(dtype, m):
    """The unfused sequence (bare GEMM, bias + activation, amax, quantise, bare GEMM, bias)
    against the oracle's stepwise reading of that sequence."""
    run_mlp(m, 256, 512, dtype, "gelu_bias", "kn", seed=39, fused=False)


@pytest.mark.parametrize("m", [16, 32, 64, 1000])
def test_mlp_block_batch_sizes(m):
    up, down = run_mlp(m, 512, 1024, "e4m3", "gelu_bias", "kn", seed=36)
    if m <= 64:
        assert up["kernel"] == g.KERNEL_SPLITK and down["kernel"] == g.KERNEL_SPLITK
    else:
        assert up["kernel"] != g.KERNEL_SPLITK and down["kernel"] != g.KERNEL_SPLITK


def test_mlp_block_fp8_full_size_sampled():
    """8192 tokens, d_model 4096, d_ff 14336 (the FP8 up-projection's shape): the oracle on 16
    seeded rows (rows of an MLP are independent)."""
    rows = np.sort(np.random.default_rng(37).choice(8192, 16, replace=False))
    rows[0], rows[-1] = 0, 8191
    up, down = run_mlp(8192, 4096, 14336, "e4m3", "gelu_bias", "kn", seed=37, rows=rows)
    assert up["kernel"] == g.KERNEL_TC2


def test_mlp_argument_errors():
    def status(fn):
        with pytest.raises(g.GemmEpiError) as e:
            fn()
        return e.value.status

    assert status(lambda: g.MlpPlan(64, 256, 512, "bf16", "tanh_bias")) == g.ERR_ARG
    with g.MlpPlan(64, 256, 512, "bf16", "gelu_bias") as mp:
        one = _f32(1.0)
        assert status(lambda: mp.set_scales(one, one, one, None, one)) == g.ERR_ARG   # 16-bit: no scales
    with g.MlpPlan(256, 256, 512, "e4m3", "gelu_bias") as mp:
        X = torch.zeros((256, 256), dtype=torch.uint8, device="cuda")
        W = torch.zeros((256, 512), dtype=torch.uint8, device="cuda")
        b = torch.zeros((512,), dtype=torch.bfloat16, device="cuda")
        H = torch.zeros((256, 512), dtype=torch.uint8, device="cuda")
        Y = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
        assert status(lambda: mp.run(X, W, b, W, b[:256], H, Y)) == g.ERR_NULL       # scales unset
        one = _f32(1.0)
        assert status(lambda: mp.set_scales(one, one, None, None, one)) == g.ERR_NULL
    torch.cuda.synchronize()
