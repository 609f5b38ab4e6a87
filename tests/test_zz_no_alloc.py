"""gemm_epi_run_noalloc: the fused run for callers that may not allocate device memory.

Some callers cannot call cudaMalloc: code running inside a host framework that
owns all device memory through its own pool and forbids side allocations, or
code on a latency-critical path that cannot pay for cudaMalloc/cudaFree and
their implicit synchronisation.  They cannot create a plan (a plan allocates
its status word), so the library offers one entry point that keeps its only
scratch -- the kernels' timeout status word -- in a static device array.

This file checks, through the C ABI, that two calls in a row of that entry
point give the same results as the plan-based gemm_epi_run on the same inputs,
within the tolerance the parity tests use, and that each call also matches the
fp64 oracle element by element.  The mask is compared bit for bit wherever the
oracle's pre-activation lies outside the tolerance band (inside it, several
roundings are correct: the no-alloc call runs without the split tail, so its
sums may be taken in another order than the plan's).  It is collected last and
builds everything it needs itself, so it passes alone in a fresh process as
well as after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from helpers import aux_padding_bits, band, tolerance, unpack_aux

from activation_epilogue_tcgen05_b200 import gemm_epi as g
from activation_epilogue_tcgen05_b200.workloads import TORCH_DTYPE, Workload, make_problem, storage

pytestmark = pytest.mark.gpu

CASES = [
    # persistent tensor-core kernel, ragged edges, mask output
    Workload("noalloc_tc", 200, 272, 328, "bf16", "relu_aux_bias", "row", "kn", seed=21),
    # small-m split-K cluster kernel (an nn.Linear weight), GELU
    Workload("noalloc_sk", 16, 512, 1024, "f16", "gelu_bias", "col", "nk", seed=22,
             dist_b=("uniform", 1 / 64), dist_bias=("uniform", 1 / 64)),
    # FP8 operands with per-tensor scales
    Workload("noalloc_fp8", 256, 384, 512, "e4m3", "gelu_bias", "col", "kn", seed=23),
]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available() or torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs an sm_100 GPU")
    from activation_epilogue_tcgen05_b200 import build
    build.build()
    oracle.build()
    g.lib()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _outputs(wl):
    D = torch.full((wl.m, wl.n), float("nan"), dtype=TORCH_DTYPE[wl.out_dtype], device="cuda")
    aux = None
    if wl.epilogue == "relu_aux_bias":
        aux = torch.full((wl.m * g.aux_pitch_words(wl.n),), -1, dtype=torch.int32, device="cuda")
    return D, aux


@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_plan_run_twice(wl):
    p = make_problem(wl)
    A, B, bias = p.A.cuda(), p.B.cuda(), p.bias.cuda()
    sa = torch.tensor([p.scale_a], dtype=torch.float32, device="cuda")
    sb = torch.tensor([p.scale_b], dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    s = ctypes.c_void_p(stream.cuda_stream)
    codes = (g.DTYPE[wl.dtype], g.EPILOGUE[wl.epilogue], g.AXIS[wl.bias_axis], g.LAYOUT[wl.b_layout])

    # the existing entry point: plan + gemm_epi_run
    D_ref, aux_ref = _outputs(wl)
    with g.Plan(wl.m, wl.n, wl.k, wl.dtype, wl.epilogue, wl.bias_axis, wl.b_layout) as plan:
        if wl.dtype == "e4m3":
            plan.set_scales(sa, sb)
        plan.run(A, B, bias, D_ref, aux_ref, stream=stream)
        plan.check(stream)
    d_plan = D_ref.double().cpu().numpy()

    # the fp64 oracle on the same stored inputs
    o_ref, o_pre, o_mask = oracle.gemm_epi(storage(p.A), storage(p.B), storage(p.bias), dtype=wl.dtype,
                                           epilogue=wl.epilogue, bias_axis=wl.bias_axis,
                                           b_layout=wl.b_layout, scale_a=p.scale_a, scale_b=p.scale_b)
    sigma_a = float(p.A.double().std(unbiased=False)) * p.scale_a
    sigma_b = float(p.B.double().std(unbiased=False)) * p.scale_b
    tol_oracle = tolerance(o_ref, wl.dtype, wl.k, sigma_a, sigma_b)
    tol_plan = tolerance(d_plan, wl.dtype, wl.k, sigma_a, sigma_b)
    exact = band(o_pre, wl.dtype, wl.k, sigma_a, sigma_b)     # mask bits that must be exact
    assert bool((np.abs(d_plan - o_ref) <= tol_oracle).all()), "gemm_epi_run disagrees with the oracle"

    for call in range(2):                       # two calls in a row share the static scratch
        D, aux = _outputs(wl)
        rc = g.lib().gemm_epi_run_noalloc(wl.m, wl.n, wl.k, *codes, _ptr(A), _ptr(B), _ptr(bias),
                                          _ptr(sa), _ptr(sb), _ptr(D), _ptr(aux), 1, s)
        assert rc == g.OK, f"call {call}: {g.gemm_epi_status_string(rc)}"
        d = D.double().cpu().numpy()            # NaN (an unwritten output) fails both checks
        bad_plan = ~(np.abs(d - d_plan) <= tol_plan)
        assert not bad_plan.any(), f"call {call}: {int(bad_plan.sum())} outputs differ from gemm_epi_run"
        bad_oracle = ~(np.abs(d - o_ref) <= tol_oracle)
        assert not bad_oracle.any(), f"call {call}: {int(bad_oracle.sum())} outputs outside the oracle's tolerance"
        if aux is not None:
            words = aux.cpu().numpy().view(np.uint32)
            words_plan = aux_ref.cpu().numpy().view(np.uint32)
            bits = unpack_aux(words, wl.m, wl.n)
            assert not (exact & (bits != o_mask)).any(), f"call {call}: mask bits differ from the oracle"
            assert not (exact & (bits != unpack_aux(words_plan, wl.m, wl.n))).any(), \
                f"call {call}: mask bits differ from gemm_epi_run"
            assert aux_padding_bits(words, wl.m, wl.n) == 0, f"call {call}: mask padding bits set"


def test_noalloc_rejects_bad_requests():
    wl = CASES[0]
    p = make_problem(wl)
    A, B, bias = p.A.cuda(), p.B.cuda(), p.bias.cuda()
    D, aux = _outputs(wl)
    L = g.lib()
    args = (g.BF16, g.RELU_AUX_BIAS, g.BIAS_ROW, g.B_KN)
    # a size beyond the entry point's limit
    assert L.gemm_epi_run_noalloc(1 << 31, wl.n, wl.k, *args, _ptr(A), _ptr(B), _ptr(bias), None,
                                  None, _ptr(D), _ptr(aux), 1, None) == g.ERR_ARG
    # the mask buffer is required for RELU_AUX_BIAS
    assert L.gemm_epi_run_noalloc(wl.m, wl.n, wl.k, *args, _ptr(A), _ptr(B), _ptr(bias), None,
                                  None, _ptr(D), None, 1, None) == g.ERR_NULL
    # E4M3 needs its scales
    wl8 = CASES[2]
    p8 = make_problem(wl8)
    A8, B8, bias8 = p8.A.cuda(), p8.B.cuda(), p8.bias.cuda()
    D8, _ = _outputs(wl8)
    assert L.gemm_epi_run_noalloc(wl8.m, wl8.n, wl8.k, g.E4M3, g.GELU_BIAS, g.BIAS_COL, g.B_KN,
                                  _ptr(A8), _ptr(B8), _ptr(bias8), None, None, _ptr(D8), None, 1,
                                  None) == g.ERR_NULL
