"""Run the CUDA path through the C ABI and compare it with the oracle.

Inputs come from the seeded generators (activation_epilogue_tcgen05_b200.workloads);
the expected values come only from ``oracle``.  Output buffers are pre-filled
with sentinels (NaN for D, 0xA5A5A5A5 for mask words) so anything the kernel
fails to write shows up as a mismatch.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from helpers import aux_padding_bits, band, tolerance, unpack_aux

from activation_epilogue_tcgen05_b200 import gemm_epi as g
from activation_epilogue_tcgen05_b200.workloads import TORCH_DTYPE, Problem, Workload, storage

SENTINEL_WORD = np.int32(np.uint32(0xA5A5A5A5).view(np.int32))


def device_inputs(prob: Problem, device="cuda"):
    return (prob.A.to(device), prob.B.to(device), prob.bias.to(device))


def alloc_outputs(wl: Workload, device="cuda"):
    D = torch.full((wl.m, wl.n), float("nan"), dtype=TORCH_DTYPE[wl.out_dtype], device=device)
    aux = None
    if wl.epilogue in g.HAS_AUX:
        words = wl.m * g.aux_pitch_words(wl.n)
        aux = torch.full((words,), int(SENTINEL_WORD), dtype=torch.int32, device=device)
    return D, aux


def make_plan(wl: Workload, prob: Problem, device="cuda", **opts):
    plan = g.Plan(wl.m, wl.n, wl.k, wl.dtype, wl.epilogue, wl.bias_axis, wl.b_layout, a_layout=wl.a_layout,
                  **opts)
    if wl.dtype == "e4m3" or prob.scale_a != 1.0 or prob.scale_b != 1.0:
        sa = torch.tensor([prob.scale_a], dtype=torch.float32, device=device)
        sb = torch.tensor([prob.scale_b], dtype=torch.float32, device=device)
        plan.set_scales(sa, sb)
    return plan


def gpu_run(wl: Workload, prob: Problem, fused=True, inputs=None, **opts):
    """One run through gemm_epi_run (or the unfused path); returns host D, aux words, plan info."""
    A, B, bias = inputs if inputs is not None else device_inputs(prob)
    if wl.epilogue not in g.HAS_BIAS:
        bias = None                      # bias-free epilogues take a NULL bias
    D, aux = alloc_outputs(wl)
    plan = make_plan(wl, prob, **opts)
    try:
        plan.run(A, B, bias, D, aux, fused=fused)
        plan.check()
        info = plan.info
    finally:
        plan.close()
    torch.cuda.synchronize()
    words = None if aux is None else aux.cpu().numpy().view(np.uint32)
    return D.cpu(), words, info


def _pop_std(t: torch.Tensor, limit: int = 1 << 24) -> float:
    flat = t.reshape(-1)
    if flat.numel() > limit:                 # large operands: a seeded 2^20-element sample
        gen = torch.Generator(device="cpu").manual_seed(0)
        idx = torch.randint(0, flat.numel(), (1 << 20,), generator=gen).to(flat.device)
        flat = flat[idx]
    return float(flat.double().std(unbiased=False))


def sigmas(prob: Problem):
    """Population std (fp64) of the operand values the product uses (dequantised)."""
    return _pop_std(prob.A) * abs(prob.scale_a), _pop_std(prob.B) * abs(prob.scale_b)


def oracle_full(wl: Workload, prob: Problem):
    return oracle.gemm_epi(storage(prob.A), storage(prob.B), storage(prob.bias), dtype=wl.dtype,
                           epilogue=wl.epilogue, bias_axis=wl.bias_axis, b_layout=wl.b_layout,
                           scale_a=prob.scale_a, scale_b=prob.scale_b, a_layout=wl.a_layout)


def compare(wl, D_gpu, words, ref, pre, mask, sa, sb, rows=None, cols=None, extra=None):
    """Assert elementwise tolerance on D and exactness of the mask outside the band.

    ``extra`` (same shape as ref) widens both bounds, for paths with an
    additional rounding step (the unfused baseline)."""
    d = D_gpu.double().numpy()
    if rows is not None:
        d = d[rows, cols]
    tol = tolerance(ref, wl.dtype, wl.k, sa, sb)
    if extra is not None:
        tol = tol + extra
    err = np.abs(d - ref)
    ok = err <= tol                       # NaN (unwritten) compares False
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        detail = [(tuple(int(v) for v in i), float(d[tuple(i)]), float(ref[tuple(i)]),
                   float(tol[tuple(i)])) for i in idx]
        raise AssertionError(f"{int((~ok).sum())} of {ok.size} outputs outside tolerance; first "
                             f"(index, gpu, ref, tol): {detail}")
    if wl.epilogue in g.HAS_AUX:
        bits = unpack_aux(words, wl.m, wl.n)
        if rows is not None:
            bits = bits[rows, cols]
        exact = band(pre, wl.dtype, wl.k, sa, sb)
        if extra is not None:
            exact &= np.abs(pre) > tolerance(pre, wl.dtype, wl.k, sa, sb) + extra
        wrong = exact & (bits != mask)
        assert not wrong.any(), f"{int(wrong.sum())} mask bits differ outside the tolerance band"
        assert aux_padding_bits(words, wl.m, wl.n) == 0, "mask padding bits are not zero"
    return float((err / np.maximum(tol, 1e-30)).max())


def check_against_oracle(wl: Workload, prob: Problem, fused=True, **opts):
    D, words, info = gpu_run(wl, prob, fused=fused, **opts)
    ref, pre, mask = oracle_full(wl, prob)
    sa, sb = sigmas(prob)
    worst = compare(wl, D, words, ref, pre, mask, sa, sb)
    return worst, info


def sampled_oracle(wl: Workload, prob: Problem, rows, cols):
    """Oracle at positions (rows, cols), passing only the needed rows of A (and bias)."""
    ur, inv = np.unique(rows, return_inverse=True)
    A_rows = storage(prob.A[torch.as_tensor(ur, device=prob.A.device)])
    Bs = storage(prob.B)
    bias = storage(prob.bias)
    if wl.bias_axis == "row":
        bias = np.ascontiguousarray(bias[ur])
    return oracle.gemm_epi_sampled(A_rows, Bs, bias, inv.astype(np.int64), np.asarray(cols, np.int64),
                                   dtype=wl.dtype, epilogue=wl.epilogue, bias_axis=wl.bias_axis,
                                   b_layout=wl.b_layout, scale_a=prob.scale_a, scale_b=prob.scale_b)


# One unit in the last place, relative, of the output type: the unfused path
# rounds alpha*A.B to the output type before the bias is added.
OUT_ULP = {"f16": 2.0 ** -10, "bf16": 2.0 ** -7, "e4m3": 2.0 ** -7}


def unfused_extra(wl: Workload, prob: Problem, pre):
    """|alpha*A.B| * ulp(out): the unfused path's additional rounding of the product."""
    from oracle import decode
    if wl.epilogue not in g.HAS_BIAS:
        return OUT_ULP[wl.out_dtype] * np.abs(pre)
    b = decode(storage(prob.bias), wl.out_dtype)
    b = b[:, None] if wl.bias_axis == "row" else b[None, :]
    return OUT_ULP[wl.out_dtype] * np.abs(pre - b)
