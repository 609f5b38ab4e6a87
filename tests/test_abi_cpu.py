"""The C-ABI library on a machine without a GPU: it loads, exports every symbol
include/gemm_epi.h declares, and its host-side validation answers without
touching a device.  No compute call is made here."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gemm_epi.h")


@pytest.fixture(scope="module")
def g():
    from activation_epilogue_tcgen05_b200 import build, gemm_epi
    build.build()
    gemm_epi.lib()
    return gemm_epi


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gemm_epi_[a-z_]+)\s*\(", text)))


def test_header_declares_expected_entry_points(g):
    assert declared_functions() == sorted(g.EXPORTS)


def test_library_exports_every_declared_symbol(g):
    lib = g.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", g.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (gemm_epi_\w+)", out))
    assert set(declared_functions()) <= exported


def test_library_exports_only_the_c_abi(g):
    out = subprocess.run(["nm", "-D", "--defined-only", g.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (gemm_epi_\w+)", out))
    assert exported == set(declared_functions())


def test_small_helpers(g):
    assert g.gemm_epi_version() >= 100
    assert g.gemm_epi_aux_pitch_bytes(1) == 16
    assert g.gemm_epi_aux_pitch_bytes(128) == 16
    assert g.gemm_epi_aux_pitch_bytes(129) == 32
    assert g.gemm_epi_aux_pitch_bytes(4096) == 512
    assert g.gemm_epi_aux_pitch_bytes(14336) == 1792
    assert g.gemm_epi_aux_pitch_bytes(0) == 0
    for code in range(-7, 1):
        s = g.gemm_epi_status_string(code)
        assert s and s != "unknown status"
    assert g.gemm_epi_status_string(-99) == "unknown status"


def _plan_rc(g, m, n, k, dt=1, epi=1, axis=0, layout=0, opts=None):
    h = ctypes.c_void_p()
    return g.lib().gemm_epi_plan_opts(m, n, k, dt, epi, axis, layout,
                                      ctypes.byref(opts) if opts else None, ctypes.byref(h))


@pytest.mark.parametrize("args", [
    (0, 64, 64), (64, 0, 64), (64, 64, 0), (-1, 64, 64), (1 << 31, 64, 64),
])
def test_plan_rejects_bad_sizes(g, args):
    assert _plan_rc(g, *args) == g.ERR_ARG


@pytest.mark.parametrize("kw", [dict(dt=3), dict(dt=-1), dict(epi=12), dict(epi=-1), dict(axis=2),
                                dict(layout=4)])
def test_plan_rejects_bad_enums(g, kw):
    assert _plan_rc(g, 64, 64, 64, **kw) == g.ERR_ARG


@pytest.mark.parametrize("opts", [
    dict(kernel=4), dict(kernel=-1), dict(block_n=64), dict(block_n=192), dict(split_k=9),
    dict(split_k=-1), dict(max_ctas=-1), dict(inject_stall=2), dict(stream_k=3), dict(stream_k=-1),
])
def test_plan_rejects_bad_options(g, opts):
    o = g.Options(**{**dict(kernel=0, block_n=0, split_k=0, max_ctas=0, inject_stall=0,
                            stream_k=0), **opts})
    assert _plan_rc(g, 64, 64, 64, opts=o) == g.ERR_ARG


@pytest.mark.parametrize("m,n,k,dt", [
    (64, 64, 60, 1),     # k*2 = 120 B: not a multiple of 16
    (64, 60, 64, 0),     # n*2 = 120 B
    (64, 64, 40, 2),     # e4m3: k = 40 bytes
    (64, 56, 64, 2),     # e4m3: n = 56 bytes (B (k, n) pitch)
])
def test_plan_rejects_unaligned_pitches(g, m, n, k, dt):
    assert _plan_rc(g, m, n, k, dt=dt) == g.ERR_ALIGN


def test_valid_plan_without_gpu_reports_no_device(g):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _plan_rc(g, 4096, 4096, 4096, dt=1, epi=3) == g.ERR_NO_DEVICE
    with pytest.raises(g.GemmEpiError) as e:
        g.Plan(128, 128, 128)
    assert e.value.status == g.ERR_NO_DEVICE


def test_null_and_unknown_handles_rejected(g):
    lib = g.lib()
    assert lib.gemm_epi_run(None, None, None, None, None, None, None) == g.ERR_ARG
    assert lib.gemm_epi_free(None) == g.ERR_ARG
    bogus = ctypes.c_void_p(0x1000)
    assert lib.gemm_epi_run(bogus, None, None, None, None, None, None) == g.ERR_ARG
    assert lib.gemm_epi_free(bogus) == g.ERR_ARG
    assert lib.gemm_epi_set_scales(bogus, None, None) == g.ERR_ARG
    assert lib.gemm_epi_check(bogus, None) == g.ERR_ARG
    info = g.PlanInfo()
    assert lib.gemm_epi_plan_query(bogus, ctypes.byref(info)) == g.ERR_ARG
    h = ctypes.c_void_p()
    assert lib.gemm_epi_plan(64, 64, 64, 1, 1, 0, None) == g.ERR_ARG
    del h


def test_binding_fails_loudly_without_library(tmp_path):
    code = (
        "import activation_epilogue_tcgen05_b200.gemm_epi as g\n"
        f"g.LIB_PATH = {str(tmp_path / 'missing.so')!r}\n"
        "try:\n    g.lib()\nexcept RuntimeError as e:\n    print('RAISED', e)\n"
    )
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert "RAISED" in r.stdout and "no fallback" in r.stdout


def test_product_does_not_import_oracle():
    """Nothing under the package imports or opens the oracle."""
    pkg = os.path.join(ROOT, "activation_epilogue_tcgen05_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text
                assert "gemm_epi_oracle" not in text and "libgemm_epi_oracle" not in text


def test_backward_entry_points_reject_bad_handles(g):
    for fn in (g.lib().gemm_epi_run_bwd, g.lib().gemm_epi_unfused_run_bwd):
        assert fn(None, None, None, None, None, None, None) == g.ERR_ARG
        assert fn(ctypes.c_void_p(0x1000), None, None, None, None, None, None) == g.ERR_ARG


@pytest.mark.parametrize("epi", [10, 11])
def test_backward_epilogues_are_valid_enums(g, epi):
    # accepted as enums: without a device the plan stops at the device check
    assert _plan_rc(g, 64, 64, 64, epi=epi) == g.ERR_NO_DEVICE


@pytest.mark.parametrize("epi", [10, 11])
def test_noalloc_refuses_backward_epilogues(g, epi):
    rc = g.lib().gemm_epi_run_noalloc(64, 64, 64, 1, epi, 0, 0, None, None, None, None, None, None, None,
                                      0, None)
    assert rc == g.ERR_ARG


def test_fp8_output_option_checks_before_the_device(g):
    o = g.Options(kernel=0, block_n=0, split_k=0, max_ctas=0, inject_stall=0, stream_k=0, out_e4m3=2)
    assert _plan_rc(g, 64, 64, 64, dt=2, epi=1, opts=o) == g.ERR_ARG
    o.out_e4m3 = 1
    assert _plan_rc(g, 64, 64, 64, dt=1, epi=1, opts=o) == g.ERR_UNSUPPORTED      # bf16 operands
    assert _plan_rc(g, 64, 64, 64, dt=2, epi=3, opts=o) == g.ERR_UNSUPPORTED      # RELU_AUX_BIAS
    assert _plan_rc(g, 64, 64, 64, dt=2, epi=4, opts=o) == g.ERR_NO_DEVICE        # GELU_BIAS: valid
    assert g.lib().gemm_epi_set_out_scale(None, None, None) == g.ERR_ARG


def test_mlp_entry_points_reject_bad_handles_and_acts(g):
    L = g.lib()
    h = ctypes.c_void_p()
    assert L.gemm_epi_mlp_plan(64, 64, 128, 1, 5, 0, ctypes.byref(h)) == g.ERR_ARG   # TANH_BIAS
    assert L.gemm_epi_mlp_plan(64, 64, 128, 1, 4, 0, None) == g.ERR_ARG
    assert L.gemm_epi_mlp_plan(64, 64, 128, 1, 4, 0, ctypes.byref(h)) == g.ERR_NO_DEVICE
    for bad in (None, ctypes.c_void_p(0x1000)):
        assert L.gemm_epi_mlp_set_scales(bad, None, None, None, None, None) == g.ERR_ARG
        assert L.gemm_epi_mlp_run(bad, None, None, None, None, None, None, None, None) == g.ERR_ARG
        assert L.gemm_epi_mlp_unfused_run(bad, None, None, None, None, None, None, None, None, None) == g.ERR_ARG
        assert L.gemm_epi_mlp_check(bad, None) == g.ERR_ARG
        assert L.gemm_epi_mlp_free(bad) == g.ERR_ARG


def test_layout_flags_checked_before_the_device(g):
    assert _plan_rc(g, 64, 64, 64, layout=4) == g.ERR_ARG                   # unknown flag
    assert _plan_rc(g, 100, 64, 64, dt=0, layout=2) == g.ERR_ALIGN          # A (k, m): m*2 = 200 B
    assert _plan_rc(g, 104, 64, 64, dt=0, layout=3) == g.ERR_NO_DEVICE      # valid: A (k, m), B (n, k)
    h = ctypes.c_void_p()
    assert g.lib().gemm_epi_mlp_plan(64, 64, 128, 1, 4, 2, ctypes.byref(h)) == g.ERR_ARG   # MLP: B layouts only


def test_plan_rejects_tile_counts_beyond_int(g):
    # m, n each below 2^31 but (m/128) * (n/128) above it
    assert _plan_rc(g, (1 << 31) - 1, 1 << 28, 64) == g.ERR_ARG
