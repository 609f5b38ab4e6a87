"""ctypes binding of the C ABI in ``include/gemm_epi.h`` (argument marshalling only).

The functions keep the C names and signatures; every step of the computation
runs in the CUDA library.  ``Plan`` is a small convenience wrapper that takes
torch tensors (device memory, the current stream) and passes their raw
pointers through the same entry points.

If ``libgemm_epi.so`` has not been built, loading raises ``RuntimeError``:
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgemm_epi.so")

# enums (include/gemm_epi.h)
F16, BF16, E4M3 = 0, 1, 2
NONE, BIAS, RELU_BIAS, RELU_AUX_BIAS, GELU_BIAS = 0, 1, 2, 3, 4
TANH_BIAS, RELU, RELU_AUX, GELU, TANH = 5, 6, 7, 8, 9
DRELU, DRELU_BGRAD = 10, 11
BIAS_ROW, BIAS_COL = 0, 1
B_KN, B_NK = 0, 1
A_KM = 2          # layout flag: A stored (k, m)
KERNEL_AUTO, KERNEL_TC1, KERNEL_TC2, KERNEL_SPLITK = 0, 1, 2, 3
OK, ERR_ARG, ERR_ALIGN, ERR_NULL, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NO_DEVICE = \
    0, -1, -2, -3, -4, -5, -6, -7

DTYPE = {"f16": F16, "bf16": BF16, "e4m3": E4M3}
EPILOGUE = {"none": NONE, "bias": BIAS, "relu_bias": RELU_BIAS, "relu_aux_bias": RELU_AUX_BIAS,
            "gelu_bias": GELU_BIAS, "tanh_bias": TANH_BIAS, "relu": RELU, "relu_aux": RELU_AUX,
            "gelu": GELU, "tanh": TANH, "drelu": DRELU, "drelu_bgrad": DRELU_BGRAD}
HAS_BIAS = {"bias", "relu_bias", "relu_aux_bias", "gelu_bias", "tanh_bias"}
HAS_AUX = {"relu_aux_bias", "relu_aux"}
BACKWARD = {"drelu", "drelu_bgrad"}
AXIS = {"row": BIAS_ROW, "col": BIAS_COL}
LAYOUT = {"kn": B_KN, "nk": B_NK}
KERNEL = {"auto": KERNEL_AUTO, "tc1": KERNEL_TC1, "tc2": KERNEL_TC2, "splitk": KERNEL_SPLITK}
STREAM_K = {"auto": 0, "off": 1, "on": 2}

# every symbol include/gemm_epi.h declares
EXPORTS = ("gemm_epi_plan", "gemm_epi_plan_ex", "gemm_epi_plan_opts", "gemm_epi_set_scales",
           "gemm_epi_run", "gemm_epi_unfused_run", "gemm_epi_check", "gemm_epi_plan_query",
           "gemm_epi_free", "gemm_epi_status_string", "gemm_epi_aux_pitch_bytes",
           "gemm_epi_version", "gemm_epi_run_noalloc", "gemm_epi_run_bwd", "gemm_epi_unfused_run_bwd",
           "gemm_epi_set_out_scale", "gemm_epi_mlp_plan", "gemm_epi_mlp_set_scales", "gemm_epi_mlp_run",
           "gemm_epi_mlp_check", "gemm_epi_mlp_query", "gemm_epi_mlp_free", "gemm_epi_mlp_unfused_run",
           "gemm_epi_plan_preview")


class Options(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("block_n", ctypes.c_int32),
                ("split_k", ctypes.c_int32), ("max_ctas", ctypes.c_int32),
                ("inject_stall", ctypes.c_int32), ("stream_k", ctypes.c_int32),
                ("out_e4m3", ctypes.c_int32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in
                ("kernel", "block_m", "block_n", "block_k", "stages", "split_k", "grid", "cluster",
                 "threads", "smem_bytes", "tiles", "sk_tiles", "sk_split", "group_m", "group_n")]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class GemmEpiError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None
_lock = threading.Lock()


def lib():
    """Load libgemm_epi.so (raises RuntimeError when it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m activation_epilogue_tcgen05_b200.build` (no fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
            pp = ctypes.POINTER(vp)
            L.gemm_epi_plan.argtypes = [i64, i64, i64, i32, i32, i32, pp]
            L.gemm_epi_plan_ex.argtypes = [i64, i64, i64, i32, i32, i32, i32, pp]
            L.gemm_epi_plan_opts.argtypes = [i64, i64, i64, i32, i32, i32, i32,
                                             ctypes.POINTER(Options), pp]
            L.gemm_epi_set_scales.argtypes = [vp, vp, vp]
            L.gemm_epi_run.argtypes = [vp, vp, vp, vp, vp, vp, vp]
            L.gemm_epi_unfused_run.argtypes = [vp, vp, vp, vp, vp, vp, vp]
            L.gemm_epi_run_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp]
            L.gemm_epi_unfused_run_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp]
            L.gemm_epi_set_out_scale.argtypes = [vp, vp, vp]
            L.gemm_epi_mlp_plan.argtypes = [i64, i64, i64, i32, i32, i32, pp]
            L.gemm_epi_mlp_set_scales.argtypes = [vp, vp, vp, vp, vp, vp]
            L.gemm_epi_mlp_run.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.gemm_epi_mlp_unfused_run.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.gemm_epi_mlp_check.argtypes = [vp, vp]
            L.gemm_epi_mlp_query.argtypes = [vp, ctypes.POINTER(PlanInfo), ctypes.POINTER(PlanInfo)]
            L.gemm_epi_mlp_free.argtypes = [vp]
            L.gemm_epi_check.argtypes = [vp, vp]
            L.gemm_epi_plan_query.argtypes = [vp, ctypes.POINTER(PlanInfo)]
            L.gemm_epi_plan_preview.argtypes = [i64, i64, i64, i32, i32, i32, i32,
                                                ctypes.POINTER(Options), i32, ctypes.POINTER(PlanInfo)]
            L.gemm_epi_free.argtypes = [vp]
            L.gemm_epi_status_string.argtypes = [i32]
            L.gemm_epi_status_string.restype = ctypes.c_char_p
            L.gemm_epi_aux_pitch_bytes.argtypes = [i64]
            L.gemm_epi_aux_pitch_bytes.restype = i64
            L.gemm_epi_version.argtypes = []
            L.gemm_epi_run_noalloc.argtypes = [i64, i64, i64, i32, i32, i32, i32, vp, vp, vp, vp,
                                               vp, vp, vp, i32, vp]
            for name in ("gemm_epi_plan", "gemm_epi_plan_ex", "gemm_epi_plan_opts",
                         "gemm_epi_set_scales", "gemm_epi_run", "gemm_epi_unfused_run",
                         "gemm_epi_check", "gemm_epi_plan_query", "gemm_epi_free",
                         "gemm_epi_version", "gemm_epi_run_noalloc", "gemm_epi_run_bwd",
                         "gemm_epi_unfused_run_bwd", "gemm_epi_set_out_scale", "gemm_epi_mlp_plan",
                         "gemm_epi_mlp_set_scales", "gemm_epi_mlp_run", "gemm_epi_mlp_check",
                         "gemm_epi_mlp_query", "gemm_epi_mlp_free", "gemm_epi_mlp_unfused_run"):
                getattr(L, name).restype = i32
            _lib = L
    return _lib


# ---------------------------------------------------------------- C-named wrappers
def gemm_epi_plan(m, n, k, dtype, epilogue, bias_axis) -> int:
    h = ctypes.c_void_p()
    _check(lib().gemm_epi_plan(m, n, k, dtype, epilogue, bias_axis, ctypes.byref(h)), "gemm_epi_plan")
    return h.value


def gemm_epi_plan_ex(m, n, k, dtype, epilogue, bias_axis, b_layout) -> int:
    h = ctypes.c_void_p()
    _check(lib().gemm_epi_plan_ex(m, n, k, dtype, epilogue, bias_axis, b_layout, ctypes.byref(h)),
           "gemm_epi_plan_ex")
    return h.value


def gemm_epi_plan_opts(m, n, k, dtype, epilogue, bias_axis, b_layout, opts: Options | None) -> int:
    h = ctypes.c_void_p()
    _check(lib().gemm_epi_plan_opts(m, n, k, dtype, epilogue, bias_axis, b_layout,
                                    ctypes.byref(opts) if opts is not None else None,
                                    ctypes.byref(h)), "gemm_epi_plan_opts")
    return h.value


def gemm_epi_set_scales(plan, d_scale_a, d_scale_b) -> None:
    _check(lib().gemm_epi_set_scales(plan, d_scale_a, d_scale_b), "gemm_epi_set_scales")


def gemm_epi_run(plan, A, B, bias, D, aux, stream) -> None:
    _check(lib().gemm_epi_run(plan, A, B, bias, D, aux, stream), "gemm_epi_run")


def gemm_epi_unfused_run(plan, A, B, bias, D, aux, stream) -> None:
    _check(lib().gemm_epi_unfused_run(plan, A, B, bias, D, aux, stream), "gemm_epi_unfused_run")


def gemm_epi_run_bwd(plan, A, B, aux, D, dbias, stream) -> None:
    _check(lib().gemm_epi_run_bwd(plan, A, B, aux, D, dbias, stream), "gemm_epi_run_bwd")


def gemm_epi_unfused_run_bwd(plan, A, B, aux, D, dbias, stream) -> None:
    _check(lib().gemm_epi_unfused_run_bwd(plan, A, B, aux, D, dbias, stream), "gemm_epi_unfused_run_bwd")


def gemm_epi_set_out_scale(plan, d_scale_out, d_amax) -> None:
    _check(lib().gemm_epi_set_out_scale(plan, d_scale_out, d_amax), "gemm_epi_set_out_scale")


def gemm_epi_mlp_plan(m, d_model, d_ff, dtype, act, w_layout) -> int:
    h = ctypes.c_void_p()
    _check(lib().gemm_epi_mlp_plan(m, d_model, d_ff, dtype, act, w_layout, ctypes.byref(h)),
           "gemm_epi_mlp_plan")
    return h.value


def gemm_epi_mlp_set_scales(mlp, d_scale_x, d_scale_w1, d_scale_h, d_amax_h, d_scale_w2) -> None:
    _check(lib().gemm_epi_mlp_set_scales(mlp, d_scale_x, d_scale_w1, d_scale_h, d_amax_h, d_scale_w2),
           "gemm_epi_mlp_set_scales")


def gemm_epi_mlp_run(mlp, X, W1, b1, W2, b2, H, Y, stream) -> None:
    _check(lib().gemm_epi_mlp_run(mlp, X, W1, b1, W2, b2, H, Y, stream), "gemm_epi_mlp_run")


def gemm_epi_mlp_unfused_run(mlp, X, W1, b1, W2, b2, H, Y, H_wide, stream) -> None:
    _check(lib().gemm_epi_mlp_unfused_run(mlp, X, W1, b1, W2, b2, H, Y, H_wide, stream),
           "gemm_epi_mlp_unfused_run")


def gemm_epi_mlp_check(mlp, stream) -> None:
    _check(lib().gemm_epi_mlp_check(mlp, stream), "gemm_epi_mlp_check")


def gemm_epi_mlp_query(mlp) -> tuple:
    up, down = PlanInfo(), PlanInfo()
    _check(lib().gemm_epi_mlp_query(mlp, ctypes.byref(up), ctypes.byref(down)), "gemm_epi_mlp_query")
    return up.as_dict(), down.as_dict()


def gemm_epi_mlp_free(mlp) -> None:
    _check(lib().gemm_epi_mlp_free(mlp), "gemm_epi_mlp_free")


def gemm_epi_check(plan, stream) -> None:
    _check(lib().gemm_epi_check(plan, stream), "gemm_epi_check")


def gemm_epi_plan_query(plan) -> dict:
    info = PlanInfo()
    _check(lib().gemm_epi_plan_query(plan, ctypes.byref(info)), "gemm_epi_plan_query")
    return info.as_dict()


def gemm_epi_plan_preview(m, n, k, dtype, epilogue, bias_axis, b_layout, opts: Options | None,
                          num_sms: int) -> dict:
    info = PlanInfo()
    _check(lib().gemm_epi_plan_preview(m, n, k, dtype, epilogue, bias_axis, b_layout,
                                       ctypes.byref(opts) if opts is not None else None, num_sms,
                                       ctypes.byref(info)), "gemm_epi_plan_preview")
    return info.as_dict()


def plan_preview(m, n, k, dtype="bf16", epilogue="bias", bias_axis="row", b_layout="kn", num_sms=148,
                 kernel="auto", block_n=0, split_k=0, max_ctas=0, stream_k="auto", out_e4m3=False,
                 a_layout="mk") -> dict:
    """The kernel choice a plan would make on a device with ``num_sms`` SMs, computed on the
    host (no device needed); the same names as :class:`Plan`, the same keys as ``Plan.info``."""
    opts = Options(KERNEL[kernel], int(block_n), int(split_k), int(max_ctas), 0, STREAM_K[stream_k],
                   1 if out_e4m3 else 0)
    layout = LAYOUT[b_layout] | (A_KM if a_layout == "km" else 0)
    return gemm_epi_plan_preview(int(m), int(n), int(k), DTYPE[dtype], EPILOGUE[epilogue], AXIS[bias_axis],
                                 layout, opts, int(num_sms))


def gemm_epi_free(plan) -> None:
    _check(lib().gemm_epi_free(plan), "gemm_epi_free")


def gemm_epi_status_string(status: int) -> str:
    return lib().gemm_epi_status_string(status).decode()


def gemm_epi_aux_pitch_bytes(n: int) -> int:
    return lib().gemm_epi_aux_pitch_bytes(n)


def gemm_epi_version() -> int:
    return lib().gemm_epi_version()


def gemm_epi_run_noalloc(m, n, k, dtype, epilogue, bias_axis, b_layout, A, B, bias, d_scale_a,
                         d_scale_b, D, aux, wait, stream) -> None:
    """Allocation-free fused run (see include/gemm_epi.h); raises on a non-zero status."""
    _check(lib().gemm_epi_run_noalloc(m, n, k, dtype, epilogue, bias_axis, b_layout, A, B, bias,
                                      d_scale_a, d_scale_b, D, aux, wait, stream),
           "gemm_epi_run_noalloc")


def status_string(status: int) -> str:
    try:
        return gemm_epi_status_string(status)
    except Exception:  # library not loadable: still report the number
        return "status"


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise GemmEpiError(rc, what)


# ---------------------------------------------------------------- torch convenience
def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class Plan:
    """Owns one gemm_epi plan; ``run`` passes torch tensors' device pointers.

    ``dtype``/``epilogue``/``bias_axis``/``b_layout``/``kernel`` take the
    names used across the package ("bf16", "relu_aux_bias", "row", "kn", ...).
    """

    def __init__(self, m, n, k, dtype="bf16", epilogue="bias", bias_axis="row", b_layout="kn",
                 kernel="auto", block_n=0, split_k=0, max_ctas=0, inject_stall=0, stream_k="auto",
                 out_e4m3=False, a_layout="mk"):
        self.m, self.n, self.k = int(m), int(n), int(k)
        self.dtype, self.epilogue, self.bias_axis, self.b_layout = dtype, epilogue, bias_axis, b_layout
        opts = Options(KERNEL[kernel], int(block_n), int(split_k), int(max_ctas), int(inject_stall),
                       STREAM_K[stream_k], 1 if out_e4m3 else 0)
        layout = LAYOUT[b_layout] | (A_KM if a_layout == "km" else 0)
        self.handle = gemm_epi_plan_opts(self.m, self.n, self.k, DTYPE[dtype], EPILOGUE[epilogue],
                                         AXIS[bias_axis], layout, opts)
        self._scales = None

    @property
    def info(self) -> dict:
        return gemm_epi_plan_query(self.handle)

    def set_scales(self, scale_a, scale_b):
        """fp32 device scalars (torch tensors); kept alive by the plan object."""
        self._scales = (scale_a, scale_b)
        gemm_epi_set_scales(self.handle, _ptr(scale_a), _ptr(scale_b))

    def set_out_scale(self, scale_out, amax=None):
        """FP8-output plans: fp32 device scalars (the output scale; the amax word or None)."""
        self._out = (scale_out, amax)
        gemm_epi_set_out_scale(self.handle, _ptr(scale_out), _ptr(amax))

    def run(self, A, B, bias, D, aux=None, stream=None, fused=True):
        s = _stream_ptr(stream)
        f = gemm_epi_run if fused else gemm_epi_unfused_run
        f(self.handle, _ptr(A), _ptr(B), _ptr(bias), _ptr(D), _ptr(aux), s)

    def run_bwd(self, A, B, aux, D, dbias=None, stream=None, fused=True):
        """Backward plans (``drelu``/``drelu_bgrad``): D = mask ? alpha*A.B : 0 (+ dbias)."""
        s = _stream_ptr(stream)
        f = gemm_epi_run_bwd if fused else gemm_epi_unfused_run_bwd
        f(self.handle, _ptr(A), _ptr(B), _ptr(aux), _ptr(D), _ptr(dbias), s)

    def check(self, stream=None):
        gemm_epi_check(self.handle, _stream_ptr(stream))

    def close(self):
        if getattr(self, "handle", None):
            gemm_epi_free(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _stream_ptr(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream) if hasattr(stream, "cuda_stream") else stream


def aux_pitch_words(n: int) -> int:
    return gemm_epi_aux_pitch_bytes(n) // 4


class MlpPlan:
    """Owns one MLP-block handle (gemm_epi_mlp_*): H = act(X.W1 + b1), Y = H.W2 + b2."""

    def __init__(self, m, d_model, d_ff, dtype="bf16", act="gelu_bias", w_layout="kn"):
        self.m, self.d_model, self.d_ff = int(m), int(d_model), int(d_ff)
        self.dtype, self.act, self.w_layout = dtype, act, w_layout
        self.handle = gemm_epi_mlp_plan(self.m, self.d_model, self.d_ff, DTYPE[dtype], EPILOGUE[act],
                                        LAYOUT[w_layout])
        self._scales = None

    @property
    def info(self) -> tuple:
        return gemm_epi_mlp_query(self.handle)

    def set_scales(self, scale_x, scale_w1, scale_h, amax_h, scale_w2):
        self._scales = (scale_x, scale_w1, scale_h, amax_h, scale_w2)
        gemm_epi_mlp_set_scales(self.handle, _ptr(scale_x), _ptr(scale_w1), _ptr(scale_h), _ptr(amax_h),
                                _ptr(scale_w2))

    def run(self, X, W1, b1, W2, b2, H, Y, stream=None, fused=True, H_wide=None):
        """fused=False: the unfused baseline (H_wide: bf16 (m, d_ff) scratch, e4m3 plans)."""
        if fused:
            gemm_epi_mlp_run(self.handle, _ptr(X), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(H), _ptr(Y),
                             _stream_ptr(stream))
        else:
            gemm_epi_mlp_unfused_run(self.handle, _ptr(X), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(H),
                                     _ptr(Y), _ptr(H_wide), _stream_ptr(stream))

    def check(self, stream=None):
        gemm_epi_mlp_check(self.handle, _stream_ptr(stream))

    def close(self):
        if getattr(self, "handle", None):
            gemm_epi_mlp_free(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
