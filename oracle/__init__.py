"""fp64 CPU oracle for D = act(alpha * A.B + bias) and its ReLU sign mask.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg (``cpu_baseline`` / ``--impl reference``) may
import this package.  The product path (the C-ABI library and its binding)
never imports, links or runs anything here, and this package never imports the
product: the two meet only at the seeded input generators, which hold no
arithmetic of the method.

The arithmetic lives in ``gemm_epi_oracle.c`` (plain C, IEEE double, OpenMP
over output rows); this module compiles it with gcc on first use and marshals
numpy arrays through ctypes.  Inputs are raw storage arrays (``uint16`` for
fp16/bf16 bit patterns, ``uint8`` for e4m3 bytes); the C code decodes them
itself.  Every function's docstring names the page passage it follows; the
file header of ``gemm_epi_oracle.c`` lists them all.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gemm_epi_oracle.c")
_LIB = os.path.join(_HERE, "libgemm_epi_oracle.so")
_lock = threading.Lock()
_lib = None

DTYPES = ("f16", "bf16", "e4m3")
EPILOGUES = ("none", "bias", "relu_bias", "relu_aux_bias", "gelu_bias", "tanh_bias", "relu",
             "relu_aux", "gelu", "tanh")
AXES = ("row", "col")
LAYOUTS = ("kn", "nk")
A_LAYOUTS = ("mk", "km")   # A stored (m, k) row-major, or transposed: (k, m) row-major


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (no fast-math: IEEE double)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Werror",
             _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # A test may point the loader at a deliberately mutated build of the
            # same source (tests/test_oracle_mutants.py) to check that the pins
            # catch the mutation.
            path = os.environ.get("GEMM_EPI_ORACLE_LIB") or build()
            lib = ctypes.CDLL(path)
            i64, vp, dp, cp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double, ctypes.c_char_p
            lib.oracle_decode_f16.argtypes = [ctypes.c_uint16]
            lib.oracle_decode_f16.restype = dp
            lib.oracle_decode_bf16.argtypes = [ctypes.c_uint16]
            lib.oracle_decode_bf16.restype = dp
            lib.oracle_decode_e4m3.argtypes = [ctypes.c_uint8]
            lib.oracle_decode_e4m3.restype = dp
            lib.oracle_gelu.argtypes = [dp]
            lib.oracle_gelu.restype = dp
            lib.oracle_gemm_epi.argtypes = [i64, i64, i64, cp, cp, cp, cp, vp, vp, vp, dp, dp,
                                            vp, vp, vp]
            lib.oracle_gemm_epi.restype = ctypes.c_int
            lib.oracle_gemm_epi_sampled.argtypes = [i64, i64, i64, cp, cp, cp, cp, vp, vp, vp,
                                                    dp, dp, i64, vp, vp, vp, vp, vp]
            lib.oracle_gemm_epi_sampled.restype = ctypes.c_int
            lib.oracle_gemm_epi_bwd.argtypes = [i64, i64, i64, cp, cp, cp, cp, vp, vp, vp, dp, dp,
                                                vp, vp]
            lib.oracle_gemm_epi_bwd.restype = ctypes.c_int
            lib.oracle_encode_e4m3.argtypes = [dp]
            lib.oracle_encode_e4m3.restype = ctypes.c_uint8
            lib.oracle_encode_f16.argtypes = [dp]
            lib.oracle_encode_f16.restype = ctypes.c_uint16
            lib.oracle_encode_bf16.argtypes = [dp]
            lib.oracle_encode_bf16.restype = ctypes.c_uint16
            lib.oracle_encode.argtypes = [i64, cp, vp, dp, vp]
            lib.oracle_encode.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _storage(a, dtype):
    """Check a raw storage array against the input format and make it contiguous."""
    want = np.uint8 if dtype == "e4m3" else np.uint16
    a = np.ascontiguousarray(a)
    if a.dtype != want:
        raise TypeError(f"{dtype} storage must be {np.dtype(want).name}, got {a.dtype}")
    return a


def decode(bits, dtype: str) -> np.ndarray:
    """Decode raw fp16 / bf16 / e4m3 bit patterns to float64 with the C decoders."""
    lib = _load()
    fn = {"f16": lib.oracle_decode_f16, "bf16": lib.oracle_decode_bf16,
          "e4m3": lib.oracle_decode_e4m3}[dtype]
    flat = np.asarray(bits).ravel()
    return np.array([fn(int(v)) for v in flat], dtype=np.float64).reshape(np.shape(bits))


def gelu(x: float) -> float:
    """Exact GELU x*Phi(x) (erf form), as the oracle applies it."""
    return _load().oracle_gelu(float(x))


def _names(dtype, epilogue, bias_axis, b_layout, a_layout="mk"):
    if dtype not in DTYPES or epilogue not in EPILOGUES or bias_axis not in AXES \
            or b_layout not in LAYOUTS or a_layout not in A_LAYOUTS:
        raise ValueError(f"unknown oracle option {(dtype, epilogue, bias_axis, b_layout, a_layout)}")
    return tuple(s.encode() for s in (dtype, epilogue, bias_axis, _layout(b_layout, a_layout)))


def _layout(b_layout, a_layout):
    """The C side's layout string: B's layout, prefixed "at_" when A is stored (k, m)."""
    return ("at_" if a_layout == "km" else "") + b_layout


def _a_shape(A, a_layout):
    """(m, k) of the operand A from its storage array."""
    return (A.shape[1], A.shape[0]) if a_layout == "km" else A.shape


def gemm_epi(A, B, bias, *, dtype: str, epilogue: str, bias_axis: str = "row",
             b_layout: str = "kn", scale_a: float = 1.0, scale_b: float = 1.0, a_layout: str = "mk"):
    """Full fp64 result (D, pre-activation, mask) of act(alpha*A.B + bias).

    A is (m, k) row-major storage (``a_layout="mk"``) or its transpose, (k, m)
    row-major (``"km"``); B is (k, n) for ``b_layout="kn"`` or (n, k)
    for ``"nk"``; bias has length m (``"row"``: one value per output row,
    added to every column -- the pages' default broadcast) or n (``"col"``).
    Returns float64 D and pre (m, n) and a uint8 0/1 mask (m, n).
    """
    A = _storage(A, dtype)
    B = _storage(B, dtype)
    m, k = _a_shape(A, a_layout)
    n = B.shape[1] if b_layout == "kn" else B.shape[0]
    if (B.shape[0] if b_layout == "kn" else B.shape[1]) != k:
        raise ValueError("inner dimensions differ")
    if bias is not None:
        bias = _storage(bias, "bf16" if dtype == "e4m3" else dtype)
        if bias.size != (m if bias_axis == "row" else n):
            raise ValueError("bias length does not match its axis")
    D = np.empty((m, n), np.float64)
    pre = np.empty((m, n), np.float64)
    mask = np.empty((m, n), np.uint8)
    rc = _load().oracle_gemm_epi(m, n, k, *_names(dtype, epilogue, bias_axis, b_layout, a_layout),
                                 _ptr(A), _ptr(B), _ptr(bias), float(scale_a), float(scale_b),
                                 _ptr(D), _ptr(pre), _ptr(mask))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_epi failed with status {rc}")
    return D, pre, mask


def gemm_epi_sampled(A, B, bias, rows, cols, *, dtype: str, epilogue: str,
                     bias_axis: str = "row", b_layout: str = "kn", scale_a: float = 1.0,
                     scale_b: float = 1.0, m: int | None = None, k: int | None = None,
                     a_layout: str = "mk"):
    """(D, pre, mask) at positions (rows[s], cols[s]); one fp64 dot product each.

    ``A`` may be given as the full (m, k) storage array.  Same conventions as
    :func:`gemm_epi`.
    """
    A = _storage(A, dtype)
    B = _storage(B, dtype)
    m_, k_ = _a_shape(A, a_layout)
    m = m_ if m is None else m
    k = k_ if k is None else k
    n = B.shape[1] if b_layout == "kn" else B.shape[0]
    if bias is not None:
        bias = _storage(bias, "bf16" if dtype == "e4m3" else dtype)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    if rows.shape != cols.shape:
        raise ValueError("rows and cols differ in length")
    cnt = rows.size
    D = np.empty(cnt, np.float64)
    pre = np.empty(cnt, np.float64)
    mask = np.empty(cnt, np.uint8)
    rc = _load().oracle_gemm_epi_sampled(m, n, k, *_names(dtype, epilogue, bias_axis, b_layout, a_layout),
                                         _ptr(A), _ptr(B), _ptr(bias), float(scale_a),
                                         float(scale_b), cnt, _ptr(rows), _ptr(cols), _ptr(D),
                                         _ptr(pre), _ptr(mask))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_epi_sampled failed with status {rc}")
    return D, pre, mask


def gemm_epi_bwd(A, B, mask, *, dtype: str, epilogue: str, bias_axis: str = "row",
                 b_layout: str = "kn", scale_a: float = 1.0, scale_b: float = 1.0):
    """ReLU backward epilogues: D = mask * (alpha*A.B) and, for "drelu_bgrad", the bias
    gradient (sums of D along the bias axis).  mask is an (m, n) 0/1 array.

    Returns float64 D (m, n) and dbias (length m for "row", n for "col"; None for "drelu").
    """
    if epilogue not in ("drelu", "drelu_bgrad") or dtype not in DTYPES or bias_axis not in AXES \
            or b_layout not in LAYOUTS:
        raise ValueError(f"unknown oracle option {(dtype, epilogue, bias_axis, b_layout)}")
    A = _storage(A, dtype)
    B = _storage(B, dtype)
    m, k = A.shape
    n = B.shape[1] if b_layout == "kn" else B.shape[0]
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    if mask.shape != (m, n):
        raise ValueError("mask must be (m, n)")
    D = np.empty((m, n), np.float64)
    dbias = np.empty(m if bias_axis == "row" else n, np.float64) if epilogue == "drelu_bgrad" else None
    rc = _load().oracle_gemm_epi_bwd(m, n, k, dtype.encode(), epilogue.encode(), bias_axis.encode(),
                                     b_layout.encode(), _ptr(A), _ptr(B), _ptr(mask),
                                     float(scale_a), float(scale_b), _ptr(D), _ptr(dbias))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_epi_bwd failed with status {rc}")
    return D, dbias


def threads() -> int:
    """OpenMP threads the oracle will use (OMP_NUM_THREADS, else the CPU count)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def encode(x, dtype: str, scale: float = 1.0):
    """Storage codes of x / scale in `dtype` (uint8 for e4m3, uint16 bit patterns for fp16 /
    bf16): round to nearest even from the format definitions, e4m3 saturating at +-448.

    The MLP block's intermediate stored in a narrower type ("nvmath-python cuBLASLt bias
    fusion for PyTorch inference", paragraphs 1 and 5; "PyTorch 2.14 NVGEMM epilogue
    fusion", section "why epilogue fusion matters": scaling and type conversion)."""
    if dtype not in DTYPES:
        raise ValueError(f"unknown dtype {dtype}")
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint8 if dtype == "e4m3" else np.uint16)
    rc = _load().oracle_encode(x.size, dtype.encode(), _ptr(x), float(scale), _ptr(out))
    if rc != 0:
        raise RuntimeError(f"oracle_encode failed with status {rc}")
    return out


def mlp(X, W1, b1, W2, b2, *, dtype: str, act: str = "gelu_bias", w_layout: str = "kn",
        scale_x: float = 1.0, scale_w1: float = 1.0, scale_h: float = 1.0, scale_w2: float = 1.0,
        stepwise: bool = False):
    """MLP block ("nvmath-python cuBLASLt bias fusion for PyTorch inference", paragraph 1):

        H = act(scale_x*scale_w1 * X.W1 + b1)          (bias along the d_ff columns)
        Hs = encode(H / scale_h) in the storage type    (e4m3: the per-tensor requantisation)
        Y = scale_h*scale_w2 * decode(Hs).W2 + b2       (bias along the d_model columns)

    For fp16 / bf16, scale_h is 1 and Hs is H rounded to that type.  X is (m, d_model); W1
    is (d_model, d_ff) for w_layout "kn" or (d_ff, d_model) for "nk" (an nn.Linear weight);
    W2 likewise (d_ff, d_model) or (d_model, d_ff).

    ``stepwise=True`` follows the unfused sequence instead ("nvmath-python epilog bias fusion
    parameters", body paragraph 1: the product is written back in the output type, then a
    separate kernel adds the bias and applies the activation): every product is rounded to
    the 16-bit output type (bf16 for e4m3) before its bias is added, H is rounded to that
    type before it is quantised, and Y's product is rounded before b2 is added.

    Returns (Y, H, Hs, amax) with Y and H in float64 (H before encoding), Hs the stored
    codes, and amax = max |H|."""
    if dtype != "e4m3" and scale_h != 1.0:
        raise ValueError("scale_h applies to e4m3 only")
    if not stepwise:
        H, _, _ = gemm_epi(X, W1, b1, dtype=dtype, epilogue=act, bias_axis="col", b_layout=w_layout,
                           scale_a=scale_x, scale_b=scale_w1)
        amax = float(np.abs(H).max())
        Hs = encode(H, dtype, scale_h)
        Y, _, _ = gemm_epi(Hs, W2, b2, dtype=dtype, epilogue="bias", bias_axis="col", b_layout=w_layout,
                           scale_a=scale_h, scale_b=scale_w2)
        return Y, H, Hs, amax
    out = "bf16" if dtype == "e4m3" else dtype
    rnd = lambda v: decode(encode(v, out), out)            # round to the 16-bit output type
    f = {"bias": lambda z: z, "relu_bias": lambda z: np.where(z > 0.0, z, 0.0),
         "gelu_bias": np.vectorize(gelu, otypes=[np.float64])}[act]
    P, _, _ = gemm_epi(X, W1, None, dtype=dtype, epilogue="none", b_layout=w_layout, scale_a=scale_x,
                       scale_b=scale_w1)
    H = rnd(f(rnd(P) + decode(_storage(b1, out), out)[None, :]))
    amax = float(np.abs(H).max())
    Hs = encode(H, dtype, scale_h)
    Q, _, _ = gemm_epi(Hs, W2, None, dtype=dtype, epilogue="none", b_layout=w_layout, scale_a=scale_h,
                       scale_b=scale_w2)
    Y = rnd(rnd(Q) + decode(_storage(b2, out), out)[None, :])
    return Y, H, Hs, amax
