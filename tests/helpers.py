"""Shared test helpers: golden loading, tolerance, aux-mask unpacking.

No arithmetic of the method lives here: the tolerance is the acceptance
bound, the unpacking reads the library's documented aux layout.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# Acceptance bound per element: |gpu - ref| <= RTOL*|ref| + ATOL*sqrt(k)*sigma_A*sigma_B
TOL = {"f16": (4e-3, 2e-3), "bf16": (4e-3, 2e-3), "e4m3": (6e-2, 2e-2)}


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def to_storage_values(values, dtype):
    """Exact real values -> raw storage array (uint16 bit patterns / e4m3 bytes)."""
    t = torch.tensor(values, dtype=torch.float64)
    if dtype == "f16":
        return t.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    if dtype == "bf16":
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if dtype == "e4m3":
        return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    raise ValueError(dtype)


def operand_sigma(values_f64: np.ndarray) -> float:
    """Population standard deviation in fp64 of the operand values the product uses."""
    v = np.asarray(values_f64, dtype=np.float64)
    return float(v.std())


def tolerance(ref: np.ndarray, dtype: str, k: int, sigma_a: float, sigma_b: float) -> np.ndarray:
    rt, at = TOL[dtype]
    return rt * np.abs(ref) + at * np.sqrt(k) * sigma_a * sigma_b


def band(ref_pre: np.ndarray, dtype: str, k: int, sigma_a: float, sigma_b: float) -> np.ndarray:
    """True where the mask bit must be exact: |pre| outside the tolerance band."""
    return np.abs(ref_pre) > tolerance(ref_pre, dtype, k, sigma_a, sigma_b)


def unpack_aux(words: np.ndarray, m: int, n: int) -> np.ndarray:
    """Library aux layout -> (m, n) 0/1 array.

    Row-major uint32 words, row pitch ceil(n/128)*4 words, bit b of word w in
    row i is element (i, 32*w + b).
    """
    pitch = ((n + 127) // 128) * 4
    w = np.ascontiguousarray(words, dtype=np.uint32).reshape(m, pitch)
    bits = np.unpackbits(w.view(np.uint8).reshape(m, pitch * 4), axis=1, bitorder="little")
    return bits[:, :n]


def aux_padding_bits(words: np.ndarray, m: int, n: int) -> int:
    """Number of set bits beyond column n (must be 0)."""
    pitch = ((n + 127) // 128) * 4
    w = np.ascontiguousarray(words, dtype=np.uint32).reshape(m, pitch)
    bits = np.unpackbits(w.view(np.uint8).reshape(m, pitch * 4), axis=1, bitorder="little")
    return int(bits[:, n:].sum())


def pack_aux(mask: np.ndarray, pad_fill: int = 0) -> np.ndarray:
    """(m, n) 0/1 array -> library aux layout (the seeded-input module's packer)."""
    from activation_epilogue_tcgen05_b200.workloads import pack_mask
    return pack_mask(mask, pad_fill)
