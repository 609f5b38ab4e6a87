"""Seeded synthetic inputs for the fused GEMM + bias + activation path.

This module only draws random numbers and casts them to the storage types: it
holds none of the method's arithmetic, and both the CUDA path's tests/bench and
the CPU oracle consume what it produces.

Recipe (one ``torch.Generator`` per problem, seeded, drawing A, then B, then
the bias, each in fp32, then cast with round-to-nearest-even):

* normal(std):   ``randn * std``
* uniform(a):    ``(rand * 2 - 1) * a``  -> U(-a, a)
* int(r):        integers drawn uniformly from {-r..r} (exact in every type)
* fp8 e4m3 operands are drawn in fp32, given a per-tensor scale
  ``s = amax(|x|) / 448`` and stored as ``clamp(x / s, -448, 448)`` cast to
  e4m3 (round to nearest even, saturating); the scales are returned beside
  them as fp32.

The five named workloads follow the shapes, dtypes and distributions of the
pages' examples (the nvmath-python worked example, the Linear(4096,4096)+GELU
batch-16 latency script, the RELU_AUX_BIAS and large RELU_BIAS shapes, and an
FP8 MLP up-projection).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}
E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    name: str
    m: int
    n: int
    k: int
    dtype: str                  # "f16" | "bf16" | "e4m3" (operand type)
    epilogue: str               # "none" | "bias" | "relu_bias" | "relu_aux_bias" | "gelu_bias"
    bias_axis: str = "row"      # "row": length m, one value per output row; "col": length n
    b_layout: str = "kn"        # "kn": B stored (k, n) row-major; "nk": (n, k), an nn.Linear weight
    dist_a: tuple = ("normal", 1.0)
    dist_b: tuple = ("normal", 1.0)
    dist_bias: tuple = ("normal", 1.0)
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False)
    a_layout: str = "mk"        # "mk": A stored (m, k) row-major; "km": stored transposed, (k, m)

    @property
    def out_dtype(self) -> str:
        return "bf16" if self.dtype == "e4m3" else self.dtype

    @property
    def flops(self) -> int:
        return 2 * self.m * self.n * self.k

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "gemm_bias_f16_1024x512x2048": Workload(
        "gemm_bias_f16_1024x512x2048", 1024, 512, 2048, "f16", "bias", "row", "kn",
        ("normal", 1.0), ("normal", 1.0), ("normal", 1.0)),
    "linear_gelu_f16_16x4096x4096": Workload(
        "linear_gelu_f16_16x4096x4096", 16, 4096, 4096, "f16", "gelu_bias", "col", "nk",
        ("normal", 1.0), ("uniform", 1.0 / 64), ("uniform", 1.0 / 64)),
    "relu_aux_bias_bf16_4096x4096x4096": Workload(
        "relu_aux_bias_bf16_4096x4096x4096", 4096, 4096, 4096, "bf16", "relu_aux_bias", "row",
        "kn", ("normal", 1.0 / 64), ("normal", 1.0 / 64), ("normal", 1.0)),
    "relu_bias_bf16_65536x8192x16384": Workload(
        "relu_bias_bf16_65536x8192x16384", 65536, 8192, 16384, "bf16", "relu_bias", "row", "kn",
        ("normal", 1.0 / 128), ("normal", 1.0 / 128), ("normal", 1.0)),
    "fp8_gelu_bias_8192x14336x4096": Workload(
        "fp8_gelu_bias_8192x14336x4096", 8192, 14336, 4096, "e4m3", "gelu_bias", "col", "kn",
        ("normal", 1.0), ("normal", 1.0), ("normal", 0.02)),
}
# The five workloads in the order the benchmark's configuration list gives them.
ORDER = list(WORKLOADS)

# Calibration shape (not one of the five): the size at which the measured bf16
# dense peak of this GPU pool was taken, for a like-for-like comparison.
WORKLOADS["gemm_bias_bf16_8192x8192x8192"] = Workload(
    "gemm_bias_bf16_8192x8192x8192", 8192, 8192, 8192, "bf16", "bias", "row", "kn",
    ("normal", 1.0 / 64), ("normal", 1.0 / 64), ("normal", 1.0))


def _draw(shape, dist, gen, device):
    kind, p = dist
    if kind == "normal":
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * p
    if kind == "uniform":
        return (torch.rand(shape, generator=gen, device=device, dtype=torch.float32) * 2 - 1) * p
    if kind == "int":
        r = int(p)
        return torch.randint(-r, r + 1, shape, generator=gen, device=device).to(torch.float32)
    if kind == "zeros":
        return torch.zeros(shape, device=device, dtype=torch.float32)
    raise ValueError(f"unknown distribution {dist}")


def _to_e4m3(x):
    amax = float(x.abs().max())
    s = amax / E4M3_MAX if amax > 0 else 1.0
    s32 = torch.tensor(s, dtype=torch.float32)
    q = (x / s32.to(x.device)).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return q, float(s32)


@dataclass
class Problem:
    """Inputs of one problem: torch tensors on ``device`` plus fp8 scales."""
    wl: Workload
    A: torch.Tensor
    B: torch.Tensor
    bias: torch.Tensor | None
    scale_a: float = 1.0
    scale_b: float = 1.0


def make_problem(wl: Workload, device="cpu", int_scales: bool = False) -> Problem:
    """Draw A, B, bias for ``wl`` (seeded) on ``device``.

    ``int_scales``: for e4m3 with an ``("int", r)`` distribution, store the
    integers themselves (exact in e4m3 for |x| <= 16) with unit scales.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    b_shape = (wl.k, wl.n) if wl.b_layout == "kn" else (wl.n, wl.k)
    a = _draw((wl.m, wl.k), wl.dist_a, gen, device)
    b = _draw(b_shape, wl.dist_b, gen, device)
    blen = wl.m if wl.bias_axis == "row" else wl.n
    bias = _draw((blen,), wl.dist_bias, gen, device)
    bias_t = bias.to(TORCH_DTYPE[wl.out_dtype])
    # A stored transposed holds the same values, (k, m) row-major
    lay = (lambda x: x.t().contiguous()) if wl.a_layout == "km" else (lambda x: x)
    if wl.dtype == "e4m3":
        if int_scales:
            return Problem(wl, lay(a.to(torch.float8_e4m3fn)), b.to(torch.float8_e4m3fn), bias_t)
        qa, sa = _to_e4m3(a)
        qb, sb = _to_e4m3(b)
        return Problem(wl, lay(qa), qb, bias_t, sa, sb)
    t = TORCH_DTYPE[wl.dtype]
    return Problem(wl, lay(a.to(t)), b.to(t), bias_t)


def make_mask(m: int, n: int, seed: int = 0, kind: str = "bernoulli", p: float = 0.5) -> np.ndarray:
    """Seeded (m, n) 0/1 uint8 mask for the ReLU backward epilogues.

    kind: "bernoulli" (each bit 1 with probability p, from one seeded
    ``torch.Generator``), "zeros", "ones", or "checker" (bit = (i + j) odd).
    """
    if kind == "bernoulli":
        gen = torch.Generator(device="cpu")
        gen.manual_seed(seed)
        return (torch.rand((m, n), generator=gen) < p).to(torch.uint8).numpy()
    if kind == "zeros":
        return np.zeros((m, n), np.uint8)
    if kind == "ones":
        return np.ones((m, n), np.uint8)
    if kind == "checker":
        return ((np.arange(m)[:, None] + np.arange(n)[None, :]) & 1).astype(np.uint8)
    raise ValueError(f"unknown mask kind {kind}")


def pack_mask(mask: np.ndarray, pad_fill: int = 0) -> np.ndarray:
    """(m, n) 0/1 array -> the library's aux storage: row-major uint32 words, row
    pitch ceil(n/128)*4 words, bit b of word w in row i = element (i, 32w + b).

    ``pad_fill`` = 1 sets every bit past column n-1 (which readers ignore).
    """
    m, n = mask.shape
    pitch = ((n + 127) // 128) * 4
    bits = np.full((m, pitch * 32), 1 if pad_fill else 0, np.uint8)
    bits[:, :n] = mask
    return np.packbits(bits, axis=1, bitorder="little").view(np.uint32).reshape(-1).copy()


def storage(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a fp16/bf16 (uint16) or e4m3 (uint8) tensor, on the host."""
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    raise TypeError(f"no storage view for {t.dtype}")


def sample_positions(m: int, n: int, count_rows: int = 64, count_cols: int = 64, seed: int = 0,
                     tile_m: int = 128, tile_n: int = 128):
    """Seeded output positions for sampled checks at full size.

    ``count_rows`` rows x ``count_cols`` columns (a grid), always containing
    row/column 0 and m-1/n-1 and the first and last index of each of a few
    tile boundaries.  Returns (rows, cols) int64 arrays of equal length.
    """
    rng = np.random.default_rng(seed)

    def pick(size, count, tile):
        must = {0, size - 1}
        for b in range(tile, size, tile):
            if len(must) >= count // 2:
                break
            must.update({b - 1, b})
        must = sorted(x for x in must if 0 <= x < size)
        rest = count - len(must)
        pool = np.setdiff1d(np.arange(size), must)
        extra = rng.choice(pool, size=min(rest, pool.size), replace=False) if rest > 0 else []
        return np.sort(np.concatenate([np.array(must, np.int64), np.asarray(extra, np.int64)]))

    r = pick(m, count_rows, tile_m)
    c = pick(n, count_cols, tile_n)
    rr, cc = np.meshgrid(r, c, indexing="ij")
    return rr.ravel().astype(np.int64), cc.ravel().astype(np.int64)
