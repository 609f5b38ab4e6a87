"""GPU parity on seeded random problems: shapes, types, epilogues, layouts and the
automatic kernel choice drawn together, so combinations no hand-written case
lists are exercised as well (each case against the fp64 oracle)."""
import numpy as np
import pytest
import torch

import oracle
from parity import check_against_oracle

from activation_epilogue_tcgen05_b200 import gemm_epi as g
from activation_epilogue_tcgen05_b200.workloads import Workload, make_problem

pytestmark = pytest.mark.gpu

FORWARD = ["none", "bias", "relu_bias", "relu_aux_bias", "gelu_bias", "tanh_bias", "relu", "relu_aux",
           "gelu", "tanh"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability() != (10, 0):
        pytest.skip("needs sm_100")
    from activation_epilogue_tcgen05_b200 import build
    build.build()
    oracle.build()


def draw_case(i):
    rng = np.random.default_rng(1000 + i)
    dtype = ["f16", "bf16", "e4m3"][rng.integers(3)]
    step = 16 if dtype == "e4m3" else 8                   # 16-byte row pitches
    # A stored (k, m) (a quarter of the cases) needs a 16-byte pitch along m as well
    a_layout = "km" if rng.random() < 0.25 else "mk"
    m = int(rng.choice([rng.integers(1, 65), rng.integers(65, 700)]))
    if a_layout == "km":
        m = step * max(1, m // step)
    n = int(step * rng.integers(1, 800 // step + 1))
    k = int(step * rng.integers(1, 1200 // step + 1))
    epi = FORWARD[rng.integers(len(FORWARD))]
    axis = ["row", "col"][rng.integers(2)]
    b_layout = ["kn", "nk"][rng.integers(2)]
    return Workload(f"rand{i}", m, n, k, dtype, epi, axis, b_layout, seed=2000 + i, a_layout=a_layout)


def draw_long_k_case(i):
    """Few tiles and a long k: the automatic plan splits every tile into three or four parts."""
    rng = np.random.default_rng(5000 + i)
    dtype = ["f16", "bf16", "e4m3"][rng.integers(3)]
    step = 16 if dtype == "e4m3" else 8
    m = int(rng.integers(65, 520))          # above the split-K kernel's range
    n = int(step * rng.integers(1, 640 // step + 1))
    k = int(step * rng.integers(2048 // step, 4096 // step + 1))
    epi = FORWARD[rng.integers(len(FORWARD))]
    axis = ["row", "col"][rng.integers(2)]
    b_layout = ["kn", "nk"][rng.integers(2)]
    return Workload(f"randk{i}", m, n, k, dtype, epi, axis, b_layout, seed=6000 + i)


CASES = [draw_case(i) for i in range(64)] + [draw_long_k_case(i) for i in range(16)]


@pytest.mark.parametrize("wl", CASES, ids=[f"{w.name}-{w.m}x{w.n}x{w.k}-{w.dtype}-{w.epilogue}-{w.bias_axis}-"
                                           f"{w.b_layout}-{w.a_layout}" for w in CASES])
def test_random_problem_matches_oracle(wl):
    worst, info = check_against_oracle(wl, make_problem(wl))
    assert worst <= 1.0
    # the automatic choice: split-K for small m where it applies, else a persistent kernel
    small = wl.m <= 64 and wl.a_layout == "mk"
    assert (info["kernel"] == g.KERNEL_SPLITK) == small
