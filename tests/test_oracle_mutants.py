"""The oracle's pins must catch plausible slips in the oracle.

Each case below plants one mistake in a temporary copy of the oracle's C
source (on the CPU, never touching the committed file), compiles it, and runs
the pin suite (test_oracle_pins.py) against the mutant in a subprocess.  The
suite must FAIL for every mutant: a mutant that survives is a gap in the pins.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gemm_epi_oracle.c")

# (id, text to replace, replacement, which occurrence (0-based) or None for all)
MUTANTS = [
    ("bias_axis_swapped", "axis == OR_ROW ? i : j", "axis == OR_ROW ? j : i", None),
    ("bias_dropped", "if (has_bias(epi)) p += load", "if (0) p += load", None),
    ("bias_on_none_too", "if (has_bias(epi)) p += load", "if (epi == OR_NONE || has_bias(epi)) p += load", None),
    ("b_transposed_full", "lay == OR_KN ? t * n + j : j * k + t",
     "lay == OR_KN ? j * k + t : t * n + j", 0),
    ("b_transposed_sampled", "lay == OR_KN ? t * n + j : j * k + t",
     "lay == OR_KN ? j * k + t : t * n + j", 1),
    ("a_index_wrong", "return la == OR_MK ? i * k + t : t * m + i;", "return la == OR_MK ? t * m + i : t * m + i;", None),
    ("a_transposed_index_wrong", "return la == OR_MK ? i * k + t : t * m + i;", "return la == OR_MK ? i * k + t : i * k + t;", None),
    ("a_layout_ignored", "return (s && !strncmp(s, \"at_\", 3)) ? OR_KM : OR_MK;", "return OR_MK;", None),
    ("gelu_sign", "0.5 * x * (1.0 + erf(", "0.5 * x * (1.0 - erf(", None),
    ("gelu_tanh_form", "0.5 * x * (1.0 + erf(x / sqrt(2.0)))",
     "0.5 * x * (1.0 + tanh(0.7978845608028654 * (x + 0.044715 * x * x * x)))", None),
    ("mask_ge", "(uint8_t)(p > 0.0)", "(uint8_t)(p >= 0.0)", None),
    ("relu_dropped", "y = p > 0.0 ? p : 0.0", "y = p", None),
    ("alpha_dropped", "p = alpha * p;", "p = p;", None),
    ("alpha_after_bias", "p = alpha * p;\n    if (has_bias(epi)) p += load(bias, bdt, axis == OR_ROW ? i : j);",
     "if (has_bias(epi)) p += load(bias, bdt, axis == OR_ROW ? i : j);\n    p = alpha * p;", None),
    ("e4m3_exponent_bias", "ldexp(1.0 + (double)f / 8.0, e - 7)", "ldexp(1.0 + (double)f / 8.0, e - 8)", None),
    ("e4m3_subnormal", "ldexp((double)f, -9)", "ldexp((double)f, -10)", None),
    ("f16_subnormal", "ldexp((double)f, -24)", "ldexp((double)f, -25)", None),
    ("bf16_exponent_bias", "e - 127)", "e - 126)", None),
    ("bias_dtype_for_fp8", "return dt == OR_E4M3 ? OR_BF16 : dt;", "return dt;", None),
    ("accumulate_dropped_term", "for (int64_t t = 0; t < k; ++t) {", "for (int64_t t = 1; t < k; ++t) {", None),
    ("tanh_sign", "y = tanh(p);", "y = -tanh(p);", None),
    ("tanh_as_relu", "case OR_TANH: y = tanh(p); break;", "case OR_TANH: y = p > 0.0 ? p : 0.0; break;", None),
    ("bias_free_adds_bias", "return epi == OR_BIAS ||", "return epi == OR_RELU || epi == OR_BIAS ||", None),
    ("alpha_fp8_only", "double alpha = scale_a * scale_b;", "double alpha = dt == OR_E4M3 ? scale_a * scale_b : 1.0;", None),
    ("bwd_mask_inverted", "D_ref[i * n + j] = mask[i * n + j] ? alpha * row[j] : 0.0;",
     "D_ref[i * n + j] = mask[i * n + j] ? 0.0 : alpha * row[j];", None),
    ("bwd_alpha_dropped", "D_ref[i * n + j] = mask[i * n + j] ? alpha * row[j] : 0.0;",
     "D_ref[i * n + j] = mask[i * n + j] ? row[j] : 0.0;", None),
    ("encode_ties_up", "else code = (lo & 1u) ? hi : lo;", "else code = hi;", None),
    ("encode_truncates", "if (dl < dh) code = lo;", "if (1) code = lo;", None),
    ("encode_no_saturation", "code = max_code;\n        } else {", "code = 0x7Fu;\n        } else {", None),
    ("encode_sign_dropped", "return neg ? (code | sign_bit) : code;", "return code;", None),
    ("encode_scale_multiplies", "encode_value(dt, x[i] / scale)", "encode_value(dt, x[i] * scale)", None),
    ("encode_f16_overflow_early", "code = a < vmax + half ? max_code : inf_code;",
     "code = a < vmax ? max_code : inf_code;", None),
    ("bwd_bgrad_wrong_axis", "if (axis == OR_ROW) {\n            for (int64_t i = 0; i < m; ++i) {\n                double s",
     "if (axis != OR_ROW) {\n            for (int64_t i = 0; i < m; ++i) {\n                double s", None),
]


def _mutate(text, old, new, which):
    assert old in text, f"mutation anchor not found: {old!r}"
    if which is None:
        return text.replace(old, new)
    parts = text.split(old)
    assert which < len(parts) - 1
    return old.join(parts[: which + 1]) + new + old.join(parts[which + 1:])


@pytest.mark.parametrize("mid,old,new,which", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_kill_mutant(mid, old, new, which):
    with open(SRC) as f:
        text = f.read()
    mutated = _mutate(text, old, new, which)
    assert mutated != text
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "mutant.c")
        lib = os.path.join(td, "libmutant.so")
        with open(src, "w") as f:
            f.write(mutated)
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", src,
                               "-o", lib, "-lm"])
        env = dict(os.environ, GEMM_EPI_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                           env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"mutant {mid} survived the pins:\n{r.stdout[-2000:]}"
