/*
 * gemm_epi_oracle.c -- plain, slow, obviously correct CPU reference for
 *
 *     D = act(alpha * (A . B) + bias)      and     mask = (alpha * (A . B) + bias) > 0
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or call this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with the
 * CUDA library: it decodes every input format itself from the format's
 * definition and does all arithmetic in IEEE double.
 *
 * What is computed, and where the pages define it:
 *   - the product A.B with a wide accumulator ("compute type 32F"): page
 *     "PyTorch inference: cuBLASLt bias fusion optimization" (blog.hotdry.top),
 *     paragraph 3.  The oracle accumulates in double, wider than the method.
 *   - a bias vector added to the product: same page, paragraph 2 (EPILOGUE_BIAS);
 *     its broadcast -- a length-m bias is added to every column of the (m,n)
 *     result, a (1,n) bias to every row -- from "nvmath-python epilog bias
 *     fusion parameters" (blog.hotdry.top), body paragraph 3, and
 *     "nvmath-python cuBLASLt bias fusion for PyTorch inference"
 *     (blog.hotdry.top), paragraph 5 (shape constraints).
 *   - ReLU applied after the bias (RELU_BIAS): "nvmath-python epilog bias
 *     fusion parameters", body paragraph 2.
 *   - the auxiliary output of RELU_AUX_BIAS, the sign mask of the ReLU input
 *     kept for the backward pass: same paragraph, and "nvmath-python cuBLASLt
 *     bias fusion for PyTorch inference", paragraph 6.  Read as: bit set
 *     exactly when the pre-activation is strictly greater than zero.
 *   - GELU after the bias: "PyTorch inference: cuBLASLt bias fusion
 *     optimization", paragraph 2; torch.nn.GELU() in "PyTorch 2.14 NVGEMM
 *     epilogue fusion" (zdabc.icu), section "verifying torch.compile".  Read
 *     as the exact erf form, 0.5 x (1 + erf(x / sqrt 2)).
 *   - tanh after the bias (TANH_BIAS), and the same activations without a bias
 *     (RELU, RELU_AUX, GELU, TANH): the predefined epilogue list of
 *     "nvmath-python cuBLASLt bias fusion for PyTorch inference", paragraph 6
 *     (Bias, ReLU, Tanh and so on).
 *   - a scaling factor applied in the epilogue: "PyTorch 2.14 NVGEMM epilogue
 *     fusion", section "why epilogue fusion matters".  Read as alpha = s_A * s_B
 *     multiplying the product before the bias, for every input type (the FP8
 *     per-tensor dequantisation scales, or a plain scale for 16-bit inputs;
 *     callers pass 1 and 1 for no scaling).
 *
 * Formats decoded here (from their definitions, not from any library):
 *   fp16  IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.
 *   bf16  upper half of IEEE binary32: 1 sign, 8 exponent (bias 127), 7 fraction.
 *   e4m3  OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 fraction,
 *         no infinities, S.1111.111 is NaN, largest finite 448.
 *
 * Result of the full variant: D_ref (double, m x n, row-major) holds the
 * activation output before any rounding to the output type; pre_ref (double,
 * optional) holds the pre-activation p; mask_ref (uint8, optional) holds
 * 1 where p > 0 else 0 for every epilogue.  The sampled variant computes the
 * same three quantities at a list of (row, col) positions, one dot product
 * each.
 *
 * Status codes: 0 ok, -1 bad argument (unknown name, non-positive size, NULL
 * buffer where one is required), -2 out of memory.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- the oracle's own vocabulary (independent of the CUDA library's enums) --- */
enum { OR_F16 = 1, OR_BF16 = 2, OR_E4M3 = 3 };
enum { OR_NONE = 10, OR_BIAS = 11, OR_RELU_BIAS = 12, OR_RELU_AUX_BIAS = 13, OR_GELU_BIAS = 14,
       OR_TANH_BIAS = 15, OR_RELU = 16, OR_RELU_AUX = 17, OR_GELU = 18, OR_TANH = 19 };
enum { OR_ROW = 20, OR_COL = 21 };
enum { OR_KN = 30, OR_NK = 31 };

static int dtype_code(const char *s) {
    if (!s) return 0;
    if (!strcmp(s, "f16")) return OR_F16;
    if (!strcmp(s, "bf16")) return OR_BF16;
    if (!strcmp(s, "e4m3")) return OR_E4M3;
    return 0;
}
static int epi_code(const char *s) {
    if (!s) return 0;
    if (!strcmp(s, "none")) return OR_NONE;
    if (!strcmp(s, "bias")) return OR_BIAS;
    if (!strcmp(s, "relu_bias")) return OR_RELU_BIAS;
    if (!strcmp(s, "relu_aux_bias")) return OR_RELU_AUX_BIAS;
    if (!strcmp(s, "gelu_bias")) return OR_GELU_BIAS;
    if (!strcmp(s, "tanh_bias")) return OR_TANH_BIAS;
    if (!strcmp(s, "relu")) return OR_RELU;
    if (!strcmp(s, "relu_aux")) return OR_RELU_AUX;
    if (!strcmp(s, "gelu")) return OR_GELU;
    if (!strcmp(s, "tanh")) return OR_TANH;
    return 0;
}
static int axis_code(const char *s) {
    if (!s) return 0;
    if (!strcmp(s, "row")) return OR_ROW;
    if (!strcmp(s, "col")) return OR_COL;
    return 0;
}
/* Operand storage.  B: "kn" = (k, n) row-major, "nk" = (n, k) row-major.  A is
 * (m, k) row-major unless the layout string carries the prefix "at_" ("at_kn",
 * "at_nk"): then A is stored transposed, (k, m) row-major. */
enum { OR_MK = 40, OR_KM = 41 };
static int a_layout_of(const char *s) { return (s && !strncmp(s, "at_", 3)) ? OR_KM : OR_MK; }
static int layout_code(const char *s) {
    if (!s) return 0;
    if (!strncmp(s, "at_", 3)) s += 3;
    if (!strcmp(s, "kn")) return OR_KN;
    if (!strcmp(s, "nk")) return OR_NK;
    return 0;
}
/* Where element (i, t) of the (m, k) operand A is stored. */
static int64_t a_index(int la, int64_t i, int64_t t, int64_t m, int64_t k) {
    return la == OR_MK ? i * k + t : t * m + i;
}

/* ---- format decoding, written from each format's bit-level definition ----- */

double oracle_decode_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^(1-15-10) */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp(1.0 + (double)f / 1024.0, e - 15);
    }
    return sign ? -v : v;
}

double oracle_decode_bf16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -133);                /* subnormal: f * 2^(1-127-7) */
    } else if (e == 255) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp(1.0 + (double)f / 128.0, e - 127);
    }
    return sign ? -v : v;
}

double oracle_decode_e4m3(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xf;
    int f = b & 0x7;
    double v;
    if (e == 15 && f == 7) {
        v = NAN;                                   /* the only NaN pattern; no infinities */
    } else if (e == 0) {
        v = ldexp((double)f, -9);                  /* subnormal: f * 2^(1-7-3) */
    } else {
        v = ldexp(1.0 + (double)f / 8.0, e - 7);
    }
    return sign ? -v : v;
}

/* GELU, exact form: x * Phi(x) with Phi the standard normal CDF. */
double oracle_gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }

static double load(const void *base, int dt, int64_t idx) {
    switch (dt) {
    case OR_F16: return oracle_decode_f16(((const uint16_t *)base)[idx]);
    case OR_BF16: return oracle_decode_bf16(((const uint16_t *)base)[idx]);
    case OR_E4M3: return oracle_decode_e4m3(((const uint8_t *)base)[idx]);
    }
    return NAN;
}

/* The bias and the output share the input type for 16-bit inputs; for e4m3
 * inputs they are bf16. */
static int bias_dtype(int dt) { return dt == OR_E4M3 ? OR_BF16 : dt; }

/* Epilogues that add a bias vector. */
static int has_bias(int epi) {
    return epi == OR_BIAS || epi == OR_RELU_BIAS || epi == OR_RELU_AUX_BIAS || epi == OR_GELU_BIAS ||
           epi == OR_TANH_BIAS;
}

/* One output element after the product p = sum_t a(i,t) b(t,j) is known. */
static void finish(double p, int epi, int axis, int bdt, const void *bias, int64_t i, int64_t j,
                   double alpha, double *d, double *pre, uint8_t *mask) {
    p = alpha * p;
    if (has_bias(epi)) p += load(bias, bdt, axis == OR_ROW ? i : j);
    double y;
    switch (epi) {
    case OR_RELU_BIAS:
    case OR_RELU_AUX_BIAS:
    case OR_RELU:
    case OR_RELU_AUX: y = p > 0.0 ? p : 0.0; break;
    case OR_GELU_BIAS:
    case OR_GELU: y = oracle_gelu(p); break;
    case OR_TANH_BIAS:
    case OR_TANH: y = tanh(p); break;
    default: y = p; break;                         /* NONE and BIAS */
    }
    *d = y;
    if (pre) *pre = p;
    if (mask) *mask = (uint8_t)(p > 0.0);
}

static int check_args(int64_t m, int64_t n, int64_t k, int dt, int epi, int axis, int lay,
                      const void *A, const void *B, const void *bias) {
    if (m <= 0 || n <= 0 || k <= 0) return -1;
    if (!dt || !epi || !axis || !lay) return -1;
    if (!A || !B) return -1;
    if (has_bias(epi) && !bias) return -1;
    return 0;
}

/*
 * Full result.  Loop order i (rows, OpenMP) -> t (reduction) -> j (columns):
 * each output row is accumulated in a double row buffer; B is decoded once
 * into a (k, n) double array whatever its stored layout.
 */
int oracle_gemm_epi(int64_t m, int64_t n, int64_t k, const char *dtype, const char *epilogue,
                    const char *bias_axis, const char *b_layout, const void *A, const void *B,
                    const void *bias, double scale_a, double scale_b, double *D_ref,
                    double *pre_ref, uint8_t *mask_ref) {
    int dt = dtype_code(dtype), epi = epi_code(epilogue), axis = axis_code(bias_axis);
    int lay = layout_code(b_layout), la = a_layout_of(b_layout);
    if (check_args(m, n, k, dt, epi, axis, lay, A, B, bias) || !D_ref) return -1;
    double alpha = scale_a * scale_b;
    int bdt = bias_dtype(dt);

    double *Bd = (double *)malloc((size_t)k * (size_t)n * sizeof(double));
    if (!Bd) return -2;
    for (int64_t t = 0; t < k; ++t)
        for (int64_t j = 0; j < n; ++j)
            Bd[t * n + j] = load(B, dt, lay == OR_KN ? t * n + j : j * k + t);

    int err = 0;
#pragma omp parallel
    {
        double *row = (double *)malloc((size_t)n * sizeof(double));
        if (!row) {
#pragma omp atomic write
            err = -2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < m; ++i) {
            if (!row) continue;
            for (int64_t j = 0; j < n; ++j) row[j] = 0.0;
            for (int64_t t = 0; t < k; ++t) {
                double a = load(A, dt, a_index(la, i, t, m, k));
                const double *brow = Bd + t * n;
                for (int64_t j = 0; j < n; ++j) row[j] += a * brow[j];
            }
            for (int64_t j = 0; j < n; ++j)
                finish(row[j], epi, axis, bdt, bias, i, j, alpha, &D_ref[i * n + j],
                       pre_ref ? &pre_ref[i * n + j] : NULL,
                       mask_ref ? &mask_ref[i * n + j] : NULL);
        }
        free(row);
    }
    free(Bd);
    return err;
}

/*
 * The same quantities at `count` positions (rows[s], cols[s]): one plain dot
 * product over t per position, read straight from the stored operands.
 */
int oracle_gemm_epi_sampled(int64_t m, int64_t n, int64_t k, const char *dtype,
                            const char *epilogue, const char *bias_axis, const char *b_layout,
                            const void *A, const void *B, const void *bias, double scale_a,
                            double scale_b, int64_t count, const int64_t *rows,
                            const int64_t *cols, double *D_ref, double *pre_ref,
                            uint8_t *mask_ref) {
    int dt = dtype_code(dtype), epi = epi_code(epilogue), axis = axis_code(bias_axis);
    int lay = layout_code(b_layout), la = a_layout_of(b_layout);
    if (check_args(m, n, k, dt, epi, axis, lay, A, B, bias) || !D_ref || !rows || !cols ||
        count < 0)
        return -1;
    for (int64_t s = 0; s < count; ++s)
        if (rows[s] < 0 || rows[s] >= m || cols[s] < 0 || cols[s] >= n) return -1;
    double alpha = scale_a * scale_b;
    int bdt = bias_dtype(dt);
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t s = 0; s < count; ++s) {
        int64_t i = rows[s], j = cols[s];
        double p = 0.0;
        for (int64_t t = 0; t < k; ++t)
            p += load(A, dt, a_index(la, i, t, m, k)) * load(B, dt, lay == OR_KN ? t * n + j : j * k + t);
        finish(p, epi, axis, bdt, bias, i, j, alpha, &D_ref[s], pre_ref ? &pre_ref[s] : NULL,
               mask_ref ? &mask_ref[s] : NULL);
    }
    return 0;
}

/*
 * Backward epilogues (the mask of a forward RELU_AUX(_BIAS) fed back in).
 * "nvmath-python cuBLASLt bias fusion for PyTorch inference" (blog.hotdry.top),
 * paragraph 6: the auxiliary output of RELU_AUX_BIAS is the mask the backward
 * pass needs; paragraph 7: fusing dBias is the next step.  Read as the usual
 * ReLU backward of a layer z = alpha*A.B + bias, y = relu(z):
 *
 *   "drelu":        D(i,j) = mask(i,j) ? alpha * sum_t a(i,t) b(t,j) : 0
 *   "drelu_bgrad":  the same D, plus the bias gradient, the sum of D over the
 *                   axis the bias was broadcast along:
 *                     ROW bias (length m): dbias(i) = sum_j D(i,j)
 *                     COL bias (length n): dbias(j) = sum_i D(i,j)
 *
 * mask is m x n bytes (0/1, row-major); dbias may be NULL for "drelu".
 * Everything is accumulated in double; D_ref is not rounded.
 */
int oracle_gemm_epi_bwd(int64_t m, int64_t n, int64_t k, const char *dtype, const char *epilogue,
                        const char *bias_axis, const char *b_layout, const void *A, const void *B,
                        const uint8_t *mask, double scale_a, double scale_b, double *D_ref,
                        double *dbias_ref) {
    int dt = dtype_code(dtype), axis = axis_code(bias_axis), lay = layout_code(b_layout);
    int la = a_layout_of(b_layout);
    int bgrad;
    if (!epilogue) return -1;
    if (!strcmp(epilogue, "drelu")) bgrad = 0;
    else if (!strcmp(epilogue, "drelu_bgrad")) bgrad = 1;
    else return -1;
    if (m <= 0 || n <= 0 || k <= 0 || !dt || !axis || !lay || !A || !B || !mask || !D_ref) return -1;
    if (bgrad && !dbias_ref) return -1;
    const double alpha = scale_a * scale_b;

    double *Bd = (double *)malloc((size_t)k * (size_t)n * sizeof(double));
    if (!Bd) return -2;
    for (int64_t t = 0; t < k; ++t)
        for (int64_t j = 0; j < n; ++j)
            Bd[t * n + j] = load(B, dt, lay == OR_KN ? t * n + j : j * k + t);
    int err = 0;
#pragma omp parallel
    {
        double *row = (double *)malloc((size_t)n * sizeof(double));
        if (!row) {
#pragma omp atomic write
            err = -2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < m; ++i) {
            if (!row) continue;
            for (int64_t j = 0; j < n; ++j) row[j] = 0.0;
            for (int64_t t = 0; t < k; ++t) {
                double a = load(A, dt, a_index(la, i, t, m, k));
                const double *brow = Bd + t * n;
                for (int64_t j = 0; j < n; ++j) row[j] += a * brow[j];
            }
            for (int64_t j = 0; j < n; ++j)
                D_ref[i * n + j] = mask[i * n + j] ? alpha * row[j] : 0.0;
        }
        free(row);
    }
    free(Bd);
    if (err) return err;
    if (bgrad) {
        if (axis == OR_ROW) {
            for (int64_t i = 0; i < m; ++i) {
                double s = 0.0;
                for (int64_t j = 0; j < n; ++j) s += D_ref[i * n + j];
                dbias_ref[i] = s;
            }
        } else {
            for (int64_t j = 0; j < n; ++j) dbias_ref[j] = 0.0;
            for (int64_t i = 0; i < m; ++i)
                for (int64_t j = 0; j < n; ++j) dbias_ref[j] += D_ref[i * n + j];
        }
    }
    return 0;
}

/*
 * Encoding a real value into a storage format (the inverse of the decoders
 * above), for results that are stored in a narrower type: the intermediate H
 * of an MLP block (up-projection, then down-projection; "nvmath-python
 * cuBLASLt bias fusion for PyTorch inference" (blog.hotdry.top), paragraph 1:
 * the MLP is where the GEMM + bias time goes) and its FP8 form (paragraph 5:
 * FP8 inputs; "PyTorch 2.14 NVGEMM epilogue fusion" (zdabc.icu), section "why
 * epilogue fusion matters": scaling and type conversion in the epilogue).
 *
 * Written from the formats' definitions only: the non-negative finite codes
 * 0 .. max_code of each format decode (with the decoders above) to strictly
 * increasing values, so |x| is located between two neighbouring codes by
 * bisection and rounded to the nearer; a tie goes to the code whose last
 * fraction bit is 0 (round to nearest, ties to even).  Beyond the largest
 * finite value, e4m3 saturates to it (+-448); fp16 and bf16 round to
 * infinity once |x| reaches the largest finite value plus half its spacing.
 * The sign bit is copied from x (so -0.0 and tiny negatives give -0).
 */
static double decode_code(int dt, uint32_t c) {
    switch (dt) {
    case OR_F16: return oracle_decode_f16((uint16_t)c);
    case OR_BF16: return oracle_decode_bf16((uint16_t)c);
    case OR_E4M3: return oracle_decode_e4m3((uint8_t)c);
    }
    return NAN;
}

static uint32_t encode_value(int dt, double x) {
    const uint32_t max_code = dt == OR_E4M3 ? 0x7Eu : dt == OR_F16 ? 0x7BFFu : 0x7F7Fu;
    const uint32_t inf_code = dt == OR_F16 ? 0x7C00u : 0x7F80u;     /* 16-bit formats only */
    const uint32_t sign_bit = dt == OR_E4M3 ? 0x80u : 0x8000u;
    const int neg = signbit(x) != 0;
    const double a = fabs(x);
    const double vmax = decode_code(dt, max_code);
    uint32_t code;
    if (!(a < vmax)) {
        if (dt == OR_E4M3) {
            code = max_code;
        } else {
            /* half the spacing below the largest finite value equals half the spacing above it */
            const double half = 0.5 * (vmax - decode_code(dt, max_code - 1));
            code = a < vmax + half ? max_code : inf_code;
        }
    } else {
        uint32_t lo = 0, hi = max_code;         /* decode(lo) <= a < decode(hi) */
        while (hi - lo > 1) {
            const uint32_t mid = lo + (hi - lo) / 2;
            if (decode_code(dt, mid) <= a) lo = mid;
            else hi = mid;
        }
        const double dl = a - decode_code(dt, lo), dh = decode_code(dt, hi) - a;
        if (dl < dh) code = lo;
        else if (dh < dl) code = hi;
        else code = (lo & 1u) ? hi : lo;
    }
    return neg ? (code | sign_bit) : code;
}

uint8_t oracle_encode_e4m3(double x) { return (uint8_t)encode_value(OR_E4M3, x); }
uint16_t oracle_encode_f16(double x) { return (uint16_t)encode_value(OR_F16, x); }
uint16_t oracle_encode_bf16(double x) { return (uint16_t)encode_value(OR_BF16, x); }

/*
 * codes[i] = encode(x[i] / scale) in `dtype` storage (uint8 for e4m3, uint16
 * otherwise): the per-tensor quantisation of the MLP block's intermediate,
 * scale > 0 (s = amax / 448 is the usual choice for e4m3; 1 stores the values
 * themselves).  Returns 0, or -1 on a bad argument.
 */
int oracle_encode(int64_t count, const char *dtype, const double *x, double scale, void *codes) {
    const int dt = dtype_code(dtype);
    if (!dt || count < 0 || !x || !codes || !(scale > 0.0)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        const uint32_t c = encode_value(dt, x[i] / scale);
        if (dt == OR_E4M3) ((uint8_t *)codes)[i] = (uint8_t)c;
        else ((uint16_t *)codes)[i] = (uint16_t)c;
    }
    return 0;
}
