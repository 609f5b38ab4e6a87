/*
 * gemm_epi.h -- fused GEMM + bias + activation for NVIDIA B200 (sm_100a).
 *
 *     D = act(alpha * (A . B) + bias)          aux = packed bits of (alpha*(A.B) + bias) > 0
 *
 * One persistent kernel computes the product on the tcgen05 tensor cores with
 * the fp32 accumulator in tensor memory, finishes every accumulator tile in
 * registers (scale, bias, activation, sign mask, rounding to the output type)
 * and writes it to HBM once.
 *
 * Where the pages define the operation
 *   [bias-fusion]   "PyTorch inference: cuBLASLt bias fusion optimization"
 *                   (blog.hotdry.top/posts/2025/09/22/pytorch-inference-cublaslt-bias-fusion-optimization)
 *   [nvmath-fusion] "nvmath-python cuBLASLt bias fusion for PyTorch inference"
 *                   (blog.hotdry.top/posts/2025/09/22/nvmath-python-cublaslt-bias-fusion-for-pytorch-inference)
 *   [epilog-params] "nvmath-python epilog bias fusion parameters"
 *                   (blog.hotdry.top/agent/posts/2025/09/22/nvmath-python-epilog-bias-fusion-parameters)
 *   [nvgemm]        "PyTorch 2.14 NVGEMM epilogue fusion" (zdabc.icu/article/2026/9/3/3582.html)
 *
 * Conventions for every entry point
 *   - A is row-major (m, k) (or (k, m) with the GEMM_EPI_A_KM layout flag).  B is row-major (k, n) (GEMM_EPI_B_KN, default)
 *     or row-major (n, k) (GEMM_EPI_B_NK: an nn.Linear weight, D = A . B^T).
 *   - D is row-major (m, n), densely packed (row pitch n elements).
 *   - Accumulation and all epilogue arithmetic are fp32; D is rounded to
 *     nearest even.  fp16 inputs give fp16 bias and D; bf16 gives bf16; e4m3
 *     inputs give bf16 bias and D ([nvmath-fusion] paragraph 5: input, weight
 *     and bias types agree; FP8 keeps a 16-bit output).
 *   - Every pointer passed to run() is a DEVICE pointer into memory of the
 *     current CUDA device, owned by the caller, 16-byte aligned ([epilog-params]
 *     body paragraph 3).  Row pitches k*esize and n*esize must be multiples of
 *     16 bytes: k and n multiples of 8 for 16-bit types, of 16 for e4m3.
 *   - Calls are asynchronous on the given stream (a cudaStream_t passed as
 *     void*, NULL = legacy default stream) and never synchronise.
 *   - The GEMM kernels are launched with programmatic stream serialisation:
 *     their launch and on-chip setup may overlap the previous kernel on the
 *     stream, but they read and write no global memory before that kernel has
 *     completed, so stream order is kept.  GEMM_EPI_PDL=0 in the environment
 *     (read when a plan is created) launches them plainly.
 *   - On any error nothing is launched and a negative status is returned.
 */
#ifndef GEMM_EPI_H
#define GEMM_EPI_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- enumerations -------------------------------------------------------- */

/* Operand types ([nvmath-fusion] paragraph 5: FP16, BF16, FP8). */
enum gemm_epi_dtype { GEMM_EPI_F16 = 0, GEMM_EPI_BF16 = 1, GEMM_EPI_E4M3 = 2 };

/* Epilogues ([epilog-params] body paragraph 2; [bias-fusion] paragraph 2 for GELU;
 * [nvmath-fusion] paragraph 6 lists Tanh among the predefined ones).  x = alpha*A.B + bias
 * for the *_BIAS epilogues and x = alpha*A.B for the others, which ignore the bias
 * argument (it may be NULL).
 *   NONE           D = alpha*A.B                   (the bare GEMM)
 *   BIAS           D = x
 *   RELU_BIAS      D = max(x, 0)
 *   RELU_AUX_BIAS  as RELU_BIAS, plus aux = sign mask of the ReLU input x
 *   GELU_BIAS      D = GELU(x) = 0.5 x (1 + erf(x / sqrt 2))
 *   TANH_BIAS      D = tanh(x)
 *   RELU, RELU_AUX, GELU, TANH: the same without a bias
 * Backward epilogues (run with gemm_epi_run_bwd / gemm_epi_unfused_run_bwd only): the
 * ReLU backward of a layer z = alpha*A.B + bias, y = relu(z), fed the aux mask that the
 * forward RELU_AUX(_BIAS) wrote ([nvmath-fusion] paragraph 6: the mask is kept for the
 * backward pass; paragraph 7: fusing dBias is the next step).  g = alpha*A.B is the
 * incoming gradient (for example dY . W of the next layer):
 *   DRELU          D = mask ? g : 0
 *   DRELU_BGRAD    as DRELU, plus dbias = the sum of D over the axis the forward bias
 *                  was broadcast along: ROW (bias length m): dbias[i] = sum_j D[i][j];
 *                  COL (bias length n): dbias[j] = sum_i D[i][j].  The sums are taken in
 *                  fp32 on the unrounded values of D, in an order fixed by the shapes
 *                  (identical results from run to run), and rounded once to the bias type. */
enum gemm_epi_epilogue {
    GEMM_EPI_NONE = 0,
    GEMM_EPI_BIAS = 1,
    GEMM_EPI_RELU_BIAS = 2,
    GEMM_EPI_RELU_AUX_BIAS = 3,
    GEMM_EPI_GELU_BIAS = 4,
    GEMM_EPI_TANH_BIAS = 5,
    GEMM_EPI_RELU = 6,
    GEMM_EPI_RELU_AUX = 7,
    GEMM_EPI_GELU = 8,
    GEMM_EPI_TANH = 9,
    GEMM_EPI_DRELU = 10,
    GEMM_EPI_DRELU_BGRAD = 11
};

/* Bias broadcast ([epilog-params] body paragraph 3; [nvmath-fusion] paragraph 5):
 *   ROW  bias has length m; bias[i] is added to every column of output row i
 *        (a (m,1) bias -- the pages' default).
 *   COL  bias has length n; bias[j] is added to every row of output column j
 *        (a (1,n) bias). */
enum gemm_epi_bias_axis { GEMM_EPI_BIAS_ROW = 0, GEMM_EPI_BIAS_COL = 1 };

/* Operand storage, passed as `b_layout`: GEMM_EPI_B_KN or GEMM_EPI_B_NK for B, optionally
 * OR-ed with GEMM_EPI_A_KM for an A stored transposed, (k, m) row-major (m contiguous; its
 * row pitch m*esize must be a multiple of 16 bytes).  A stored (k, m) runs on the persistent
 * kernels with 256-wide tiles (block_n 128 is ERR_UNSUPPORTED; small m uses TC1) and the
 * forward epilogues, not with the backward epilogues or an e4m3 output. */
enum gemm_epi_b_layout { GEMM_EPI_B_KN = 0, GEMM_EPI_B_NK = 1, GEMM_EPI_A_KM = 2 };

/* Kernel families a plan can use.  GEMM_EPI_KERNEL_AUTO lets the plan choose: SPLITK for
 * m <= 64 (forward epilogues, A stored (m, k)), TC2 when there is a 256 x 256 tile for every SM
 * pair, TC1 otherwise. */
enum gemm_epi_kernel {
    GEMM_EPI_KERNEL_AUTO = 0,
    GEMM_EPI_KERNEL_TC1 = 1,    /* persistent, one CTA per 128 x block_n tile           */
    GEMM_EPI_KERNEL_TC2 = 2,    /* persistent, CTA pair (cta_group::2) per 256 x block_n */
    GEMM_EPI_KERNEL_SPLITK = 3  /* small m: operand roles swapped, K split over a cluster */
};

/* Status codes. */
enum gemm_epi_status {
    GEMM_EPI_OK = 0,
    GEMM_EPI_ERR_ARG = -1,          /* size <= 0, unknown enum, bad option, bad plan handle */
    GEMM_EPI_ERR_ALIGN = -2,        /* pointer not 16-byte aligned, or row pitch not a multiple of 16 B */
    GEMM_EPI_ERR_NULL = -3,         /* required pointer NULL (A, B, D; bias for a bias epilogue;
                                       aux for RELU_AUX(_BIAS) and the backward epilogues; dbias
                                       for DRELU_BGRAD; scales unset for E4M3) */
    GEMM_EPI_ERR_UNSUPPORTED = -4,  /* valid request this library cannot serve (option combination) */
    GEMM_EPI_ERR_CUDA = -5,         /* a CUDA runtime/driver call failed (launch, tensor map) */
    GEMM_EPI_ERR_TIMEOUT = -6,      /* a kernel gave up on a bounded wait (reported by check()) */
    GEMM_EPI_ERR_NO_DEVICE = -7     /* current device is not sm_100 (B200 class) */
};

/* Opaque plan.  Created by gemm_epi_plan*, owned by the caller until
 * gemm_epi_free; holds host metadata, a tensor-map cache, one 256-byte
 * device status word and, when the plan uses stream-K, a workspace for
 * partial tiles plus their flags; a DRELU_BGRAD plan also owns an fp32 workspace for
 * the bias-gradient partial sums (ROW: m x ceil(n/block_n) floats; COL: n x
 * ceil(m/32) floats).  A plan may be run any number of times, on any stream,
 * from one host thread at a time. */
typedef struct gemm_epi_plan_s *gemm_epi_plan_t;

/* Optional tuning knobs; zero-initialise for automatic choices. */
typedef struct gemm_epi_options {
    int32_t kernel;    /* enum gemm_epi_kernel                                        */
    int32_t block_n;   /* output tile width (128, 256, or 512 for TC2 forward plans; 0 =
                          auto, which takes 512 for TC2 with 16-bit operands, an epilogue
                          without GELU / tanh and at least four waves of 256 x 512 tiles).  TC2 with e4m3 and B stored (k, n) supports
                          256 and 512 only (128 is ERR_UNSUPPORTED)                       */
    int32_t split_k;   /* SPLITK: CTAs per cluster along k (1..8; 0 = auto: 8 when there are
                          at most 8 tiles of 128 columns, else the largest of 4, 3, 2, 1 that
                          keeps the launch at or under 128 CTAs, so that every cluster is
                          resident at once; capped at the split the batch tile allows).  TC1/TC2:
                          cap on the parts a tail tile is split into (0 = auto: 2 behind
                          whole waves; with fewer tiles than SMs up to 4, at least 8
                          128-byte k-atoms a part).  The parts are whole ring stages
                          (gemm_epi_plan_info.block_k of k each), so a value above the
                          number of stages k makes, or above the idle units, is lowered
                          to that number (gemm_epi_plan_info.sk_split reports it)      */
    int32_t max_ctas;  /* persistent kernels: cap on resident CTAs (0 = one per SM)    */
    int32_t inject_stall; /* testing only (TC1/TC2): 1 = the MMA issuer never publishes an
                             accumulator, so the epilogue's bounded wait runs out after about
                             one second and gemm_epi_check() reports GEMM_EPI_ERR_TIMEOUT;
                             D is left unwritten.  0 for real work.                        */
    int32_t stream_k;  /* TC1/TC2: 0 = auto, 1 = off, 2 = on.  Splits the tiles of an
                          incomplete last wave (or all tiles, when there are fewer tiles than
                          SMs) along k over several SMs (stream-K style); partial tiles pass
                          through a workspace the plan allocates (SMs x 128 x block_n fp32). */
    int32_t out_e4m3;  /* 1 = D is e4m3, quantised in the epilogue: D = e4m3(y / s_out) with
                          round to nearest even, saturating at +-448, y the epilogue's fp32
                          result; max |y| is reported (gemm_epi_set_out_scale).  E4M3 plans
                          with epilogue NONE, BIAS, RELU_BIAS, GELU_BIAS, RELU or GELU, on every
                          kernel family; else ERR_UNSUPPORTED.
                          0 = D in the 16-bit output type.                              */
} gemm_epi_options;

/* What a plan decided (for logging and tests). */
typedef struct gemm_epi_plan_info {
    int32_t kernel, block_m, block_n, block_k, stages, split_k;
    int32_t grid, cluster, threads, smem_bytes, tiles;
    int32_t sk_tiles, sk_split;   /* split tail: tiles split along k, parts per split tile */
    int32_t group_m, group_n;     /* TC tile raster: groups of group_m tile-rows walked column by
                                     column, or (group_m == 0) groups of group_n tile-columns
                                     walked row by row; 0, 0 for SPLITK */
} gemm_epi_plan_info;

/* ---- entry points -------------------------------------------------------- */

/* Create a plan for D = act(alpha*A.B + bias) with B stored (k, n).
 * The stateful plan / execute / free life cycle follows [nvmath-fusion]
 * paragraphs 3 and 5 (Matmul.plan(epilog=..., epilog_inputs={"bias": ...}),
 * execute(), free()).
 * m, n, k >= 1; dtype/epilogue/bias_axis from the enums above.
 * Returns GEMM_EPI_OK and *out, or ERR_ARG / ERR_ALIGN (pitch rule) /
 * ERR_NO_DEVICE / ERR_CUDA; *out is untouched on error.  Needs a current CUDA
 * device of compute capability 10.0 (allocates the status word there). */
int gemm_epi_plan(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis,
                  gemm_epi_plan_t *out);

/* As gemm_epi_plan, with the storage of B given explicitly. */
int gemm_epi_plan_ex(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis,
                     int b_layout, gemm_epi_plan_t *out);

/* As gemm_epi_plan_ex, with tuning options (opts may be NULL). */
int gemm_epi_plan_opts(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis,
                       int b_layout, const gemm_epi_options *opts, gemm_epi_plan_t *out);

/* Per-tensor fp32 scales s_A, s_B as DEVICE pointers to one float each, read
 * by every run; alpha = s_A * s_B multiplies the product before the bias (the
 * epilogue scaling factor of [nvgemm], section "why epilogue fusion matters").
 * Required for E4M3 plans (the dequantisation scales); optional for 16-bit
 * plans, whose alpha is 1 until set (both NULL resets it).  The pointers are
 * borrowed, not owned.  ERR_NULL if only one is given. */
int gemm_epi_set_scales(gemm_epi_plan_t plan, const float *d_scale_a, const float *d_scale_b);

/* For plans created with options.out_e4m3 = 1: the output scale s_out (DEVICE pointer to
 * one float, > 0; D = e4m3(y / s_out), the usual choice being amax / 448 from an earlier
 * run) and, optionally, d_amax (DEVICE pointer to one float): each run sets it to 0 on the
 * stream before the launch and the kernel max-reduces |y| into it, so after the run it
 * holds max |y| over D before quantisation (exact: a maximum does not depend on order).
 * Borrowed, not owned.  ERR_ARG for other plans, ERR_NULL without d_scale_out, ERR_ALIGN
 * for pointers not 4-byte aligned.  A run of such a plan without a scale is ERR_NULL; its
 * unfused run is ERR_UNSUPPORTED. */
int gemm_epi_set_out_scale(gemm_epi_plan_t plan, const float *d_scale_out, float *d_amax);

/* Enqueue the fused kernel: one launch, D (and aux) written once.
 *   A     (m, k) operand, B (k, n) or (n, k) operand, device pointers.
 *   bias  length m (ROW) or n (COL), output type; ignored (may be NULL) for the
 *         epilogues without a bias.
 *   D     (m, n) output.
 *   aux   RELU_AUX_BIAS and RELU_AUX only (else ignored, may be NULL): packed sign mask,
 *         row-major uint32 words, row pitch gemm_epi_aux_pitch_bytes(n);
 *         bit b of word w in row i is 1 iff the fp32 pre-activation of
 *         element (i, 32w + b) is > 0 (taken before rounding to the output
 *         type); bits past column n-1 are 0.  ([epilog-params] body
 *         paragraph 2: the ReLU input's sign mask kept for the backward pass.)
 *   stream  cudaStream_t as void*.
 * Returns OK, ERR_ARG (bad plan, or a current device other than the one the
 * plan was created on), ERR_NULL, ERR_ALIGN or ERR_CUDA.  A kernel that gives
 * up on a bounded internal wait records it in the plan's status word;
 * gemm_epi_check() reports it.  The same device rule holds for every run entry
 * point below. */
int gemm_epi_run(gemm_epi_plan_t plan, const void *A, const void *B, const void *bias, void *D,
                 uint32_t *aux, void *stream);

/* The library's own UNFUSED baseline on the same plan and arguments: the bare
 * GEMM (epilogue NONE) writes alpha*A.B to D in the output type, then a
 * separate elementwise kernel reads D back, adds the bias, applies the
 * activation, writes D (in place) and aux.  Two launches and one extra round
 * trip of D through HBM: the sequence the pages' fusion removes ([epilog-params]
 * body paragraphs 1 and 5: validate the stepwise result first).  It rounds
 * alpha*A.B to the output type before adding the bias, so where the bias
 * cancels a large product its error can exceed the fused path's by up to one
 * unit in the last place of alpha*A.B in the output type. */
int gemm_epi_unfused_run(gemm_epi_plan_t plan, const void *A, const void *B, const void *bias,
                         void *D, uint32_t *aux, void *stream);

/* Enqueue a backward plan (epilogue DRELU or DRELU_BGRAD).
 *   A, B   operands of g = alpha*A.B (as for gemm_epi_run).
 *   aux    the forward pass's packed mask for the (m, n) output, read only: row-major
 *          uint32 words, row pitch gemm_epi_aux_pitch_bytes(n), bit b of word w in row i
 *          for element (i, 32w + b) -- the layout gemm_epi_run writes.  Bits past
 *          column n-1 are ignored.
 *   D      (m, n) output in the output type: D = mask ? alpha*A.B : 0.
 *   dbias  DRELU_BGRAD: output, length m (ROW plan) or n (COL plan), bias type (fp16 for
 *          F16, bf16 for BF16 and E4M3).  DRELU: ignored (may be NULL).
 * Fused: one GEMM launch whose epilogue applies the mask, writes D once and (BGRAD)
 * writes fp32 partial sums of each tile to the plan's workspace, then one small launch
 * that adds the partials in a fixed order and writes dbias.  Every pointer is a 16-byte
 * aligned device pointer.  Returns OK, ERR_ARG (bad handle, or a forward plan),
 * ERR_NULL, ERR_ALIGN or ERR_CUDA; gemm_epi_run with a backward plan returns ERR_ARG.
 * The small-m split-K kernel has no backward epilogue: AUTO plans use TC1 there, and a
 * plan that forces GEMM_EPI_KERNEL_SPLITK fails with ERR_UNSUPPORTED. */
int gemm_epi_run_bwd(gemm_epi_plan_t plan, const void *A, const void *B, const uint32_t *aux, void *D,
                     void *dbias, void *stream);

/* The UNFUSED baseline of gemm_epi_run_bwd on the same plan and arguments: the bare
 * GEMM writes alpha*A.B to D, an elementwise kernel reads D back and zeroes it where
 * the mask is 0, and (BGRAD) a third kernel reads D again and sums it along the bias
 * axis (so dbias here adds values already rounded to the output type). */
int gemm_epi_unfused_run_bwd(gemm_epi_plan_t plan, const void *A, const void *B, const uint32_t *aux,
                             void *D, void *dbias, void *stream);

/* Synchronise `stream`, read and clear the plan's device status word.
 * Returns OK, ERR_TIMEOUT (some kernel of this plan gave up waiting since the
 * last check), ERR_CUDA (a sticky CUDA error) or ERR_ARG. */
int gemm_epi_check(gemm_epi_plan_t plan, void *stream);

/* Fill *info with the plan's kernel choice.  ERR_ARG on a bad handle. */
int gemm_epi_plan_query(gemm_epi_plan_t plan, gemm_epi_plan_info *info);

/* The kernel choice gemm_epi_plan_opts would make on a compute-capability 10.0 device
 * with num_sms SMs, computed on the host alone: no device is needed or touched, nothing is
 * allocated or launched.  Arguments as gemm_epi_plan_opts (opts may be NULL); num_sms in
 * 2..1024 (148 on a B200); info is a HOST pointer, filled as by gemm_epi_plan_query.
 * Returns OK, or the status gemm_epi_plan_opts returns for these arguments before it
 * looks at the device (ERR_ARG / ERR_ALIGN / ERR_UNSUPPORTED); ERR_ARG for a NULL info
 * or num_sms out of range.  *info is untouched on error.  (A service of this library;
 * the pages have no counterpart.) */
int gemm_epi_plan_preview(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis,
                          int b_layout, const gemm_epi_options *opts, int num_sms,
                          gemm_epi_plan_info *info);

/* Fused run that allocates nothing (the pages have no counterpart; this is a
 * service of this library).  For callers that must not allocate device memory:
 * code inside a host framework that hands out all device memory from its own
 * pool and forbids side allocations, or code on a latency-critical path that
 * cannot afford cudaMalloc/cudaFree and their implicit synchronisation.  Such
 * callers cannot create a plan (a plan allocates its status word), so this
 * call takes the problem description and the buffers directly and computes
 * what gemm_epi_plan_ex + gemm_epi_run would (same kernels, same automatic
 * kernel choice, same argument rules and errors), except that the split tail
 * (options.stream_k), which needs a workspace, is off: where a plan would
 * split its last wave's tiles along k, the sums are taken in another order and
 * the results agree with gemm_epi_run within the library's tolerance rather
 * than bit for bit.  Forward epilogues only (NONE .. TANH); the backward ones
 * return GEMM_EPI_ERR_ARG.
 *
 * Arguments: as gemm_epi_plan_ex and gemm_epi_run; d_scale_a/d_scale_b as in
 * gemm_epi_set_scales (E4M3 only, else ignored).  wait = 0: enqueue and
 * return; a kernel that gives up on a bounded wait goes unreported.  wait = 1:
 * also synchronise `stream` and return GEMM_EPI_ERR_TIMEOUT if it did.
 *
 * Scratch and its limits: the kernels' only scratch is a 4-byte status word,
 * kept in a 256-byte static device array that every GPU which loads this
 * library holds until the process exits.  A call that needed more than 256
 * bytes would be refused with GEMM_EPI_ERR_UNSUPPORTED; m, n and k are limited
 * to 2^31 - 1 (GEMM_EPI_ERR_ARG beyond).  Every call on a device shares the
 * array and clears the status word on `stream` before its launch, so calls
 * that overlap on the GPU (other streams, other host threads) race on it: one
 * call's timeout may be reported by another, or lost.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current and keeps it for the life of the process; make that first
 * call before any stream capture.  A cudaDeviceReset between calls is not
 * supported (it unloads the module, and the kept address would go stale).  No
 * cudaMalloc, cudaFree or allocating library routine is called. */
int gemm_epi_run_noalloc(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis,
                         int b_layout, const void *A, const void *B, const void *bias,
                         const float *d_scale_a, const float *d_scale_b, void *D, uint32_t *aux,
                         int wait, void *stream);

/* ---- MLP block ------------------------------------------------------------ */

/* Two fused GEMMs of a transformer MLP ([nvmath-fusion] paragraph 1: the MLP layers are
 * where GEMM + bias time goes):
 *     H = act(alpha1 * X . W1 + b1)     up-projection, act = BIAS, RELU_BIAS or GELU_BIAS
 *     Y = alpha2 * H . W2 + b2          down-projection (BIAS)
 * X is (m, d_model); W1 is (d_model, d_ff) and W2 (d_ff, d_model) for GEMM_EPI_B_KN, or
 * nn.Linear weights (d_ff, d_model) and (d_model, d_ff) for GEMM_EPI_B_NK; b1 has length
 * d_ff, b2 length d_model (per output feature); H (m, d_ff) is caller-owned scratch.
 * fp16 / bf16: alpha1 = alpha2 = 1 and H, Y are in the input type.
 * e4m3: X, W1, W2 are e4m3 with per-tensor scales; the up-projection's epilogue stores H
 * in e4m3 as e4m3(h / s_H) and reports max |h| (the per-tensor requantisation), so
 * alpha1 = s_X * s_W1, alpha2 = s_H * s_W2, and b1, b2, Y are bf16.  Two launches, the
 * second a programmatic dependent of the first; no kernel between them.
 * The handle owns two plans (see gemm_epi_plan); errors as there. */
typedef struct gemm_epi_mlp_s *gemm_epi_mlp_t;

int gemm_epi_mlp_plan(int64_t m, int64_t d_model, int64_t d_ff, int dtype, int act, int w_layout,
                      gemm_epi_mlp_t *out);

/* E4M3 only (ERR_ARG otherwise); all four scales required (ERR_NULL), d_amax_h optional.
 * DEVICE pointers to one float each, borrowed. */
int gemm_epi_mlp_set_scales(gemm_epi_mlp_t mlp, const float *d_scale_x, const float *d_scale_w1,
                            const float *d_scale_h, float *d_amax_h, const float *d_scale_w2);

/* Enqueue both GEMMs on `stream` (all arguments are checked before either is enqueued). */
int gemm_epi_mlp_run(gemm_epi_mlp_t mlp, const void *X, const void *W1, const void *b1, const void *W2,
                     const void *b2, void *H, void *Y, void *stream);

/* The UNFUSED baseline of gemm_epi_mlp_run, same plan and arguments: bare GEMM writing the
 * up-projection in the 16-bit type, a separate bias + activation kernel, and for e4m3 an amax
 * pass and a quantisation pass (H_wide: caller-owned bf16 scratch, (m, d_ff); ignored, may be
 * NULL, for 16-bit plans); then the down-projection as bare GEMM plus bias kernel.  The same
 * result as the fused run up to the roundings it adds; the sequence the epilogues remove. */
int gemm_epi_mlp_unfused_run(gemm_epi_mlp_t mlp, const void *X, const void *W1, const void *b1,
                             const void *W2, const void *b2, void *H, void *Y, void *H_wide,
                             void *stream);

/* gemm_epi_check on both plans (the first non-OK status). */
int gemm_epi_mlp_check(gemm_epi_mlp_t mlp, void *stream);

/* The two plans' choices. */
int gemm_epi_mlp_query(gemm_epi_mlp_t mlp, gemm_epi_plan_info *up, gemm_epi_plan_info *down);

int gemm_epi_mlp_free(gemm_epi_mlp_t mlp);

/* Release the plan (host metadata, tensor maps, status word).  Must not
 * overlap a run still executing on the GPU that uses this plan's status word:
 * synchronise first.  ERR_ARG for an unknown or already freed handle. */
int gemm_epi_free(gemm_epi_plan_t plan);

/* Static description of a status code (never NULL). */
const char *gemm_epi_status_string(int status);

/* Row pitch of the aux mask in bytes: ceil(n / 128) * 16 (0 for n <= 0). */
int64_t gemm_epi_aux_pitch_bytes(int64_t n);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gemm_epi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GEMM_EPI_H */
