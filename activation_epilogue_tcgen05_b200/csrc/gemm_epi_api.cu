// gemm_epi_api.cu -- the C ABI declared in include/gemm_epi.h: plan creation
// and kernel choice, argument and alignment checks, TMA tensor-map encoding
// (cached per plan), launches, status-word handling.
//
// The plan / run / free life cycle mirrors the stateful interface of
// "nvmath-python cuBLASLt bias fusion for PyTorch inference" (blog.hotdry.top),
// paragraphs 3 and 5 (Matmul.plan(epilog=..., epilog_inputs=...), execute(),
// free()); the epilogue set, the bias broadcast and the 16-byte alignment rule
// follow "nvmath-python epilog bias fusion parameters" (blog.hotdry.top), body
// paragraphs 2-3.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_set>

#include "../../include/gemm_epi.h"
#include "kernels.h"

using namespace gemm_epi;

namespace {

constexpr uint64_t kPlanMagic = 0x67656d6d5f657069ull;   // "gemm_epi"

struct Plan {
    uint64_t magic;
    int64_t m, n, k;
    int dtype, epilogue, axis, b_layout;   // b_layout: GEMM_EPI_B_KN or GEMM_EPI_B_NK
    bool a_km;           // A stored (k, m) row-major (layout flag GEMM_EPI_A_KM)
    int kepi;            // kernel epilogue (EPI_*): the activation
    bool has_bias;       // the public epilogue adds a bias
    bool bwd, bgrad;     // backward epilogue (DRELU*); with a bias gradient (DRELU_BGRAD)
    bool qout;           // e4m3 output quantised in the epilogue (options.out_e4m3)
    gemm_epi_options opts;
    int device, num_sms;
    // kernel choice
    int kernel;          // GEMM_EPI_KERNEL_TC1 / TC2 / SPLITK
    int block_n;         // TC: tile width; SPLITK: 128
    int nm;              // SPLITK: MMA N (batch rows rounded up)
    int split;           // SPLITK: cluster size along k (cluster form); k-parts per tile, rounded up (grid form)
    bool sk_grid = false;      // SPLITK: the grid-wide form (workspace reduction) rather than clusters
    bool no_workspace = false; // the plan may not own device memory beyond its status word (no-alloc runs)
    int kb_per_cta;
    int katoms = 1;      // TC: 128-byte k-atoms per ring stage (the kernel's KATOMS)
    int grid;
    int group_m, group_n = 0;   // TC raster (TcParams::group_m / group_n)
    int l2_mode = 1;     // TcParams::l2_mode (GEMM_EPI_L2=0/1/2 overrides)
    int prefetch = 0;    // TcParams::prefetch (GEMM_EPI_PREFETCH=n overrides)
    int sk_pre_kb = 4;   // SkParams::pre_kb (GEMM_EPI_SK_PRE=n overrides)
    int sk_pre_x = 0;    // SkParams::pre_x (GEMM_EPI_SK_PRE_X=1)
    bool fused = false;  // TcParams::fused: stage-wide 3-D / 4-D operand copies (GEMM_EPI_FUSED_COPIES=1 enables)
    bool pdl;            // programmatic dependent launch (GEMM_EPI_PDL=0 turns it off)
    // split tail (TC kernels): tiles [0, sk_tiles) cut along k into sk_split parts
    int sk_tiles = 0, sk_split = 0;
    float *workspace = nullptr;          // owned: units x CG x 128 x block_n fp32
    unsigned int *flags = nullptr;       // owned: units x CG x 4 words, zero between launches
    size_t flags_bytes = 0;
    // DRELU_BGRAD: fp32 partial sums [dbias_parts][dbias_len] (owned)
    float *dbias_ws = nullptr;
    int64_t dbias_parts = 0, dbias_len = 0;
    TcLauncher tc_launch = nullptr, tc_none_launch = nullptr;
    SkLauncher sk_launch = nullptr, sk_none_launch = nullptr;
    SgLauncher sg_launch = nullptr, sg_none_launch = nullptr;
    BiasActLauncher ba_launch = nullptr;
    KernelInfo info{};
    // FP8 scales (device pointers, borrowed)
    const float *scale_a = nullptr, *scale_b = nullptr;
    // FP8 output: the output scale and the optional amax word (device pointers, borrowed)
    const float *out_scale = nullptr;
    float *amax = nullptr;
    // device status word (owned)
    unsigned int *status = nullptr;
    // tensor-map cache, keyed on the operand pointers
    bool maps_valid = false;
    const void *cA = nullptr, *cB = nullptr;
    void *cD = nullptr;
    CUtensorMap tmA, tmB, tmD;
};

std::mutex g_mu;
std::unordered_set<Plan *> g_plans;

bool live(gemm_epi_plan_t h) {
    std::lock_guard<std::mutex> lk(g_mu);
    Plan *p = reinterpret_cast<Plan *>(h);
    return h && g_plans.count(p) && p->magic == kPlanMagic;
}

int esize(int dt) { return dt == GEMM_EPI_E4M3 ? 1 : 2; }

// Public epilogue -> kernel activation, and whether it adds a bias.  The
// bias-free epilogues run the bias kernels with a NULL bias pointer.
int kernel_epi(int e) {
    switch (e) {
    case GEMM_EPI_BIAS: return EPI_BIAS;
    case GEMM_EPI_RELU_BIAS: case GEMM_EPI_RELU: return EPI_RELU;
    case GEMM_EPI_RELU_AUX_BIAS: case GEMM_EPI_RELU_AUX: return EPI_RELU_AUX;
    case GEMM_EPI_GELU_BIAS: case GEMM_EPI_GELU: return EPI_GELU;
    case GEMM_EPI_TANH_BIAS: case GEMM_EPI_TANH: return EPI_TANH;
    case GEMM_EPI_DRELU: case GEMM_EPI_DRELU_BGRAD: return EPI_DRELU;
    default: return EPI_NONE;
    }
}
bool epi_has_bias(int e) {
    return e == GEMM_EPI_BIAS || e == GEMM_EPI_RELU_BIAS || e == GEMM_EPI_RELU_AUX_BIAS || e == GEMM_EPI_GELU_BIAS ||
           e == GEMM_EPI_TANH_BIAS;
}

// ----------------------------------------------------------------- tensor maps
using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                              CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                              CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(ptr);
    });
    return fn;
}

CUtensorMapDataType tmap_type(int dt) {
    switch (dt) {
    case GEMM_EPI_F16: return CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    case GEMM_EPI_BF16: return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    default: return CU_TENSOR_MAP_DATA_TYPE_UINT8;
    }
}

// Row-major 2-D tensor: `inner` contiguous elements per row, `outer` rows.
bool make_map(CUtensorMap *map, int dt, const void *ptr, int64_t inner, int64_t outer, uint32_t box_inner,
              uint32_t box_outer, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)(inner * esize(dt))};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, tmap_type(dt), 2, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// N-D view (rank 3 or 4) of a row-major tensor, 128-byte swizzle: dims[0] is contiguous,
// strides_bytes[i] is the byte distance between consecutive indices of dims[i + 1].
bool make_map_nd(CUtensorMap *map, int dt, const void *ptr, uint32_t rank, const cuuint64_t *dims,
                 const cuuint64_t *strides_bytes, const cuuint32_t *box) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, tmap_type(dt), rank, const_cast<void *>(ptr), dims, strides_bytes, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ----------------------------------------------------------------- kernel choice
int num_sms_of(int dev) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
}

int round_nm(int64_t m) {
    if (m <= 16) return 16;
    if (m <= 32) return 32;
    if (m <= 64) return 64;
    return 128;
}

bool getenv_flag(const char *name) {
    const char *e = getenv(name);
    return e && e[0] == '1';
}

int choose(Plan *P) {
    const int64_t m = P->m, n = P->n;
    // The GEMM kernels do only on-chip setup before waiting on the previous grid, so they are
    // launched as programmatic dependents: their launch and setup overlap the previous
    // kernel's tail.  GEMM_EPI_PDL=0 launches them plainly (for comparison).
    {
        const char *e = getenv("GEMM_EPI_PDL");
        P->pdl = !(e && e[0] == '0');
    }
    int kernel = P->opts.kernel;
    if (kernel == GEMM_EPI_KERNEL_AUTO) {
        // small m: swapped split-K; enough 256 x 256 tiles for every SM pair: CTA pairs
        // (half the operand traffic per SM); otherwise single CTAs.  Split-K up to m = 64,
        // where it streams the weight faster than the single CTAs with a four-part split tail
        // (m = 64, fp16 GELU: 10.3 vs 17.1 us at 4096 x 4096, 23.5 vs 31.4 us at n = 4096,
        // k = 14336, 28.3 vs 29.1 us at n = 14336, k = 4096; e4m3 7.5 vs 14.2 us); above, its
        // ring holds too few stages (m = 96: 17.5 vs 16.7 us).  (The split-K kernel has no
        // backward epilogue.)
        const int64_t pair_tiles = ((m + 255) / 256) * ((n + 255) / 256);
        const int sms_auto = P->opts.max_ctas > 0 ? std::min(P->opts.max_ctas, P->num_sms) : P->num_sms;
        if (m <= 64 && P->kepi != EPI_DRELU && !P->a_km) kernel = GEMM_EPI_KERNEL_SPLITK;
        else if (pair_tiles >= sms_auto / 2) kernel = GEMM_EPI_KERNEL_TC2;
        else kernel = GEMM_EPI_KERNEL_TC1;
    }
    if (kernel == GEMM_EPI_KERNEL_SPLITK && (m > 128 || P->kepi == EPI_DRELU || P->a_km))
        return GEMM_EPI_ERR_UNSUPPORTED;
    P->kernel = kernel;
    const bool b_mn = P->b_layout == GEMM_EPI_B_KN;
    const int bk = 128 / esize(P->dtype);
    const int64_t num_kb = (P->k + bk - 1) / bk;
    const int sms = P->opts.max_ctas > 0 ? std::min(P->opts.max_ctas, P->num_sms) : P->num_sms;

    if (kernel == GEMM_EPI_KERNEL_SPLITK && !P->no_workspace && getenv_flag("GEMM_EPI_SK_GRID")) {
        // grid-wide form: every SM takes an equal share of the (tile, k-block) units; a split
        // tile is finished by the CTA holding its first k-block, from partials the others
        // publish in a plan-owned workspace
        P->sk_grid = true;
        P->nm = round_nm(m);
        P->block_n = 128;
        const int64_t tiles_n = (n + 127) / 128;
        const int64_t units = tiles_n * num_kb;
        int64_t g = sms;
        if (P->opts.split_k > 0) g = std::min<int64_t>(g, tiles_n * P->opts.split_k);   // k-parts per tile
        g = std::max<int64_t>(1, std::min<int64_t>(g, units));
        P->grid = (int)g;
        P->split = (int)((g + tiles_n - 1) / tiles_n);
        P->kb_per_cta = (int)((units + g - 1) / g);
        KernelInfo none_info;
        if (!find_sg(P->dtype, GEMM_EPI_NONE, 0, b_mn, P->nm, false, &P->sg_none_launch, &none_info))
            return GEMM_EPI_ERR_UNSUPPORTED;
        if (!find_sg(P->dtype, P->kepi, P->axis, b_mn, P->nm, P->qout, &P->sg_launch, &P->info))
            return GEMM_EPI_ERR_UNSUPPORTED;
    } else if (kernel == GEMM_EPI_KERNEL_SPLITK) {
        P->nm = round_nm(m);
        P->block_n = 128;
        const int64_t tiles_n = (n + 127) / 128;
        const int max_split = sk_max_split(P->nm);
        int split = P->opts.split_k;
        if (split <= 0) {
            // Every cluster of the launch must be resident at once, or the last ones wait for a
            // second wave.  Measured (m = 16, k = 4096, fp16): clusters of up to 4 CTAs, at most
            // 128 CTAs, all fit (n = 2048: 4 x 16 CTAs 7.9 us against 8 x 16 11.1 us; n = 3072:
            // 4 x 24 8.1 against 6 x 24 13.1; n = 6144: 2 x 48 12.8 against 3 x 48 20.1), and
            // so do 8 clusters of 8 (n = 1024: 5.1 us).
            const int64_t cap = std::min<int64_t>(128, sms);
            if (tiles_n * 8 <= 64 && max_split >= 8 && 64 <= cap) {
                split = 8;
            } else {
                split = std::min(4, max_split);
                while (split > 1 && tiles_n * split > cap) --split;
            }
        }
        if (split > max_split || split < 1) return GEMM_EPI_ERR_ARG;
        if (split > num_kb) split = (int)num_kb;
        P->kb_per_cta = (int)((num_kb + split - 1) / split);
        split = (int)((num_kb + P->kb_per_cta - 1) / P->kb_per_cta);   // no CTA without work
        P->split = split;
        P->grid = (int)(tiles_n * split);
        // the first 4 k-blocks of each CTA's weight slice are asked of L2 before the dependency
        // wait: measured 9.58 us a step for 16 x 4096 x 4096 fp16 GELU against 10.80 us for the
        // whole slice (which floods the memory queues ahead of the first demand loads, and L2
        // itself for large weights: 30.8 against 24.4 us at n = 14336) and 10.05 us for none
        P->sk_pre_kb = 4;
        if (const char *g = getenv("GEMM_EPI_SK_PRE")) P->sk_pre_kb = atoi(g);   // tuning knob (< 0: all)
        P->sk_pre_x = getenv_flag("GEMM_EPI_SK_PRE_X") ? 1 : 0;
        KernelInfo none_info;
        if (!find_sk(P->dtype, GEMM_EPI_NONE, 0, b_mn, P->nm, false, &P->sk_none_launch, &none_info))
            return GEMM_EPI_ERR_UNSUPPORTED;
        if (!find_sk(P->dtype, P->kepi, P->axis, b_mn, P->nm, P->qout, &P->sk_launch, &P->info))
            return GEMM_EPI_ERR_UNSUPPORTED;
    } else {
        const int cg = kernel == GEMM_EPI_KERNEL_TC2 ? 2 : 1;
        const int bm = 128 * cg;
        int bn = P->opts.block_n;
        if (bn == 0) {
            const int64_t tiles256 = ((m + bm - 1) / bm) * ((n + 255) / 256);
            bn = tiles256 >= sms / cg ? 256 : 128;
            // a pair's e4m3 B half-tile stored (k, n) must be a whole 128-byte box: 128 columns
            if (cg == 2 && P->dtype == GEMM_EPI_E4M3 && b_mn) bn = 256;
            if (P->a_km) bn = 256;     // A stored (k, m) is built with 256-wide tiles only
            // Many waves of 16-bit work with a light epilogue: 512-wide pair tiles.  They move a
            // quarter fewer operand bytes per flop into each SM, which under the power cap buys
            // clock (+7 % at 8192^3 and 65536 x 8192 x 16384), but hold a single accumulator, so
            // the epilogue is not overlapped: they need >= 4 waves, and they lose with GELU / tanh
            // or with e4m3's twice-as-short mainloop (-7 % on the FP8 GELU shape).
            const int64_t tiles512 = ((m + 255) / 256) * ((n + 511) / 512);
            const bool light = P->kepi == EPI_NONE || P->kepi == EPI_BIAS || P->kepi == EPI_RELU ||
                               P->kepi == EPI_RELU_AUX;
            if (cg == 2 && light && P->dtype != GEMM_EPI_E4M3 && !P->a_km && !P->qout && tiles512 >= 4 * (sms / 2))
                bn = 512;
        }
        if (bn != 128 && bn != 256 && bn != 512) return GEMM_EPI_ERR_ARG;
        P->block_n = bn;
        // the kernel's ring stages hold katoms k-atoms; its k-blocks are stages
        P->katoms = tc_katoms(128 * 128 + (bn / cg) * 128);
        const int64_t num_kb_tc = (P->k + (int64_t)bk * P->katoms - 1) / ((int64_t)bk * P->katoms);
        const int64_t tiles = ((m + bm - 1) / bm) * ((n + bn - 1) / bn);
        const int64_t units_max = cg == 2 ? sms / 2 : sms;
        // split tail: the tiles of an incomplete last wave (or all tiles, when there are fewer
        // tiles than units) are cut along k into `split` parts on separate units, so the last
        // wave costs 1/split of a tile.  Behind whole waves, two parts: the finishing unit then
        // adds a single partial, which overlaps its next tile's mainloop.  With fewer tiles than
        // units nothing follows the parts, so up to four parts (at least 8 k-blocks each) put
        // more SMs on the operand stream: 128 x 4096 x 4096 fp16 19.7 -> 17.3 us, 128 x 4096 x
        // 14336 43.5 -> 33.4 us, 1024 x 512 x 2048 12.5 -> 11.9 us.
        int64_t sk_tiles = 0, split = 0;
        const int sk_mode = P->opts.stream_k;          // 0 auto, 1 off, 2 on
        if (sk_mode != 1 && tiles % units_max != 0) {
            const int64_t rem = tiles < units_max ? tiles : tiles % units_max;
            const int64_t waves = (tiles + units_max - 1) / units_max;
            const double loss = 1.0 - (double)tiles / (double)(waves * units_max);
            // (part sizes in 128-byte k-atoms, so that the rule does not depend on the stage size)
            const int64_t parts = tiles < units_max ? std::max<int64_t>(2, std::min<int64_t>(4, num_kb / 8)) : 2;
            split = std::min<int64_t>({units_max / rem, P->opts.split_k > 0 ? P->opts.split_k : parts, num_kb_tc});
            const bool worth = tiles < units_max ? num_kb >= 8 : loss > 0.02;
            if (split >= 2 && (sk_mode == 2 || worth)) sk_tiles = rem;
        }
        if (sk_tiles > 0) {
            P->sk_tiles = (int)sk_tiles;
            P->sk_split = (int)split;
            // whole waves of tiles remain for every unit, or only the split parts need units
            const int64_t units = tiles > sk_tiles ? units_max : sk_tiles * split;
            P->grid = (int)(units * cg);
        } else {
            const int64_t units = std::min<int64_t>(tiles, units_max);
            P->grid = (int)(units * cg);
        }
        // Raster from the L2 capacity.  If all of A's panels (or all of B's) fit in a budget
        // of about 40 % of the 126 MB L2, the whole matrix is walked with that operand resident
        // and the other streamed once: column by column over every tile-row when A is the
        // smaller, row by row over every tile-column when B is.  Otherwise groups of 8
        // tile-rows: with panels this long (large k) the resident tiles only share panels within
        // a wave.  (FP8 8192 x 14336 x 4096: A 32 MB resident, DRAM reads 3.0x the operands with
        // groups of 8, where B was re-read by each of the four groups.)
        {
            const int64_t kb_bytes = P->k * esize(P->dtype);
            const int64_t tiles_m = (m + bm - 1) / bm, tiles_n = (n + bn - 1) / bn;
            const int64_t total_a = tiles_m * bm * kb_bytes, total_b = tiles_n * bn * kb_bytes;
            const int64_t budget = 50ll << 20;
            P->group_m = 8;
            P->group_n = 0;
            if (std::min(total_a, total_b) <= budget) {
                if (total_a <= total_b) P->group_m = (int)std::min<int64_t>(tiles_m, 1 << 30);
                else P->group_n = (int)std::min<int64_t>(tiles_n, 1 << 30);
            }
        }
        if (const char *g = getenv("GEMM_EPI_GROUP_M")) {   // tuning knob: tile-raster group height
            const int v = atoi(g);
            if (v >= 1 && v <= 1 << 20) { P->group_m = v; P->group_n = 0; }
        }
        P->l2_mode = 1;
        if (const char *g = getenv("GEMM_EPI_L2")) {        // tuning knob: L2 cache policy (TcParams)
            const int v = atoi(g);
            if (v >= 0 && v <= 2) P->l2_mode = v;
        }
        P->prefetch = 0;
        if (const char *g = getenv("GEMM_EPI_PREFETCH")) {
            const int v = atoi(g);
            if (v >= 0 && v <= 64) P->prefetch = v;
        }
        // Stage-wide copies: a ring stage of A (all its k-atoms) and of each MMA half of B lands
        // with one 3-D / 4-D copy instead of one copy per 128-byte box.  The N-D views split k
        // into atoms (and n or m into 128-byte blocks for an MN-major operand), so those extents
        // must divide exactly; otherwise the 2-D maps are used.
        {
            const int64_t box_el = 128 / esize(P->dtype);
            const bool ok_k = P->k % bk == 0;
            const bool ok_b = !b_mn || n % box_el == 0;
            const bool ok_a = !P->a_km || m % box_el == 0;
            // Off unless GEMM_EPI_FUSED_COPIES=1: at 4096^3 the per-atom full barriers of the 2-D
            // copies turn a stage over faster (1110 against 1160 SM clocks on average).
            const char *g = getenv("GEMM_EPI_FUSED_COPIES");
            P->fused = ok_k && ok_b && ok_a && g && g[0] == '1';
        }
        KernelInfo none_info;
        if (!find_tc(cg, P->dtype, GEMM_EPI_NONE, 0, b_mn, bn, false, P->a_km, &P->tc_none_launch, &none_info))
            return GEMM_EPI_ERR_UNSUPPORTED;
        if (!find_tc(cg, P->dtype, P->kepi, P->axis, b_mn, bn, P->qout, P->a_km, &P->tc_launch, &P->info))
            return GEMM_EPI_ERR_UNSUPPORTED;
        if (P->info.katoms != P->katoms || none_info.katoms != P->katoms) return GEMM_EPI_ERR_UNSUPPORTED;
        P->split = 1;
    }
    if (P->kepi != EPI_NONE && !P->qout && !find_bias_act(P->dtype, P->kepi, P->axis, &P->ba_launch))
        return GEMM_EPI_ERR_UNSUPPORTED;
    return GEMM_EPI_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Timeline buffer of a tracing build (GEMM_EPI_TRACE=1 or 2); NULL in a normal build.
unsigned long long *trace_buffer() {
#if GEMM_EPI_TRACE
    static unsigned long long *buf = nullptr;
    if (!buf) {
        const size_t bytes = (2 + 2 * (size_t)TRACE_CAP) * sizeof(unsigned long long);
        if (cudaMalloc(&buf, bytes) != cudaSuccess || cudaMemset(buf, 0, bytes) != cudaSuccess) buf = nullptr;
    }
    return buf;
#else
    return nullptr;
#endif
}
// The trace pointer a launch is given: the whole buffer (level 1), or the next of its
// per-launch slots (level 2).
unsigned long long *trace_for_launch() {
    unsigned long long *buf = trace_buffer();
#if GEMM_EPI_TRACE == 2
    static unsigned int next = 0;
    if (buf) buf += 2 + 2 * (size_t)TRACE_LAUNCH_RECS * (next++ % (TRACE_CAP / TRACE_LAUNCH_RECS));
#endif
    return buf;
}

// A plan's status word and workspaces live on the device it was created on: its runs must be
// issued with that device current.
bool on_plan_device(const Plan *P) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return dev == P->device;
}

int check_run_args(Plan *P, const void *A, const void *B, const void *bias, void *D, uint32_t *aux) {
    if (!on_plan_device(P)) return GEMM_EPI_ERR_ARG;
    if (P->bwd) return GEMM_EPI_ERR_ARG;          // backward plans run through gemm_epi_run_bwd
    if (!A || !B || !D) return GEMM_EPI_ERR_NULL;
    if (P->has_bias && !bias) return GEMM_EPI_ERR_NULL;
    if (P->kepi == EPI_RELU_AUX && !aux) return GEMM_EPI_ERR_NULL;
    if (P->dtype == GEMM_EPI_E4M3 && (!P->scale_a || !P->scale_b)) return GEMM_EPI_ERR_NULL;
    if (P->qout && !P->out_scale) return GEMM_EPI_ERR_NULL;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return GEMM_EPI_ERR_ALIGN;
    if (P->has_bias && !aligned16(bias)) return GEMM_EPI_ERR_ALIGN;
    if (P->kepi == EPI_RELU_AUX && !aligned16(aux)) return GEMM_EPI_ERR_ALIGN;
    return GEMM_EPI_OK;
}

int check_bwd_args(Plan *P, const void *A, const void *B, const uint32_t *aux, void *D, void *dbias) {
    if (!on_plan_device(P)) return GEMM_EPI_ERR_ARG;
    if (!P->bwd) return GEMM_EPI_ERR_ARG;
    if (!A || !B || !D || !aux) return GEMM_EPI_ERR_NULL;
    if (P->bgrad && !dbias) return GEMM_EPI_ERR_NULL;
    if (P->dtype == GEMM_EPI_E4M3 && (!P->scale_a || !P->scale_b)) return GEMM_EPI_ERR_NULL;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(aux)) return GEMM_EPI_ERR_ALIGN;
    if (P->bgrad && !aligned16(dbias)) return GEMM_EPI_ERR_ALIGN;
    return GEMM_EPI_OK;
}

int ensure_maps(Plan *P, const void *A, const void *B, void *D) {
    if (P->maps_valid && P->cA == A && P->cB == B && P->cD == D) return GEMM_EPI_OK;
    const int dt = P->dtype;
    const int64_t m = P->m, n = P->n, k = P->k;
    const int bk = 128 / esize(dt);
    const bool b_kn = P->b_layout == GEMM_EPI_B_KN;
    const int box_n = 128 / esize(dt);            // elements in one 128-byte row
    bool ok = true;
    if (P->kernel == GEMM_EPI_KERNEL_SPLITK) {
        // operand "W" = B (128 output columns per tile), operand "X" = A (nm rows)
        ok = ok && (b_kn ? make_map(&P->tmA, dt, B, n, k, box_n, bk) : make_map(&P->tmA, dt, B, k, n, bk, 128));
        ok = ok && make_map(&P->tmB, dt, A, k, m, bk, P->nm);
    } else {
        const int cg = P->kernel == GEMM_EPI_KERNEL_TC2 ? 2 : 1;
        const int bn_local = std::min(P->block_n, 256) / cg;   // B rows of one MMA in this CTA
        if (P->fused) {
            // stage-wide views: [atom][row][128 B] for a K-major operand, [atom][block][k row][128 B]
            // for an MN-major one -- the shared-memory layout of the 2-D copies, in one copy
            const int es = esize(dt);
            const cuuint32_t ka = (cuuint32_t)P->katoms;
            if (P->a_km) {
                const cuuint64_t d[4] = {(cuuint64_t)box_n, (cuuint64_t)bk, (cuuint64_t)(m / box_n), (cuuint64_t)(k / bk)};
                const cuuint64_t st[3] = {(cuuint64_t)(m * es), 128, (cuuint64_t)(bk * m * es)};
                const cuuint32_t bx[4] = {(cuuint32_t)box_n, (cuuint32_t)bk, (cuuint32_t)(128 / box_n), ka};
                ok = ok && make_map_nd(&P->tmA, dt, A, 4, d, st, bx);
            } else {
                const cuuint64_t d[3] = {(cuuint64_t)bk, (cuuint64_t)m, (cuuint64_t)(k / bk)};
                const cuuint64_t st[2] = {(cuuint64_t)(k * es), (cuuint64_t)(bk * es)};
                const cuuint32_t bx[3] = {(cuuint32_t)bk, 128, ka};
                ok = ok && make_map_nd(&P->tmA, dt, A, 3, d, st, bx);
            }
            if (b_kn) {
                const cuuint64_t d[4] = {(cuuint64_t)box_n, (cuuint64_t)bk, (cuuint64_t)(n / box_n), (cuuint64_t)(k / bk)};
                const cuuint64_t st[3] = {(cuuint64_t)(n * es), 128, (cuuint64_t)(bk * n * es)};
                const cuuint32_t bx[4] = {(cuuint32_t)box_n, (cuuint32_t)bk, (cuuint32_t)(bn_local / box_n), ka};
                ok = ok && make_map_nd(&P->tmB, dt, B, 4, d, st, bx);
            } else {
                const cuuint64_t d[3] = {(cuuint64_t)bk, (cuuint64_t)n, (cuuint64_t)(k / bk)};
                const cuuint64_t st[2] = {(cuuint64_t)(k * es), (cuuint64_t)(bk * es)};
                const cuuint32_t bx[3] = {(cuuint32_t)bk, (cuuint32_t)bn_local, ka};
                ok = ok && make_map_nd(&P->tmB, dt, B, 3, d, st, bx);
            }
        } else {
            ok = ok && (P->a_km ? make_map(&P->tmA, dt, A, m, k, box_n, bk) : make_map(&P->tmA, dt, A, k, m, bk, 128));
            ok = ok && (b_kn ? make_map(&P->tmB, dt, B, n, k, box_n, bk) : make_map(&P->tmB, dt, B, k, n, bk, bn_local));
        }
        const int out_dt = dt == GEMM_EPI_E4M3 ? GEMM_EPI_BF16 : dt;
        if (P->qout)   // e4m3 output goes out with direct stores; the map is valid but unused
            ok = ok && make_map(&P->tmD, GEMM_EPI_E4M3, D, n, m, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
        else           // the epilogue stages 32 rows x 32 outputs (64 bytes a row, 64-byte swizzle) per store
            ok = ok && make_map(&P->tmD, out_dt, D, n, m, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    }
    if (!ok) {
        P->maps_valid = false;
        return GEMM_EPI_ERR_CUDA;
    }
    P->cA = A;
    P->cB = B;
    P->cD = D;
    P->maps_valid = true;
    return GEMM_EPI_OK;
}

int launch_main(Plan *P, bool fused, const void *bias, void *D, uint32_t *aux, cudaStream_t stream,
                float *dbias_ws = nullptr) {
    if (!P->has_bias) bias = nullptr;
    const int bk = 128 / esize(P->dtype);
    const int num_kb = (int)((P->k + bk - 1) / bk);
    const int64_t pitch_words = ((P->n + 127) / 128) * 4;
    cudaError_t e;
    if (P->kernel == GEMM_EPI_KERNEL_SPLITK && P->sk_grid) {
        SgLaunch L{};
        L.tmW = P->tmA;
        L.tmX = P->tmB;
        L.p.m = (int)P->m;
        L.p.n = (int)P->n;
        L.p.k = (int)P->k;
        L.p.num_kb = num_kb;
        L.p.tiles_n = (int)((P->n + 127) / 128);
        L.p.grid = P->grid;
        L.p.bias = bias;
        L.p.D = D;
        L.p.aux = aux;
        L.p.aux_pitch_words = pitch_words;
        L.p.scale_a = P->scale_a;
        L.p.scale_b = P->scale_b;
        L.p.status = P->status;
        L.p.dq = P->qout ? static_cast<uint8_t *>(D) : nullptr;
        L.p.out_scale = P->out_scale;
        L.p.amax = reinterpret_cast<unsigned int *>(P->amax);
        L.p.workspace = P->workspace;
        L.p.flags = P->flags;
        L.p.trace = trace_for_launch();
        L.pdl = P->pdl;
        L.stream = stream;
        e = (fused ? P->sg_launch : P->sg_none_launch)(L);
    } else if (P->kernel == GEMM_EPI_KERNEL_SPLITK) {
        SkLaunch L{};
        L.tmW = P->tmA;
        L.tmX = P->tmB;
        L.p.m = (int)P->m;
        L.p.n = (int)P->n;
        L.p.k = (int)P->k;
        L.p.num_kb = num_kb;
        L.p.kb_per_cta = P->kb_per_cta;
        L.p.bias = bias;
        L.p.D = D;
        L.p.aux = aux;
        L.p.aux_pitch_words = pitch_words;
        L.p.scale_a = P->scale_a;
        L.p.scale_b = P->scale_b;
        L.p.status = P->status;
        L.p.dq = P->qout ? static_cast<uint8_t *>(D) : nullptr;
        L.p.out_scale = P->out_scale;
        L.p.amax = reinterpret_cast<unsigned int *>(P->amax);
        L.p.trace = trace_for_launch();
        L.p.pre_kb = P->sk_pre_kb;
        L.p.pre_x = P->sk_pre_x;
        L.grid = P->grid;
        L.cluster = P->split;
        L.pdl = P->pdl;
        L.stream = stream;
        e = (fused ? P->sk_launch : P->sk_none_launch)(L);
    } else {
        const int cg = P->kernel == GEMM_EPI_KERNEL_TC2 ? 2 : 1;
        TcLaunch L{};
        L.tmA = P->tmA;
        L.tmB = P->tmB;
        L.tmD = P->tmD;
        L.p.m = (int)P->m;
        L.p.n = (int)P->n;
        L.p.k = (int)P->k;
        L.p.tiles_m = (int)((P->m + 128 * cg - 1) / (128 * cg));
        L.p.tiles_n = (int)((P->n + P->block_n - 1) / P->block_n);
        L.p.num_tiles = L.p.tiles_m * L.p.tiles_n;
        L.p.num_kb = (int)((P->k + (int64_t)bk * P->katoms - 1) / ((int64_t)bk * P->katoms));   // ring stages
        L.p.group_m = P->group_m;
        L.p.group_n = P->group_n;
        L.p.bias = bias;
        L.p.aux = aux;
        L.p.aux_pitch_words = pitch_words;
        L.p.scale_a = P->scale_a;
        L.p.scale_b = P->scale_b;
        L.p.status = P->status;
        L.p.inject_stall = P->opts.inject_stall;
        L.p.sk_tiles = P->sk_tiles;
        L.p.sk_split = P->sk_split;
        L.p.workspace = P->workspace;
        L.p.flags = P->flags;
        L.p.trace = trace_for_launch();
        L.p.dbias_ws = fused ? dbias_ws : nullptr;
        L.p.dq = P->qout ? static_cast<uint8_t *>(D) : nullptr;
        L.p.out_scale = P->out_scale;
        L.p.amax = reinterpret_cast<unsigned int *>(P->amax);
        L.p.l2_mode = P->l2_mode;
        L.p.prefetch = P->prefetch;
        L.p.fused = P->fused ? 1 : 0;
        L.grid = P->grid;
        L.pdl = P->pdl;
        L.stream = stream;
        e = (fused ? P->tc_launch : P->tc_none_launch)(L);
    }
    if (e != cudaSuccess && getenv("GEMM_EPI_LOG")) fprintf(stderr, "gemm_epi launch: %s (%d)\n", cudaGetErrorString(e), (int)e);
    return e == cudaSuccess ? GEMM_EPI_OK : GEMM_EPI_ERR_CUDA;
}

// Argument checks that need no device, and the plan's problem fields.
int plan_fields(Plan *P, int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis, int b_layout,
                const gemm_epi_options *opts) {
    if (m <= 0 || n <= 0 || k <= 0) return GEMM_EPI_ERR_ARG;
    if (m > 0x7fffffffll || n > 0x7fffffffll || k > 0x7fffffffll) return GEMM_EPI_ERR_ARG;
    if (((m + 127) / 128) * ((n + 127) / 128) > 0x7fffffffll) return GEMM_EPI_ERR_ARG;   // tile count is an int
    if (dtype < GEMM_EPI_F16 || dtype > GEMM_EPI_E4M3) return GEMM_EPI_ERR_ARG;
    if (epilogue < GEMM_EPI_NONE || epilogue > GEMM_EPI_DRELU_BGRAD) return GEMM_EPI_ERR_ARG;
    if (bias_axis != GEMM_EPI_BIAS_ROW && bias_axis != GEMM_EPI_BIAS_COL) return GEMM_EPI_ERR_ARG;
    if (b_layout & ~(GEMM_EPI_B_NK | GEMM_EPI_A_KM)) return GEMM_EPI_ERR_ARG;
    const bool a_km = (b_layout & GEMM_EPI_A_KM) != 0;
    b_layout &= GEMM_EPI_B_NK;
    gemm_epi_options o{};
    if (opts) o = *opts;
    if (o.kernel < GEMM_EPI_KERNEL_AUTO || o.kernel > GEMM_EPI_KERNEL_SPLITK) return GEMM_EPI_ERR_ARG;
    if (o.block_n != 0 && o.block_n != 128 && o.block_n != 256 && o.block_n != 512) return GEMM_EPI_ERR_ARG;
    if (o.split_k < 0 || o.split_k > 8 || o.max_ctas < 0) return GEMM_EPI_ERR_ARG;
    if (o.inject_stall != 0 && o.inject_stall != 1) return GEMM_EPI_ERR_ARG;
    if (o.stream_k < 0 || o.stream_k > 2) return GEMM_EPI_ERR_ARG;
    if (o.inject_stall && o.kernel == GEMM_EPI_KERNEL_SPLITK) return GEMM_EPI_ERR_UNSUPPORTED;
    if (o.out_e4m3 != 0 && o.out_e4m3 != 1) return GEMM_EPI_ERR_ARG;
    if (o.out_e4m3) {
        // FP8 output: e4m3 operands, forward epilogues without a mask or tanh
        const bool epi_ok = epilogue == GEMM_EPI_NONE || epilogue == GEMM_EPI_BIAS || epilogue == GEMM_EPI_RELU_BIAS ||
                            epilogue == GEMM_EPI_GELU_BIAS || epilogue == GEMM_EPI_RELU || epilogue == GEMM_EPI_GELU;
        if (dtype != GEMM_EPI_E4M3 || !epi_ok) return GEMM_EPI_ERR_UNSUPPORTED;
    }
    // 16-byte row pitches (TMA strides; the pages' 16-byte alignment rule)
    const int es = esize(dtype);
    const int out_es = 2;
    if ((k * es) % 16 != 0) return GEMM_EPI_ERR_ALIGN;
    if ((n * es) % 16 != 0 || (n * out_es) % 16 != 0) return GEMM_EPI_ERR_ALIGN;
    if (a_km && (m * es) % 16 != 0) return GEMM_EPI_ERR_ALIGN;     // A (k, m): row pitch m * esize

    P->m = m;
    P->n = n;
    P->k = k;
    P->dtype = dtype;
    P->epilogue = epilogue;
    P->kepi = kernel_epi(epilogue);
    P->has_bias = epi_has_bias(epilogue);
    P->bwd = P->kepi == EPI_DRELU;
    P->bgrad = epilogue == GEMM_EPI_DRELU_BGRAD;
    P->qout = o.out_e4m3 == 1;
    P->axis = (P->has_bias || P->bgrad) ? bias_axis : GEMM_EPI_BIAS_ROW;
    P->b_layout = b_layout;
    P->a_km = a_km;
    P->opts = o;
    return GEMM_EPI_OK;
}

int make_plan(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis, int b_layout,
              const gemm_epi_options *opts, gemm_epi_plan_t *out) {
    if (!out) return GEMM_EPI_ERR_ARG;
    Plan *P = new (std::nothrow) Plan();
    if (!P) return GEMM_EPI_ERR_CUDA;
    int rc = plan_fields(P, m, n, k, dtype, epilogue, bias_axis, b_layout, opts);
    if (rc != GEMM_EPI_OK) {
        delete P;
        return rc;
    }
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        delete P;
        return GEMM_EPI_ERR_NO_DEVICE;
    }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) {
        delete P;
        return GEMM_EPI_ERR_NO_DEVICE;
    }
    P->magic = kPlanMagic;
    P->device = dev;
    P->num_sms = num_sms_of(dev);
    rc = choose(P);
    if (rc != GEMM_EPI_OK) {
        delete P;
        return rc;
    }
    if (cudaMalloc(&P->status, 256) != cudaSuccess || cudaMemset(P->status, 0, 256) != cudaSuccess) {
        cudaGetLastError();
        if (P->status) cudaFree(P->status);
        delete P;
        return GEMM_EPI_ERR_CUDA;
    }
    const int64_t sg_tiles = (n + 127) / 128;
    if (P->sk_tiles > 0 || (P->sk_grid && P->grid != sg_tiles)) {
        size_t ws_bytes, fl_bytes;
        if (P->sk_grid) {
            // per CTA one partial tile (of its first piece) of NM x 128 fp32 and one flag per
            // TMEM lane quadrant
            ws_bytes = (size_t)P->grid * 128 * (size_t)P->nm * sizeof(float);
            fl_bytes = (size_t)P->grid * 4 * sizeof(unsigned int);
        } else {
            const int cg = P->kernel == GEMM_EPI_KERNEL_TC2 ? 2 : 1;
            const size_t units = (size_t)P->grid / cg;
            ws_bytes = units * cg * 128 * (size_t)P->block_n * sizeof(float);
            fl_bytes = units * cg * 4 * sizeof(unsigned int);
        }
        P->flags_bytes = fl_bytes;
        if (cudaMalloc(&P->workspace, ws_bytes) != cudaSuccess || cudaMalloc(&P->flags, fl_bytes) != cudaSuccess ||
            cudaMemset(P->flags, 0, fl_bytes) != cudaSuccess) {
            cudaGetLastError();
            if (P->workspace) cudaFree(P->workspace);
            if (P->flags) cudaFree(P->flags);
            cudaFree(P->status);
            delete P;
            return GEMM_EPI_ERR_CUDA;
        }
    }
    if (P->bgrad) {
        // one fp32 partial per (row, tile column) for ROW, per (32-row block, column) for COL
        P->dbias_len = P->axis == GEMM_EPI_BIAS_ROW ? m : n;
        P->dbias_parts = P->axis == GEMM_EPI_BIAS_ROW ? (n + P->block_n - 1) / P->block_n : (m + 31) / 32;
        if (cudaMalloc(&P->dbias_ws, (size_t)P->dbias_parts * (size_t)P->dbias_len * sizeof(float)) != cudaSuccess) {
            cudaGetLastError();
            if (P->workspace) cudaFree(P->workspace);
            if (P->flags) cudaFree(P->flags);
            cudaFree(P->status);
            delete P;
            return GEMM_EPI_ERR_CUDA;
        }
    }
    if (getenv("GEMM_EPI_LOG")) {
        fprintf(stderr,
                "gemm_epi plan m=%lld n=%lld k=%lld dtype=%d epi=%d axis=%d b=%d -> kernel=%d bn=%d nm=%d "
                "split=%d grid=%d stages=%d smem=%d sk_tiles=%d sk_split=%d\n",
                (long long)m, (long long)n, (long long)k, dtype, epilogue, bias_axis, b_layout, P->kernel,
                P->block_n, P->nm, P->split, P->grid, P->info.stages, P->info.smem_bytes, P->sk_tiles, P->sk_split);
    }
    {
        std::lock_guard<std::mutex> lk(g_mu);
        g_plans.insert(P);
    }
    *out = reinterpret_cast<gemm_epi_plan_t>(P);
    return GEMM_EPI_OK;
}

}  // namespace

// ----------------------------------------------------------------- lookups
namespace gemm_epi {
bool find_tc(int cg, int dt, int epi, int axis, bool b_mn, int bn, bool qout, bool a_mn, TcLauncher *l,
             KernelInfo *i) {
    KernelInfo tmp;
    if (!i) i = &tmp;
    if (qout) return !a_mn && dt == DT_E4M3 && find_tc_e4m3_q(cg, epi, axis, b_mn, bn, l, i);
    if (a_mn) {
        switch (dt) {
        case DT_F16: return find_tc_f16_at(cg, epi, axis, b_mn, bn, l, i);
        case DT_BF16: return find_tc_bf16_at(cg, epi, axis, b_mn, bn, l, i);
        case DT_E4M3: return find_tc_e4m3_at(cg, epi, axis, b_mn, bn, l, i);
        }
        return false;
    }
    switch (dt) {
    case DT_F16: return find_tc_f16(cg, epi, axis, b_mn, bn, l, i);
    case DT_BF16: return find_tc_bf16(cg, epi, axis, b_mn, bn, l, i);
    case DT_E4M3: return find_tc_e4m3(cg, epi, axis, b_mn, bn, l, i);
    }
    return false;
}
bool find_sg(int dt, int epi, int axis, bool w_mn, int nm, bool qout, SgLauncher *l, KernelInfo *i) {
    KernelInfo tmp;
    if (!i) i = &tmp;
    if (qout) return dt == DT_E4M3 && find_sg_e4m3_q(epi, axis, w_mn, nm, l, i);
    switch (dt) {
    case DT_F16: return find_sg_f16(epi, axis, w_mn, nm, l, i);
    case DT_BF16: return find_sg_bf16(epi, axis, w_mn, nm, l, i);
    case DT_E4M3: return find_sg_e4m3(epi, axis, w_mn, nm, l, i);
    }
    return false;
}
bool find_sk(int dt, int epi, int axis, bool w_mn, int nm, bool qout, SkLauncher *l, KernelInfo *i) {
    KernelInfo tmp;
    if (!i) i = &tmp;
    if (qout) return dt == DT_E4M3 && find_sk_e4m3_q(epi, axis, w_mn, nm, l, i);
    switch (dt) {
    case DT_F16: return find_sk_f16(epi, axis, w_mn, nm, l, i);
    case DT_BF16: return find_sk_bf16(epi, axis, w_mn, nm, l, i);
    case DT_E4M3: return find_sk_e4m3(epi, axis, w_mn, nm, l, i);
    }
    return false;
}
}  // namespace gemm_epi

// ----------------------------------------------------------------- C ABI
extern "C" {

int gemm_epi_plan(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis,
                  gemm_epi_plan_t *out) {
    return make_plan(m, n, k, dtype, epilogue, bias_axis, GEMM_EPI_B_KN, nullptr, out);
}

int gemm_epi_plan_ex(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis, int b_layout,
                     gemm_epi_plan_t *out) {
    return make_plan(m, n, k, dtype, epilogue, bias_axis, b_layout, nullptr, out);
}

int gemm_epi_plan_opts(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis, int b_layout,
                       const gemm_epi_options *opts, gemm_epi_plan_t *out) {
    return make_plan(m, n, k, dtype, epilogue, bias_axis, b_layout, opts, out);
}

int gemm_epi_set_scales(gemm_epi_plan_t plan, const float *d_scale_a, const float *d_scale_b) {
    if (!live(plan)) return GEMM_EPI_ERR_ARG;
    Plan *P = reinterpret_cast<Plan *>(plan);
    if (!d_scale_a && !d_scale_b && P->dtype != GEMM_EPI_E4M3) {   // 16-bit: back to alpha = 1
        P->scale_a = P->scale_b = nullptr;
        return GEMM_EPI_OK;
    }
    if (!d_scale_a || !d_scale_b) return GEMM_EPI_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(d_scale_a) & 3u) || (reinterpret_cast<uintptr_t>(d_scale_b) & 3u))
        return GEMM_EPI_ERR_ALIGN;
    P->scale_a = d_scale_a;
    P->scale_b = d_scale_b;
    return GEMM_EPI_OK;
}

int gemm_epi_set_out_scale(gemm_epi_plan_t plan, const float *d_scale_out, float *d_amax) {
    if (!live(plan)) return GEMM_EPI_ERR_ARG;
    Plan *P = reinterpret_cast<Plan *>(plan);
    if (!P->qout) return GEMM_EPI_ERR_ARG;
    if (!d_scale_out) return GEMM_EPI_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(d_scale_out) & 3u) || (reinterpret_cast<uintptr_t>(d_amax) & 3u))
        return GEMM_EPI_ERR_ALIGN;
    P->out_scale = d_scale_out;
    P->amax = d_amax;
    return GEMM_EPI_OK;
}

int gemm_epi_run(gemm_epi_plan_t plan, const void *A, const void *B, const void *bias, void *D, uint32_t *aux,
                 void *stream) {
    if (!live(plan)) return GEMM_EPI_ERR_ARG;
    Plan *P = reinterpret_cast<Plan *>(plan);
    int rc = check_run_args(P, A, B, bias, D, aux);
    if (rc != GEMM_EPI_OK) return rc;
    rc = ensure_maps(P, A, B, D);
    if (rc != GEMM_EPI_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the amax word is this run's maximum: start it at 0 (the kernel max-reduces into it)
    if (P->qout && P->amax && cudaMemsetAsync(P->amax, 0, sizeof(float), s) != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    return launch_main(P, true, bias, D, aux, s);
}

int gemm_epi_unfused_run(gemm_epi_plan_t plan, const void *A, const void *B, const void *bias, void *D,
                         uint32_t *aux, void *stream) {
    if (!live(plan)) return GEMM_EPI_ERR_ARG;
    Plan *P = reinterpret_cast<Plan *>(plan);
    if (P->qout) return GEMM_EPI_ERR_UNSUPPORTED;
    int rc = check_run_args(P, A, B, bias, D, aux);
    if (rc != GEMM_EPI_OK) return rc;
    rc = ensure_maps(P, A, B, D);
    if (rc != GEMM_EPI_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = launch_main(P, false, bias, D, aux, s);
    if (rc != GEMM_EPI_OK || P->kepi == EPI_NONE) return rc;
    if (!P->has_bias) bias = nullptr;
    const int64_t pitch_words = ((P->n + 127) / 128) * 4;
    const int64_t total = P->m * pitch_words;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, (int64_t)P->num_sms * 16);
    cudaError_t e = P->ba_launch(D, bias, aux, (int)P->m, (int)P->n, pitch_words, (int)blocks, s);
    return e == cudaSuccess ? GEMM_EPI_OK : GEMM_EPI_ERR_CUDA;
}

int gemm_epi_run_bwd(gemm_epi_plan_t plan, const void *A, const void *B, const uint32_t *aux, void *D,
                     void *dbias, void *stream) {
    if (!live(plan)) return GEMM_EPI_ERR_ARG;
    Plan *P = reinterpret_cast<Plan *>(plan);
    int rc = check_bwd_args(P, A, B, aux, D, dbias);
    if (rc != GEMM_EPI_OK) return rc;
    rc = ensure_maps(P, A, B, D);
    if (rc != GEMM_EPI_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = launch_main(P, true, nullptr, D, const_cast<uint32_t *>(aux), s, P->bgrad ? P->dbias_ws : nullptr);
    if (rc != GEMM_EPI_OK || !P->bgrad) return rc;
    const int out_dt = P->dtype == GEMM_EPI_E4M3 ? DT_BF16 : P->dtype;
    const cudaError_t e = launch_sum_parts_f32(out_dt, P->dbias_ws, P->dbias_parts, P->dbias_len, dbias, P->pdl, s);
    return e == cudaSuccess ? GEMM_EPI_OK : GEMM_EPI_ERR_CUDA;
}

int gemm_epi_unfused_run_bwd(gemm_epi_plan_t plan, const void *A, const void *B, const uint32_t *aux, void *D,
                             void *dbias, void *stream) {
    if (!live(plan)) return GEMM_EPI_ERR_ARG;
    Plan *P = reinterpret_cast<Plan *>(plan);
    int rc = check_bwd_args(P, A, B, aux, D, dbias);
    if (rc != GEMM_EPI_OK) return rc;
    rc = ensure_maps(P, A, B, D);
    if (rc != GEMM_EPI_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = launch_main(P, false, nullptr, D, nullptr, s);
    if (rc != GEMM_EPI_OK) return rc;
    const int64_t pitch_words = ((P->n + 127) / 128) * 4;
    const int64_t total = P->m * pitch_words;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, (int64_t)P->num_sms * 16);
    cudaError_t e = P->ba_launch(D, nullptr, const_cast<uint32_t *>(aux), (int)P->m, (int)P->n, pitch_words,
                                 (int)blocks, s);
    if (e != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    if (!P->bgrad) return GEMM_EPI_OK;
    const int out_dt = P->dtype == GEMM_EPI_E4M3 ? DT_BF16 : P->dtype;
    if (P->axis == GEMM_EPI_BIAS_ROW) {
        const int64_t g = std::min<int64_t>((P->m + 7) / 8, (int64_t)P->num_sms * 16);
        e = launch_sum_rows(out_dt, D, P->m, P->n, dbias, (int)g, s);
    } else {
        e = launch_sum_cols(out_dt, D, P->m, P->n, dbias, s);
    }
    return e == cudaSuccess ? GEMM_EPI_OK : GEMM_EPI_ERR_CUDA;
}

int gemm_epi_check(gemm_epi_plan_t plan, void *stream) {
    if (!live(plan)) return GEMM_EPI_ERR_ARG;
    Plan *P = reinterpret_cast<Plan *>(plan);
    const cudaError_t se = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (se != cudaSuccess) {
        if (getenv("GEMM_EPI_LOG")) fprintf(stderr, "gemm_epi_check: %s (%d)\n", cudaGetErrorString(se), (int)se);
        return GEMM_EPI_ERR_CUDA;
    }
    unsigned int word = 0;
    if (cudaMemcpy(&word, P->status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GEMM_EPI_ERR_CUDA;
    if (word != 0) {
        cudaMemset(P->status, 0, sizeof(word));
        // an aborted launch may have left stream-K flags raised: start the next one clean
        if (P->flags) cudaMemset(P->flags, 0, P->flags_bytes);
        return GEMM_EPI_ERR_TIMEOUT;
    }
    return GEMM_EPI_OK;
}

namespace {
void fill_info(const Plan *P, gemm_epi_plan_info *info) {
    info->kernel = P->kernel;
    info->block_m = P->kernel == GEMM_EPI_KERNEL_SPLITK ? P->nm : P->info.block_m;
    info->block_n = P->block_n;
    info->block_k = P->info.block_k;
    info->stages = P->info.stages;
    info->split_k = P->split;
    info->grid = P->grid;
    info->cluster = P->kernel == GEMM_EPI_KERNEL_SPLITK ? (P->sk_grid ? 1 : P->split)
                                                         : (P->kernel == GEMM_EPI_KERNEL_TC2 ? 2 : 1);
    info->threads = P->info.threads;
    info->smem_bytes = P->info.smem_bytes;
    info->sk_tiles = P->sk_tiles;
    info->sk_split = P->sk_split;
    info->group_m = P->kernel == GEMM_EPI_KERNEL_SPLITK ? 0 : (P->group_n > 0 ? 0 : P->group_m);
    info->group_n = P->kernel == GEMM_EPI_KERNEL_SPLITK ? 0 : P->group_n;
    if (P->kernel == GEMM_EPI_KERNEL_SPLITK) {
        info->tiles = (int)((P->n + 127) / 128);
    } else {
        const int bm = P->kernel == GEMM_EPI_KERNEL_TC2 ? 256 : 128;
        info->tiles = (int)(((P->m + bm - 1) / bm) * ((P->n + P->block_n - 1) / P->block_n));
    }
}
}  // namespace

int gemm_epi_plan_query(gemm_epi_plan_t plan, gemm_epi_plan_info *info) {
    if (!live(plan) || !info) return GEMM_EPI_ERR_ARG;
    fill_info(reinterpret_cast<Plan *>(plan), info);
    return GEMM_EPI_OK;
}

int gemm_epi_plan_preview(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis, int b_layout,
                          const gemm_epi_options *opts, int num_sms, gemm_epi_plan_info *info) {
    if (!info || num_sms < 2 || num_sms > 1024) return GEMM_EPI_ERR_ARG;
    Plan P;
    int rc = plan_fields(&P, m, n, k, dtype, epilogue, bias_axis, b_layout, opts);
    if (rc != GEMM_EPI_OK) return rc;
    P.device = -1;
    P.num_sms = num_sms;
    rc = choose(&P);
    if (rc != GEMM_EPI_OK) return rc;
    fill_info(&P, info);
    return GEMM_EPI_OK;
}

int gemm_epi_free(gemm_epi_plan_t plan) {
    Plan *P = reinterpret_cast<Plan *>(plan);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!plan || !g_plans.count(P)) return GEMM_EPI_ERR_ARG;
        g_plans.erase(P);
    }
    if (P->status) cudaFree(P->status);
    if (P->workspace) cudaFree(P->workspace);
    if (P->flags) cudaFree(P->flags);
    if (P->dbias_ws) cudaFree(P->dbias_ws);
    P->magic = 0;
    delete P;
    return GEMM_EPI_OK;
}

const char *gemm_epi_status_string(int status) {
    switch (status) {
    case GEMM_EPI_OK: return "ok";
    case GEMM_EPI_ERR_ARG: return "invalid argument (size, enum, option or plan handle)";
    case GEMM_EPI_ERR_ALIGN: return "pointer not 16-byte aligned or row pitch not a multiple of 16 bytes";
    case GEMM_EPI_ERR_NULL: return "required pointer is NULL (operand, bias, aux, dbias or FP8 scales)";
    case GEMM_EPI_ERR_UNSUPPORTED: return "combination not supported by this library";
    case GEMM_EPI_ERR_CUDA: return "CUDA runtime or driver call failed";
    case GEMM_EPI_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case GEMM_EPI_ERR_NO_DEVICE: return "no current sm_100 (B200-class) CUDA device";
    }
    return "unknown status";
}

int64_t gemm_epi_aux_pitch_bytes(int64_t n) { return n <= 0 ? 0 : ((n + 127) / 128) * 16; }

int gemm_epi_version(void) { return 100; }

}  // extern "C"

// ----------------------------------------------------------------- MLP block
//
// Up-projection H = act(X.W1 + b1) and down-projection Y = H.W2 + b2 as two plans of
// the fused kernel ("nvmath-python cuBLASLt bias fusion for PyTorch inference"
// (blog.hotdry.top), paragraph 1: the MLP is where the GEMM + bias time goes).  For
// e4m3 the up-projection's epilogue also quantises H to e4m3 with the caller's scale
// s_H and reports max |H|, so the down-projection reads H in FP8 with no kernel between
// the two GEMMs.
namespace {

constexpr uint64_t kMlpMagic = 0x6d6c705f626c6f63ull;   // "mlp_bloc"

struct Mlp {
    uint64_t magic;
    int dtype;
    gemm_epi_plan_t up = nullptr, down = nullptr;
};

std::mutex g_mlp_mu;
std::unordered_set<Mlp *> g_mlps;

Mlp *mlp_live(gemm_epi_mlp_t h) {
    std::lock_guard<std::mutex> lk(g_mlp_mu);
    Mlp *M = reinterpret_cast<Mlp *>(h);
    return (h && g_mlps.count(M) && M->magic == kMlpMagic) ? M : nullptr;
}

}  // namespace

extern "C" {

int gemm_epi_mlp_plan(int64_t m, int64_t d_model, int64_t d_ff, int dtype, int act, int w_layout,
                      gemm_epi_mlp_t *out) {
    if (!out) return GEMM_EPI_ERR_ARG;
    if (act != GEMM_EPI_BIAS && act != GEMM_EPI_RELU_BIAS && act != GEMM_EPI_GELU_BIAS) return GEMM_EPI_ERR_ARG;
    if (w_layout != GEMM_EPI_B_KN && w_layout != GEMM_EPI_B_NK) return GEMM_EPI_ERR_ARG;
    Mlp *M = new (std::nothrow) Mlp();
    if (!M) return GEMM_EPI_ERR_CUDA;
    M->magic = kMlpMagic;
    M->dtype = dtype;
    gemm_epi_options up_opts{};
    up_opts.out_e4m3 = dtype == GEMM_EPI_E4M3 ? 1 : 0;
    int rc = make_plan(m, d_ff, d_model, dtype, act, GEMM_EPI_BIAS_COL, w_layout, &up_opts, &M->up);
    if (rc == GEMM_EPI_OK) rc = make_plan(m, d_model, d_ff, dtype, GEMM_EPI_BIAS, GEMM_EPI_BIAS_COL, w_layout, nullptr,
                                          &M->down);
    if (rc != GEMM_EPI_OK) {
        if (M->up) gemm_epi_free(M->up);
        M->magic = 0;
        delete M;
        return rc;
    }
    {
        std::lock_guard<std::mutex> lk(g_mlp_mu);
        g_mlps.insert(M);
    }
    *out = reinterpret_cast<gemm_epi_mlp_t>(M);
    return GEMM_EPI_OK;
}

int gemm_epi_mlp_set_scales(gemm_epi_mlp_t mlp, const float *d_scale_x, const float *d_scale_w1,
                            const float *d_scale_h, float *d_amax_h, const float *d_scale_w2) {
    Mlp *M = mlp_live(mlp);
    if (!M || M->dtype != GEMM_EPI_E4M3) return GEMM_EPI_ERR_ARG;
    if (!d_scale_x || !d_scale_w1 || !d_scale_h || !d_scale_w2) return GEMM_EPI_ERR_NULL;
    int rc = gemm_epi_set_scales(M->up, d_scale_x, d_scale_w1);
    if (rc == GEMM_EPI_OK) rc = gemm_epi_set_out_scale(M->up, d_scale_h, d_amax_h);
    if (rc == GEMM_EPI_OK) rc = gemm_epi_set_scales(M->down, d_scale_h, d_scale_w2);
    return rc;
}

int gemm_epi_mlp_run(gemm_epi_mlp_t mlp, const void *X, const void *W1, const void *b1, const void *W2,
                     const void *b2, void *H, void *Y, void *stream) {
    Mlp *M = mlp_live(mlp);
    if (!M) return GEMM_EPI_ERR_ARG;
    Plan *U = reinterpret_cast<Plan *>(M->up), *Dn = reinterpret_cast<Plan *>(M->down);
    // every check of both launches before either is enqueued
    int rc = check_run_args(U, X, W1, b1, H, nullptr);
    if (rc == GEMM_EPI_OK) rc = check_run_args(Dn, H, W2, b2, Y, nullptr);
    if (rc == GEMM_EPI_OK) rc = ensure_maps(U, X, W1, H);
    if (rc == GEMM_EPI_OK) rc = ensure_maps(Dn, H, W2, Y);
    if (rc != GEMM_EPI_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (U->qout && U->amax && cudaMemsetAsync(U->amax, 0, sizeof(float), s) != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    rc = launch_main(U, true, b1, H, nullptr, s);
    if (rc != GEMM_EPI_OK) return rc;
    return launch_main(Dn, true, b2, Y, nullptr, s);
}

int gemm_epi_mlp_unfused_run(gemm_epi_mlp_t mlp, const void *X, const void *W1, const void *b1, const void *W2,
                             const void *b2, void *H, void *Y, void *H_wide, void *stream) {
    Mlp *M = mlp_live(mlp);
    if (!M) return GEMM_EPI_ERR_ARG;
    Plan *U = reinterpret_cast<Plan *>(M->up), *Dn = reinterpret_cast<Plan *>(M->down);
    const bool fp8 = U->qout;
    if (fp8 && !H_wide) return GEMM_EPI_ERR_NULL;
    if (fp8 && !aligned16(H_wide)) return GEMM_EPI_ERR_ALIGN;
    int rc = check_run_args(U, X, W1, b1, H, nullptr);
    if (rc == GEMM_EPI_OK) rc = check_run_args(Dn, H, W2, b2, Y, nullptr);
    if (rc != GEMM_EPI_OK) return rc;
    // the up-projection as a bare GEMM writing the 16-bit type (bf16 for e4m3 operands):
    // a copy of its plan without the FP8 output, with its own tensor maps
    Plan Uc = *U;
    Uc.qout = false;
    Uc.maps_valid = false;
    void *Hout = fp8 ? H_wide : H;
    BiasActLauncher ba = nullptr;
    if (!find_bias_act(U->dtype, U->kepi, U->axis, &ba)) return GEMM_EPI_ERR_UNSUPPORTED;
    rc = ensure_maps(&Uc, X, W1, Hout);
    if (rc == GEMM_EPI_OK) rc = ensure_maps(Dn, H, W2, Y);
    if (rc != GEMM_EPI_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = launch_main(&Uc, false, nullptr, Hout, nullptr, s);
    if (rc != GEMM_EPI_OK) return rc;
    const int64_t count = U->m * U->n;
    const int64_t pitch_words = ((U->n + 127) / 128) * 4;
    const int64_t blocks = std::min<int64_t>((U->m * pitch_words + 255) / 256, (int64_t)U->num_sms * 16);
    if (ba(Hout, b1, nullptr, (int)U->m, (int)U->n, pitch_words, (int)blocks, s) != cudaSuccess)
        return GEMM_EPI_ERR_CUDA;
    if (fp8) {
        const int grid = (int)std::min<int64_t>((count / 8 + 255) / 256, (int64_t)U->num_sms * 16);
        if (U->amax && (cudaMemsetAsync(U->amax, 0, sizeof(float), s) != cudaSuccess ||
                        launch_amax_bf16(H_wide, count, reinterpret_cast<unsigned int *>(U->amax), grid, s) !=
                            cudaSuccess))
            return GEMM_EPI_ERR_CUDA;
        if (launch_quantize_bf16_e4m3(H_wide, count, U->out_scale, static_cast<uint8_t *>(H), grid, s) != cudaSuccess)
            return GEMM_EPI_ERR_CUDA;
    }
    return gemm_epi_unfused_run(M->down, H, W2, b2, Y, nullptr, stream);
}

int gemm_epi_mlp_check(gemm_epi_mlp_t mlp, void *stream) {
    Mlp *M = mlp_live(mlp);
    if (!M) return GEMM_EPI_ERR_ARG;
    const int a = gemm_epi_check(M->up, stream);
    const int b = gemm_epi_check(M->down, stream);
    return a != GEMM_EPI_OK ? a : b;
}

int gemm_epi_mlp_query(gemm_epi_mlp_t mlp, gemm_epi_plan_info *up, gemm_epi_plan_info *down) {
    Mlp *M = mlp_live(mlp);
    if (!M || !up || !down) return GEMM_EPI_ERR_ARG;
    const int rc = gemm_epi_plan_query(M->up, up);
    return rc != GEMM_EPI_OK ? rc : gemm_epi_plan_query(M->down, down);
}

int gemm_epi_mlp_free(gemm_epi_mlp_t mlp) {
    Mlp *M = reinterpret_cast<Mlp *>(mlp);
    {
        std::lock_guard<std::mutex> lk(g_mlp_mu);
        if (!mlp || !g_mlps.count(M)) return GEMM_EPI_ERR_ARG;
        g_mlps.erase(M);
    }
    gemm_epi_free(M->up);
    gemm_epi_free(M->down);
    M->magic = 0;
    delete M;
    return GEMM_EPI_OK;
}

}  // extern "C"

// ----------------------------------------------------------------- allocation-free entry point
//
// gemm_epi_run_noalloc serves callers that may not allocate device memory
// themselves or through this library.  Its kernels still need scratch beyond
// the caller's inputs and outputs -- the 4-byte status word that a bounded
// wait writes when it gives up -- so that word lives in the file-scope array
// below instead of in a plan's cudaMalloc'd block.
namespace {

constexpr size_t kNoallocScratchBytes = 256;                  // reserved on every device
constexpr size_t kNoallocNeededBytes = sizeof(unsigned int);  // used by one call: the status word
static_assert(kNoallocNeededBytes <= kNoallocScratchBytes, "no-alloc scratch array too small");

static __device__ __align__(256) unsigned int g_noalloc_scratch[kNoallocScratchBytes / sizeof(unsigned int)];

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
unsigned int *g_noalloc_addr[kNoallocMaxDevices] = {};        // device address of the array, per device

// Device address of g_noalloc_scratch on `dev` (the current device).  In host
// code the array's name is only a host-side stand-in, so the address is taken
// once per device with cudaGetSymbolAddress and cached.
int noalloc_scratch(int dev, unsigned int **out) {
    if (dev < 0 || dev >= kNoallocMaxDevices) return GEMM_EPI_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return GEMM_EPI_ERR_CUDA;
        }
        g_noalloc_addr[dev] = static_cast<unsigned int *>(p);
    }
    *out = g_noalloc_addr[dev];
    return GEMM_EPI_OK;
}

}  // namespace

extern "C" int gemm_epi_run_noalloc(int64_t m, int64_t n, int64_t k, int dtype, int epilogue, int bias_axis,
                                    int b_layout, const void *A, const void *B, const void *bias,
                                    const float *d_scale_a, const float *d_scale_b, void *D, uint32_t *aux,
                                    int wait, void *stream) {
    // the same argument rules as a plan (sizes are limited to 2^31 - 1)
    if (m <= 0 || n <= 0 || k <= 0) return GEMM_EPI_ERR_ARG;
    if (m > 0x7fffffffll || n > 0x7fffffffll || k > 0x7fffffffll) return GEMM_EPI_ERR_ARG;
    if (((m + 127) / 128) * ((n + 127) / 128) > 0x7fffffffll) return GEMM_EPI_ERR_ARG;
    if (dtype < GEMM_EPI_F16 || dtype > GEMM_EPI_E4M3) return GEMM_EPI_ERR_ARG;
    if (epilogue < GEMM_EPI_NONE || epilogue > GEMM_EPI_TANH) return GEMM_EPI_ERR_ARG;
    if (bias_axis != GEMM_EPI_BIAS_ROW && bias_axis != GEMM_EPI_BIAS_COL) return GEMM_EPI_ERR_ARG;
    if (b_layout & ~(GEMM_EPI_B_NK | GEMM_EPI_A_KM)) return GEMM_EPI_ERR_ARG;
    if (wait != 0 && wait != 1) return GEMM_EPI_ERR_ARG;
    const int es = esize(dtype);
    if ((k * es) % 16 != 0 || (n * es) % 16 != 0 || (n * 2) % 16 != 0) return GEMM_EPI_ERR_ALIGN;
    if ((b_layout & GEMM_EPI_A_KM) && (m * es) % 16 != 0) return GEMM_EPI_ERR_ALIGN;
    // the call needs kNoallocNeededBytes of scratch; anything larger than the array is refused
    if (kNoallocNeededBytes > kNoallocScratchBytes) return GEMM_EPI_ERR_UNSUPPORTED;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return GEMM_EPI_ERR_NO_DEVICE;
    }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return GEMM_EPI_ERR_NO_DEVICE;

    Plan P{};                                   // on the stack: nothing is allocated
    P.magic = kPlanMagic;
    P.m = m;
    P.n = n;
    P.k = k;
    P.dtype = dtype;
    P.epilogue = epilogue;
    P.kepi = kernel_epi(epilogue);
    P.has_bias = epi_has_bias(epilogue);
    P.axis = P.has_bias ? bias_axis : GEMM_EPI_BIAS_ROW;
    P.b_layout = b_layout & GEMM_EPI_B_NK;
    P.a_km = (b_layout & GEMM_EPI_A_KM) != 0;
    P.device = dev;
    P.num_sms = num_sms_of(dev);
    P.opts.stream_k = 1;                        // stream-K would need a workspace: off
    P.no_workspace = true;                      // small m: the cluster split-K (no workspace)
    int rc = choose(&P);
    if (rc != GEMM_EPI_OK) return rc;
    if (dtype == GEMM_EPI_E4M3 || d_scale_a || d_scale_b) {      // 16-bit: optional alpha
        if (!d_scale_a || !d_scale_b) return GEMM_EPI_ERR_NULL;
        P.scale_a = d_scale_a;
        P.scale_b = d_scale_b;
    }
    rc = check_run_args(&P, A, B, bias, D, aux);
    if (rc != GEMM_EPI_OK) return rc;
    unsigned int *scratch = nullptr;
    rc = noalloc_scratch(dev, &scratch);
    if (rc != GEMM_EPI_OK) return rc;
    P.status = scratch;
    rc = ensure_maps(&P, A, B, D);
    if (rc != GEMM_EPI_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the status word must start at zero
    if (cudaMemsetAsync(scratch, 0, kNoallocNeededBytes, s) != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    rc = launch_main(&P, true, bias, D, aux, s);
    if (rc != GEMM_EPI_OK || !wait) return rc;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpy(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    return word != 0 ? GEMM_EPI_ERR_TIMEOUT : GEMM_EPI_OK;
}

#if GEMM_EPI_TRACE
// Tracing builds only: copy the timeline (counter word + records) to host memory and reset it.
extern "C" int gemm_epi_trace_read(void *host, size_t bytes) {
    unsigned long long *buf = trace_buffer();
    if (!buf) return GEMM_EPI_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    const size_t cap = (2 + 2 * (size_t)TRACE_CAP) * sizeof(unsigned long long);
    if (cudaMemcpy(host, buf, bytes < cap ? bytes : cap, cudaMemcpyDeviceToHost) != cudaSuccess) return GEMM_EPI_ERR_CUDA;
    return cudaMemset(buf, 0, cap) == cudaSuccess ? GEMM_EPI_OK : GEMM_EPI_ERR_CUDA;
}
#endif
