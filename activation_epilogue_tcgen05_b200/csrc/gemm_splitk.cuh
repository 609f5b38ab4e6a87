// gemm_splitk.cuh -- small-m path (a batch of up to 128 rows, e.g. the
// Linear(4096,4096)+GELU batch-16 latency case of "PyTorch 2.14 NVGEMM epilogue
// fusion" (zdabc.icu), section "verifying torch.compile").
//
// With m this small the problem is a stream over the weight B (HBM-bound),
// and a 128-row MMA tile along m would be mostly empty.  So the operand roles
// are swapped: tcgen05.mma computes D^T tiles, its M = 128 rows are 128
// output COLUMNS (rows of the weight), its N = NM (m rounded up to 16) are the
// batch rows, and the accumulator lane of a thread is one output column.
// To put enough SMs on the weight stream, K is split over a thread-block
// cluster of S CTAs: each CTA accumulates its k-range in its own tensor
// memory, the S-1 partner CTAs push their fp32 partial tiles into the leader
// CTA's shared memory (distributed shared memory, st.shared::cluster), and
// after one cluster barrier the leader sums them in rank order and runs the
// same fused epilogue (scale, bias, ReLU/GELU, sign mask, RNE cast).
// No global scratch memory is used.
#pragma once
#include "gemm_tc.cuh"

namespace gemm_epi {

// Largest K split the leader's reduction buffer is sized for, and that buffer's size.
constexpr int sk_max_split(int nm) { return nm <= 16 ? 8 : (nm <= 64 ? 4 : 2); }
constexpr int sk_red_bytes(int nm) { return (sk_max_split(nm) - 1) * 128 * (nm + 4) * 4; }
// Ring depth: fill ~200 KB of shared memory with the reduction buffer and stages, at most 8.
constexpr int sk_stages(int nm) {
    return (200 * 1024 - sk_red_bytes(nm)) / (128 * 128 + nm * 128) > 8
               ? 8
               : (200 * 1024 - sk_red_bytes(nm)) / (128 * 128 + nm * 128);
}

struct SkParams {
    int m, n, k;
    int num_kb;                  // k-blocks in total
    int kb_per_cta;              // k-blocks per CTA of a cluster
    const void *bias;
    void *D;
    uint32_t *aux;
    int64_t aux_pitch_words;
    const float *scale_a;
    const float *scale_b;
    unsigned int *status;
    // FP8 output (QOUT kernels): D = e4m3(y / *out_scale), one byte per element; amax
    // (optional) receives max |y| as float bits through an atomic max
    uint8_t *dq;
    const float *out_scale;
    unsigned int *amax;
    unsigned long long *trace;   // timeline records; used only by builds with GEMM_EPI_TRACE=2
};

template <int DT_, int EPI_, int AXIS_, bool W_MN_, int NM_, int STAGES_, bool QOUT_ = false>
struct SkCfg {
    static constexpr int DT = DT_, EPI = EPI_, AXIS = AXIS_, NM = NM_, STAGES = STAGES_;
    static constexpr bool QOUT = QOUT_;             // e4m3 output quantised in the epilogue
    static constexpr bool W_MN = W_MN_;             // weight stored (k, n): MMA operand A is MN-major
    static constexpr int ESIZE = DT == DT_E4M3 ? 1 : 2;
    static constexpr int KIND = DT == DT_E4M3 ? 1 : 0;
    static constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
    static constexpr int BK = 128 / ESIZE;
    static constexpr int UMMA_K = 32 / ESIZE;
    static constexpr int KSTEPS = BK / UMMA_K;
    static constexpr int W_BYTES = 128 * 128;       // 128 output columns x 128 bytes of k
    static constexpr int X_BYTES = NM * 128;        // NM batch rows x 128 bytes of k
    static constexpr int W_BOX_N = 128 / ESIZE;
    static constexpr int W_BOXES = W_MN ? 128 / W_BOX_N : 1;
    static constexpr int W_BOX_BYTES = W_MN ? BK * 128 : W_BYTES;
    static constexpr int THREADS = 64 + 128;
    static constexpr int TMEM_COLS = NM <= 32 ? 32 : (NM <= 64 ? 64 : 128);
    static constexpr int RED_STRIDE = NM + 4;       // floats per partial row (padded)
    static constexpr int MAX_SPLIT = sk_max_split(NM);
    static constexpr int OFF_W = 0;
    static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
    static constexpr int OFF_RED = OFF_X + STAGES * X_BYTES;
    static constexpr int RED_BYTES_PER_RANK = 128 * RED_STRIDE * 4;
    static constexpr int OFF_BAR = OFF_RED + sk_red_bytes(NM);
    static constexpr int NUM_BARS = 2 * STAGES + 2;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    static_assert(NM % 16 == 0 && NM >= 16 && NM <= 128, "MMA N for M = 128");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(X_BYTES % 1024 == 0, "stage alignment");
    static_assert(!QOUT || (DT == DT_E4M3 && EPI != EPI_RELU_AUX), "FP8 output: e4m3 forward plans");
};

// grid = tiles_n * S CTAs, cluster (S, 1, 1): cluster c owns output columns
// [128c, 128c + 128), CTA rank r of it owns k-blocks [r*kb_per_cta, ...).
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    splitk_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const SkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sb = ptx::smem_addr(smem);
    const uint32_t sW = sb + C::OFF_W, sX = sb + C::OFF_X;
    const uint32_t bar0 = sb + C::OFF_BAR;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
    const uint32_t tfull = bar0 + 8u * (2 * C::STAGES);
    const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = ptx::warp_id();
    const int lane = ptx::lane_id();
    uint32_t csize;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(csize));
    const uint32_t rank = ptx::cluster_ctarank();
    const int tile_n = blockIdx.x / (int)csize;
    const int n0 = tile_n * 128;
    const int kb_begin = (int)rank * p.kb_per_cta;
    const int kb_end = min(p.num_kb, kb_begin + p.kb_per_cta);
    const int my_kb = kb_end > kb_begin ? kb_end - kb_begin : 0;

    uint32_t tr_i = 0;
    if (warp == 0 && lane == 0) {
        trace_stage(p.trace, 0, tr_i, 10, tile_n, (int)rank);
        ptx::prefetch_tmap(&tmW);
        ptx::prefetch_tmap(&tmX);
        for (int s = 0; s < C::STAGES; ++s) {
            ptx::mbar_init(full_bar(s), 1);
            ptx::mbar_init(empty_bar(s), 1);
        }
        ptx::mbar_init(tfull, 1);
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc<1>(ptx::smem_addr(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // This CTA's slice of the weight operand is prefetched into L2 before waiting on the
    // previous grid, so its DRAM latency overlaps that grid's tail.  A prefetch writes
    // nothing and L2 is the point of coherence, so the loads below still see any value the
    // previous kernel stores.  Every other global access waits for the previous grid.
    if (warp == 0 && lane == 0) {
        for (int kb = kb_begin; kb < kb_end; ++kb) {
            if constexpr (C::W_MN) {
#pragma unroll
                for (int b = 0; b < C::W_BOXES; ++b) ptx::tma_prefetch_l2_2d(&tmW, n0 + b * C::W_BOX_N, kb * C::BK);
            } else {
                ptx::tma_prefetch_l2_2d(&tmW, kb * C::BK, n0);
            }
        }
    }
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            trace_stage(p.trace, 0, tr_i, 11, tile_n, (int)rank);
            uint32_t stage = 0, phase = 0, issued = 0;
            bool ok = true;
            const uint64_t pol = ptx::policy_evict_normal();
            for (int kb = kb_begin; kb < kb_end; ++kb) {
                if (!wait_bounded<false>(empty_bar(stage), phase ^ 1u, abort_flag, p.status, ST_TIMEOUT_SPLITK)) {
                    ok = false;
                    break;
                }
                trace_stage(p.trace, 0, tr_i, 20, tile_n, kb);
                const uint32_t fb = full_bar(stage);
                ptx::mbar_arrive_expect_tx(fb, C::W_BYTES + C::X_BYTES);
                const int k0 = kb * C::BK;
                const uint32_t w_dst = sW + stage * C::W_BYTES;
                if constexpr (C::W_MN) {
#pragma unroll
                    for (int b = 0; b < C::W_BOXES; ++b)
                        ptx::tma_load_2d(w_dst + b * C::W_BOX_BYTES, &tmW, fb, n0 + b * C::W_BOX_N, k0,
                                         pol);
                } else {
                    ptx::tma_load_2d(w_dst, &tmW, fb, k0, n0, pol);
                }
                ptx::tma_load_2d(sX + stage * C::X_BYTES, &tmX, fb, k0, 0, pol);
                ++issued;
                if (++stage == (uint32_t)C::STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) {
                const uint32_t back = issued < (uint32_t)C::STAGES ? issued : (uint32_t)C::STAGES;
                for (uint32_t j = issued - back; j < issued; ++j)
                    wait_drain(full_bar(j % C::STAGES), (j / C::STAGES) & 1u, p.status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(C::FMT, C::W_MN, false, 128, C::NM);
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int i = 0; i < my_kb; ++i) {
                if (!wait_bounded<false>(full_bar(stage), phase, abort_flag, p.status, ST_TIMEOUT_SPLITK)) {
                    ok = false;
                    break;
                }
                trace_stage(p.trace, 1, tr_i, 22, tile_n, kb_begin + i);
                ptx::tc_fence_after();
                const uint32_t w_base = sW + stage * C::W_BYTES;
                const uint32_t x_base = sX + stage * C::X_BYTES;
#pragma unroll
                for (int ks = 0; ks < C::KSTEPS; ++ks) {
                    const uint64_t ad = C::W_MN ? make_sdesc(w_base + ks * C::UMMA_K * 128, C::W_BOX_BYTES, 1024)
                                                : make_sdesc(w_base + ks * 32, 16, 1024);
                    const uint64_t bd = make_sdesc(x_base + ks * 32, 16, 1024);
                    ptx::mma<1, C::KIND>(tmem_base, ad, bd, idesc, (i | ks) != 0 ? 1u : 0u);
                }
                ptx::mma_commit(empty_bar(stage));
                if (++stage == (uint32_t)C::STAGES) { stage = 0; phase ^= 1u; }
            }
            if (ok) ptx::mma_commit(tfull);
            trace_stage(p.trace, 1, tr_i, 23, tile_n, kb_end);
            ptx::mma_commit(done_bar);
            wait_drain(done_bar, 0, p.status);
        }
    }

    // -------------------------------------------------------------- epilogue
    // warps 2..5: thread (q, lane) owns accumulator lane 32q + lane = output column n0 + 32q + lane.
    const bool epi = warp >= 2;
    const int q = warp & 3;
    float acc[C::NM];
    bool have = false;
    if (epi) {
        if (my_kb > 0 && wait_bounded<false>(tfull, 0, abort_flag, p.status, ST_TIMEOUT_SPLITK)) {
            if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 26, tile_n, (int)rank);
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16);
#pragma unroll
            for (int c = 0; c < C::NM; c += 16) {
                uint32_t v[16];
                ptx::tmem_ld_32x32b_x16(taddr + c, v);
                ptx::tmem_wait_ld16(v);
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[c + j] = __uint_as_float(v[j]);
            }
            have = true;
        }
        if (!have) {
#pragma unroll
            for (int j = 0; j < C::NM; ++j) acc[j] = 0.0f;
        }
        if (rank != 0) {
            // push this CTA's partial row into the leader's reduction slot rank-1
            const uint32_t local = sb + C::OFF_RED + (rank - 1) * C::RED_BYTES_PER_RANK +
                                   (uint32_t)((32 * q + lane) * C::RED_STRIDE * 4);
            const uint32_t remote = ptx::mapa(local, 0);
#pragma unroll
            for (int j = 0; j < C::NM; j += 4)
                ptx::st_cluster_v4(remote + j * 4, acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        }
    }
    // the leader's column bias, read before the cluster barrier so that its latency hides
    float cbias = 0.0f;
    if constexpr (C::EPI != EPI_NONE && C::AXIS == AXIS_COL) {
        const int col = n0 + 32 * q + lane;
        if (epi && rank == 0 && col < p.n && p.bias != nullptr) cbias = OutT<C::DT>::load(p.bias, col);
    }
    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();     // partials visible in the leader's shared memory
    if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 28, tile_n, (int)rank);

    if (epi && rank == 0) {
        using O = OutT<C::DT>;
        using T = typename O::type;
        const float *red = reinterpret_cast<const float *>(smem + C::OFF_RED);
        const int row_in_tile = 32 * q + lane;
        for (uint32_t r = 1; r < csize; ++r) {
            const float *src = red + (r - 1) * (C::RED_BYTES_PER_RANK / 4) + row_in_tile * C::RED_STRIDE;
#pragma unroll
            for (int j = 0; j < C::NM; j += 4) {
                const float4 f = *reinterpret_cast<const float4 *>(src + j);
                acc[j] += f.x;
                acc[j + 1] += f.y;
                acc[j + 2] += f.z;
                acc[j + 3] += f.w;
            }
        }
        const int col = n0 + row_in_tile;
        const bool col_ok = col < p.n;
        float alpha = 1.0f;
        if (p.scale_a != nullptr) alpha = __ldg(p.scale_a) * __ldg(p.scale_b);
        const bool has_bias = p.bias != nullptr;
        T *D = reinterpret_cast<T *>(p.D);
        float inv_out = 1.0f, amax_l = 0.0f;
        if constexpr (C::QOUT) inv_out = 1.0f / __ldg(p.out_scale);
        // every word of the mask pitch belongs to exactly one warp of one tile;
        // columns at or past n contribute 0 bits, so padding words come out 0
        const int64_t word = (n0 + 32 * q) / 32;
#pragma unroll
        for (int i = 0; i < C::NM; ++i) {
            if (i < p.m) {
                float x = acc[i];
                x *= alpha;
                if constexpr (C::EPI != EPI_NONE) {
                    if constexpr (C::AXIS == AXIS_COL) x += cbias;
                    else if (has_bias) x += O::load(p.bias, i);
                }
                if constexpr (C::EPI == EPI_RELU_AUX) {
                    const uint32_t bits = __ballot_sync(0xFFFFFFFFu, col_ok && x > 0.0f);
                    if (lane == 0) p.aux[(int64_t)i * p.aux_pitch_words + word] = bits;
                }
                const float y = activate<C::EPI>(x);
                if (col_ok) {
                    if constexpr (C::QOUT) {
                        // e4m3 code, round to nearest even, saturating at +-448
                        amax_l = fmaxf(amax_l, fabsf(y));
                        p.dq[(int64_t)i * p.n + col] = __nv_cvt_float_to_fp8(y * inv_out, __NV_SATFINITE, __NV_E4M3);
                    } else if constexpr (C::DT == DT_F16) {
                        D[(int64_t)i * p.n + col] = __float2half_rn(y);
                    } else {
                        D[(int64_t)i * p.n + col] = __float2bfloat16_rn(y);
                    }
                }
            }
        }
        if constexpr (C::QOUT) {
            // one atomic per warp: the launch's max |y| (non-negative floats order as their bits)
            const unsigned int wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_l));
            if (lane == 0 && p.amax != nullptr) atomicMax(p.amax, wmax);
        }
    }

    if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 27, tile_n, (int)rank);
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc<1>(tmem_base, C::TMEM_COLS);
        if (lane == 0) trace_stage(p.trace, 3, tr_i, 29, tile_n, (int)rank);
    }
}

}  // namespace gemm_epi
