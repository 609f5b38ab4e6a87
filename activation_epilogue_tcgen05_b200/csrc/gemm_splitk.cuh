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
// memory.  The tile's 128 columns form four groups of 32 (one per epilogue
// warp); group q is finished by CTA q mod S.  Every CTA sends each group's fp32
// partial to that group's owner with asynchronous remote stores
// (st.async into distributed shared memory, counted on the owner's mbarrier),
// and each owner sums the S partials of its groups in rank order and runs the
// fused epilogue (scale, bias, ReLU/GELU, sign mask, RNE cast) with all four of
// its epilogue warps.  No global scratch memory is used.
#pragma once
#include "gemm_tc.cuh"

namespace gemm_epi {

// Largest K split the reduction buffer is sized for.
constexpr int sk_max_split(int nm) { return nm <= 16 ? 8 : (nm <= 64 ? 4 : 2); }
// Receive slots a CTA needs: it owns ceil(4/S) column groups (at most) and takes S partials
// of each; the most over the allowed splits.
constexpr int sk_red_slots(int nm) {
    int most = 0;
    for (int s = 1; s <= sk_max_split(nm); ++s) {
        const int slots = (4 + s - 1) / s * s;
        if (slots > most) most = slots;
    }
    return most;
}
// One slot: a 32-column group's partial, NM rows, as NM/4 blocks of [32 lanes][4 rows] floats.
constexpr int sk_red_bytes(int nm) { return sk_red_slots(nm) * nm * 128; }
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
    int pre_kb;                  // k-blocks of this CTA's weight slice asked of L2 before the dependency wait (< 0: all)
    int pre_x;                   // nonzero: also ask L2 for this CTA's activation slice before that wait
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
    static constexpr int MAX_SPLIT = sk_max_split(NM);
    static constexpr int SLOT_BYTES = NM * 128;     // one column group's partial
    static constexpr int OFF_W = 0;
    static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
    static constexpr int OFF_RED = OFF_X + STAGES * X_BYTES;
    static constexpr int OFF_BAR = OFF_RED + sk_red_bytes(NM);
    static constexpr int NUM_BARS = 2 * STAGES + 3;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    static_assert(NM % 16 == 0 && NM >= 16 && NM <= 128, "MMA N for M = 128");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(X_BYTES % 1024 == 0, "stage alignment");
    static_assert(!QOUT || (DT == DT_E4M3 && EPI != EPI_RELU_AUX), "FP8 output: e4m3 forward plans");
};

// grid = tiles_n * S CTAs, cluster (S, 1, 1): cluster c owns output columns
// [128c, 128c + 128), CTA rank r of it owns k-blocks [r*kb_per_cta, ...) and finishes the
// column groups q (32 columns each) with q mod S = r.
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
    const uint32_t red_bar = bar0 + 8u * (2 * C::STAGES + 2);   // partials of this CTA's groups in
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
    // column groups q < 4 with q mod S == rank
    const int groups = rank < 4u ? (int)((4u - rank + csize - 1u) / csize) : 0;

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
        ptx::mbar_init(red_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
        // the one arrival of red_bar's phase, with the bytes every CTA of the cluster will send
        if (groups > 0 && csize > 1u)
            ptx::mbar_arrive_expect_tx(red_bar, (uint32_t)(groups * (int)csize * C::SLOT_BYTES));
    }
    if (warp == 1) {
        ptx::tmem_alloc<1>(ptx::smem_addr(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // peers may send into this CTA's red_bar once they are past the matching wait
    ptx::cluster_arrive();
    // This CTA's slice of the weight operand (the first p.pre_kb k-blocks of it, or all) and
    // optionally of the activations is prefetched into L2 before waiting on the previous
    // grid, so its DRAM latency overlaps that grid's tail.  A prefetch writes nothing and L2
    // is the point of coherence, so the loads below still see any value the previous kernel
    // stores.  Every other global access waits for the previous grid.
    if (warp == 0 && lane == 0) {
        if (p.pre_x)
            for (int kb = kb_begin; kb < kb_end; ++kb) ptx::tma_prefetch_l2_2d(&tmX, kb * C::BK, 0);
        const int pre_end = p.pre_kb < 0 ? kb_end : min(kb_end, kb_begin + p.pre_kb);
        for (int kb = kb_begin; kb < pre_end; ++kb) {
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

    // The epilogue's operands other than the partials (column bias of each column group this
    // CTA finishes, FP8 scales), read now by the epilogue warps, idle until the accumulator is
    // ready, so that their latency is off the reduction's path.
    const bool epi = warp >= 2;
    float cbias[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float alpha = 1.0f, inv_out = 1.0f;
    if (epi && groups > 0) {
        if constexpr (C::EPI != EPI_NONE && C::AXIS == AXIS_COL) {
#pragma unroll
            for (int gl = 0; gl < 4; ++gl) {
                const int col = n0 + 32 * ((int)rank + gl * (int)csize) + lane;
                if (gl < groups && col < p.n && p.bias != nullptr) cbias[gl] = OutT<C::DT>::load(p.bias, col);
            }
        }
        if (p.scale_a != nullptr) alpha = __ldg(p.scale_a) * __ldg(p.scale_b);
        if constexpr (C::QOUT) inv_out = 1.0f / __ldg(p.out_scale);
    }

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
    const int q = warp & 3;
    using O = OutT<C::DT>;
    using T = typename O::type;
    T *D = reinterpret_cast<T *>(p.D);
    const bool has_bias = p.bias != nullptr;
    float amax_l = 0.0f;
    // The fused epilogue of rows 4u .. 4u+3 of column group `grp` (this thread's column
    // n0 + 32 grp + lane), from their fp32 sums `part`: the four rows' values first, without
    // branches, then their stores.
    auto emit4 = [&](int grp, int u, const float (&part)[4], float cb) {
        const int col = n0 + 32 * grp + lane;
        const bool col_ok = col < p.n;
        // every word of the mask pitch belongs to exactly one group of one tile;
        // columns at or past n contribute 0 bits, so padding words come out 0
        const int64_t word = (col - lane) / 32;
        float y[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = 4 * u + c;
            float x = part[c] * alpha;
            if constexpr (C::EPI != EPI_NONE) {
                if constexpr (C::AXIS == AXIS_COL) x += cb;
                else if (has_bias && i < p.m) x += O::load(p.bias, i);
            }
            if constexpr (C::EPI == EPI_RELU_AUX) {
                const uint32_t bits = __ballot_sync(0xFFFFFFFFu, col_ok && x > 0.0f);
                if (lane == 0 && i < p.m) p.aux[(int64_t)i * p.aux_pitch_words + word] = bits;
            }
            y[c] = activate<C::EPI>(x);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = 4 * u + c;
            if (col_ok && i < p.m) {
                if constexpr (C::QOUT) {
                    // e4m3 code, round to nearest even, saturating at +-448
                    amax_l = fmaxf(amax_l, fabsf(y[c]));
                    p.dq[(int64_t)i * p.n + col] = __nv_cvt_float_to_fp8(y[c] * inv_out, __NV_SATFINITE, __NV_E4M3);
                } else if constexpr (C::DT == DT_F16) {
                    D[(int64_t)i * p.n + col] = __float2half_rn(y[c]);
                } else {
                    D[(int64_t)i * p.n + col] = __float2bfloat16_rn(y[c]);
                }
            }
        }
    };
    __syncwarp();
    ptx::cluster_wait();     // every CTA's red_bar is initialised
    if (epi) {
        float acc[C::NM];
        bool have = false;
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
        if (csize == 1u) {
            // a cluster of one CTA: the accumulator is the whole sum; each warp finishes its own
            // column group straight from its registers
            if (have) {
                float cb = 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (j == q) cb = cbias[j];
#pragma unroll
                for (int u = 0; u < C::NM / 4; ++u) {
                    const float part[4] = {acc[4 * u], acc[4 * u + 1], acc[4 * u + 2], acc[4 * u + 3]};
                    emit4(q, u, part, cb);
                }
            }
        } else {
            // this CTA's partial of group q goes to slot (q / S) * S + rank of the group's owner;
            // a CTA without work (or after an abort) sends zeros, so every owner's count completes
            const uint32_t owner = (uint32_t)q % csize;
            const uint32_t slot = ((uint32_t)q / csize) * csize + rank;
            const uint32_t dst = ptx::mapa(sb + C::OFF_RED + slot * C::SLOT_BYTES + (uint32_t)lane * 16u, owner);
            const uint32_t dbar = ptx::mapa(red_bar, owner);
#pragma unroll
            for (int u = 0; u < C::NM / 4; ++u)
                ptx::st_async_v4(dst + (uint32_t)u * 512u, acc[4 * u], acc[4 * u + 1], acc[4 * u + 2], acc[4 * u + 3], dbar);
        }
    }

    if (epi && groups > 0 && csize > 1u) {
        const int ew = warp - 2;
        if (wait_bounded<true>(red_bar, 0, abort_flag, p.status, ST_TIMEOUT_SPLITK)) {
            if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 28, tile_n, (int)rank);
            constexpr int QUADS = C::NM / 4;
            // work units (owned group, block of 4 rows), dealt round-robin to the 4 epilogue warps
            for (int unit = ew; unit < groups * QUADS; unit += 4) {
                const int gl = unit / QUADS, u = unit - gl * QUADS;
                // the S partials, all loaded first, then added in rank order
                const float *src = reinterpret_cast<const float *>(smem + C::OFF_RED) +
                                   ((gl * (int)csize) * C::SLOT_BYTES + u * 512 + lane * 16) / 4;
                float4 pv[C::MAX_SPLIT];
#pragma unroll
                for (int r = 0; r < C::MAX_SPLIT; ++r)
                    if (r < (int)csize) pv[r] = *reinterpret_cast<const float4 *>(src + r * (C::SLOT_BYTES / 4));
                float4 sum = pv[0];
#pragma unroll
                for (int r = 1; r < C::MAX_SPLIT; ++r) {
                    if (r < (int)csize) {
                        sum.x += pv[r].x;
                        sum.y += pv[r].y;
                        sum.z += pv[r].z;
                        sum.w += pv[r].w;
                    }
                }
                const float part[4] = {sum.x, sum.y, sum.z, sum.w};
                if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 33, tile_n, unit);
                float cb = 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (j == gl) cb = cbias[j];
                emit4((int)rank + gl * (int)csize, u, part, cb);
                if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 34, tile_n, unit);
            }
        }
    }
    if constexpr (C::QOUT) {
        if (epi && groups > 0) {
            // one atomic per warp: the launch's max |y| (non-negative floats order as their bits)
            const unsigned int wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_l));
            if (lane == 0 && p.amax != nullptr && wmax != 0u) atomicMax(p.amax, wmax);
        }
    }

    if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 27, tile_n, (int)rank);
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc<1>(tmem_base, C::TMEM_COLS);
    }
    // The cluster's CTAs leave together.  (Each one has already received every byte sent to
    // it, so nothing is in flight towards its shared memory; the relaxed arrival does not wait
    // for this thread's global stores.)
    ptx::cluster_arrive_relaxed();
    ptx::cluster_wait();
    if (warp == 1 && lane == 0) trace_stage(p.trace, 3, tr_i, 29, tile_n, (int)rank);
}

}  // namespace gemm_epi
