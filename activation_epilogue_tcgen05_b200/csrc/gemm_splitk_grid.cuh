// gemm_splitk_grid.cuh -- small-m path over every SM of the GPU.
//
// The same problem and operand roles as the cluster split-K kernel (gemm_splitk.cuh): a
// batch of up to 128 rows times a weight, a stream over the weight that HBM bandwidth
// bounds (the Linear(4096,4096)+GELU batch-16 case of "PyTorch 2.14 NVGEMM epilogue
// fusion" (zdabc.icu), section "verifying torch.compile").  tcgen05.mma computes D^T
// tiles: M = 128 output columns (rows of the weight), N = NM batch rows.
//
// The work is the list of (tile, k-block) units, tile-major.  Every CTA of the grid (one
// per SM) takes an equal contiguous range of it, so all SMs stream the weight whatever
// the number of tiles; a range is cut at tile boundaries into pieces.  A piece that covers
// a whole tile is finished in place.  A tile cut into pieces is finished by the CTA that
// holds its first k-block: each other piece is, by construction, the first piece of its
// CTA's range, so it is multiplied first and published early (each epilogue warp writes its
// 32 columns' fp32 partial to the CTA's workspace slot and raises a flag).  The finishing
// warp keeps its own partial in registers, waits (bounded) for the flags, adds the other
// pieces in piece order (a fixed order: run-to-run identical results), clears the flags and
// runs the fused epilogue (scale, bias, ReLU/GELU, sign mask, cast).  Waits only ever point
// to higher-numbered CTAs' first pieces, which wait on nothing lower, so they always end.
// Every flag is cleared by its one reader, so a launch leaves the flags as it found them
// (zero) and launches can be replayed from CUDA graphs.
#pragma once
#include "gemm_tc.cuh"

namespace gemm_epi {

// Ring depth: ~200 KB of stages, at most 12.  (A ring half as deep, which lets the next
// launch's CTAs sit beside this launch's and prefetch early, streamed slower: 14.9 against
// 12.9 us a step for 16 x 4096 x 4096.)
constexpr int sg_stages(int nm) {
    return (200 * 1024) / (128 * 128 + nm * 128) > 12 ? 12 : (200 * 1024) / (128 * 128 + nm * 128);
}

struct SgParams {
    int m, n, k;
    int num_kb;                  // k-blocks per output tile
    int tiles_n;                 // output tiles of 128 columns
    int grid;                    // CTAs: one contiguous range of units each
    const void *bias;
    void *D;
    uint32_t *aux;
    int64_t aux_pitch_words;
    const float *scale_a;
    const float *scale_b;
    unsigned int *status;
    uint8_t *dq;                 // FP8 output (QOUT kernels), as SkParams
    const float *out_scale;
    unsigned int *amax;
    // Partial tiles of the pieces that do not start a tile (always their CTA's first piece):
    // [cta][quadrant][NM][32] fp32.  NULL: one CTA per tile, nothing is split.
    float *workspace;
    unsigned int *flags;         // [cta][quadrant]: 1 while a published partial is unread; 0 between launches
    unsigned long long *trace;   // timeline records; used only by builds with GEMM_EPI_TRACE=2
};

template <int DT_, int EPI_, int AXIS_, bool W_MN_, int NM_, int STAGES_, bool QOUT_ = false>
struct SgCfg {
    static constexpr int DT = DT_, EPI = EPI_, AXIS = AXIS_, NM = NM_, STAGES = STAGES_;
    static constexpr bool QOUT = QOUT_;
    static constexpr bool W_MN = W_MN_;             // weight stored (k, n): MMA operand A is MN-major
    static constexpr int ESIZE = DT == DT_E4M3 ? 1 : 2;
    static constexpr int KIND = DT == DT_E4M3 ? 1 : 0;
    static constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
    static constexpr int BK = 128 / ESIZE;
    static constexpr int UMMA_K = 32 / ESIZE;
    static constexpr int KSTEPS = BK / UMMA_K;
    static constexpr int W_BYTES = 128 * 128;
    static constexpr int X_BYTES = NM * 128;
    static constexpr int W_BOX_N = 128 / ESIZE;
    static constexpr int W_BOXES = W_MN ? 128 / W_BOX_N : 1;
    static constexpr int W_BOX_BYTES = W_MN ? BK * 128 : W_BYTES;
    static constexpr int THREADS = 64 + 128;
    static constexpr int TMEM_COLS = 2 * NM <= 32 ? 32 : (2 * NM <= 64 ? 64 : (2 * NM <= 128 ? 128 : 256));
    static constexpr int OFF_W = 0;
    static constexpr int OFF_X = OFF_W + STAGES * W_BYTES;
    static constexpr int OFF_BAR = OFF_X + STAGES * X_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
    static constexpr int WS_FLOATS = 4 * NM * 32;       // workspace floats per CTA
    static constexpr int PB = NM <= 32 ? 8 : (NM <= 64 ? 4 : 2);   // partials loaded at once
    static_assert(NM % 16 == 0 && NM >= 16 && NM <= 128, "MMA N for M = 128");
    static_assert(STAGES >= 2, "the ring needs two stages");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(X_BYTES % 1024 == 0, "stage alignment");
    static_assert(!QOUT || (DT == DT_E4M3 && EPI != EPI_RELU_AUX), "FP8 output: e4m3 forward plans");
};

// A CTA's range of units [u0, u1) and the pieces it is cut into.
struct SgRange {
    int64_t units, u, u1;
    int num_kb, grid;
    __device__ SgRange(const SgParams &p, int cta) : num_kb(p.num_kb), grid(p.grid) {
        units = (int64_t)p.tiles_n * p.num_kb;
        u = (int64_t)cta * units / p.grid;
        u1 = (int64_t)(cta + 1) * units / p.grid;
    }
    __device__ int64_t start_of(int cta) const { return (int64_t)cta * units / grid; }
    // the CTA whose range holds unit v
    __device__ int owner(int64_t v) const { return (int)(((v + 1) * grid - 1) / units); }
    // next piece: tile, k-blocks [kb0, kb1) of it, and whether it starts the CTA's range
    __device__ bool next(int &tile, int &kb0, int &kb1, bool &first, int64_t u_first) {
        if (u >= u1) return false;
        tile = (int)(u / num_kb);
        kb0 = (int)(u - (int64_t)tile * num_kb);
        const int64_t left = u1 - u;
        kb1 = left < (int64_t)(num_kb - kb0) ? kb0 + (int)left : num_kb;
        first = u == u_first;
        u += kb1 - kb0;
        return true;
    }
};

// Bounded wait, by one warp, until flags[0], flags[stride], ... flags[(count - 1) * stride] are
// all set: each lane polls its own flags, so one poll round is one memory round trip whatever
// the count.  After it every lane's later loads see what the flags' writers published.
__device__ __forceinline__ bool wait_flags_warp(const unsigned int *flags, int stride, int count, int lane,
                                                volatile int *abort_flag, unsigned int *status) {
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 0;; ++it) {
        bool mine = true;
        for (int j = lane; j < count; j += 32) mine = mine && ptx::ld_acquire_gpu(flags + (size_t)j * stride) != 0u;
        if (__all_sync(0xffffffffu, mine)) break;
        if ((it & 15u) == 15u) {
            // one decision for the whole warp (lane 0's), so that every lane leaves together
            int stop = 0;
            if (lane == 0) stop = *abort_flag ? 1 : (ptx::globaltimer() - t0 > TIMEOUT_NS ? 2 : 0);
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop == 2 && lane == 0) {
                *abort_flag = 1;
                atomicOr(status, ST_TIMEOUT_SPLITK);
            }
            if (stop) return false;
        }
    }
    __syncwarp();     // orders every lane's loads after the lanes' acquires
    return true;
}

template <class C>
__device__ __forceinline__ float *sg_slot(const SgParams &p, int cta, int q) {
    return p.workspace + ((size_t)cta * C::WS_FLOATS) + (size_t)q * C::NM * 32;
}

// grid = p.grid CTAs, no cluster.
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    splitk_grid_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const SgParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sb = ptx::smem_addr(smem);
    const uint32_t sW = sb + C::OFF_W, sX = sb + C::OFF_X;
    const uint32_t bar0 = sb + C::OFF_BAR;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 2 + a); };
    const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = ptx::warp_id();
    const int lane = ptx::lane_id();
    const int cta = blockIdx.x;
    const int64_t u_first = (int64_t)cta * ((int64_t)p.tiles_n * p.num_kb) / p.grid;

    uint32_t tr_i = 0;
    if (warp == 0 && lane == 0) {
        trace_stage(p.trace, 0, tr_i, 10, 0, cta);
        ptx::prefetch_tmap(&tmW);
        ptx::prefetch_tmap(&tmX);
        for (int s = 0; s < C::STAGES; ++s) {
            ptx::mbar_init(full_bar(s), 1);
            ptx::mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(tfull_bar(a), 1);
            ptx::mbar_init(tempty_bar(a), 4);
        }
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
    // This CTA's part of the weight is prefetched into L2 before waiting on the previous
    // grid, so its DRAM latency overlaps that grid's tail (a prefetch writes nothing; L2 is
    // the point of coherence).  Every other global access waits for the previous grid.
    if (warp == 0 && lane == 0) {
        SgRange r(p, cta);
        int tile, kb0, kb1;
        bool first;
        while (r.next(tile, kb0, kb1, first, u_first)) {
            for (int kb = kb0; kb < kb1; ++kb) {
                if constexpr (C::W_MN) {
#pragma unroll
                    for (int b = 0; b < C::W_BOXES; ++b)
                        ptx::tma_prefetch_l2_2d(&tmW, tile * 128 + b * C::W_BOX_N, kb * C::BK);
                } else {
                    ptx::tma_prefetch_l2_2d(&tmW, kb * C::BK, tile * 128);
                }
            }
        }
    }
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            trace_stage(p.trace, 0, tr_i, 11, 0, cta);
            uint32_t stage = 0, phase = 0, issued = 0;
            bool ok = true;
            const uint64_t pol = ptx::policy_evict_normal();
            SgRange r(p, cta);
            int tile, kb0, kb1;
            bool first;
            while (ok && r.next(tile, kb0, kb1, first, u_first)) {
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bounded<false>(empty_bar(stage), phase ^ 1u, abort_flag, p.status,
                                             ST_TIMEOUT_SPLITK)) {
                        ok = false;
                        break;
                    }
                    trace_stage(p.trace, 0, tr_i, 20, tile, kb);
                    const uint32_t fb = full_bar(stage);
                    ptx::mbar_arrive_expect_tx(fb, C::W_BYTES + C::X_BYTES);
                    const int k0 = kb * C::BK;
                    const uint32_t w_dst = sW + stage * C::W_BYTES;
                    if constexpr (C::W_MN) {
#pragma unroll
                        for (int b = 0; b < C::W_BOXES; ++b)
                            ptx::tma_load_2d(w_dst + b * C::W_BOX_BYTES, &tmW, fb, tile * 128 + b * C::W_BOX_N, k0,
                                             pol);
                    } else {
                        ptx::tma_load_2d(w_dst, &tmW, fb, k0, tile * 128, pol);
                    }
                    ptx::tma_load_2d(sX + stage * C::X_BYTES, &tmX, fb, k0, 0, pol);
                    ++issued;
                    if (++stage == (uint32_t)C::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                const uint32_t back = issued < (uint32_t)C::STAGES ? issued : (uint32_t)C::STAGES;
                for (uint32_t j = issued - back; j < issued; ++j)
                    wait_drain(full_bar(j % C::STAGES), (j / C::STAGES) & 1u, p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(C::FMT, C::W_MN, false, 128, C::NM);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true;
            SgRange r(p, cta);
            int tile, kb0, kb1;
            bool first;
            while (ok && r.next(tile, kb0, kb1, first, u_first)) {
                if (!wait_bounded<false>(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status, ST_TIMEOUT_SPLITK)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * C::NM;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bounded<false>(full_bar(stage), phase, abort_flag, p.status, ST_TIMEOUT_SPLITK)) {
                        ok = false;
                        break;
                    }
                    trace_stage(p.trace, 1, tr_i, 22, tile, kb);
                    ptx::tc_fence_after();
                    const uint32_t w_base = sW + stage * C::W_BYTES;
                    const uint32_t x_base = sX + stage * C::X_BYTES;
#pragma unroll
                    for (int ks = 0; ks < C::KSTEPS; ++ks) {
                        const uint64_t ad = C::W_MN ? make_sdesc(w_base + ks * C::UMMA_K * 128, C::W_BOX_BYTES, 1024)
                                                    : make_sdesc(w_base + ks * 32, 16, 1024);
                        const uint64_t bd = make_sdesc(x_base + ks * 32, 16, 1024);
                        ptx::mma<1, C::KIND>(d_tmem, ad, bd, idesc, (kb > kb0 || ks > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit(empty_bar(stage));
                    if (++stage == (uint32_t)C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit(tfull_bar(acc));
                if (++acc == 2u) { acc = 0; acc_phase ^= 1u; }
            }
            trace_stage(p.trace, 1, tr_i, 23, 0, cta);
            ptx::mma_commit(done_bar);
            wait_drain(done_bar, 0, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // warps 2..5: thread (q, lane) owns accumulator lane 32q + lane = output column
        // 128 * tile + 32q + lane.
        using O = OutT<C::DT>;
        using T = typename O::type;
        const int q = warp & 3;
        float alpha = 1.0f;
        if (p.scale_a != nullptr) alpha = __ldg(p.scale_a) * __ldg(p.scale_b);
        const bool has_bias = p.bias != nullptr;
        float inv_out = 1.0f, amax_l = 0.0f;
        if constexpr (C::QOUT) inv_out = 1.0f / __ldg(p.out_scale);
        T *D = reinterpret_cast<T *>(p.D);
        uint32_t acc = 0, acc_phase = 0;
        bool ok = true;
        SgRange r(p, cta);
        int tile, kb0, kb1;
        bool first;
        while (ok && r.next(tile, kb0, kb1, first, u_first)) {
            // this lane's output column and its bias, read before the accumulator is waited for
            const int n0 = tile * 128;
            const int col = n0 + 32 * q + lane;
            const bool col_ok = col < p.n;
            float cbias = 0.0f;
            if constexpr (C::EPI != EPI_NONE && C::AXIS == AXIS_COL) {
                if (kb0 == 0 && col_ok && has_bias) cbias = O::load(p.bias, col);
            }
            if (!wait_bounded<false>(tfull_bar(acc), acc_phase, abort_flag, p.status, ST_TIMEOUT_SPLITK)) {
                ok = false;
                break;
            }
            if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 26, tile, kb0);
            ptx::tc_fence_after();
            float v[C::NM];
            const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + acc * C::NM;
#pragma unroll
            for (int c = 0; c < C::NM; c += 16) {
                uint32_t t16[16];
                ptx::tmem_ld_32x32b_x16(taddr + c, t16);
                ptx::tmem_wait_ld16(t16);
#pragma unroll
                for (int j = 0; j < 16; ++j) v[c + j] = __uint_as_float(t16[j]);
            }
            // accumulator read: hand it back to the MMA issuer
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(tempty_bar(acc));
            if (++acc == 2u) { acc = 0; acc_phase ^= 1u; }

            if (kb0 > 0) {
                // a piece after a tile's first k-block (its CTA's first piece): publish this
                // warp's partial for the CTA that finishes the tile
                float *mine = sg_slot<C>(p, cta, q);
#pragma unroll
                for (int i = 0; i < C::NM; ++i) __stcg(mine + i * 32 + lane, v[i]);
                ptx::fence_acq_rel_gpu();       // this lane's partial before the warp's flag
                __syncwarp();
                if (lane == 0) ptx::st_release_gpu(p.flags + cta * 4 + q, 1u);
                if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 32, tile, kb1);
                continue;
            }
            if (kb1 < p.num_kb) {
                // this CTA holds the tile's first k-block and finishes it: wait for the other
                // pieces (the first pieces of CTAs cta + 1 .. c_hi), then add them in order
                const int c_hi = r.owner((int64_t)tile * p.num_kb + p.num_kb - 1);
                ok = wait_flags_warp(p.flags + (cta + 1) * 4 + q, 4, c_hi - cta, lane, abort_flag, p.status);
                if (!ok) break;
                if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 30, tile, c_hi - cta);
#pragma unroll
                for (int i0 = 0; i0 < C::NM; i0 += 16) {
                    for (int cc0 = cta + 1; cc0 <= c_hi; cc0 += C::PB) {
                        float buf[C::PB][16];
#pragma unroll
                        for (int j = 0; j < C::PB; ++j) {
                            if (cc0 + j <= c_hi) {
                                const float *src = sg_slot<C>(p, cc0 + j, q) + i0 * 32 + lane;
#pragma unroll
                                for (int ii = 0; ii < 16; ++ii) buf[j][ii] = __ldcg(src + ii * 32);
                            }
                        }
#pragma unroll
                        for (int j = 0; j < C::PB; ++j) {
                            if (cc0 + j <= c_hi) {
#pragma unroll
                                for (int ii = 0; ii < 16; ++ii) v[i0 + ii] += buf[j][ii];
                            }
                        }
                    }
                }
                if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 31, tile, kb1);
                // the partials have been read: clear their flags for the next launch
                __syncwarp();
                if (lane == 0)
                    for (int cc = cta + 1; cc <= c_hi; ++cc) p.flags[cc * 4 + q] = 0u;
            }

            // fused epilogue for output column `col`, rows 0..m-1
            // every word of the mask pitch belongs to exactly one warp of one tile; columns at
            // or past n contribute 0 bits, so padding words come out 0
            const int64_t word = (n0 + 32 * q) / 32;
#pragma unroll
            for (int i = 0; i < C::NM; ++i) {
                if (i < p.m) {
                    float x = v[i];
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
            if (warp == 2 && lane == 0) trace_stage(p.trace, 2, tr_i, 27, tile, kb1);
        }
        if constexpr (C::QOUT) {
            const unsigned int wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_l));
            if (ok && lane == 0 && p.amax != nullptr) atomicMax(p.amax, wmax);
        }
    }

    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc<1>(tmem_base, C::TMEM_COLS);
        if (lane == 0) trace_stage(p.trace, 3, tr_i, 29, 0, cta);
    }
}

}  // namespace gemm_epi
