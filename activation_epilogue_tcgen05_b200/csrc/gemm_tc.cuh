// gemm_tc.cuh -- persistent, warp-specialised tcgen05 GEMM with the bias /
// ReLU / GELU / sign-mask / FP8-scale epilogue fused in.
//
//   D = act(alpha * A.B + bias),   aux bit = (alpha * A.B + bias) > 0
//
// The fused epilogue follows "PyTorch inference: cuBLASLt bias fusion
// optimization" (blog.hotdry.top), paragraph 2 (bias -- and GELU -- applied in
// the GEMM kernel itself, no separate add kernel, no write-back of the
// intermediate) and "nvmath-python epilog bias fusion parameters"
// (blog.hotdry.top), body paragraphs 2-3 (BIAS / RELU_BIAS / RELU_AUX_BIAS,
// the ReLU input's sign mask, length-m bias added to every column).  The FP8
// scale is the epilogue "scaling factor" of "PyTorch 2.14 NVGEMM epilogue
// fusion" (zdabc.icu), section "why epilogue fusion matters".  The kernel
// design is this library's own, for sm_100a.
//
// Roles (one CTA per SM, or one CTA pair per two SMs when CG == 2):
//   warp 0      TMA producer: streams A and B k-blocks into a STAGES-deep
//               ring of 128-byte-swizzled shared-memory stages.
//   warp 1      TMEM allocator and MMA issuer: one thread issues
//               tcgen05.mma (M = 128*CG, N = BN, K = 32 bytes per step) into
//               one of two fp32 accumulators in tensor memory; tcgen05.commit
//               frees ring stages and publishes finished accumulators.
//   warps 2..    epilogue (8 warps, two per TMEM lane quadrant; 4 for the ReLU
//               backward): tcgen05.ld 32 lanes x 32 columns at a time, then
//               scale, bias, activation, sign-mask bits, RNE cast, 64-byte
//               swizzled staging in shared memory and 32 x 32 TMA stores of D;
//               the mask goes out as 16-byte vector stores.  With two
//               accumulators the epilogue of tile t overlaps the mainloop of
//               tile t+1.  Variants: an e4m3 output (QOUT) written with direct
//               16-byte stores plus an amax reduction; the ReLU backward
//               (EPI_DRELU) reading the mask and writing bias-gradient partials;
//               A stored (k, m) (A_MN) loaded as MN-major boxes.
//
// Split tail (stream-K style): when the tiles do not divide evenly over the
// units (CTAs, or CTA pairs), the first sk_tiles tiles are not given out
// whole.  Tile i is cut along k into sk_split equal parts handled by units
// i*sk_split + j as their first piece of work.  Parts j < sk_split-1 write their
// fp32 partial tile to the unit's workspace slot and raise one flag per
// epilogue warp; the last part's unit waits (bounded) for those flags, adds the
// partials in part order, clears the flags and runs the epilogue.  All parts
// start together and waiters only wait on lower-indexed units.  Because every
// flag is cleared by its one reader, a launch leaves the flags as it found
// them (all zero), so launches can be replayed (CUDA graphs).
//
// Every wait is bounded: after TIMEOUT_NS without progress the waiting thread
// records a code in the caller's status word, raises a CTA-wide abort flag and
// every role winds down (waiting, again bounded, for its own copies and MMAs
// in flight) so that tensor memory is always released and the kernel returns.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "ptx.cuh"

namespace gemm_epi {

enum : int { DT_F16 = 0, DT_BF16 = 1, DT_E4M3 = 2 };
// Kernel epilogues (activation after alpha*A.B + bias).  A bias pointer of
// NULL means no bias: the bias-free public epilogues run these same kernels.
// EPI_DRELU is the ReLU backward: D = mask ? alpha*A.B : 0 with the mask read
// from aux, plus (when TcParams::dbias_ws is set) per-part bias-gradient sums.
enum : int { EPI_NONE = 0, EPI_BIAS = 1, EPI_RELU = 2, EPI_RELU_AUX = 3, EPI_GELU = 4, EPI_TANH = 5,
             EPI_DRELU = 6 };
enum : int { AXIS_ROW = 0, AXIS_COL = 1 };


// Status-word bits written by kernels that gave up waiting.
enum : unsigned int {
    ST_TIMEOUT_PRODUCER = 1u << 0,
    ST_TIMEOUT_MMA = 1u << 1,
    ST_TIMEOUT_EPILOGUE = 1u << 2,
    ST_TIMEOUT_DRAIN = 1u << 3,
    ST_TIMEOUT_SPLITK = 1u << 4,
};

constexpr uint64_t TIMEOUT_NS = 1000000000ull;    // 1 s without progress on one wait
constexpr uint64_t DRAIN_TIMEOUT_NS = 100000000ull;  // 100 ms for the wind-down waits

struct TcParams {
    int m, n, k;
    int tiles_m, tiles_n, num_tiles, num_kb;
    int group_m;                 // tile raster: groups of group_m tile-rows walked column by column,
    int group_n;                 // or (group_n > 0) groups of group_n tile-columns walked row by row
    const void *bias;            // length m (ROW) or n (COL), output type
    uint32_t *aux;               // RELU_AUX: mask written; DRELU: mask read
    int64_t aux_pitch_words;     // ceil(n/128)*4
    const float *scale_a;        // alpha = *scale_a * *scale_b when set (always for E4M3)
    const float *scale_b;
    unsigned int *status;        // device status word
    int inject_stall;            // testing only: 1 = the MMA issuer publishes no accumulator
    int sk_tiles;                // tiles [0, sk_tiles) are split along k over units
    int sk_split;                // parts per split tile (units per split tile)
    float *workspace;            // partial tiles, 128 x BN fp32 per (unit, cta rank); see ws_chunk()
    unsigned int *flags;         // [unit][cta rank][4 epilogue warps]: 1 while a partial is unread
    unsigned long long *trace;   // timeline records; used only by builds with GEMM_EPI_TRACE=1
    // DRELU with a bias gradient: fp32 partial sums of D, written once each per launch.
    //   ROW: [n-part = column / BN][row]      (m floats per part, ceil(n/BN) parts)
    //   COL: [m-part = row / 32][column]      (n floats per part, ceil(m/32) parts)
    float *dbias_ws;
    // FP8 output (QOUT kernels): D = e4m3(y / *out_scale), stored m x n bytes; amax (optional)
    // receives max |y| over the launch as float bits (an atomic max: order-independent)
    uint8_t *dq;
    const float *out_scale;
    unsigned int *amax;
    int prefetch;                // producer: L2 prefetch of the stage this many stages ahead (0: none)
    // 1: tmA / tmB are 3-D / 4-D views that land a whole ring stage of an operand (all its
    // k-atoms and 128-byte boxes) with one copy; 0: 2-D maps, one copy per box
    int fused;
    // L2 cache policy: 0 = normal for every access; 1 = the outputs (D, mask) are written
    // evict-first, so that streaming them out does not push the operands out of L2; 2 = as 1,
    // and the operands are loaded evict-last
    int l2_mode;
};

// Timeline tracing (off unless the library is compiled with -DGEMM_EPI_TRACE=1 or 2).
// Level 1: each record is two 64-bit words, %globaltimer and (cta << 40 | warp << 32 |
// event << 24 | tile << 8 | k-block), appended at trace[2 + 2*i] with i from an
// atomic counter in trace[0].
// Level 2 (per ring stage, no atomics): each launch gets its own slot of TRACE_LAUNCH_RECS
// records (the host rotates over TRACE_CAP / TRACE_LAUNCH_RECS slots and passes the slot's
// base); in it every (CTA, role) owns TRACE_ROLE_CAP records at
// base[2 * ((cta * 4 + role) * TRACE_ROLE_CAP + i)], i counted by the caller; a record is
// %globaltimer and (clock low 32 bits << 32 | event << 24 | tile & 0xFF << 16 | kb & 0xFFFF).
// The SM clock orders one CTA's roles exactly; %globaltimer relates CTAs.
#ifndef GEMM_EPI_TRACE
#define GEMM_EPI_TRACE 0
#endif
constexpr unsigned int TRACE_CAP = 1u << 22;
constexpr unsigned int TRACE_ROLE_CAP = 256;
constexpr unsigned int TRACE_LAUNCH_RECS = 256u * 4u * TRACE_ROLE_CAP;   // up to 256 CTAs a launch
__device__ __forceinline__ void trace_stage(unsigned long long *trace, int role, uint32_t &i, unsigned int ev,
                                            int tile, int kb) {
    if constexpr (GEMM_EPI_TRACE == 2) {
        if (trace == nullptr || i >= TRACE_ROLE_CAP || (blockIdx.x * 4u + role + 1u) * TRACE_ROLE_CAP > TRACE_LAUNCH_RECS)
            return;
        unsigned long long *r = trace + 2 * ((size_t)(blockIdx.x * 4u + role) * TRACE_ROLE_CAP + i);
        uint32_t clk;
        asm volatile("mov.u32 %0, %%clock;" : "=r"(clk));
        r[0] = ptx::globaltimer();
        r[1] = ((unsigned long long)clk << 32) | ((unsigned long long)(ev & 0xFFu) << 24) |
               ((unsigned long long)(tile & 0xFF) << 16) | (unsigned long long)(kb & 0xFFFF);
        ++i;
    } else {
        (void)trace; (void)role; (void)i; (void)ev; (void)tile; (void)kb;
    }
}
__device__ __forceinline__ void trace_event(unsigned long long *trace, int warp, unsigned int ev, int tile,
                                            int kb) {
    if constexpr (GEMM_EPI_TRACE == 1) {
        if (trace == nullptr) return;
        const unsigned long long i = atomicAdd(trace, 1ull);
        if (i < TRACE_CAP) {
            trace[2 + 2 * i] = ptx::globaltimer();
            trace[3 + 2 * i] = ((unsigned long long)blockIdx.x << 40) | ((unsigned long long)warp << 32) |
                               ((unsigned long long)ev << 24) | ((unsigned long long)(tile & 0xFFFF) << 8) |
                               (unsigned long long)(kb & 0xFF);
        }
    } else {
        (void)trace; (void)warp; (void)ev; (void)tile; (void)kb;
    }
}

// Bounded mbarrier wait.  Returns false when this CTA is aborting (this wait
// timed out, or another role already raised the abort flag).
template <bool CLUSTER_SCOPE>
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             unsigned int *status, unsigned int code,
                                             uint64_t limit_ns = TIMEOUT_NS) {
    auto poll = [&]() {
        return CLUSTER_SCOPE ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
    };
    if (poll()) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (poll()) return true;
        if ((i & 15u) == 0u) {
            if (*abort_flag) return false;
            if (ptx::globaltimer() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicOr(status, code);
                return false;
            }
        }
    }
}

// Wind-down wait used after an abort: waits for this CTA's own copies or MMAs
// still in flight, ignoring the abort flag, for at most DRAIN_TIMEOUT_NS.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, unsigned int *status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 0u && ptx::globaltimer() - t0 > DRAIN_TIMEOUT_NS) {
            atomicOr(status, ST_TIMEOUT_DRAIN);
            return false;
        }
    }
}

// Bounded wait until *flag is set (a partial tile published by another unit).
__device__ __forceinline__ bool wait_flag(const unsigned int *flag, volatile int *abort_flag, unsigned int *status) {
    if (ptx::ld_acquire_gpu(flag) != 0u) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (ptx::ld_acquire_gpu(flag) != 0u) return true;
        if ((i & 15u) == 0u) {
            if (*abort_flag) return false;
            if (ptx::globaltimer() - t0 > TIMEOUT_NS) {
                *abort_flag = 1;
                atomicOr(status, ST_TIMEOUT_EPILOGUE);
                return false;
            }
        }
    }
}

// Where a thread's 32 partial sums of chunk c live in a workspace slot (128 x BN
// fp32 per unit and CTA rank).  The slot is laid out [warp q][chunk c][group
// g < 8][lane][4 floats], so the eight float4 accesses of a chunk are each one
// 512-byte contiguous run per warp (fully coalesced writes and reads).
template <int BN>
__device__ __forceinline__ float4 *ws_chunk(float *workspace, int unit, int cg, int rank, int q, int c, int lane) {
    float *slot = workspace + ((size_t)unit * cg + rank) * 128 * BN;
    return reinterpret_cast<float4 *>(slot) + ((size_t)(q * (BN / 32) + c) * 8) * 32 + lane;
}

// One unit of work: k-blocks [kb0, kb1) of one output tile.
struct WorkItem {
    int tile, kb0, kb1;
};

// The work of one unit, in processing order: its part of a split tile (if
// unit < sk_tiles * sk_split), then its data-parallel tiles sk_tiles + unit,
// + units, ...
struct WorkIter {
    WorkItem s0;
    bool has_part;
    int dp_t;
    __device__ WorkIter(const TcParams &p, int unit, int units) : has_part(false), dp_t(p.sk_tiles + unit) {
        if (unit < p.sk_tiles * p.sk_split) {
            const int tile = unit / p.sk_split, part = unit - tile * p.sk_split;
            s0 = WorkItem{tile, part * p.num_kb / p.sk_split, (part + 1) * p.num_kb / p.sk_split};
            has_part = true;
        }
        (void)units;
    }
    __device__ bool next(const TcParams &p, int units, WorkItem &w) {
        if (has_part) {
            w = s0;
            has_part = false;
            return true;
        }
        if (dp_t < p.num_tiles) {
            w = WorkItem{dp_t, 0, p.num_kb};
            dp_t += units;
            return true;
        }
        return false;
    }
};

template <int DT>
struct OutT;
template <>
struct OutT<DT_F16> {
    using type = __half;
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float load(const void *p, int64_t i) {
        return __half2float(reinterpret_cast<const __half *>(p)[i]);
    }
};
template <>
struct OutT<DT_BF16> {
    using type = __nv_bfloat16;
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    static __device__ __forceinline__ float load(const void *p, int64_t i) {
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    }
};
template <>
struct OutT<DT_E4M3> : OutT<DT_BF16> {};   // e4m3 operands -> bf16 bias and output

// 16-bit bias values -> fp32 (8 packed values from one 16-byte load).
template <int DT>
__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (DT == DT_F16) {
            __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
            float2 t = __half22float2(h);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        } else {
            __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
            float2 t = __bfloat1622float2(h);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
}

// GELU(x) = x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), exact (erf) form.
// erfc(z) for z = |x|/sqrt(2) >= 0 follows Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26:
//     erfc(z) ~= t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-z^2),  t = 1 / (1 + p z),
// with p = 0.3275911, a1..a5 = 0.254829592, -0.284496736, 1.421413741,
// -1.453152027, 1.061405429 and |error| <= 1.5e-7.  Since Phi(x) = erfc(z)/2 for
// x < 0 and 1 - erfc(z)/2 for x >= 0, both sides are one expression:
//     GELU(x) = max(x, 0) - |x| erfc(z) / 2,
// with no cancellation on the negative tail.  The halves are folded into the
// coefficients (h_i = a_i / 2), p / sqrt 2 into the reciprocal's argument, and
// exp(-z^2) = 2^(-(c |x|)^2) with c = sqrt(log2(e) / 2).  Branch-free: 10 fp32
// operations and two hardware approximations (rcp.approx, ex2.approx of the PTX ISA).
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float gelu_erf(float x) {
    const float ax = fabsf(x);
    const float t = rcp_approx(fmaf(0.3275911f * 0.70710678118654752f, ax, 1.0f));
    const float half_poly =
        t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, 0.5307027145f, -0.7265760135f), 0.7107068705f), -0.142248368f),
                 0.127414796f);
    const float s = ax * 0.84932180028801907f;
    return fmaf(-ax, half_poly * ex2_approx(-s * s), fmaxf(x, 0.0f));
}

template <int EPI>
__device__ __forceinline__ float activate(float x) {
    if constexpr (EPI == EPI_RELU || EPI == EPI_RELU_AUX) {
        return x > 0.0f ? x : 0.0f;
    } else if constexpr (EPI == EPI_GELU) {
        return gelu_erf(x);
    } else if constexpr (EPI == EPI_TANH) {
        return tanhf(x);
    } else {
        return x;
    }
}

// 128-byte k-atoms per ring stage.  A stage is turned over (loaded, multiplied, released) in
// roughly the same time whatever its size, so where one atom's A and B tiles are at most 32 KB
// per CTA a stage holds two atoms: twice the MMA work per turnover (pair 256 x 256 tiles: 64 KB
// and 1024 MMA clocks a stage, three stages).  48 KB atoms (the 512-wide pair tile, the
// single-CTA 256-wide tile) stay at one atom, keeping enough stages in flight.
constexpr int tc_katoms(int atom_bytes) { return atom_bytes <= 32768 ? 2 : 1; }

template <int DT_, int EPI_, int AXIS_, bool B_MN_, int BN_, int CG_, int STAGES_, bool QOUT_ = false,
          bool A_MN_ = false>
struct TcCfg {
    static constexpr int DT = DT_, EPI = EPI_, AXIS = AXIS_, BN = BN_, CG = CG_, STAGES = STAGES_;
    static constexpr bool B_MN = B_MN_;             // B stored (k, n): N contiguous
    static constexpr bool A_MN = A_MN_;             // A stored (k, m): M contiguous
    static constexpr int ESIZE = DT == DT_E4M3 ? 1 : 2;
    static constexpr int KIND = DT == DT_E4M3 ? 1 : 0;
    static constexpr uint32_t FMT = DT == DT_BF16 ? 1u : 0u;
    static constexpr int BM = 128;                  // output rows per CTA
    static constexpr int BK = 128 / ESIZE;          // k per stage: one 128-byte swizzle row
    static constexpr int UMMA_K = 32 / ESIZE;       // k per tcgen05.mma
    static constexpr int KSTEPS = BK / UMMA_K;      // 4
    static constexpr int BN_LOCAL = BN / CG;        // B rows (n) this CTA loads
    static constexpr int A_BYTES = BM * 128;                 // one k-atom of A (128 bytes of k a row)
    static constexpr int B_BYTES = BN_LOCAL * 128;           // one k-atom of this CTA's B rows
    static constexpr int KATOMS = tc_katoms(A_BYTES + B_BYTES);
    static constexpr int A_STAGE = KATOMS * A_BYTES, B_STAGE = KATOMS * B_BYTES;
    static constexpr int B_BOX_N = 128 / ESIZE;     // n per 128-byte MN-major box
    static constexpr int B_BOXES = B_MN ? BN_LOCAL / B_BOX_N : 1;
    // A 512-wide pair tile is two N = 256 MMAs per k-step, each writing its own 256 TMEM
    // columns; tensor memory then holds one accumulator, not two.  Each CTA's B tile is the
    // two MMAs' local halves, 128 rows each, one after the other.
    static constexpr int MMA_N = BN <= 256 ? BN : 256;      // N of one tcgen05.mma
    static constexpr int N_MMAS = BN / MMA_N;                // MMAs per k-step
    static constexpr int MMA_N_LOCAL = MMA_N / CG;           // B rows of one MMA in this CTA
    static constexpr int HALF_B_BYTES = MMA_N_LOCAL * 128;   // shared-memory bytes of those rows
    static constexpr int NUM_ACC = BN <= 256 ? 2 : 1;        // accumulators in tensor memory
    // One accumulator in two halves (a 512-wide pair tile, forward epilogues): the epilogue
    // drains columns 0-255 first and hands them back (tempty barrier 0), then 256-511 (barrier 1).
    // The next tile's MMAs start on the first half and keep each stage's shared memory until
    // the second half is free, then issue the deferred second-half MMAs in order.
    static constexpr bool SPLIT_HALVES = NUM_ACC == 1 && N_MMAS == 2;
    static constexpr int B_BOX_BYTES = B_MN ? BK * 128 : B_BYTES;
    static constexpr int A_BOX_M = 128 / ESIZE;     // m per 128-byte MN-major box
    static constexpr int A_BOXES = A_MN ? BM / A_BOX_M : 1;
    static constexpr int A_BOX_BYTES = A_MN ? BK * 128 : A_BYTES;
    // Two epilogue warps per TMEM lane quadrant (each taking half the columns): GELU and
    // tanh cost ~20 instructions an element and must keep up with the next tile's
    // mainloop, and for every epilogue the last wave's drain, which nothing overlaps, is
    // halved (a small launch gains 4.5 %; large ones are unchanged).  The ReLU backward
    // keeps one warp per quadrant (its mask words are read one 16-byte load per 128 columns).
    static constexpr bool HEAVY_EPI = EPI != EPI_DRELU;
    static constexpr bool BWD = EPI == EPI_DRELU;             // reads the mask, adds no bias
    static constexpr bool FWD_BIAS = EPI != EPI_NONE && !BWD;  // may add a bias
    // e4m3 output quantised with a per-tensor scale (the MLP block's intermediate): written
    // with direct 16-byte stores from registers, no staging
    static constexpr bool QOUT = QOUT_;
    static constexpr int EPI_WARPS = HEAVY_EPI ? 8 : 4;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr int COLS_W = BN * 4 / EPI_WARPS;       // columns of a tile one epilogue warp handles
    static constexpr int NCH_W = COLS_W / 32;                // its 32-column chunks
    static constexpr int CPG = NCH_W < 4 ? NCH_W : 4;        // chunks per mask-word group
    static_assert(NCH_W % CPG == 0 && (CPG == 2 || CPG == 4), "chunk grouping");
    static constexpr int TMEM_COLS = (NUM_ACC * BN <= 32) ? 32 : (NUM_ACC * BN <= 64) ? 64 : (NUM_ACC * BN <= 128) ? 128
                                   : (NUM_ACC * BN <= 256) ? 256 : 512;
    static constexpr int STG_BYTES = QOUT ? 0 : 32 * 64;   // per epilogue warp: 32 rows x 32 16-bit outputs
    // shared-memory layout (offsets from a 1024-byte aligned base)
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
    static constexpr int OFF_STG = OFF_B + STAGES * B_STAGE;
    static constexpr int OFF_BIAS = OFF_STG + EPI_WARPS * STG_BYTES;
    static constexpr int BIAS_FLOATS = (FWD_BIAS && AXIS == AXIS_COL) ? COLS_W : 0;
    static constexpr int OFF_BAR = OFF_BIAS + EPI_WARPS * BIAS_FLOATS * 4;
    // a full barrier per (stage, k-atom): the MMA starts on a stage's first atom while the
    // second is still landing; an empty barrier per stage; two accumulator pairs; done
    static constexpr int NUM_BARS = (KATOMS + 1) * STAGES + 4 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + alignment slack
    static_assert(BN == 128 || BN == 256 || (BN == 512 && CG == 2), "BN is 128 or 256 (512 for CTA pairs)");
    static_assert(NUM_ACC * BN <= 512, "the accumulators must fit in tensor memory");
    static_assert(!B_MN || MMA_N_LOCAL % B_BOX_N == 0, "an MMA's B half must be whole boxes");
    static_assert(B_MN == false || BN_LOCAL % B_BOX_N == 0, "MN-major B tile must be whole boxes");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(STAGES >= 2, "the ring needs two stages: one loading while one is multiplied");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "stage alignment");
    static_assert(!BWD || (EPI_WARPS == 4 && CPG == 4), "backward epilogue: one mask uint4 per chunk group");
    static_assert(!QOUT || (DT == DT_E4M3 && !BWD && EPI != EPI_RELU_AUX), "FP8 output: e4m3 forward plans");
    static_assert(!A_MN || BM % A_BOX_M == 0, "MN-major A tile must be whole boxes");
    static_assert(EPI_WARPS * NCH_W * 2048 <= STAGES * (A_STAGE + B_STAGE),
                  "the last tile's output staging fits in the operand ring");
    static_assert(KATOMS == 1 || N_MMAS == 1, "a stage-wide copy of B lands its atoms one after another");
};

// The tile's 32-column chunk that chunk cl of epilogue warp ew covers.  Two warps share each TMEM
// lane quadrant and split its columns; with SPLIT_HALVES each takes a quarter of either half,
// first-half chunks first, so the first half is read out before the second.
template <class C>
__device__ __forceinline__ int chunk_of(int ew, int cl) {
    if constexpr (C::SPLIT_HALVES) {
        constexpr int H = C::NCH_W / 2;            // chunks a warp takes from each half
        constexpr int HALF = C::MMA_N / 32;        // chunks in a half
        return cl < H ? (ew >> 2) * H + cl : HALF + (ew >> 2) * H + (cl - H);
    } else {
        return (ew >> 2) * C::NCH_W + cl;
    }
}

// Tile index -> (tile_m, tile_n) with a grouped raster.  group_n == 0: groups of group_m
// tile-rows, each walked column by column, so the group's A panels are reused by every
// column while B panels stream through; group_n > 0: groups of group_n tile-columns walked
// row by row (B panels reused, A streamed).  The plan sizes the group from the L2 capacity.
__device__ __forceinline__ void tile_coords(const TcParams &p, int t, int &tm, int &tn) {
    if (p.group_n > 0) {
        const int per_group = p.group_n * p.tiles_m;
        const int g = t / per_group;
        const int first = g * p.group_n;
        const int cols = min(p.group_n, p.tiles_n - first);
        const int r = t - g * per_group;
        tn = first + r % cols;
        tm = r / cols;
        return;
    }
    const int per_group = p.group_m * p.tiles_n;
    const int g = t / per_group;
    const int first = g * p.group_m;
    const int rows = min(p.group_m, p.tiles_m - first);
    const int r = t - g * per_group;
    tm = first + r % rows;
    tn = r / rows;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmD, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sb = ptx::smem_addr(smem);
    const uint32_t sA = sb + C::OFF_A, sB = sb + C::OFF_B, sStg = sb + C::OFF_STG;
    float *bias_smem = reinterpret_cast<float *>(smem + C::OFF_BIAS);
    const uint32_t bar0 = sb + C::OFF_BAR;
    auto full_bar = [&](int s, int at) { return bar0 + 8u * (s * C::KATOMS + at); };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::KATOMS * C::STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * ((C::KATOMS + 1) * C::STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * ((C::KATOMS + 1) * C::STAGES + 2 + a); };
    const uint32_t done_bar = bar0 + 8u * ((C::KATOMS + 1) * C::STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = ptx::warp_id();
    const int lane = ptx::lane_id();
    const uint32_t rank = C::CG == 2 ? ptx::cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = C::CG == 2 ? (blockIdx.x >> 1) : blockIdx.x;        // tile-processing unit
    const int units = C::CG == 2 ? (gridDim.x >> 1) : gridDim.x;

    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
        if constexpr (!C::QOUT) ptx::prefetch_tmap(&tmD);
        for (int s = 0; s < C::STAGES; ++s) {
            for (int at = 0; at < C::KATOMS; ++at) ptx::mbar_init(full_bar(s, at), 1);
            ptx::mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(tfull_bar(a), 1);
            ptx::mbar_init(tempty_bar(a), C::EPI_WARPS * C::CG);
        }
        ptx::mbar_init(done_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc<C::CG>(ptx::smem_addr(tmem_slot), C::TMEM_COLS);
        ptx::tmem_relinquish<C::CG>();
    }
    ptx::tc_fence_before();
    if constexpr (C::CG == 2) ptx::cluster_sync(); else __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // L2 prefetch of stage kb of the tile at (m0_, nb_): the same boxes as its loads, no
    // shared-memory destination, no barrier (only a hint to L2)
    auto prefetch_stage = [&](int m0_, int nb_, int kb_) {
        if (p.fused) {
            if constexpr (C::A_MN) ptx::tma_prefetch_l2_4d(&tmA, 0, 0, m0_ / C::A_BOX_M, kb_ * C::KATOMS);
            else ptx::tma_prefetch_l2_3d(&tmA, 0, m0_, kb_ * C::KATOMS);
#pragma unroll
            for (int h = 0; h < C::N_MMAS; ++h) {
                if constexpr (C::B_MN) ptx::tma_prefetch_l2_4d(&tmB, 0, 0, (nb_ + h * C::MMA_N) / C::B_BOX_N, kb_ * C::KATOMS);
                else ptx::tma_prefetch_l2_3d(&tmB, 0, nb_ + h * C::MMA_N, kb_ * C::KATOMS);
            }
            return;
        }
#pragma unroll
        for (int at = 0; at < C::KATOMS; ++at) {
            const int k0 = (kb_ * C::KATOMS + at) * C::BK;
            if constexpr (C::A_MN) {
#pragma unroll
                for (int b = 0; b < C::A_BOXES; ++b) ptx::tma_prefetch_l2_2d(&tmA, m0_ + b * C::A_BOX_M, k0);
            } else {
                ptx::tma_prefetch_l2_2d(&tmA, k0, m0_);
            }
            if constexpr (C::B_MN) {
                constexpr int PER_HALF = C::MMA_N_LOCAL / C::B_BOX_N;
#pragma unroll
                for (int b = 0; b < C::B_BOXES; ++b)
                    ptx::tma_prefetch_l2_2d(&tmB, nb_ + (b / PER_HALF) * C::MMA_N + (b % PER_HALF) * C::B_BOX_N, k0);
            } else {
#pragma unroll
                for (int h = 0; h < C::N_MMAS; ++h) ptx::tma_prefetch_l2_2d(&tmB, k0, nb_ + h * C::MMA_N);
            }
        }
    };
    auto origin = [&](int tile, int &m0_, int &nb_) {
        int tm, tn;
        tile_coords(p, tile, tm, tn);
        m0_ = tm * (C::BM * C::CG) + (int)rank * C::BM;
        // local B row r (MMA half h = r / MMA_N_LOCAL) holds global column
        // tn*BN + h*MMA_N + rank*MMA_N_LOCAL + r % MMA_N_LOCAL
        nb_ = tn * C::BN + (int)rank * C::MMA_N_LOCAL;
    };
    // Everything above touches only on-chip state, so under programmatic dependent launch
    // it overlaps the previous kernel's tail.  Before waiting for that kernel, the producer
    // asks L2 for the first ring's worth of this unit's operand boxes: a prefetch writes
    // nothing and brings nothing into the SM, and L2 is the point of coherence, so the loads
    // below still see every value the previous kernel stores.  No other global memory is read
    // or written before the previous kernel has completed; the next kernel may be scheduled
    // from here on.
    if (warp == 0 && lane == 0) {
        WorkIter it0(p, unit, units);
        WorkItem w0;
        if (it0.next(p, units, w0)) {
            int m0, nb;
            origin(w0.tile, m0, nb);
            const int last = min(w0.kb1, w0.kb0 + C::STAGES);
            for (int kb = w0.kb0; kb < last; ++kb) prefetch_stage(m0, nb, kb);
        }
    }
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t issued = 0, tr_i = 0;
            bool ok = true;
            const uint64_t pol_ab = p.l2_mode == 2 ? ptx::policy_evict_last() : ptx::policy_evict_normal();
            trace_stage(p.trace, 0, tr_i, 10, 0, 0);
            WorkIter it(p, unit, units);
            WorkItem w;
            while (ok && it.next(p, units, w)) {
                trace_event(p.trace, warp, 1, w.tile, w.kb0);
                int m0, nb;
                origin(w.tile, m0, nb);
                // the next work item, for prefetches that run past this one's last stage
                WorkIter peek = it;
                WorkItem w2;
                const bool has_next = peek.next(p, units, w2);
                int m0n = 0, nbn = 0;
                if (has_next) origin(w2.tile, m0n, nbn);
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!wait_bounded<false>(empty_bar(stage), phase ^ 1u, abort_flag, p.status,
                                             ST_TIMEOUT_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    trace_stage(p.trace, 0, tr_i, 20, w.tile, kb);
                    if (p.fused) {
                        // one copy per operand (per MMA half of B) for the whole stage, counted on
                        // the stage's first full barrier; the other atoms' barriers get a plain arrive
                        uint32_t fb = full_bar(stage, 0);
                        if constexpr (C::CG == 2) {
                            fb = ptx::mapa(fb, 0);
                            if (leader) {
                                ptx::mbar_arrive_expect_tx(full_bar(stage, 0), 2 * (C::A_STAGE + C::B_STAGE));
                                for (int at = 1; at < C::KATOMS; ++at) ptx::mbar_arrive(full_bar(stage, at));
                            }
                        } else {
                            ptx::mbar_arrive_expect_tx(fb, C::A_STAGE + C::B_STAGE);
                            for (int at = 1; at < C::KATOMS; ++at) ptx::mbar_arrive(full_bar(stage, at));
                        }
                        const uint32_t a_dst = sA + stage * C::A_STAGE;
                        const uint32_t b_dst = sB + stage * C::B_STAGE;
                        const int a0 = kb * C::KATOMS;          // first k-atom of the stage
                        if constexpr (C::CG == 2) {
                            if constexpr (C::A_MN) ptx::tma_load_4d_pair(a_dst, &tmA, fb, 0, 0, m0 / C::A_BOX_M, a0, pol_ab);
                            else ptx::tma_load_3d_pair(a_dst, &tmA, fb, 0, m0, a0, pol_ab);
                        } else {
                            if constexpr (C::A_MN) ptx::tma_load_4d(a_dst, &tmA, fb, 0, 0, m0 / C::A_BOX_M, a0, pol_ab);
                            else ptx::tma_load_3d(a_dst, &tmA, fb, 0, m0, a0, pol_ab);
                        }
#pragma unroll
                        for (int h = 0; h < C::N_MMAS; ++h) {
                            const uint32_t bd = b_dst + h * C::HALF_B_BYTES;
                            const int n1 = nb + h * C::MMA_N;
                            if constexpr (C::CG == 2) {
                                if constexpr (C::B_MN) ptx::tma_load_4d_pair(bd, &tmB, fb, 0, 0, n1 / C::B_BOX_N, a0, pol_ab);
                                else ptx::tma_load_3d_pair(bd, &tmB, fb, 0, n1, a0, pol_ab);
                            } else {
                                if constexpr (C::B_MN) ptx::tma_load_4d(bd, &tmB, fb, 0, 0, n1 / C::B_BOX_N, a0, pol_ab);
                                else ptx::tma_load_3d(bd, &tmB, fb, 0, n1, a0, pol_ab);
                            }
                        }
                    } else
                    for (int at = 0; at < C::KATOMS; ++at) {    // the stage's k-atoms
                    uint32_t fb = full_bar(stage, at);
                    if constexpr (C::CG == 2) {
                        fb = ptx::mapa(fb, 0);      // the pair's leader counts both CTAs' bytes
                        if (leader) ptx::mbar_arrive_expect_tx(full_bar(stage, at), 2 * (C::A_BYTES + C::B_BYTES));
                    } else {
                        ptx::mbar_arrive_expect_tx(fb, C::A_BYTES + C::B_BYTES);
                    }
                    const int k0 = (kb * C::KATOMS + at) * C::BK;
                    const uint32_t a_dst = sA + stage * C::A_STAGE + at * C::A_BYTES;
                    const uint32_t b_dst = sB + stage * C::B_STAGE + at * C::B_BYTES;
                    auto load = [&](uint32_t dst, const CUtensorMap *map, int c0, int c1) {
                        if constexpr (C::CG == 2)
                            ptx::tma_load_2d_pair(dst, map, fb, c0, c1, pol_ab);
                        else
                            ptx::tma_load_2d(dst, map, fb, c0, c1, pol_ab);
                    };
                    if constexpr (C::A_MN) {
#pragma unroll
                        for (int b = 0; b < C::A_BOXES; ++b)
                            load(a_dst + b * C::A_BOX_BYTES, &tmA, m0 + b * C::A_BOX_M, k0);
                    } else {
                        load(a_dst, &tmA, k0, m0);
                    }
                    if constexpr (C::B_MN) {
                        constexpr int PER_HALF = C::MMA_N_LOCAL / C::B_BOX_N;
#pragma unroll
                        for (int b = 0; b < C::B_BOXES; ++b)
                            load(b_dst + b * C::B_BOX_BYTES, &tmB,
                                 nb + (b / PER_HALF) * C::MMA_N + (b % PER_HALF) * C::B_BOX_N, k0);
                    } else {
#pragma unroll
                        for (int h = 0; h < C::N_MMAS; ++h)
                            load(b_dst + h * C::HALF_B_BYTES, &tmB, k0, nb + h * C::MMA_N);
                    }
                    }
                    if (p.prefetch > 0) {
                        // warm L2 for the stage p.prefetch ahead (in this work item or the next), so
                        // that its load, issued once a ring slot frees, finds the data in L2
                        const int ahead = kb + p.prefetch;
                        if (ahead < w.kb1) prefetch_stage(m0, nb, ahead);
                        else if (has_next && w2.kb0 + (ahead - w.kb1) < w2.kb1)
                            prefetch_stage(m0n, nbn, w2.kb0 + (ahead - w.kb1));
                    }
                    ++issued;
                    if (++stage == (uint32_t)C::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok && (C::CG == 1 || leader)) {
                // wind down: wait (bounded) until the loads still in flight have landed
                const uint32_t back = issued < (uint32_t)C::STAGES ? issued : (uint32_t)C::STAGES;
                for (uint32_t j = issued - back; j < issued; ++j)
                    for (int at = 0; at < C::KATOMS; ++at)
                        wait_drain(full_bar(j % C::STAGES, at), (j / C::STAGES) & 1u, p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && leader) {
            constexpr uint32_t idesc = make_idesc(C::FMT, C::A_MN, C::B_MN, 128 * C::CG, C::MMA_N);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0, tr_i = 0;
            bool ok = true;
            // with inject_stall nothing is issued or committed: the epilogue's
            // bounded wait for the first accumulator runs out (failure-path test)
            WorkIter it(p, unit, units);
            WorkItem w;
            while (ok && !p.inject_stall && it.next(p, units, w)) {
                trace_stage(p.trace, 1, tr_i, 24, w.tile, w.kb0);
                if (!wait_bounded<C::CG == 2>(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status,
                                              ST_TIMEOUT_MMA)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                trace_event(p.trace, warp, 3, w.tile, w.kb0);
                trace_stage(p.trace, 1, tr_i, 25, w.tile, w.kb0);
                const uint32_t d_tmem = tmem_base + acc * C::BN;
                // the MMAs of k-atom `at` of ring stage `st` (this tile's stage kb_) into halves [h_lo, h_hi)
                auto issue_atom = [&](uint32_t st, int kb_, int at, int h_lo, int h_hi) {
                    const uint32_t a_base = sA + st * C::A_STAGE + at * C::A_BYTES;
                    const uint32_t b_base = sB + st * C::B_STAGE + at * C::B_BYTES;
#pragma unroll
                    for (int ks = 0; ks < C::KSTEPS; ++ks) {
                        const uint64_t ad = C::A_MN ? make_sdesc(a_base + ks * C::UMMA_K * 128, C::A_BOX_BYTES, 1024)
                                                    : make_sdesc(a_base + ks * 32, 16, 1024);
#pragma unroll
                        for (int h = 0; h < C::N_MMAS; ++h) {
                            if (h < h_lo || h >= h_hi) continue;
                            const uint32_t bh = b_base + h * C::HALF_B_BYTES;
                            const uint64_t bd = C::B_MN ? make_sdesc(bh + ks * C::UMMA_K * 128, C::B_BOX_BYTES, 1024)
                                                        : make_sdesc(bh + ks * 32, 16, 1024);
                            ptx::mma<C::CG, C::KIND>(d_tmem + h * C::MMA_N, ad, bd, idesc,
                                                     (kb_ > w.kb0 || at > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                };
                auto release = [&](uint32_t st) {
                    if constexpr (C::CG == 2) ptx::mma_commit_pair_mc(empty_bar(st), 0x3);
                    else ptx::mma_commit(empty_bar(st));
                };
                // SPLIT_HALVES: is the accumulator's second half free yet?  Stages whose second-half
                // MMAs wait for it (in order; their ring slots are not released meanwhile).
                bool h1_free = !C::SPLIT_HALVES;
                uint32_t def_st[C::STAGES];
                int def_kb[C::STAGES];
                int ndef = 0;
                auto flush = [&]() {
                    for (int i = 0; i < ndef; ++i) {
#pragma unroll
                        for (int at = 0; at < C::KATOMS; ++at) issue_atom(def_st[i], def_kb[i], at, 1, 2);
                        release(def_st[i]);
                    }
                    ndef = 0;
                };
                auto h1_probe = [&]() {
                    return C::CG == 2 ? ptx::mbar_test_wait_cluster(tempty_bar(1), acc_phase ^ 1u)
                                      : ptx::mbar_test_wait(tempty_bar(1), acc_phase ^ 1u);
                };
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
#pragma unroll
                    for (int at = 0; at < C::KATOMS; ++at) {
                    if (!wait_bounded<false>(full_bar(stage, at), phase, abort_flag, p.status, ST_TIMEOUT_MMA)) {
                        ok = false;
                        break;
                    }
                    if (at == 0) trace_stage(p.trace, 1, tr_i, 22, w.tile, kb);
                    ptx::tc_fence_after();
                    issue_atom(stage, kb, at, 0, h1_free ? C::N_MMAS : 1);
                    }
                    if (!ok) break;
                    if constexpr (C::SPLIT_HALVES) {
                        if (!h1_free && h1_probe()) {
                            h1_free = true;
                            ptx::tc_fence_after();
                            flush();
                            // this stage's first half went out above; now its second half
#pragma unroll
                            for (int at = 0; at < C::KATOMS; ++at) issue_atom(stage, kb, at, 1, 2);
                            release(stage);
                        } else if (!h1_free) {
                            def_st[ndef] = stage;
                            def_kb[ndef] = kb;
                            if (++ndef == C::STAGES) {
                                // every ring slot is held: wait for the second half
                                if (!wait_bounded<C::CG == 2>(tempty_bar(1), acc_phase ^ 1u, abort_flag, p.status,
                                                              ST_TIMEOUT_MMA)) {
                                    ok = false;
                                    break;
                                }
                                ptx::tc_fence_after();
                                h1_free = true;
                                flush();
                            }
                        } else {
                            release(stage);
                        }
                    } else {
                        release(stage);
                    }
                    if (++stage == (uint32_t)C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (ok && ndef > 0) {
                    if (!wait_bounded<C::CG == 2>(tempty_bar(1), acc_phase ^ 1u, abort_flag, p.status, ST_TIMEOUT_MMA)) {
                        ok = false;
                    } else {
                        ptx::tc_fence_after();
                        flush();
                    }
                }
                if (!ok) break;
                if constexpr (C::CG == 2) ptx::mma_commit_pair_mc(tfull_bar(acc), 0x3);
                else ptx::mma_commit(tfull_bar(acc));
                trace_event(p.trace, warp, 4, w.tile, w.kb1);
                if (++acc == (uint32_t)C::NUM_ACC) { acc = 0; acc_phase ^= 1u; }
            }
            // every MMA issued by this thread has completed once done_bar flips
            if constexpr (C::CG == 2) ptx::mma_commit_pair_mc(done_bar, 0x1);
            else ptx::mma_commit(done_bar);
            wait_drain(done_bar, 0, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        using O = OutT<C::DT>;
        const int ew = warp - 2;                 // epilogue warp 0..EPI_WARPS-1
        const int q = warp & 3;                  // TMEM lane quadrant this warp may access
        const int cbase = (ew >> 2) * C::NCH_W;  // its first 32-column chunk of the tile
        const uint32_t stg = sStg + ew * C::STG_BYTES;
        float *bsm = bias_smem + ew * C::BIAS_FLOATS;
        float alpha = 1.0f;
        if (p.scale_a != nullptr) alpha = __ldg(p.scale_a) * __ldg(p.scale_b);
        const bool has_bias = p.bias != nullptr;
        const bool bgrad = C::BWD && p.dbias_ws != nullptr;   // backward: bias-gradient partials
        float inv_out = 1.0f, amax_l = 0.0f;                  // FP8 output: 1 / scale, running max |y|
        const uint64_t pol_d = p.l2_mode >= 1 ? ptx::policy_evict_first() : ptx::policy_evict_normal();
        if constexpr (C::QOUT) inv_out = 1.0f / __ldg(p.out_scale);
        uint32_t acc = 0, acc_phase = 0, tr_i = 0;
        bool ok = true;
        WorkIter it(p, unit, units);
        WorkItem w;
        while (ok && it.next(p, units, w)) {
            // the unit's last work item: its MMAs are the last to read the operand ring, so once
            // its accumulator is complete the ring can hold the output staging
            WorkIter peek = it;
            WorkItem wn;
            const bool last_item = !peek.next(p, units, wn);
            // partial_out: this unit holds a non-final slice of the tile -> publish a partial.
            // Otherwise units [c_first, unit) published the slices before ours.
            const bool partial_out = w.kb1 < p.num_kb;
            const int c_first = w.kb0 > 0 ? w.tile * p.sk_split : unit;
            int tm, tn;
            tile_coords(p, w.tile, tm, tn);
            const int m0 = tm * (C::BM * C::CG) + (int)rank * C::BM;
            const int n0 = tn * C::BN;
            const int nw = n0 + 32 * cbase;      // this warp's first output column
            const int row = m0 + 32 * q + lane;
            const bool row_ok = row < p.m;
            float rbias = 0.0f;
            if constexpr (C::FWD_BIAS && C::AXIS == AXIS_ROW) {
                if (row_ok && has_bias) rbias = O::load(p.bias, row);
            }
            // backward: this lane's mask words for columns [nw, nw + COLS_W), one uint4 per
            // 128 columns, fetched before the accumulator wait so that their latency hides
            uint4 mk0 = make_uint4(0u, 0u, 0u, 0u), mk1 = mk0;
            if constexpr (C::BWD) if (!partial_out && row_ok) {
                const int64_t w0 = nw / 32;
                const uint32_t *mrow = p.aux + (int64_t)row * p.aux_pitch_words + w0;
                if (w0 < p.aux_pitch_words) mk0 = __ldg(reinterpret_cast<const uint4 *>(mrow));
                if constexpr (C::NCH_W == 8)
                    if (w0 + 4 < p.aux_pitch_words) mk1 = __ldg(reinterpret_cast<const uint4 *>(mrow + 4));
            }
            float rsum = 0.0f;                   // backward, ROW axis: this row's sum over the tile
            if constexpr (C::BIAS_FLOATS > 0) if (!partial_out) {
                // this warp's copy of bias[nw .. nw+COLS_W) as fp32 (read once per tile)
                __syncwarp();
                // (bsm[j] holds the bias of the warp's j-th column: chunk j / 32, column j % 32)
                if (!has_bias) {
                    for (int j = lane; j < C::COLS_W; j += 32) bsm[j] = 0.0f;
                } else {
#pragma unroll
                    for (int j = lane * 8; j < C::COLS_W; j += 256) {
                        const int col = n0 + 32 * chunk_of<C>(ew, j >> 5) + (j & 31);
                        if (col + 8 <= p.n) {
                            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(
                                reinterpret_cast<const typename O::type *>(p.bias) + col));
                            float f[8];
                            unpack8<C::DT == DT_F16 ? DT_F16 : DT_BF16>(u, f);
#pragma unroll
                            for (int e = 0; e < 8; ++e) bsm[j + e] = f[e];
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) bsm[j + e] = col + e < p.n ? O::load(p.bias, col + e) : 0.0f;
                        }
                    }
                }
                __syncwarp();
            }
            if (lane == 0) trace_event(p.trace, warp, 5, w.tile, w.kb0);
            if (!wait_bounded<false>(tfull_bar(acc), acc_phase, abort_flag, p.status, ST_TIMEOUT_EPILOGUE)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            if (lane == 0) trace_event(p.trace, warp, 6, w.tile, w.kb0);
            if (lane == 0 && ew == 0) trace_stage(p.trace, 2, tr_i, 26, w.tile, w.kb0);
            // this warp's rows of each earlier slice are published by the same warp quadrant
            for (int v = c_first; ok && v < unit && !partial_out; ++v)
                ok = wait_flag(p.flags + ((size_t)v * C::CG + rank) * 4 + q, abort_flag, p.status);
            if (!ok) break;
            if (lane == 0) trace_event(p.trace, warp, 7, w.tile, c_first);
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + acc * C::BN;
            // two register buffers: the next chunk's TMEM load is in flight while this one is
            // processed (CPG is even, so a chunk's buffer is fixed by its position in its group)
            uint32_t vb[2][32];
            ptx::tmem_ld_32x32b_x32(tbase + chunk_of<C>(ew, 0) * 32, vb[0]);
#pragma unroll 1
            for (int g = 0; g < C::NCH_W / C::CPG; ++g) {    // CPG chunks share a mask store
                uint32_t words[C::CPG];
                const uint4 mk = g == 0 ? mk0 : mk1;
#pragma unroll
                for (int cc = 0; cc < C::CPG; ++cc) {          // 32 columns per chunk
                    const int cl = C::CPG * g + cc;            // chunk index within this warp
                    const int c = chunk_of<C>(ew, cl);         // chunk index within the tile
                    uint32_t(&v)[32] = vb[cc & 1];
                    ptx::tmem_wait_ld(v);                      // the only load in flight: this chunk's
                    if (cl + 1 < C::NCH_W) ptx::tmem_ld_32x32b_x32(tbase + chunk_of<C>(ew, cl + 1) * 32, vb[(cc + 1) & 1]);
                    // accumulator (or, SPLIT_HALVES, one half of it) fully read by this warp: hand
                    // it back to the MMA issuer
                    const bool last_chunk = cc == C::CPG - 1 && g == C::NCH_W / C::CPG - 1;
                    const bool half_done = C::SPLIT_HALVES && cl == C::NCH_W / 2 - 1;
                    if (last_chunk || half_done) {
                        const uint32_t tb = tempty_bar(C::SPLIT_HALVES ? (last_chunk ? 1 : 0) : (int)acc);
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (C::CG == 2) ptx::mbar_arrive_cluster(ptx::mapa(tb, 0));
                            else ptx::mbar_arrive(tb);
                        }
                    }
                    if (partial_out) {
                        // non-final slice: hand the fp32 partial to the tile's finishing unit
                        float4 *dst = ws_chunk<C::BN>(p.workspace, unit, C::CG, rank, q, c, lane);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            dst[32 * j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                      __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                        continue;
                    }
                    for (int u = c_first; u < unit; ++u) {       // earlier slices, in unit order
                        const float4 *src = ws_chunk<C::BN>(p.workspace, u, C::CG, rank, q, c, lane);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float4 f = __ldcg(src + 32 * j);
                            v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + f.x);
                            v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + f.y);
                            v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + f.z);
                            v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + f.w);
                        }
                    }
                    const int col0 = n0 + 32 * c;
                    uint32_t packed[16];
                    uint32_t bits = 0;
                    const uint32_t mbits = cc == 0 ? mk.x : cc == 1 ? mk.y : cc == 2 ? mk.z : mk.w;
                    (void)mbits;
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float x0 = __uint_as_float(v[j]), x1 = __uint_as_float(v[j + 1]);
                        x0 *= alpha;
                        x1 *= alpha;
                        if constexpr (C::FWD_BIAS) {
                            if constexpr (C::AXIS == AXIS_ROW) { x0 += rbias; x1 += rbias; }
                            else { x0 += bsm[32 * cl + j]; x1 += bsm[32 * cl + j + 1]; }
                        }
                        if constexpr (C::BWD) {
                            // ReLU backward: the gradient passes where the forward input was > 0
                            x0 = ((mbits >> j) & 1u) ? x0 : 0.0f;
                            x1 = ((mbits >> (j + 1)) & 1u) ? x1 : 0.0f;
                            if constexpr (C::AXIS == AXIS_ROW) {
                                rsum += x0;
                                rsum += x1;
                            } else {
                                v[j] = __float_as_uint(x0);
                                v[j + 1] = __float_as_uint(x1);
                            }
                        }
                        if constexpr (C::EPI == EPI_RELU_AUX) {
                            bits |= (x0 > 0.0f ? 1u : 0u) << j;
                            bits |= (x1 > 0.0f ? 1u : 0u) << (j + 1);
                        }
                        const float y0 = activate<C::EPI>(x0), y1 = activate<C::EPI>(x1);
                        if constexpr (C::QOUT) {
                            amax_l = fmaxf(amax_l, fmaxf(fabsf(y0), fabsf(y1)));
                            // two e4m3 codes, round to nearest even, saturating at +-448; y0 low byte
                            packed[j / 2] = __nv_cvt_float2_to_fp8x2(make_float2(y0 * inv_out, y1 * inv_out),
                                                                     __NV_SATFINITE, __NV_E4M3);
                        } else {
                            packed[j / 2] = O::pack(y0, y1);
                        }
                    }
                    if constexpr (C::EPI == EPI_RELU_AUX) {
                        const int valid = p.n - col0;
                        const uint32_t keep = valid >= 32 ? 0xFFFFFFFFu : (valid <= 0 ? 0u : ((1u << valid) - 1u));
                        words[cc] = bits & keep;
                    }
                    if constexpr (C::QOUT) {
                        // this lane's 32 codes are 32 contiguous bytes of its row (n is a multiple of 16)
                        if (row_ok) {
                            uint8_t *dst = p.dq + (int64_t)row * p.n + col0;
                            if (col0 + 16 <= p.n)
                                *reinterpret_cast<uint4 *>(dst) =
                                    make_uint4(packed[0] | (packed[1] << 16), packed[2] | (packed[3] << 16),
                                               packed[4] | (packed[5] << 16), packed[6] | (packed[7] << 16));
                            if (col0 + 32 <= p.n)
                                *reinterpret_cast<uint4 *>(dst + 16) =
                                    make_uint4(packed[8] | (packed[9] << 16), packed[10] | (packed[11] << 16),
                                               packed[12] | (packed[13] << 16), packed[14] | (packed[15] << 16));
                        }
                    } else {
                        // stage 32 rows x 32 outputs in the 64-byte swizzled layout the TMA store reads:
                        // 16-byte piece j of row r sits at r*64 + ((j ^ ((r >> 1) & 3)) * 16).  The
                        // unit's last tile stages every chunk in its own 2 KB of the (by then idle)
                        // operand ring, so no chunk waits for the previous one's store to be read;
                        // otherwise the warp's single staging buffer is reused.
                        uint32_t stg_c = stg;
                        uint8_t *stg_row = smem + C::OFF_STG + ew * C::STG_BYTES + lane * 64;
                        if (last_item) {
                            const int slot = ew * C::NCH_W + cl;
                            stg_c = sA + slot * 2048;
                            stg_row = smem + C::OFF_A + slot * 2048 + lane * 64;
                        } else if (lane == 0) {
                            ptx::bulk_wait_read<0>();     // previous store has read the buffer
                        }
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int piece = i ^ ((lane >> 1) & 3);
                            *reinterpret_cast<uint4 *>(stg_row + piece * 16) =
                                make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                        }
                        ptx::fence_proxy_async_smem();
                        __syncwarp();
                        // boxes starting past the last row or column hold nothing to store
                        if (lane == 0 && m0 + 32 * q < p.m && col0 < p.n) {
                            ptx::tma_store_2d_hint(&tmD, stg_c, col0, m0 + 32 * q, pol_d);
                            ptx::bulk_commit();
                        }
                    }
                    if constexpr (C::BWD && C::AXIS == AXIS_COL) if (bgrad) {
                        // column sums over this warp's 32 rows: a butterfly that halves the
                        // live values at each of 5 exchange steps (31 shuffles for 32 columns);
                        // afterwards lane l holds the sum of column col0 + l, in a fixed order
                        float f[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
#pragma unroll
                        for (int sh = 16; sh >= 1; sh >>= 1) {
                            const bool upper = (lane & sh) != 0;
#pragma unroll
                            for (int j = 0; j < sh; ++j) {
                                const float send = upper ? f[j] : f[j + sh];
                                const float keep = upper ? f[j + sh] : f[j];
                                f[j] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
                            }
                        }
                        if (m0 + 32 * q < p.m && col0 + lane < p.n)
                            p.dbias_ws[(size_t)((m0 + 32 * q) >> 5) * p.n + col0 + lane] = f[0];
                    }
                }
                if (partial_out) continue;
                if constexpr (C::EPI == EPI_RELU_AUX) {
                    const int wcol = n0 + 32 * chunk_of<C>(ew, C::CPG * g);
                    if (row_ok && wcol < p.aux_pitch_words * 32) {      // padding words too (zero bits)
                        uint32_t *dst = p.aux + (int64_t)row * p.aux_pitch_words + wcol / 32;
                        if constexpr (C::CPG == 4)
                            ptx::st_global_v4_hint(dst, make_uint4(words[0], words[1], words[2], words[3]), pol_d);
                        else
                            *reinterpret_cast<uint2 *>(dst) = make_uint2(words[0], words[1]);
                    }
                }
            }
            if constexpr (C::BWD && C::AXIS == AXIS_ROW)
                if (bgrad && !partial_out && row_ok) p.dbias_ws[(size_t)(nw / C::COLS_W) * p.m + row] = rsum;
            if (lane == 0) trace_event(p.trace, warp, 8, w.tile, partial_out ? 1 : 0);
            if (partial_out) {
                // publish: every lane's stores are ordered before the warp's flag
                __threadfence();
                __syncwarp();
                if (lane == 0) ptx::st_release_gpu(p.flags + ((size_t)unit * C::CG + rank) * 4 + q, 1u);
            } else if (lane == 0) {
                // the earlier slices have been read: clear their flags for the next launch
                for (int v = c_first; v < unit; ++v) p.flags[((size_t)v * C::CG + rank) * 4 + q] = 0u;
            }
            if (lane == 0) trace_event(p.trace, warp, 9, w.tile, 0);
            if (lane == 0 && ew == 0) trace_stage(p.trace, 2, tr_i, 27, w.tile, w.kb1);
            if (++acc == (uint32_t)C::NUM_ACC) { acc = 0; acc_phase ^= 1u; }
        }
        if (lane == 0) ptx::bulk_wait<0>();
        __syncwarp();
        if constexpr (C::QOUT) {
            // one atomic per warp: the launch's max |y| (non-negative floats order as their bits)
            const unsigned int wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_l));
            if (ok && lane == 0 && p.amax != nullptr) atomicMax(p.amax, wmax);
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    ptx::tc_fence_before();
    if constexpr (C::CG == 2) ptx::cluster_sync(); else __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc<C::CG>(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm_epi
