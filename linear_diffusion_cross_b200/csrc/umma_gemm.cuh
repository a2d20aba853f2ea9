// umma_gemm.cuh -- persistent tcgen05 GEMM for sm_100a with pluggable epilogues.
//
// D[m, n] = sum_k A[m, k] * B[n, k] over bf16 operands with an fp32
// accumulator that lives in tensor memory (TMEM).  One CTA per SM walks a
// static round-robin list of BM x BN output tiles:
//
//   warp 0      TMA producer: 128B-swizzled tiles of A and B into a
//               STAGES-deep shared-memory ring (full/empty mbarriers).
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=BN,
//               K=16) into one of two TMEM accumulators, commits the ring
//               slot back to the producer and the finished accumulator to
//               the epilogue.
//   warps 2..5  epilogue: each thread owns one accumulator row (TMEM lane),
//               reads it 32 columns at a time with tcgen05.ld and hands the
//               values to the epilogue functor; the accumulator is released
//               as soon as it is read, so the next tile's MMAs overlap the
//               current tile's epilogue.
//
// Operands may be K-major (K contiguous) or MN-major (M/N contiguous); both
// are consumed straight from their row-major HBM layout through the TMA
// tensor map, so no transposed copy of any operand is ever made.
//
// Every mbarrier wait is bounded by global time; on time-out the CTA records
// FLDCE_DEV_ERR_TIMEOUT in `err`, stops issuing work and frees its TMEM.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace fldce {

constexpr int kGemmThreads = 192;
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s per wait
constexpr int32_t FLDCE_DEV_ERR_TIMEOUT = 1;

template <int BN_, int STAGES_, bool A_MN_, bool B_MN_>
struct GemmCfg {
    static constexpr int BM = 128;
    static constexpr int BN = BN_;
    static constexpr int BK = 64;                 // one 128-byte swizzle span of bf16
    static constexpr int STAGES = STAGES_;
    static constexpr bool A_MN = A_MN_;
    static constexpr bool B_MN = B_MN_;
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulators
    static constexpr uint32_t BAR_BYTES = 256;
    static constexpr uint32_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
    static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, A_MN, B_MN);
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
    static_assert(TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns");
};

struct GemmGeom {
    int tiles_m;
    int tiles_n;
    int k_iters;          // ceil(K / 64)
    int num_tiles;
    int n_fastest;        // 1: consecutive tiles walk n first (share the A panel)
};

__device__ __forceinline__ void tile_coords(const GemmGeom& g, int tile, int& mt, int& nt) {
    if (g.n_fastest) {
        nt = tile % g.tiles_n;
        mt = tile / g.tiles_n;
    } else {
        mt = tile % g.tiles_m;
        nt = tile / g.tiles_m;
    }
}

// Per-thread view of one accumulator row handed to an epilogue functor.
struct AccRow {
    uint32_t taddr;       // TMEM address of this thread's lane, column 0 of the tile
    uint32_t tempty_bar;  // mbarrier to arrive on once every column has been read
    int lane;

    // Load columns [32*j, 32*j + 32) of the row (waits for completion).
    __device__ __forceinline__ void load(int j, uint32_t (&r)[32]) const {
        tmem_ld_32x32b_x32(taddr + (uint32_t)(32 * j), r);
        tmem_ld_wait();
    }
    // Hand the accumulator back to the MMA warp (one arrive per warp).
    __device__ __forceinline__ void release() const {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar);
    }
};

template <class Cfg, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmGeom geom, const typename Epi::Params ep, int32_t* err) {
    constexpr int S = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * Cfg::STAGE_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
    auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * S + b); };
    auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * S + 2 + b); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    auto fail = [&]() {
        *abort_flag = 1;
        if (lane == 0) atomicOr(err, FLDCE_DEV_ERR_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        const uint64_t pol = l2_policy_evict_normal();
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < geom.num_tiles && !*abort_flag; tile += gridDim.x) {
            int mt, nt;
            tile_coords(geom, tile, mt, nt);
            for (int k = 0; k < geom.k_iters; ++k, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1u;
                if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, kWaitLimitNs)) { fail(); break; }
                if (lane == 0) {
                    const uint32_t sa = sbase + s * Cfg::STAGE_BYTES;
                    const uint32_t sb = sa + Cfg::A_BYTES;
                    mbar_arrive_expect_tx(full_bar(s), Cfg::STAGE_BYTES);
                    if (Cfg::A_MN) {
#pragma unroll
                        for (int j = 0; j < Cfg::BM / 64; ++j)
                            tma_load_2d(sa + j * 8192, &tmA, full_bar(s), mt * Cfg::BM + 64 * j,
                                        k * Cfg::BK, pol);
                    } else {
                        tma_load_2d(sa, &tmA, full_bar(s), k * Cfg::BK, mt * Cfg::BM, pol);
                    }
                    if (Cfg::B_MN) {
#pragma unroll
                        for (int j = 0; j < Cfg::BN / 64; ++j)
                            tma_load_2d(sb + j * 8192, &tmB, full_bar(s), nt * Cfg::BN + 64 * j,
                                        k * Cfg::BK, pol);
                    } else {
                        tma_load_2d(sb, &tmB, full_bar(s), k * Cfg::BK, nt * Cfg::BN, pol);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        uint32_t it = 0, lt = 0;
        for (int tile = blockIdx.x; tile < geom.num_tiles && !*abort_flag;
             tile += gridDim.x, ++lt) {
            const int b = lt & 1;
            const uint32_t use = lt >> 1;
            if (!mbar_wait_bounded(tempty_bar(b), (use & 1u) ^ 1u, kWaitLimitNs)) { fail(); break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(b * Cfg::BN);
            bool ok = true;
            for (int k = 0; k < geom.k_iters; ++k, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1u;
                if (!mbar_wait_bounded(full_bar(s), ph, kWaitLimitNs)) { fail(); ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sa = sbase + s * Cfg::STAGE_BYTES;
                    const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < Cfg::BK / 16; ++kk) {
                        const uint64_t ad = Cfg::A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                                      : smem_desc_sw128(sa + kk * 32, 16, 1024);
                        const uint64_t bd = Cfg::B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                                      : smem_desc_sw128(sb + kk * 32, 16, 1024);
                        tc_mma_f16(d_tmem, ad, bd, Cfg::IDESC, (k | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(empty_bar(s));
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) tc_commit(tfull_bar(b));
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int row = q * 32 + lane;          // accumulator row owned by this thread
        uint32_t lt = 0;
        for (int tile = blockIdx.x; tile < geom.num_tiles && !*abort_flag;
             tile += gridDim.x, ++lt) {
            const int b = lt & 1;
            const uint32_t use = lt >> 1;
            if (!mbar_wait_bounded(tfull_bar(b), use & 1u, kWaitLimitNs)) { fail(); break; }
            tc_fence_after();
            int mt, nt;
            tile_coords(geom, tile, mt, nt);
            AccRow acc{tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * Cfg::BN),
                       tempty_bar(b), lane};
            Epi::template run<Cfg::BN>(ep, mt, nt, row, acc);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace fldce
