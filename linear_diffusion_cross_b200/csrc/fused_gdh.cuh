// fused_gdh.cuh -- sweep 2 fused with the dH GEMM on CTA pairs (sm_100a): the
// gradient tile G is formed in shared memory and consumed there, as the A
// operand of the dH tensor-core MMAs, instead of making a round trip through
// HBM.
//
// The page "fused_linear_diffusion_cross_entropy.py" writes the logit
// gradient over the logits (cross_entropy_kernel steps 5-6) and then runs
// dx = dlogits @ weight on it (the chunk loop of
// fused_linear_cross_entropy_forward).  Here, per unit of the persistent
// walk (a 256-token x 256-vocabulary tile of the token chunk):
//   1. S = H W^T over K = D: tcgen05.mma.cta_group::2 (M = N = 256) into TMEM
//      columns [0, 256), both operands K-major, streamed by TMA;
//   2. the epilogue warps turn S into G (bf16) exactly as sweep 2 does and
//      write it into shared memory in the 128B-swizzled K-major layout of a
//      UMMA A operand: CTA r keeps its 128 token rows x 256 vocabulary
//      columns as four 64-column blocks (64 KB).  The same tile is stored to
//      HBM by TMA for the dW GEMM, which needs G transposed across the pair;
//   3. dH[tile rows, :] += G W[tile columns, :] in chunks of 128 d columns:
//      M = 256, N = 128, K = 256 vocabulary rows, A = G from shared memory,
//      B = W read MN-major.  Two 128-column TMEM accumulators alternate, so
//      the epilogue flushes chunk j (fp32 TMA reduce-add into a dH
//      accumulator) while the MMAs of chunk j + 1 run.  Each epilogue warp
//      stages a whole chunk (four 32 x 32 fp32 boxes) before one proxy fence
//      and one bulk group of four reduce-adds.
// No dH accumulator fits on chip across the whole vocabulary (a 256 x D fp32
// row block is 2.6 MB at D = 2560, TMEM holds 512 KB per pair), so each
// unit's dH partial is flushed: 256 x D x 4 bytes of reduce-add traffic per
// 2 x 256 x 256 x D flop, 128 flop per byte.  This kernel exists to measure
// that trade against the staged G of sweep 2 + the dH GEMM.
//
// Roles as in umma_gemm.cuh (192 threads per CTA): warp 0 TMA producer,
// warp 1 MMA issuer (leader CTA), warps 2..5 epilogue.  Every wait is bounded;
// no load uses cluster multicast.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace fldce {

struct FusedGdhCfg {
    static constexpr int STAGES = 3;
    static constexpr int BM = 128;                 // token rows per CTA
    static constexpr int PAIR_M = 256;
    static constexpr int BN = 256;                 // vocabulary columns of a unit
    static constexpr int BK = 64;
    static constexpr int DH_N = 128;               // d columns of one dH chunk
    static constexpr uint32_t A_BYTES = BM * BK * 2;            // H box, 16 KB
    static constexpr uint32_t B_BYTES = 128 * BK * 2;           // W box, 16 KB
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;  // sweep stage
    static constexpr uint32_t DH_STAGE_BYTES = 64 * BK * 2;     // W [64 vocab][64 d], 8 KB
    static constexpr uint32_t G_BLOCK_BYTES = BM * 64 * 2;      // 64 vocabulary columns
    static constexpr uint32_t G_BYTES = 4 * G_BLOCK_BYTES;      // 64 KB
    static constexpr uint32_t EPI_BUF_BYTES = 32 * 128;         // one 32 x 32 fp32 box
    static constexpr uint32_t EPI_WARP_BYTES = (DH_N / 32) * EPI_BUF_BYTES;   // a whole chunk
    static constexpr uint32_t EPI_BYTES = 4 * EPI_WARP_BYTES;
    static constexpr uint32_t BAR_BYTES = 256;
    static constexpr uint32_t SMEM_BYTES =
        1024 + STAGES * STAGE_BYTES + G_BYTES + EPI_BYTES + BAR_BYTES;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_S = 0;            // S accumulator, 256 columns
    static constexpr uint32_t TM_DH = 256;         // dH buffers at 256 + 128 b
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(PAIR_M, BN, false, false);
    static constexpr uint32_t IDESC_DH = idesc_bf16_f32(PAIR_M, DH_N, false, true);
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(TM_DH + 2 * DH_N == TMEM_COLS, "accumulators fill TMEM");
};

// Pack 32 fp32 values as bf16 and write them as columns [32 j, 32 j + 32) of
// row `row` of the G tile: block j / 2, 16-byte chunks 4 (j & 1) .. + 3,
// chunk c of a row at ((c ^ (row & 7)) << 4) -- the 128-byte swizzle of the
// K-major operand layout (and of the TMA store boxes).
__device__ __forceinline__ void put_g_row(uint32_t gbase, int row, int j, const float (&g)[32]) {
    uint4 v[4];
    pack16(g, v[0], v[1]);
    pack16(g + 16, v[2], v[3]);
    const uint32_t line = gbase + (uint32_t)(j >> 1) * FusedGdhCfg::G_BLOCK_BYTES + (uint32_t)row * 128u;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int chunk = (j & 1) * 4 + c;
        st_shared_v4(line + (uint32_t)((chunk ^ (row & 7)) << 4), v[c]);
    }
}

template <class Cfg>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
fused_gdh_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ CUtensorMap tmWmn,
                 const __grid_constant__ CUtensorMap tmDh, const GemmGeom geom, const int d_chunks,
                 const int64_t D, const __grid_constant__ GEpi::Params gp, int32_t* err) {
    constexpr int S = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* g_smem = smem + S * Cfg::STAGE_BYTES;
    uint8_t* epi_smem = g_smem + Cfg::G_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi_smem + Cfg::EPI_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t pair = cluster_id_x();
    const uint32_t npairs = cluster_count_x();
    const uint32_t sbase = smem_u32(smem);
    const uint32_t gbase = smem_u32(g_smem);
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
    const uint32_t s_full = smem_u32(bars + 2 * S);        // S accumulator ready
    const uint32_t g_ready = smem_u32(bars + 2 * S + 1);   // G in shared memory, S drained
    const uint32_t g_free = smem_u32(bars + 2 * S + 2);    // dH MMAs done reading G
    auto dh_full = [&](int b) { return smem_u32(bars + 2 * S + 3 + b); };
    auto dh_empty = [&](int b) { return smem_u32(bars + 2 * S + 5 + b); };
    const uint32_t drain_bar = smem_u32(bars + 2 * S + 7);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(s_full, 1);
        mbar_init(g_ready, 8);                 // 4 epilogue warps x 2 CTAs
        mbar_init(g_free, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(dh_full(b), 1);
            mbar_init(dh_empty(b), 8);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmWmn);
        tma_prefetch_desc(&tmDh);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int units = geom.num_tiles;
    const int kps = geom.k_iters;
    auto fail = [&]() {
        *abort_flag = 1;
        if (lane == 0) atomicOr(err, FLDCE_DEV_ERR_TIMEOUT);
    };

    uint32_t loads_issued = 0;
    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        const uint64_t pol = l2_policy_evict_normal();
        const uint32_t lead_full0 = mapa_shared(full_bar(0), 0);
        uint32_t& it = loads_issued;
        bool ok = true;
        // wait for a free stage; false on time-out
        auto next_stage = [&](int& s) {
            s = (int)(it % S);
            const uint32_t ph = (it / S) & 1u;
            if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, kWaitLimitNs)) {
                fail();
                return false;
            }
            return true;
        };
        for (int u = pair; ok && u < units && !*abort_flag; u += npairs) {
            int mt, nt, split, k0, k1;
            walk_unit(geom, kps, u, mt, nt, split, k0, k1);
            const int arow = mt * Cfg::PAIR_M + (int)rank * Cfg::BM;
            const int brow = nt * Cfg::BN + (int)rank * 128;
            // S = H W^T: this CTA's 128 rows of H and of the W tile
            for (int k = 0; ok && k < geom.k_iters; ++k, ++it) {
                int s;
                if (!(ok = next_stage(s))) break;
                if (lane == 0) {
                    const uint32_t sa = sbase + s * Cfg::STAGE_BYTES;
                    const uint32_t fb = lead_full0 + 8u * (uint32_t)s;
                    if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2 * Cfg::STAGE_BYTES);
                    tma_load_2d_pair(sa, &tmH, fb, k * Cfg::BK, arow, pol);
                    tma_load_2d_pair(sa + Cfg::A_BYTES, &tmW, fb, k * Cfg::BK, brow, pol);
                }
                __syncwarp();
            }
            // dH: W [64 vocabulary rows][64 d columns] MN-major boxes; CTA r
            // holds d columns [128 j + 64 r, 128 j + 64 r + 64) of chunk j
            for (int j = 0; ok && j < d_chunks; ++j) {
                for (int kk = 0; kk < Cfg::BN / Cfg::BK; ++kk, ++it) {
                    int s;
                    if (!(ok = next_stage(s))) break;
                    if (lane == 0) {
                        const uint32_t sa = sbase + s * Cfg::STAGE_BYTES;
                        const uint32_t fb = lead_full0 + 8u * (uint32_t)s;
                        if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2 * Cfg::DH_STAGE_BYTES);
                        tma_load_2d_pair(sa, &tmWmn, fb, j * Cfg::DH_N + (int)rank * 64,
                                         nt * Cfg::BN + kk * Cfg::BK, pol);
                    }
                    __syncwarp();
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader)
        if (rank == 0) {
            uint32_t it = 0, c = 0, lt = 0;
            bool ok = true;
            auto take_stage = [&](int& s) {
                s = (int)(it % S);
                const uint32_t ph = (it / S) & 1u;
                if (!mbar_wait_bounded(full_bar(s), ph, kWaitLimitNs)) {
                    fail();
                    return false;
                }
                tc_fence_after();
                return true;
            };
            for (int u = pair; ok && u < units && !*abort_flag; u += npairs, ++lt) {
                for (int k = 0; k < geom.k_iters; ++k, ++it) {
                    int s;
                    if (!(ok = take_stage(s))) break;
                    if (lane == 0) {
                        const uint32_t sa = sbase + s * Cfg::STAGE_BYTES;
                        const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < Cfg::BK / 16; ++kk)
                            tc_mma_f16_pair(tmem_base + Cfg::TM_S,
                                            smem_desc_sw128(sa + kk * 32, 16, 1024),
                                            smem_desc_sw128(sb + kk * 32, 16, 1024), Cfg::IDESC_S,
                                            (k > 0 || kk > 0) ? 1u : 0u);
                        tc_commit_pair_mc(empty_bar(s), 0x3);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) tc_commit_pair_mc(s_full, 0x3);
                __syncwarp();
                // G of this unit is in both CTAs' shared memory, S is drained
                if (!mbar_wait_bounded(g_ready, lt & 1u, kWaitLimitNs)) {
                    fail();
                    break;
                }
                tc_fence_after();
                for (int j = 0; ok && j < d_chunks; ++j, ++c) {
                    const int b = (int)(c & 1u);
                    const uint32_t use = c >> 1;
                    if (!mbar_wait_bounded(dh_empty(b), (use & 1u) ^ 1u, kWaitLimitNs)) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int kk = 0; kk < Cfg::BN / Cfg::BK; ++kk, ++it) {
                        int s;
                        if (!(ok = take_stage(s))) break;
                        if (lane == 0) {
                            const uint32_t sb = sbase + s * Cfg::STAGE_BYTES;
#pragma unroll
                            for (int k16 = 0; k16 < Cfg::BK / 16; ++k16)
                                tc_mma_f16_pair(
                                    tmem_base + Cfg::TM_DH + (uint32_t)(Cfg::DH_N * b),
                                    smem_desc_sw128(gbase + kk * Cfg::G_BLOCK_BYTES + k16 * 32, 16,
                                                    1024),
                                    smem_desc_sw128(sb + k16 * 2048, 8192, 1024), Cfg::IDESC_DH,
                                    (kk > 0 || k16 > 0) ? 1u : 0u);
                            tc_commit_pair_mc(empty_bar(s), 0x3);
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    if (lane == 0) tc_commit_pair_mc(dh_full(b), 0x3);
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) tc_commit_pair_mc(g_free, 0x3);
                __syncwarp();
            }
        }
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int row = q * 32 + lane;
        // this warp's four staging boxes, 128B-swizzled like the store maps
        const uint32_t stage0 = smem_u32(epi_smem) + (uint32_t)q * Cfg::EPI_WARP_BYTES;
        auto put_box = [&](int sub, const uint32_t (&r)[32]) {
            const uint32_t line = stage0 + (uint32_t)sub * Cfg::EPI_BUF_BYTES + (uint32_t)lane * 128u;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                st_shared_v4(line + (uint32_t)((cc ^ (lane & 7)) << 4),
                             make_uint4(r[4 * cc], r[4 * cc + 1], r[4 * cc + 2], r[4 * cc + 3]));
        };
        const uint32_t lead_gready = mapa_shared(g_ready, 0);
        const uint32_t lead_dhe0 = mapa_shared(dh_empty(0), 0);
        const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16);
        uint32_t c = 0, lt = 0;
        bool ok = true;
        for (int u = pair; ok && u < units && !*abort_flag; u += npairs, ++lt) {
            int mt, nt, split, k0, k1;
            walk_unit(geom, kps, u, mt, nt, split, k0, k1);
            const int row0 = mt * Cfg::PAIR_M + (int)rank * Cfg::BM;
            const int64_t n0 = (int64_t)nt * Cfg::BN;
            const bool rows_live = row0 + 32 * q < gp.rows;     // this warp's 32 rows
            if (!mbar_wait_bounded(s_full, lt & 1u, kWaitLimitNs) ||
                !mbar_wait_bounded(g_free, (lt & 1u) ^ 1u, kWaitLimitNs)) {
                fail();
                break;
            }
            tc_fence_after();
            if (lane == 0) bulk_wait_group_read<0>();   // the last G store has read the tile
            __syncwarp();
            // S -> G -> shared memory, 32 columns at a time, the next TMEM load
            // in flight while the current chunk is processed
            const GEpi::Row w = GEpi::row_setup<Cfg::BN>(gp, row0 + row, -1, n0);
            {
                uint32_t ra[32], rb[32];
                tmem_ld_32x32b_x32(trow + Cfg::TM_S, ra);
                tmem_ld_wait_regs(ra);
#pragma unroll 1
                for (int j = 0; j < Cfg::BN / 32; j += 2) {
                    tmem_ld_32x32b_x32(trow + Cfg::TM_S + 32u * (j + 1), rb);
                    float g[32];
                    GEpi::chunk(gp, w, ra, n0, j, g);
                    put_g_row(gbase, row, j, g);
                    tmem_ld_wait_regs(rb);
                    if (j + 2 < Cfg::BN / 32) tmem_ld_32x32b_x32(trow + Cfg::TM_S + 32u * (j + 2), ra);
                    GEpi::chunk(gp, w, rb, n0, j + 1, g);
                    put_g_row(gbase, row, j + 1, g);
                    if (j + 2 < Cfg::BN / 32) tmem_ld_wait_regs(ra);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_cluster(lead_gready);
                // the same tile to HBM for the dW GEMM: this warp's 32 rows
                if (rows_live) {
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (n0 + 64 * b < gp.V)
                            tma_store_2d_hint(&gp.gmap, gbase + b * Cfg::G_BLOCK_BYTES + q * 4096u,
                                              (int)(n0 + 64 * b), row0 + 32 * q,
                                              l2_policy_evict_first());
                    bulk_commit_group();
                }
            }
            __syncwarp();
            // dH chunks: TMEM -> staging -> fp32 reduce-add
            for (int j = 0; j < d_chunks; ++j, ++c) {
                const int b = (int)(c & 1u);
                const uint32_t use = c >> 1;
                if (!mbar_wait_bounded(dh_full(b), use & 1u, kWaitLimitNs)) {
                    fail();
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tcol = trow + Cfg::TM_DH + (uint32_t)(Cfg::DH_N * b);
                // the previous chunk's reduce-adds (and the G stores) have read
                // their shared-memory sources
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
                uint32_t ra[32], rb[32];
                tmem_ld_32x32b_x32(tcol, ra);
                tmem_ld_wait_regs(ra);
#pragma unroll 1
                for (int sub = 0; sub < Cfg::DH_N / 32; sub += 2) {
                    tmem_ld_32x32b_x32(tcol + 32u * (sub + 1), rb);
                    put_box(sub, ra);
                    tmem_ld_wait_regs(rb);
                    const bool more = sub + 2 < Cfg::DH_N / 32;
                    if (more) tmem_ld_32x32b_x32(tcol + 32u * (sub + 2), ra);
                    else {
                        // every column of the buffer is in registers: hand it back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(lead_dhe0 + 8u * (uint32_t)b);
                    }
                    put_box(sub + 1, rb);
                    if (more) tmem_ld_wait_regs(ra);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && rows_live) {
#pragma unroll
                    for (int sub = 0; sub < Cfg::DH_N / 32; ++sub) {
                        const int x = j * Cfg::DH_N + 32 * sub;
                        if (x < D)
                            tma_reduce_add_2d(&tmDh, stage0 + (uint32_t)sub * Cfg::EPI_BUF_BYTES, x,
                                              row0 + 32 * q);
                    }
                    bulk_commit_group();
                }
                __syncwarp();
            }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // as in umma_gemm_kernel: let the MMAs and loads already issued finish
        // (bounded) before TMEM is freed and the CTAs exit
        if (rank == 0 && warp == 1 && lane == 0) {
            tc_commit_pair_mc(drain_bar, 0x1);
            mbar_wait_bounded(drain_bar, 0u, kWaitLimitNs);
        }
        if (rank == 0 && warp == 0 && lane == 0) {
            const uint32_t first = loads_issued > (uint32_t)S ? loads_issued - S : 0u;
            for (uint32_t i = first; i < loads_issued; ++i)
                mbar_wait_bounded(full_bar((int)(i % S)), (i / S) & 1u, kWaitLimitNs);
        }
        __syncwarp();
        tc_fence_before();
        __syncthreads();
    }
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace fldce
