// umma_gemm.cuh -- persistent tcgen05 GEMM on CTA pairs for sm_100a, with
// pluggable epilogues.
//
// D[m, n] = sum_k A[m, k] * B[n, k] over bf16 operands with an fp32
// accumulator in tensor memory (TMEM).  Work is cut into 256 x 256 output
// tiles (256 x 512 with GemmCfg NSUB = 2), optionally also into K splits,
// and walked in a fixed order by a persistent grid of CTA pairs.  Each tile
// belongs to a cluster of two CTAs on neighbouring SMs that issue
// tcgen05.mma.cta_group::2 (M = 256, N = 256) per K step of 16: CTA r of the
// pair holds rows [128 r, 128 r + 128) of the A tile and of each 256-row B
// block in its shared memory, and receives rows [128 r, 128 r + 128) of the
// accumulator in its TMEM.  Each SM therefore streams 32 KB of operands per
// 64-wide K step instead of the 48 KB a single-CTA 128 x 256 tile needs, a
// third less L2 -> SM traffic for the same tensor work (a quarter less again
// with NSUB = 2, whose A tile feeds two MMAs).
//
// Roles (192 threads per CTA):
//   warp 0      TMA producer (both CTAs): loads this CTA's halves into a
//               STAGES-deep ring; completion is counted on the pair leader's
//               "full" mbarrier, which expects the bytes of both CTAs.
//   warp 1      MMA issuer (leader CTA only issues; both allocate TMEM):
//               waits for a full stage, issues 4 x NSUB M=256 N=256 K=16 MMAs
//               and commits the stage back to both producers (multicast
//               commit), then commits a finished accumulator to both
//               epilogues.
//   warps 2..5  epilogue (both CTAs): one accumulator row per thread, read
//               with tcgen05.ld while the next tile's MMAs run into the other
//               of the two TMEM accumulators (NSUB = 1; with NSUB = 2 the one
//               512-column accumulator is drained before the next tile
//               starts); output tiles leave through a
//               per-warp 128B-swizzled staging buffer and TMA bulk stores (or
//               bulk reduce-adds).
//
// Operands are consumed K-major or MN-major straight from row-major HBM
// through the tensor maps; no transposed copy of any operand is made.  Loads
// carry no cluster multicast.  Every mbarrier wait is bounded by global time;
// on time-out the CTA records FLDCE_DEV_ERR_TIMEOUT, stops issuing work,
// waits (bounded again) for the MMAs and loads it already issued, and frees
// its TMEM.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace fldce {

constexpr int kGemmThreads = 192;
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s per wait
constexpr int32_t FLDCE_DEV_ERR_TIMEOUT = 1;

// NSUB_ MMAs of N = 256 per K step make one tile NSUB_ x 256 columns wide.
// NSUB_ = 1: two 256-column accumulators in TMEM, so the epilogue of one tile
// overlaps the MMAs of the next.  NSUB_ = 2: one 512-column accumulator (all
// of TMEM); each A tile in shared memory feeds two MMAs, which halves the
// pipeline stages per MMA and cuts the L2 -> SM operand traffic by a quarter,
// at the price of an epilogue that no longer overlaps (worth it only where
// the K loop is long).
template <int STAGES_, bool A_MN_, bool B_MN_, int NSUB_ = 1>
struct GemmCfg {
    static constexpr int BM = 128;                 // accumulator rows per CTA
    static constexpr int PAIR_M = 256;             // rows of a pair tile
    static constexpr int NSUB = NSUB_;
    static constexpr int MMA_N = 256;              // columns of one MMA
    static constexpr int BN = MMA_N * NSUB;        // columns of a tile
    static constexpr int BN_HALF = 128 * NSUB;     // B rows held per CTA
    static constexpr int BK = 64;                  // one 128-byte swizzle span of bf16
    static constexpr int STAGES = STAGES_;
    static constexpr bool A_MN = A_MN_;
    static constexpr bool B_MN = B_MN_;
    static constexpr int NBUF = NSUB == 1 ? 2 : 1; // accumulators in TMEM
    static constexpr int NCHUNK = BN / 32;         // 32-column epilogue chunks
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BLOCK_BYTES = 128 * BK * 2;   // one MMA's B rows of this CTA
    static constexpr uint32_t B_BYTES = NSUB * B_BLOCK_BYTES;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t EPI_BUF_BYTES = 32 * 128;       // 32 rows x 128 B
    static constexpr uint32_t EPI_BYTES = 4 * 2 * EPI_BUF_BYTES;
    static constexpr uint32_t BAR_BYTES = 256;
    static constexpr uint32_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
    static constexpr uint32_t IDESC = idesc_bf16_f32(PAIR_M, MMA_N, A_MN, B_MN);
    static_assert(NSUB == 1 || NSUB == 2, "one or two MMAs per K step");
    static_assert(NBUF * BN == (int)TMEM_COLS, "accumulators fill TMEM");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

struct GemmGeom {
    int tiles_m;          // ceil(M / 256)
    int tiles_n;          // ceil(N / 256)
    int k_iters;          // ceil(K / 64)
    int k_splits;         // K ranges per tile (1 to 4)
    int num_tiles;        // tiles_m * tiles_n
    int n_fastest;        // 1: consecutive tiles walk n first (share the A panel)
    // The walk covers the fast dimension in blocks of `group` tiles: all
    // tiles of one block along the slow dimension, then the next block.  The
    // operand panels of one block stay in L2 while the other operand
    // streams past them; group >= the fast dimension's tiles is one block.
    int group;
    // Optional row count known only on the device (compacted tokens): the
    // live rows are clamp(*dyn_count - dyn_base, 0, dyn_cap), bounding M
    // (dyn_dim == 1) or K (dyn_dim == 2).  The host sizes the launch for
    // dyn_cap rows; every CTA reads the same count at start.
    const int32_t* dyn_count;
    int dyn_base;
    int dyn_cap;
    int dyn_dim;
};

// Apply the device-side row count of `g` (if any); returns the live rows or -1.
__device__ __forceinline__ int apply_dyn_rows(GemmGeom& g) {
    if (g.dyn_dim == 0) return -1;
    int n = *g.dyn_count - g.dyn_base;
    n = n < 0 ? 0 : (n > g.dyn_cap ? g.dyn_cap : n);
    if (g.dyn_dim == 1) {
        g.tiles_m = (n + 255) / 256;
        g.num_tiles = g.tiles_m * g.tiles_n;
    } else {
        g.k_iters = (n + 63) / 64;
        if (g.k_iters < 2 * g.k_splits) g.k_splits = 1;
        if (g.k_iters == 0) g.num_tiles = 0;
    }
    return n;
}

// Coordinates of unit u of the persistent walk: output tile (mt, nt), K
// split and its K-step range [k0, k1) (kps = K steps per split).  Units of
// one split cover the tiles in blocks of `group` tiles along the fast
// dimension: every tile of a block along the slow dimension, then the next
// block.
__device__ __forceinline__ void walk_unit(const GemmGeom& g, int kps, int u, int& mt, int& nt,
                                          int& split, int& k0, int& k1) {
    const int n_fast = g.n_fastest ? g.tiles_n : g.tiles_m;
    const int n_slow = g.n_fastest ? g.tiles_m : g.tiles_n;
    const int grp = max(1, min(g.group, n_fast));
    split = u / g.num_tiles;
    const int tile = u - split * g.num_tiles;
    const int blk = tile / (grp * n_slow);
    const int r = tile - blk * (grp * n_slow);
    const int f0 = blk * grp;
    const int gb = min(grp, n_fast - f0);          // the last block may be narrower
    const int f = f0 + r % gb, sl = r / gb;
    if (g.n_fastest) {
        nt = f;
        mt = sl;
    } else {
        mt = f;
        nt = sl;
    }
    k0 = split * kps;
    k1 = min(g.k_iters, k0 + kps);
}

// Where the current tile of this thread sits.
struct TileCtx {
    int rows_dyn;         // live rows from the device-side count, or -1
    int row0;             // output row of TMEM lane 0 of this CTA
    int64_t col0;         // first output column of the tile
    int split;            // K split index
    int row;              // this thread's accumulator row (TMEM lane), 0..127
    int q;                // warp quadrant: rows [32 q, 32 q + 32)
    int lane;
};

// Per-thread view of one accumulator row handed to an epilogue functor.
struct AccRow {
    uint32_t taddr;       // TMEM address of this thread's lane, column 0 of the tile
    uint32_t tempty_bar;  // leader's accumulator-empty mbarrier (cluster address)
    int lane;

    // Issue loads of columns [32 j, 32 j + 32); complete them with wait().
    __device__ __forceinline__ void issue(int j, uint32_t (&r)[32]) const {
        tmem_ld_32x32b_x32(taddr + (uint32_t)(32 * j), r);
    }
    __device__ __forceinline__ void wait(uint32_t (&r)[32]) const { tmem_ld_wait_regs(r); }
    __device__ __forceinline__ void load(int j, uint32_t (&r)[32]) const {
        issue(j, r);
        wait(r);
    }
    // Hand the accumulator back to the pair's MMA warp (one arrive per warp).
    __device__ __forceinline__ void release() const {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_bar);
    }
};

// One warp's two 32-row x 128-byte staging buffers and its TMA stores.  Row
// r's 16-byte chunk c lives at r*128 + ((c ^ (r & 7)) * 16): the 128-byte
// swizzle the store tensor maps use, which also keeps the 32 lanes' writes
// free of bank conflicts.
struct Stager {
    uint32_t buf0;
    int lane;
    int phase;

    __device__ __forceinline__ uint32_t cur() const { return buf0 + (uint32_t)phase * 4096u; }
    // Make sure the buffer about to be written is no longer read by a store.
    __device__ __forceinline__ void acquire() {
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
    }
    __device__ __forceinline__ void put(int c, uint4 v) {
        st_shared_v4(cur() + (uint32_t)lane * 128u + (uint32_t)((c ^ (lane & 7)) << 4), v);
    }
    // Store (or reduce-add) the staged 32 x 128 B box at (x, y) of `m`.
    // Stored tiles (G, dH, dW, fp32 partials) are marked evict_first in L2:
    // the kernel never reads them back, and the operand tiles it re-reads
    // from L2 stay resident longer (measured: 2.6 GB less DRAM traffic per
    // headline step, about 1% less time).
    __device__ __forceinline__ void flush(const CUtensorMap* m, int x, int y, bool add) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            if (add) tma_reduce_add_2d(m, cur(), x, y);
            else tma_store_2d_hint(m, cur(), x, y, l2_policy_evict_first());
            bulk_commit_group();
        }
        phase ^= 1;
    }
    __device__ __forceinline__ void drain() {
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }
};

template <class Cfg, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmGeom geom_in, const __grid_constant__ typename Epi::Params ep,
                 int32_t* err) {
    constexpr int S = Cfg::STAGES;
    GemmGeom geom = geom_in;
    const int rows_dyn = apply_dyn_rows(geom);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* epi_smem = smem + S * Cfg::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(epi_smem + Cfg::EPI_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0 = pair leader
    const uint32_t pair = cluster_id_x();
    const uint32_t npairs = cluster_count_x();
    const uint32_t sbase = smem_u32(smem);
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
    auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * S + b); };
    auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * S + 2 + b); };
    const uint32_t drain_bar = smem_u32(bars + 2 * S + 4);   // abort path only

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 8);       // 4 epilogue warps x 2 CTAs
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                            // the peer's barriers exist before use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int units = geom.num_tiles * geom.k_splits;
    const int kps = (geom.k_iters + geom.k_splits - 1) / geom.k_splits;

    auto fail = [&]() {
        *abort_flag = 1;
        if (lane == 0) atomicOr(err, FLDCE_DEV_ERR_TIMEOUT);
    };
    auto unit_coords = [&](int u, int& mt, int& nt, int& split, int& k0, int& k1) {
        walk_unit(geom, kps, u, mt, nt, split, k0, k1);
    };

    uint32_t loads_issued = 0;                 // producer: stages loaded so far
    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        // evict_first on the streamed operand / evict_last on the reused one
        // measured more HBM traffic than the default priority, not less
        const uint64_t pol = l2_policy_evict_normal();
        const uint32_t lead_full0 = mapa_shared(full_bar(0), 0);
        uint32_t& it = loads_issued;
        bool ok = true;
        for (int u = pair; ok && u < units && !*abort_flag; u += npairs) {
            int mt, nt, split, k0, k1;
            unit_coords(u, mt, nt, split, k0, k1);
            const int arow = mt * Cfg::PAIR_M + (int)rank * Cfg::BM;
            // this CTA's B rows for MMA j: [brow + 256 j, brow + 256 j + 128)
            const int brow = nt * Cfg::BN + (int)rank * 128;
            for (int k = k0; k < k1; ++k, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1u;
                if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, kWaitLimitNs)) {
                    fail();
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t sa = sbase + s * Cfg::STAGE_BYTES;
                    const uint32_t sb = sa + Cfg::A_BYTES;
                    const uint32_t fb = lead_full0 + 8u * (uint32_t)s;
                    if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2 * Cfg::STAGE_BYTES);
                    if (Cfg::A_MN) {
#pragma unroll
                        for (int j = 0; j < Cfg::BM / 64; ++j)
                            tma_load_2d_pair(sa + j * 8192, &tmA, fb, arow + 64 * j, k * Cfg::BK,
                                             pol);
                    } else {
                        tma_load_2d_pair(sa, &tmA, fb, k * Cfg::BK, arow, pol);
                    }
                    if (Cfg::B_MN) {
#pragma unroll
                        for (int i = 0; i < Cfg::BN_HALF / 64; ++i)   // 64-column boxes
                            tma_load_2d_pair(sb + i * 8192, &tmB, fb,
                                             brow + Cfg::MMA_N * (i >> 1) + 64 * (i & 1),
                                             k * Cfg::BK, pol);
                    } else {
#pragma unroll
                        for (int j = 0; j < Cfg::NSUB; ++j)          // 128-row boxes
                            tma_load_2d_pair(sb + j * Cfg::B_BLOCK_BYTES, &tmB, fb, k * Cfg::BK,
                                             brow + Cfg::MMA_N * j, pol);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader)
        if (rank == 0) {
            uint32_t it = 0, lt = 0;
            for (int u = pair; u < units && !*abort_flag; u += npairs, ++lt) {
                int mt, nt, split, k0, k1;
                unit_coords(u, mt, nt, split, k0, k1);
                const int b = Cfg::NBUF == 2 ? (int)(lt & 1u) : 0;
                const uint32_t use = Cfg::NBUF == 2 ? lt >> 1 : lt;
                if (!mbar_wait_bounded(tempty_bar(b), (use & 1u) ^ 1u, kWaitLimitNs)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * Cfg::BN);
                bool ok = true;
                for (int k = k0; k < k1; ++k, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (!mbar_wait_bounded(full_bar(s), ph, kWaitLimitNs)) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t sa = sbase + s * Cfg::STAGE_BYTES;
                        const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < Cfg::BK / 16; ++kk) {
                            const uint64_t ad =
                                Cfg::A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                          : smem_desc_sw128(sa + kk * 32, 16, 1024);
#pragma unroll
                            for (int j = 0; j < Cfg::NSUB; ++j) {
                                const uint32_t bj = sb + (uint32_t)j * Cfg::B_BLOCK_BYTES;
                                const uint64_t bd =
                                    Cfg::B_MN ? smem_desc_sw128(bj + kk * 2048, 8192, 1024)
                                              : smem_desc_sw128(bj + kk * 32, 16, 1024);
                                tc_mma_f16_pair(d_tmem + (uint32_t)(j * Cfg::MMA_N), ad, bd,
                                                Cfg::IDESC, (k > k0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        tc_commit_pair_mc(empty_bar(s), 0x3);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) tc_commit_pair_mc(tfull_bar(b), 0x3);
                __syncwarp();
            }
        }
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int row = q * 32 + lane;          // accumulator row owned by this thread
        Stager st{smem_u32(epi_smem) + (uint32_t)(q * 2) * Cfg::EPI_BUF_BYTES, lane, 0};
        const uint32_t lead_tempty0 = mapa_shared(tempty_bar(0), 0);
        uint32_t lt = 0;
        for (int u = pair; u < units && !*abort_flag; u += npairs, ++lt) {
            int mt, nt, split, k0, k1;
            unit_coords(u, mt, nt, split, k0, k1);
            const int b = Cfg::NBUF == 2 ? (int)(lt & 1u) : 0;
            const uint32_t use = Cfg::NBUF == 2 ? lt >> 1 : lt;
            if (!mbar_wait_bounded(tfull_bar(b), use & 1u, kWaitLimitNs)) {
                fail();
                break;
            }
            tc_fence_after();
            TileCtx t{rows_dyn, mt * Cfg::PAIR_M + (int)rank * Cfg::BM, (int64_t)nt * Cfg::BN,
                      split, row, q, lane};
            AccRow acc{tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * Cfg::BN),
                       lead_tempty0 + 8u * (uint32_t)b, lane};
            Epi::template run<Cfg>(ep, t, acc, st);
        }
        st.drain();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // A wait timed out somewhere in the pair.  Before TMEM is freed and
        // the CTAs exit, let the asynchronous work already issued finish
        // (each wait again bounded): the leader's MMA lane commits every MMA
        // it issued to a local barrier and waits for it, and the leader's
        // producer lane waits until the loads of the last S stages it issued
        // (both CTAs' bytes are counted on its barriers) have landed.  The
        // results of the call are invalid either way (FLDCE_DEV_ERR_TIMEOUT).
        if (rank == 0 && warp == 1 && lane == 0) {
            // (cta_group::2 like every tcgen05 op of this kernel; leader only)
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
    cluster_sync();            // every MMA of the pair has completed and been read
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace fldce
