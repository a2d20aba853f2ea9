// fldce_api.cu -- host side of the C ABI declared in include/fldce.h.
//
// One fwd+bwd call enqueues, on the caller's stream and without any host
// synchronisation:
//   k_count_targets                  all N tokens (the normaliser T, bad targets)
//   [SKIP_IGNORED] k_compact_valid, k_gather_rows   compact the valid tokens
//   per token chunk [r0, r0 + rows):
//     sweep 1  GEMM H W^T (+b), LseEpi      per (row, vocab tile) partial lse
//     k_merge_rows                          lse, loss[n], gradient coefficient
//     sweep 2  GEMM H W^T (+b), GEpi        G (bf16) for the chunk
//     [bias] k_colsum_*                     db (+)= column sums of G
//     dH GEMM  G W       (+ k_sum_splits when the vocabulary is split in k ranges)
//     dW GEMM  G^T H     (fp32 across chunks, converted after the last)
//   [SKIP_IGNORED] k_scatter_rows       dH and per-token outputs back in place
//   k_finish                             fixed-order loss sum, error counts
// The vocabulary-parallel entry points run the same pipeline on one shard of
// W: fldce_vp_stats stops after sweep 1 and writes the shard's per-token
// statistics; fldce_vp_fwd_bwd skips sweep 1 and merges every shard's.
// The chunk loop is the page's fused_linear_cross_entropy_forward loop over
// token chunks; it bounds the workspace.  bf16 runs on tcgen05 tensor cores;
// fp32 runs the CUDA-core GEMM of kernels.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/fldce.h"
#include "fused_gdh.cuh"
#include "kernels.cuh"

using namespace fldce;

namespace {

constexpr int kVersion = 100;          // 0.1.0
constexpr int kBN = 256;               // vocab tile of the tensor-core sweeps
constexpr int kStages = 6;
constexpr size_t kAlign = 256;
constexpr size_t kGBudget = size_t(1) << 32;   // G buffer per chunk: at most 4 GiB
constexpr int kMaxKSplits = 4;                  // K splits of the dH GEMM
// L2 bytes the sweeps' tile walk keeps resident for H: a third of the
// 126 MB L2, leaving the rest to the streamed W tiles and the G stores.  With
// a token-tile block wider than this (ragged: 64 tiles x 2 MB of H) every
// round re-read all of H from HBM (43 GB per sweep instead of 8.5 GB).
constexpr size_t kL2BudgetSweep = size_t(42) << 20;
constexpr int kColsumSegs = 8;                  // row segments of the db column sums

using CfgKK = GemmCfg<kStages, false, false>;   // sweeps 1 and 2: H (K-major), W (K-major)
using CfgKM = GemmCfg<kStages, false, true>;    // dH: G (K-major), W (MN-major)
// dH with 256 x 512 tiles: two MMAs per staged A tile (48 KB stages, 4 deep).
// Its K loop runs over the whole vocabulary, so the epilogue that no longer
// overlaps the MMAs costs little, while the stages per MMA and the operand
// traffic from L2 drop.
using CfgKM2 = GemmCfg<4, false, true, 2>;
using CfgMM = GemmCfg<kStages, true, true>;     // dW: G^T (MN-major), H (MN-major)

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct DeviceInfo {
    int major = -1;
    int sms = 0;
};

// Compute capability and SM count of the current device (cached per device;
// calls may come from several host threads).
bool device_info(DeviceInfo* out) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 64 && cache[dev].major >= 0) {
            *out = cache[dev];
            return true;
        }
    }
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return false;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 64) cache[dev] = d;
    *out = d;
    return true;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's cuTensorMapEncodeTiled, looked up once (no link-time libcuda).
EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D tensor map over a row-major [outer, inner] matrix of `elt`-byte
// elements (bf16 or fp32) with row stride `ld` elements; box = [box_outer,
// box_inner], 128-byte swizzle, zero fill outside the extent.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
              uint32_t box_inner, uint32_t box_outer, int elt = 2) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld * (uint64_t)elt};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt =
        elt == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Store map of an output: bf16 boxes of 32 rows x 64 columns, fp32 boxes of
// 32 rows x 32 columns (128 bytes either way).
bool make_store_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld,
                    int elt) {
    return make_map(m, base, cols, rows, ld, elt == 4 ? 32 : 64, 32, elt);
}

// K splits of a GEMM with `tiles` output tiles and `k_iters` K steps on
// `pairs` CTA pairs.  The persistent schedule runs ceil(k tiles / pairs)
// rounds of ceil(k_iters / k) steps; a split is taken only when it shortens
// that by more than 2% (each split costs an fp32 partial buffer and its
// share of the fixed-order sum) and keeps >= 16 K steps per split.
int choose_k_splits(int64_t tiles, int64_t k_iters, int pairs) {
    auto cost = [&](int64_t k) { return cdiv(k * tiles, pairs) * cdiv(k_iters, k); };
    int best = 1;
    for (int k = 2; k <= kMaxKSplits; ++k)
        if (k_iters >= 16 * k && (double)cost(k) < 0.98 * (double)cost(best)) best = k;
    return best;
}

struct DynRows {
    const int32_t* count = nullptr;   // device-side row count, or null
    int base = 0;
    int dim = 0;                      // 1: bounds M, 2: bounds K
};

// Fast-dimension tiles per block of the tile walk: as many as keep one
// block's panels of the reused operand (panel_bytes each) within `budget`,
// with the blocks balanced in width.
int walk_group(int64_t n_fast, size_t panel_bytes, size_t budget) {
    if (n_fast <= 0) return 1;
    const int64_t gmax = std::max<int64_t>(1, (int64_t)(budget / std::max<size_t>(panel_bytes, 1)));
    return (int)cdiv(n_fast, cdiv(n_fast, gmax));
}

// dH's tile width and K splits.  Both widths are costed with the schedule
// model of choose_k_splits, in units of one 256-column MMA step: a 512-wide
// unit does twice the MMA work per K step but, with a quarter less operand
// traffic from L2 and half the pipeline stages per MMA, measured about 4%
// less time per MMA under the power cap (kWideDhCost).  The wide tiles are
// not used when they pad D by more than 10% over 256-wide ones.
constexpr double kWideDhCost = 0.96;

struct DhPlan {
    bool wide;
    int k_splits;
};

DhPlan plan_dh(int64_t rows, int64_t D, int64_t V, int pairs) {
    const int64_t k_iters = cdiv(V, 64);
    const int64_t mt = cdiv(rows, 256);
    auto cost = [&](int64_t tiles, int ks) {
        return (double)(cdiv(ks * tiles, pairs) * cdiv(k_iters, ks));
    };
    const int64_t nt = mt * cdiv(D, 256);
    const int kn = choose_k_splits(nt, k_iters, pairs);
    DhPlan p{false, kn};
    if (round_up((size_t)D, 512) * 10 > round_up((size_t)D, 256) * 11) return p;
    const int64_t wt = mt * cdiv(D, 512);
    const int kw = choose_k_splits(wt, k_iters, pairs);
    if (2.0 * kWideDhCost * cost(wt, kw) < cost(nt, kn)) p = DhPlan{true, kw};
    return p;
}

// One block: the walk covers every tile of the fast dimension per step of
// the slow one.  dH streams both of its operands (K = V); dW's reused H
// panels measured no gain from blocking (G, the larger operand, is then
// re-read once per block).
constexpr int kOneBlock = std::numeric_limits<int>::max();

// How a GEMM's units are walked.
struct Walk {
    int n_fastest;        // 1: consecutive tiles share the A panel
    int k_splits;         // K ranges per tile
    int group;            // fast-dimension tiles per block of the walk
};

template <class Cfg, class Epi>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, int M, int64_t N, int64_t K,
                        const Walk& w, const typename Epi::Params& ep, int32_t* err, int sms,
                        cudaStream_t st, DynRows dyn = DynRows()) {
    GemmGeom g;
    g.dyn_count = dyn.count;
    g.dyn_base = dyn.base;
    g.dyn_dim = dyn.count != nullptr ? dyn.dim : 0;
    g.dyn_cap = dyn.dim == 2 ? (int)K : M;
    g.tiles_m = (int)cdiv(M, Cfg::PAIR_M);
    g.tiles_n = (int)cdiv(N, Cfg::BN);
    g.k_iters = (int)cdiv(K, Cfg::BK);
    g.k_splits = w.k_splits;
    g.num_tiles = g.tiles_m * g.tiles_n;
    g.n_fastest = w.n_fastest;
    g.group = w.group;
    if (g.num_tiles == 0 || g.k_iters == 0) return cudaSuccess;
    auto kern = umma_gemm_kernel<Cfg, Epi>;
    // The shared-memory opt-in is set once per kernel and device, so calls
    // after the first make no host-side CUDA calls besides the launch (a
    // call can then be captured into a CUDA graph).
    static std::atomic<uint64_t> attr_set{0};
    int devid = 0;
    cudaError_t e = cudaGetDevice(&devid);
    if (e != cudaSuccess) return e;
    const uint64_t bit = devid < 64 ? (uint64_t(1) << devid) : 0;
    if (bit == 0 || (attr_set.load(std::memory_order_acquire) & bit) == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit, std::memory_order_release);
    }
    const int pairs = std::min(g.num_tiles * g.k_splits, std::max(1, sms / 2));
    kern<<<2 * pairs, kGemmThreads, Cfg::SMEM_BYTES, st>>>(a, b, g, ep, err);
    return cudaGetLastError();
}

// Sweep 2 fused with the dH GEMM (FLDCE_FLAG_FUSED_DH): G tiles to HBM
// through gp.gmap, dH partials reduce-added into the fp32 map mDh.
cudaError_t launch_fused_gdh(const CUtensorMap& mH, const CUtensorMap& mW, const CUtensorMap& mWmn,
                             const CUtensorMap& mDh, int rows, int64_t V, int64_t D,
                             const Walk& w, const GEpi::Params& gp, int32_t* err, int sms,
                             cudaStream_t st) {
    using Cfg = FusedGdhCfg;
    GemmGeom g{};
    g.tiles_m = (int)cdiv(rows, Cfg::PAIR_M);
    g.tiles_n = (int)cdiv(V, Cfg::BN);
    g.k_iters = (int)cdiv(D, Cfg::BK);
    g.k_splits = 1;
    g.num_tiles = g.tiles_m * g.tiles_n;
    g.n_fastest = w.n_fastest;
    // token tiles in blocks whose fp32 dH rows (the reduce-add targets) and H
    // panels stay in L2 together; W is read once per block
    g.group = walk_group(g.tiles_m, (size_t)Cfg::PAIR_M * D * (4 + 2), kL2BudgetSweep);
    if (g.num_tiles == 0 || g.k_iters == 0) return cudaSuccess;
    auto kern = fused_gdh_kernel<Cfg>;
    static std::atomic<uint64_t> attr_set{0};
    int devid = 0;
    cudaError_t e = cudaGetDevice(&devid);
    if (e != cudaSuccess) return e;
    const uint64_t bit = devid < 64 ? (uint64_t(1) << devid) : 0;
    if (bit == 0 || (attr_set.load(std::memory_order_acquire) & bit) == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit, std::memory_order_release);
    }
    const int pairs = std::min(g.num_tiles, std::max(1, sms / 2));
    const int d_chunks = (int)cdiv(D, Cfg::DH_N);
    kern<<<2 * pairs, kGemmThreads, Cfg::SMEM_BYTES, st>>>(mH, mW, mWmn, mDh, g, d_chunks, D, gp,
                                                          err);
    return cudaGetLastError();
}

// db (+)= column sums of the chunk's G, in a fixed order (two passes).
cudaError_t launch_colsum(const void* G, bool g_bf16, int64_t ldg, int rows, int64_t V,
                          float* part, float* acc, bool add, cudaStream_t st,
                          const int32_t* dyn_count = nullptr, int dyn_base = 0) {
    const int nseg = (int)std::min<int64_t>(kColsumSegs, std::max<int64_t>(1, cdiv(rows, 256)));
    const int seg_rows = (int)cdiv(rows, nseg);
    const dim3 grid((unsigned)cdiv(cdiv(V, 2), 128), (unsigned)nseg);
    if (g_bf16)
        k_colsum_partial<__nv_bfloat16><<<grid, 128, 0, st>>>(
            static_cast<const __nv_bfloat16*>(G), ldg, rows, V, seg_rows, part, dyn_count,
            dyn_base);
    else
        k_colsum_partial<float><<<grid, 128, 0, st>>>(static_cast<const float*>(G), ldg, rows, V,
                                                      seg_rows, part, dyn_count, dyn_base);
    k_colsum_final<<<(unsigned)cdiv(V, 256), 256, 0, st>>>(part, nseg, V, acc, add ? 1 : 0);
    return cudaGetLastError();
}

// dst = sum of k fp32 partials `stride` floats apart (bf16 or fp32 out).
cudaError_t launch_sum_splits(const float* part, int64_t stride, int k, void* dst, bool to_bf16,
                              int64_t n, int sms, cudaStream_t st) {
    const int64_t n8 = n / 8;
    if (n8 == 0) return cudaSuccess;
    const int blocks = (int)std::min<int64_t>(cdiv(n8, 256), 8 * (int64_t)sms);
    if (to_bf16)
        k_sum_splits<__nv_bfloat16><<<blocks, 256, 0, st>>>(
            part, stride, k, static_cast<__nv_bfloat16*>(dst), n8);
    else
        k_sum_splits<float><<<blocks, 256, 0, st>>>(part, stride, k, static_cast<float*>(dst), n8);
    return cudaGetLastError();
}

// dst = bf16(src), or bf16(dst + src) with add.
cudaError_t launch_to_bf16(const float* src, void* dst, int64_t n, bool add, int sms,
                           cudaStream_t st) {
    const int64_t n8 = n / 8;
    if (n8 == 0) return cudaSuccess;
    const int blocks = (int)std::min<int64_t>(cdiv(n8, 256), 8 * (int64_t)sms);
    k_f32_to_bf16<<<blocks, 256, 0, st>>>(src, static_cast<__nv_bfloat16*>(dst), n8, add ? 1 : 0);
    return cudaGetLastError();
}

template <class Epi>
cudaError_t launch_simt(const float* A, int64_t sam, int64_t sak, const float* B, int64_t sbn,
                        int64_t sbk, int M, int64_t N, int K, const Epi& epi, cudaStream_t st) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    dim3 grid((unsigned)cdiv(N, kSimtTile), (unsigned)cdiv(M, kSimtTile));
    simt_gemm_kernel<Epi><<<grid, 256, 0, st>>>(A, sam, sak, B, sbn, sbk, M, N, K, epi);
    return cudaGetLastError();
}

struct Layout {
    size_t cnt, part_ml, part_sz, part_am, zy, row_lse2, row_gcoef, row_y, loss_tok, G, dh_acc,
        dw_acc, db_part, db_acc;
    size_t c_idx, c_pos, c_H, c_y, c_p, c_loss, c_lse, c_am, c_dH;   // compaction
    size_t total;
    int64_t C;        // rows per chunk buffer
    int64_t nchunks;
};

}  // namespace

enum ProfKind {
    PK_COUNT = 0, PK_LSE = 1, PK_MERGE = 2, PK_G = 3, PK_DH = 4, PK_DW = 5, PK_FINISH = 6,
    PK_CONVERT = 7, PK_DB = 8, PK_GAP = -1
};
static_assert(FLDCE_PROF_KINDS == 9, "kinds");

struct fldce_plan {
    fldce_config cfg;
    int64_t v0;       // first vocabulary id of this plan's W (0 unsharded)
    int64_t Vtot;     // total vocabulary (== V unsharded)
    bool sharded;
    int64_t chunk;    // tokens per chunk
    int64_t Vpad;     // row stride of G (elements)
    int tile_v;       // vocab tile width of the partial statistics
    int64_t n_vt;     // number of vocab tiles
    size_t elt;       // bytes per element of H / W / G
    // profiling window
    std::vector<cudaEvent_t> ev;
    std::vector<int> ev_kind;
    size_t ev_used = 0;
    bool prof_on = false;
};

namespace {
// Record an event after a launch of `kind` (or a call-start gap marker).
void prof_mark(fldce_plan* h, int kind, cudaStream_t st) {
    if (!h->prof_on || h->ev_used >= h->ev.size()) return;
    if (cudaEventRecord(h->ev[h->ev_used], st) != cudaSuccess) return;
    h->ev_kind[h->ev_used++] = kind;
}
}  // namespace

namespace {

bool dw_out_fp32(const fldce_plan* p) {
    return p->cfg.dtype == FLDCE_FP32 || (p->cfg.flags & FLDCE_FLAG_DW_FP32) != 0;
}

bool dw_accumulate(const fldce_plan* p) { return (p->cfg.flags & FLDCE_FLAG_DW_ACCUMULATE) != 0; }

Layout make_layout(const fldce_plan* p, int64_t N) {
    Layout L{};
    const int64_t C = std::max<int64_t>(1, std::min<int64_t>(p->chunk, N));
    L.C = C;
    L.nchunks = N > 0 ? cdiv(N, p->chunk) : 0;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = round_up(off + bytes, kAlign);
        return o;
    };
    const size_t nv = (size_t)p->n_vt * (size_t)C;
    L.cnt = take(sizeof(Counters));
    L.part_ml = take(nv * 8);
    L.part_sz = take(nv * 4);
    L.part_am = take(nv * 4);
    L.zy = take(C * 4);
    L.row_lse2 = take(C * 4);
    L.row_gcoef = take(C * 4);
    L.row_y = take(C * 4);
    L.loss_tok = take(std::max<int64_t>(N, 1) * 4);
    L.G = take((size_t)C * p->Vpad * p->elt);
    // one fp32 partial per K split of dH, each padded to whole pair tiles
    L.dh_acc = take(p->cfg.dtype == FLDCE_BF16
                        ? (size_t)kMaxKSplits * round_up((size_t)C, 256) * p->cfg.D * 4
                        : 0);
    // fp32 dW partials across chunks, or before adding into a bf16 dW
    const bool acc = (L.nchunks > 1 || (dw_accumulate(p) && N > 0)) && !dw_out_fp32(p);
    L.dw_acc = take(acc ? (size_t)p->cfg.V * p->cfg.D * 4 : 0);
    L.db_part = take((size_t)kColsumSegs * p->cfg.V * 4);
    L.db_acc = take((size_t)p->cfg.V * 4);
    const bool skip = (p->cfg.flags & FLDCE_FLAG_SKIP_IGNORED) != 0;
    const size_t n = skip ? (size_t)std::max<int64_t>(N, 1) : 0;
    L.c_idx = take(n * 4);
    L.c_pos = take(n * 4);
    L.c_H = take(n * p->cfg.D * 2);
    L.c_y = take(n * 8);
    L.c_p = take(n * 4);
    L.c_loss = take(n * 4);
    L.c_lse = take(n * 4);
    L.c_am = take(n * 4);
    L.c_dH = take(n * p->cfg.D * 2);
    L.total = off;
    return L;
}

bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }
bool aligned_to(const void* q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; }

int check_device(DeviceInfo* d) {
    if (!device_info(d)) return FLDCE_ERR_CUDA;
    if (d->major != 10) return FLDCE_ERR_DEVICE;
    return FLDCE_OK;
}

// The shared body of fldce_fwd_bwd and fldce_forward.
// mode: MERGE_LOCAL (the whole vocabulary in this plan), MERGE_EMIT_STATS
// (a shard's sweep 1 and statistics only), MERGE_GATHERED (a shard's
// backward from every shard's statistics).
int run(fldce_handle h, const fldce_call& call, bool backward, int mode = MERGE_LOCAL,
        float* stats_out = nullptr, const float* all_stats = nullptr, int n_shards = 0) {
    const void* H = call.H;
    const void* W = call.W;
    const int64_t* target = call.target;
    const float* p_mask = call.p_mask;
    const int64_t N = call.N;
    const float total = call.total, grad_out = call.grad_out;
    float* loss = call.loss;
    float* loss_tok_out = call.loss_per_token;
    float* lse_out = call.lse;
    int32_t* argmax_out = call.argmax;
    void* dH = call.dH;
    void* dW = call.dW;
    void* workspace = call.workspace;
    const size_t workspace_bytes = call.workspace_bytes;
    int32_t* err_count = call.err_count;
    void* stream = call.stream;
    const void* bias = call.bias;
    void* db = call.db;
    if (backward && bias != nullptr && db == nullptr) return FLDCE_ERR_INVALID_ARG;
    if (h != nullptr && h->sharded != (mode != MERGE_LOCAL)) return FLDCE_ERR_INVALID_ARG;
    if (mode == MERGE_EMIT_STATS && stats_out == nullptr) return FLDCE_ERR_INVALID_ARG;
    if (mode == MERGE_GATHERED && (all_stats == nullptr || n_shards <= 0))
        return FLDCE_ERR_INVALID_ARG;
    if (!aligned16(bias) || (backward && !aligned16(db))) return FLDCE_ERR_ALIGN;
    if (h == nullptr || (loss == nullptr && mode != MERGE_EMIT_STATS) || N < 0 ||
        N > h->cfg.max_N)
        return FLDCE_ERR_INVALID_ARG;
    if (N > 0 && (H == nullptr || W == nullptr || target == nullptr)) return FLDCE_ERR_INVALID_ARG;
    if (backward && (dW == nullptr || (N > 0 && dH == nullptr))) return FLDCE_ERR_INVALID_ARG;
    if (!std::isfinite(total) || !std::isfinite(grad_out)) return FLDCE_ERR_INVALID_ARG;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return FLDCE_ERR_WORKSPACE;
    if (!aligned16(H) || !aligned16(W) || (backward && (!aligned16(dH) || !aligned16(dW))))
        return FLDCE_ERR_ALIGN;
    // natural alignment of the per-token arrays (the row kernels read and
    // write them as 128-bit vectors where they are 16-byte aligned)
    if (!aligned_to(target, 8) || !aligned_to(p_mask, 4) || !aligned_to(loss_tok_out, 4) ||
        !aligned_to(lse_out, 4) || !aligned_to(argmax_out, 4) || !aligned16(stats_out))
        return FLDCE_ERR_ALIGN;
    const Layout L = make_layout(h, N);
    if (workspace_bytes < L.total) return FLDCE_ERR_WORKSPACE;
    DeviceInfo dev;
    if (int s = check_device(&dev)) return s;

    const fldce_config& cfg = h->cfg;
    const int64_t D = cfg.D, V = cfg.V;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    Counters* cnt = reinterpret_cast<Counters*>(ws + L.cnt);
    float2* part_ml = reinterpret_cast<float2*>(ws + L.part_ml);
    float* part_sz = reinterpret_cast<float*>(ws + L.part_sz);
    int32_t* part_am = reinterpret_cast<int32_t*>(ws + L.part_am);
    float* zy = reinterpret_cast<float*>(ws + L.zy);
    float* row_lse2 = reinterpret_cast<float*>(ws + L.row_lse2);
    float* row_gcoef = reinterpret_cast<float*>(ws + L.row_gcoef);
    int32_t* row_y = reinterpret_cast<int32_t*>(ws + L.row_y);
    float* db_part = reinterpret_cast<float*>(ws + L.db_part);
    float* db_acc = reinterpret_cast<float*>(ws + L.db_acc);
    float* loss_tok = loss_tok_out != nullptr ? loss_tok_out
                                              : reinterpret_cast<float*>(ws + L.loss_tok);
    const bool bf16 = cfg.dtype == FLDCE_BF16;
    const bool skip = (cfg.flags & FLDCE_FLAG_SKIP_IGNORED) != 0;
    const bool accum = dw_accumulate(h);     // dW (and db) += this call's gradient
    // compaction buffers (FLDCE_FLAG_SKIP_IGNORED) and the caller's outputs
    int32_t* c_idx = reinterpret_cast<int32_t*>(ws + L.c_idx);
    int32_t* c_pos = reinterpret_cast<int32_t*>(ws + L.c_pos);
    __nv_bfloat16* c_H = reinterpret_cast<__nv_bfloat16*>(ws + L.c_H);
    int64_t* c_y = reinterpret_cast<int64_t*>(ws + L.c_y);
    float* c_p = reinterpret_cast<float*>(ws + L.c_p);
    float* c_loss = reinterpret_cast<float*>(ws + L.c_loss);
    float* c_lse = reinterpret_cast<float*>(ws + L.c_lse);
    int32_t* c_am = reinterpret_cast<int32_t*>(ws + L.c_am);
    __nv_bfloat16* c_dH = reinterpret_cast<__nv_bfloat16*>(ws + L.c_dH);
    float* const user_loss_tok = loss_tok_out;
    float* const user_lse = lse_out;
    int32_t* const user_am = argmax_out;
    void* const user_dH = dH;
    const int32_t* dynp = nullptr;           // device-side row count of the compacted tokens
    const float s = cfg.logit_scale, eps = cfg.label_smoothing;
    const float c = s * 1.4426950408889634f;

#define FLDCE_CUDA(x)                                  \
    do {                                               \
        if ((x) != cudaSuccess) return FLDCE_ERR_CUDA; \
    } while (0)

    FLDCE_CUDA(cudaMemsetAsync(cnt, 0, sizeof(Counters), st));
    prof_mark(h, PK_GAP, st);
    if (N > 0) {
        const int blocks = (int)std::min<int64_t>(cdiv(N, 256), 4 * (int64_t)dev.sms);
        k_count_targets<<<blocks, 256, 0, st>>>(target, N, h->Vtot, cfg.ignore_index, cnt);
        FLDCE_CUDA(cudaGetLastError());
        prof_mark(h, PK_COUNT, st);
        if (skip) {
            // compact the tokens that carry a loss; everything below runs on
            // them, with row counts read on the device (no host sync)
            k_compact_valid<<<1, 1024, 0, st>>>(target, N, h->Vtot, cfg.ignore_index, c_idx,
                                                c_pos, &cnt->n_compact);
            FLDCE_CUDA(cudaGetLastError());
            const int gb = (int)std::min<int64_t>(cdiv(N * (D / 8), 256), 8 * (int64_t)dev.sms);
            k_gather_rows<<<gb, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(H), target,
                                              p_mask, c_idx, &cnt->n_compact, N, D, c_H, c_y,
                                              c_p);
            FLDCE_CUDA(cudaGetLastError());
            prof_mark(h, PK_COUNT, st);
            H = c_H;
            target = c_y;
            p_mask = c_p;
            loss_tok = c_loss;
            lse_out = user_lse != nullptr ? c_lse : nullptr;
            argmax_out = user_am != nullptr ? c_am : nullptr;
            if (backward) dH = c_dH;
            dynp = &cnt->n_compact;
        }
    } else if (backward && !accum) {
        FLDCE_CUDA(cudaMemsetAsync(dW, 0, (size_t)V * D * (dw_out_fp32(h) ? 4 : h->elt), st));
        if (bias != nullptr)
            FLDCE_CUDA(cudaMemsetAsync(db, 0, (size_t)V * (dw_out_fp32(h) ? 4 : h->elt), st));
    }

    const bool fp32_dw = dw_out_fp32(h);
    float* dw_ws = fp32_dw ? static_cast<float*>(dW) : reinterpret_cast<float*>(ws + L.dw_acc);

    if (skip && backward && N > 0 && !(accum && fp32_dw)) {
        // with no token to carry a loss the dW GEMM has no K rows: zero the
        // buffer its first chunk would have written (an fp32 dW accumulated
        // into is left as it is)
        const bool direct = L.nchunks == 1 && !fp32_dw && !accum;
        void* dst = direct ? dW : static_cast<void*>(dw_ws);
        const int64_t b16 = (int64_t)V * D * (direct ? 2 : 4) / 16;
        k_zero_if_none<<<(unsigned)std::min<int64_t>(cdiv(b16, 256), 8 * (int64_t)dev.sms), 256, 0,
                         st>>>(dynp, dst, b16);
        FLDCE_CUDA(cudaGetLastError());
    }

    CUtensorMap mW_k, mW_mn;
    if (bf16 && N > 0) {
        if (!make_map(&mW_k, W, D, V, D, 64, 128)) return FLDCE_ERR_CUDA;
        if (backward && !make_map(&mW_mn, W, D, V, D, 64, 64)) return FLDCE_ERR_CUDA;
    }

    for (int64_t ci = 0; ci < L.nchunks; ++ci) {
        const int64_t r0 = ci * h->chunk;
        const int rows = (int)std::min<int64_t>(h->chunk, N - r0);
        const int64_t* tgt = target + r0;

        LseEpi::Params lp;
        lp.c = c;
        lp.s = s;
        lp.V = V;
        lp.rows = rows;
        lp.ld_part = (int)L.C;
        lp.target = tgt;
        lp.part_ml = part_ml;
        lp.part_sz = eps > 0.f ? part_sz : nullptr;
        const bool want_am = argmax_out != nullptr || mode == MERGE_EMIT_STATS;
        lp.part_am = want_am ? part_am : nullptr;
        lp.zy = zy;
        lp.bias = bf16 ? static_cast<const __nv_bfloat16*>(bias) : nullptr;
        lp.v0 = h->v0;

        CUtensorMap mH_k, mH_mn, mG_k, mG_mn;
        // the sweeps walk vocabulary tiles under a block of token tiles
        // whose H panels stay in L2 (H is re-read from L2, not HBM)
        const Walk sweep_walk{0, 1,
                              walk_group(cdiv(rows, CfgKK::PAIR_M),
                                         (size_t)CfgKK::PAIR_M * D * 2, kL2BudgetSweep)};
        if (bf16) {
            const void* Hc = static_cast<const __nv_bfloat16*>(H) + r0 * D;
            if (!make_map(&mH_k, Hc, D, rows, D, 64, 128)) return FLDCE_ERR_CUDA;
        }
        // sweep 1 (not needed when every shard's statistics are given)
        if (mode != MERGE_GATHERED) {
            if (bf16) {
                FLDCE_CUDA((launch_gemm<CfgKK, LseEpi>(mH_k, mW_k, rows, V, D, sweep_walk, lp,
                                                       &cnt->dev_err, dev.sms, st,
                                                       DynRows{dynp, (int)r0, 1})));
            } else {
                const float* Hc = static_cast<const float*>(H) + r0 * D;
                SimtLse e{lp, static_cast<const float*>(bias)};
                FLDCE_CUDA(launch_simt(Hc, D, 1, static_cast<const float*>(W), D, 1, rows, V,
                                       (int)D, e, st));
            }
            prof_mark(h, PK_LSE, st);
        }

        MergeParams mp;
        mp.mode = mode;
        mp.v0 = h->v0;
        mp.Vtot = h->Vtot;
        mp.stats_out = stats_out;
        mp.all_stats = all_stats;
        mp.n_shards = n_shards;
        mp.stats_N = N;
        mp.stats_row0 = r0;
        mp.rows = rows;
        mp.ld_part = (int)L.C;
        mp.n_vt = (int)h->n_vt;
        mp.V = V;
        mp.ignore_index = cfg.ignore_index;
        mp.s = s;
        mp.eps = eps;
        mp.total = total;
        mp.grad_out = grad_out;
        mp.target = tgt;
        mp.p_mask = p_mask != nullptr ? p_mask + r0 : nullptr;
        mp.part_ml = part_ml;
        mp.part_sz = eps > 0.f ? part_sz : nullptr;
        mp.part_am = want_am ? part_am : nullptr;
        mp.zy = zy;
        mp.cnt = cnt;
        mp.count_dev = call.count_dev;
        mp.dyn_count = dynp;
        mp.dyn_base = (int)r0;
        mp.loss_tok = loss_tok + r0;
        mp.lse_out = lse_out != nullptr ? lse_out + r0 : nullptr;
        mp.am_out = argmax_out != nullptr ? argmax_out + r0 : nullptr;
        mp.row_lse2 = backward && mode != MERGE_EMIT_STATS ? row_lse2 : nullptr;
        mp.row_gcoef = row_gcoef;
        mp.row_y = row_y;
        mp.vec = aligned16(mp.target) && aligned16(mp.p_mask) && aligned16(mp.loss_tok) &&
                 aligned16(mp.lse_out) && aligned16(mp.am_out);
        k_merge_rows<<<(unsigned)cdiv((int64_t)rows * kMergeSub, 256), 256, 0, st>>>(mp);
        FLDCE_CUDA(cudaGetLastError());
        prof_mark(h, PK_MERGE, st);
        if (!backward || mode == MERGE_EMIT_STATS) continue;

        // dW: one chunk writes the output directly; several chunks store, then
        // reduce-add, fp32 partial sums (into dW itself when it is fp32).
        const int simt_mode = accum ? 2 : (L.nchunks == 1 ? 0 : (ci == 0 ? 1 : 2));
        const bool dw_first = call.dw_ready_event != nullptr && ci + 1 == L.nchunks;
        // db is final once the last chunk's column sums are in: cast it out
        auto finish_db = [&]() -> int {
            if (bias == nullptr || ci + 1 != L.nchunks) return FLDCE_OK;
            k_cast_out<<<(unsigned)cdiv(V, 256), 256, 0, st>>>(db_acc, db, V,
                                                              dw_out_fp32(h) ? 0 : 1,
                                                              accum ? 1 : 0);
            FLDCE_CUDA(cudaGetLastError());
            prof_mark(h, PK_DB, st);
            return FLDCE_OK;
        };
        if (bf16) {
            __nv_bfloat16* G = reinterpret_cast<__nv_bfloat16*>(ws + L.G);
            GEpi::Params gp;
            if (!make_store_map(&gp.gmap, G, V, rows, h->Vpad, 2)) return FLDCE_ERR_CUDA;
            gp.c = c;
            gp.V = V;
            gp.rows = rows;
            gp.lse2 = row_lse2;
            gp.gcoef = row_gcoef;
            gp.ycol = row_y;
            gp.eps_over_V = eps / (float)h->Vtot;
            gp.one_minus_eps = 1.f - eps;
            gp.bias = static_cast<const __nv_bfloat16*>(bias);
            const bool fused_dh = (cfg.flags & FLDCE_FLAG_FUSED_DH) != 0;
            float* dh_part = reinterpret_cast<float*>(ws + L.dh_acc);
            if (fused_dh) {
                // sweep 2 and dH in one kernel: G from shared memory into the
                // dH MMAs, fp32 partials reduce-added into dh_part
                CUtensorMap mDh;
                if (!make_store_map(&mDh, dh_part, D, rows, D, 4)) return FLDCE_ERR_CUDA;
                FLDCE_CUDA(cudaMemsetAsync(dh_part, 0, (size_t)rows * D * 4, st));
                FLDCE_CUDA(launch_fused_gdh(mH_k, mW_k, mW_mn, mDh, rows, V, D, sweep_walk, gp,
                                            &cnt->dev_err, dev.sms, st));
            } else {
                FLDCE_CUDA((launch_gemm<CfgKK, GEpi>(mH_k, mW_k, rows, V, D, sweep_walk, gp,
                                                     &cnt->dev_err, dev.sms, st,
                                                     DynRows{dynp, (int)r0, 1})));
            }
            prof_mark(h, PK_G, st);
            if (bias != nullptr) {
                FLDCE_CUDA(launch_colsum(G, true, h->Vpad, rows, V, db_part, db_acc, ci > 0, st,
                                         dynp, (int)r0));
                prof_mark(h, PK_DB, st);
                if (int e = finish_db()) return e;
            }
            if (!make_map(&mG_k, G, V, rows, h->Vpad, 64, 128)) return FLDCE_ERR_CUDA;
            if (!make_map(&mG_mn, G, V, rows, h->Vpad, 64, 64)) return FLDCE_ERR_CUDA;
            const void* Hc = static_cast<const __nv_bfloat16*>(H) + r0 * D;
            if (!make_map(&mH_mn, Hc, D, rows, D, 64, 64)) return FLDCE_ERR_CUDA;

            // dH = G W (K = V).  When one pass over the tiles leaves many SMs
            // idle in its last round, the vocabulary is split into k ranges;
            // split j stores its fp32 partial in its own buffer and one pass
            // sums them in split order (deterministic) into dH.
            auto do_dh = [&]() -> int {
                if (fused_dh) {
                    // the fused kernel left dH in fp32: round (or copy) it out
                    const bool dh_fp32 = (cfg.flags & FLDCE_FLAG_DH_FP32) != 0;
                    void* dHc = static_cast<uint8_t*>(dH) + (size_t)r0 * D * (dh_fp32 ? 4 : 2);
                    FLDCE_CUDA(launch_sum_splits(dh_part, 0, 1, dHc, !dh_fp32, (int64_t)rows * D,
                                                 dev.sms, st));
                    prof_mark(h, PK_CONVERT, st);
                    return FLDCE_OK;
                }
                const DhPlan dp = plan_dh(rows, D, V, std::max(1, dev.sms / 2));
                const bool wide = dp.wide;
                const int ks = dp.k_splits;
                StoreEpi::Params hp;
                const bool dh_fp32 = (cfg.flags & FLDCE_FLAG_DH_FP32) != 0;
                float* part = reinterpret_cast<float*>(ws + L.dh_acc);
                const int split_rows = (int)round_up((size_t)rows, 256);
                void* dHc = static_cast<uint8_t*>(dH) + (size_t)r0 * D * (dh_fp32 ? 4 : 2);
                if (ks > 1) {
                    if (!make_store_map(&hp.omap, part, D, (uint64_t)ks * split_rows, D, 4))
                        return FLDCE_ERR_CUDA;
                    hp.mode = WS_STORE;
                    hp.split_rows = split_rows;
                } else if (dh_fp32) {
                    if (!make_store_map(&hp.omap, dHc, D, rows, D, 4)) return FLDCE_ERR_CUDA;
                    hp.mode = WS_STORE;
                } else {
                    if (!make_store_map(&hp.omap, dHc, D, rows, D, 2)) return FLDCE_ERR_CUDA;
                    hp.mode = OUT_BF16;
                }
                const Walk dh_walk{1, ks, kOneBlock};
                if (wide)
                    FLDCE_CUDA((launch_gemm<CfgKM2, StoreEpi>(mG_k, mW_mn, rows, D, V, dh_walk,
                                                              hp, &cnt->dev_err, dev.sms, st,
                                                              DynRows{dynp, (int)r0, 1})));
                else
                    FLDCE_CUDA((launch_gemm<CfgKM, StoreEpi>(mG_k, mW_mn, rows, D, V, dh_walk,
                                                             hp, &cnt->dev_err, dev.sms, st,
                                                             DynRows{dynp, (int)r0, 1})));
                prof_mark(h, PK_DH, st);
                if (ks > 1) {
                    FLDCE_CUDA(launch_sum_splits(part, (int64_t)split_rows * D, ks, dHc,
                                                 !dh_fp32, (int64_t)rows * D, dev.sms, st));
                    prof_mark(h, PK_CONVERT, st);
                }
                return FLDCE_OK;
            };
            // dW = G^T H (K = tokens of the chunk): one chunk writes dW
            // directly; several store, then reduce-add, fp32 partial sums.
            auto do_dw = [&]() -> int {
                StoreEpi::Params wp;
                if (L.nchunks == 1 && !fp32_dw && !accum) {
                    if (!make_store_map(&wp.omap, dW, D, V, D, 2)) return FLDCE_ERR_CUDA;
                    wp.mode = OUT_BF16;
                } else {
                    // fp32 partial sums; an fp32 dW accumulated into takes
                    // every chunk's reduce-add directly
                    if (!make_store_map(&wp.omap, dw_ws, D, V, D, 4)) return FLDCE_ERR_CUDA;
                    wp.mode = (ci == 0 && !(accum && fp32_dw)) ? WS_STORE : WS_ADD;
                }
                const Walk dw_walk{1, 1, kOneBlock};
                FLDCE_CUDA((launch_gemm<CfgMM, StoreEpi>(mG_mn, mH_mn, (int)V, D, rows, dw_walk,
                                                         wp, &cnt->dev_err, dev.sms, st,
                                                         DynRows{dynp, (int)r0, 2})));
                prof_mark(h, PK_DW, st);
                if ((L.nchunks > 1 || accum) && !fp32_dw && ci + 1 == L.nchunks) {
                    FLDCE_CUDA(launch_to_bf16(dw_ws, dW, V * D, accum, dev.sms, st));
                    prof_mark(h, PK_CONVERT, st);
                }
                return FLDCE_OK;
            };
            if (dw_first) {
                if (int e = do_dw()) return e;
                FLDCE_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(call.dw_ready_event), st));
                if (int e = do_dh()) return e;
            } else {
                if (int e = do_dh()) return e;
                if (int e = do_dw()) return e;
            }
        } else {
            float* G = reinterpret_cast<float*>(ws + L.G);
            const float* Hc = static_cast<const float*>(H) + r0 * D;
            SimtG ge{c,     V,         h->Vpad,          rows,
                     row_lse2, row_gcoef, row_y,   eps / (float)h->Vtot, 1.f - eps, G,
                     static_cast<const float*>(bias)};
            FLDCE_CUDA(launch_simt(Hc, D, 1, static_cast<const float*>(W), D, 1, rows, V, (int)D,
                                   ge, st));
            prof_mark(h, PK_G, st);
            if (bias != nullptr) {
                FLDCE_CUDA(launch_colsum(G, false, h->Vpad, rows, V, db_part, db_acc, ci > 0, st));
                prof_mark(h, PK_DB, st);
                if (int e = finish_db()) return e;
            }
            SimtStore hs{rows, D, D, static_cast<float*>(dH) + r0 * D, nullptr, 0};
            SimtStore wsd{(int)V, D, D, static_cast<float*>(dW), dw_ws, simt_mode};
            if (dw_first) {
                FLDCE_CUDA(launch_simt(G, 1, h->Vpad, Hc, 1, D, (int)V, D, rows, wsd, st));
                prof_mark(h, PK_DW, st);
                FLDCE_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(call.dw_ready_event), st));
            }
            FLDCE_CUDA(launch_simt(G, h->Vpad, 1, static_cast<const float*>(W), 1, D, rows, D,
                                   (int)V, hs, st));
            prof_mark(h, PK_DH, st);
            if (!dw_first) {
                FLDCE_CUDA(launch_simt(G, 1, h->Vpad, Hc, 1, D, (int)V, D, rows, wsd, st));
                prof_mark(h, PK_DW, st);
            }
        }
    }

    if (skip && N > 0) {
        const int sb = (int)std::min<int64_t>(cdiv(N * (D / 8), 256), 8 * (int64_t)dev.sms);
        k_scatter_rows<<<sb, 256, 0, st>>>(c_pos, N, D, c_dH,
                                           backward ? static_cast<__nv_bfloat16*>(user_dH) : nullptr,
                                           c_loss, user_loss_tok, c_lse, user_lse, c_am, user_am);
        FLDCE_CUDA(cudaGetLastError());
        prof_mark(h, PK_CONVERT, st);
    }
    if (backward && N == 0 && call.dw_ready_event != nullptr)
        FLDCE_CUDA(cudaEventRecord(reinterpret_cast<cudaEvent_t>(call.dw_ready_event), st));
    if (mode == MERGE_EMIT_STATS) return FLDCE_OK;
    k_finish<<<1, 1024, 0, st>>>(loss_tok, N, cnt, loss, err_count);
    FLDCE_CUDA(cudaGetLastError());
    prof_mark(h, PK_FINISH, st);
#undef FLDCE_CUDA
    return FLDCE_OK;
}

}  // namespace

extern "C" {

int fldce_create(fldce_handle* out, const fldce_config* cfg, size_t* workspace_bytes) {
    if (out == nullptr || cfg == nullptr) return FLDCE_ERR_INVALID_ARG;
    if (cfg->D <= 0 || cfg->V <= 0 || cfg->max_N <= 0 || cfg->chunk_N < 0)
        return FLDCE_ERR_INVALID_ARG;
    if (!(cfg->label_smoothing >= 0.f && cfg->label_smoothing <= 1.f))
        return FLDCE_ERR_INVALID_ARG;
    if (!std::isfinite(cfg->logit_scale) || cfg->logit_scale == 0.f) return FLDCE_ERR_INVALID_ARG;
    if (cfg->dtype != FLDCE_BF16 && cfg->dtype != FLDCE_FP32) return FLDCE_ERR_UNSUPPORTED;
    if ((cfg->flags & ~(FLDCE_FLAG_DW_FP32 | FLDCE_FLAG_SKIP_IGNORED | FLDCE_FLAG_DH_FP32 |
                        FLDCE_FLAG_DW_ACCUMULATE | FLDCE_FLAG_FUSED_DH)) != 0)
        return FLDCE_ERR_UNSUPPORTED;
    if ((cfg->flags & FLDCE_FLAG_FUSED_DH) != 0 &&
        (cfg->dtype != FLDCE_BF16 || (cfg->flags & FLDCE_FLAG_SKIP_IGNORED) != 0))
        return FLDCE_ERR_UNSUPPORTED;
    if ((cfg->flags & FLDCE_FLAG_SKIP_IGNORED) != 0 &&
        (cfg->dtype != FLDCE_BF16 || (cfg->flags & FLDCE_FLAG_DH_FP32) != 0))
        return FLDCE_ERR_UNSUPPORTED;
    if (cfg->vocab_total > 0 && (cfg->flags & FLDCE_FLAG_SKIP_IGNORED) != 0)
        return FLDCE_ERR_UNSUPPORTED;
    if (cfg->vocab_total < 0 || cfg->vocab_start < 0 ||
        (cfg->vocab_total > 0 && cfg->vocab_start + cfg->V > cfg->vocab_total) ||
        (cfg->vocab_total == 0 && cfg->vocab_start != 0))
        return FLDCE_ERR_INVALID_ARG;
    if (cfg->D % 8 != 0) return FLDCE_ERR_UNSUPPORTED;
    if (cfg->V > (int64_t(1) << 31) - 1 || cfg->max_N > (int64_t(1) << 31) - 1 ||
        cfg->D > (int64_t(1) << 31) - 1)
        return FLDCE_ERR_UNSUPPORTED;
    fldce_plan* p = new (std::nothrow) fldce_plan;
    if (p == nullptr) return FLDCE_ERR_INVALID_ARG;
    p->cfg = *cfg;
    p->sharded = cfg->vocab_total > 0;
    p->v0 = cfg->vocab_start;
    p->Vtot = p->sharded ? cfg->vocab_total : cfg->V;
    p->elt = cfg->dtype == FLDCE_BF16 ? 2 : 4;
    // G rows start on 128-byte boundaries so every TMA box row of G is one
    // whole cache line (a 16-byte-aligned but ragged stride costs an extra
    // sector per box row in both gradient GEMMs).
    p->Vpad = (int64_t)round_up((size_t)cfg->V, cfg->dtype == FLDCE_BF16 ? 64 : 32);
    p->tile_v = cfg->dtype == FLDCE_BF16 ? kBN : kSimtTile;
    p->n_vt = cdiv(cfg->V, p->tile_v);
    int64_t chunk = cfg->chunk_N;
    if (chunk == 0) {
        // whole 256-row pair tiles, so no chunk but the last ends in a
        // partly empty M tile
        chunk = (int64_t)(kGBudget / ((size_t)p->Vpad * p->elt)) / 256 * 256;
        chunk = std::max<int64_t>(chunk, 256);
    }
    p->chunk = std::min<int64_t>(chunk, cfg->max_N);
    if (workspace_bytes != nullptr) *workspace_bytes = make_layout(p, cfg->max_N).total;
    *out = p;
    return FLDCE_OK;
}

int fldce_workspace_size(fldce_handle h, int64_t N, size_t* bytes) {
    if (h == nullptr || bytes == nullptr || N < 0 || N > h->cfg.max_N) return FLDCE_ERR_INVALID_ARG;
    *bytes = make_layout(h, N).total;
    return FLDCE_OK;
}

int fldce_chunk_size(fldce_handle h, int64_t* chunk_N) {
    if (h == nullptr || chunk_N == nullptr) return FLDCE_ERR_INVALID_ARG;
    *chunk_N = h->chunk;
    return FLDCE_OK;
}

int fldce_fwd_bwd(fldce_handle h, const void* H, const void* W, const int64_t* target,
                  const float* p_mask, int64_t N, float total, float grad_out, float* loss,
                  float* loss_per_token, float* lse, int32_t* argmax, void* dH, void* dW,
                  void* workspace, size_t workspace_bytes, int32_t* err_count, void* stream) {
    fldce_call c{};
    c.H = H;
    c.W = W;
    c.target = target;
    c.p_mask = p_mask;
    c.N = N;
    c.total = total;
    c.grad_out = grad_out;
    c.loss = loss;
    c.loss_per_token = loss_per_token;
    c.lse = lse;
    c.argmax = argmax;
    c.dH = dH;
    c.dW = dW;
    c.workspace = workspace;
    c.workspace_bytes = workspace_bytes;
    c.err_count = err_count;
    c.stream = stream;
    return run(h, c, true);
}

int fldce_fwd_bwd_ex(fldce_handle h, const fldce_call* call) {
    if (call == nullptr) return FLDCE_ERR_INVALID_ARG;
    return run(h, *call, true);
}

int fldce_forward_ex(fldce_handle h, const fldce_call* call) {
    if (call == nullptr) return FLDCE_ERR_INVALID_ARG;
    fldce_call c = *call;
    c.dH = nullptr;
    c.dW = nullptr;
    c.db = nullptr;
    c.grad_out = 1.f;
    return run(h, c, false);
}

int fldce_vp_stats(fldce_handle h, const fldce_call* call, float* stats) {
    if (call == nullptr) return FLDCE_ERR_INVALID_ARG;
    return run(h, *call, false, MERGE_EMIT_STATS, stats);
}

int fldce_vp_fwd_bwd(fldce_handle h, const fldce_call* call, const float* all_stats,
                     int32_t n_shards) {
    if (call == nullptr) return FLDCE_ERR_INVALID_ARG;
    return run(h, *call, true, MERGE_GATHERED, nullptr, all_stats, n_shards);
}

int fldce_count_valid(fldce_handle h, const int64_t* target, int64_t N, int32_t* count,
                      void* stream) {
    if (h == nullptr || count == nullptr || N < 0 || (N > 0 && target == nullptr))
        return FLDCE_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int s = check_device(&dev)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(count, 0, sizeof(int32_t), st) != cudaSuccess) return FLDCE_ERR_CUDA;
    if (N > 0) {
        const int blocks = (int)std::min<int64_t>(cdiv(N, 256), 4 * (int64_t)dev.sms);
        k_count_valid_only<<<blocks, 256, 0, st>>>(target, N, h->Vtot, h->cfg.ignore_index,
                                                   count);
        if (cudaGetLastError() != cudaSuccess) return FLDCE_ERR_CUDA;
    }
    return FLDCE_OK;
}

}  // extern "C"

// Scratch of fldce_fwd_bwd_noalloc.  In host code `g_static_scratch` names a
// host-side shadow, not device memory; the device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) uint8_t g_static_scratch[FLDCE_STATIC_SCRATCH_BYTES];

namespace {
int static_scratch(void** out) {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return FLDCE_ERR_CUDA;
    if (dev >= 64) return FLDCE_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
            return FLDCE_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return FLDCE_OK;
}
}  // namespace

extern "C" {

int fldce_fwd_bwd_noalloc(fldce_handle h, const void* H, const void* W, const int64_t* target,
                          const float* p_mask, int64_t N, float total, float grad_out, float* loss,
                          float* loss_per_token, float* lse, int32_t* argmax, void* dH, void* dW,
                          int32_t* err_count, void* stream) {
    if (h == nullptr || N < 0 || N > h->cfg.max_N) return FLDCE_ERR_INVALID_ARG;
    if (make_layout(h, N).total > FLDCE_STATIC_SCRATCH_BYTES) return FLDCE_ERR_TOO_LARGE;
    DeviceInfo dev;
    if (int s = check_device(&dev)) return s;
    void* scratch = nullptr;
    if (int s = static_scratch(&scratch)) return s;
    return fldce_fwd_bwd(h, H, W, target, p_mask, N, total, grad_out, loss, loss_per_token, lse,
                         argmax, dH, dW, scratch, FLDCE_STATIC_SCRATCH_BYTES, err_count, stream);
}

int fldce_forward(fldce_handle h, const void* H, const void* W, const int64_t* target,
                  const float* p_mask, int64_t N, float total, float* loss, float* loss_per_token,
                  float* lse, int32_t* argmax, void* workspace, size_t workspace_bytes,
                  int32_t* err_count, void* stream) {
    fldce_call c{};
    c.H = H;
    c.W = W;
    c.target = target;
    c.p_mask = p_mask;
    c.N = N;
    c.total = total;
    c.grad_out = 1.f;
    c.loss = loss;
    c.loss_per_token = loss_per_token;
    c.lse = lse;
    c.argmax = argmax;
    c.workspace = workspace;
    c.workspace_bytes = workspace_bytes;
    c.err_count = err_count;
    c.stream = stream;
    return run(h, c, false);
}

int fldce_scale(void* x, int64_t n, int32_t dtype, const float* g, void* stream) {
    if (n < 0) return FLDCE_ERR_INVALID_ARG;
    if (n == 0) return FLDCE_OK;
    if (x == nullptr || g == nullptr) return FLDCE_ERR_INVALID_ARG;
    if (dtype != FLDCE_BF16 && dtype != FLDCE_FP32) return FLDCE_ERR_UNSUPPORTED;
    if (!aligned16(x)) return FLDCE_ERR_ALIGN;
    DeviceInfo dev;
    if (int s = check_device(&dev)) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(n / 8, 256), 8 * (int64_t)dev.sms));
    if (dtype == FLDCE_BF16)
        k_scale<__nv_bfloat16><<<blocks, 256, 0, st>>>(static_cast<__nv_bfloat16*>(x), n, g);
    else
        k_scale<float><<<blocks, 256, 0, st>>>(static_cast<float*>(x), n, g);
    return cudaGetLastError() == cudaSuccess ? FLDCE_OK : FLDCE_ERR_CUDA;
}

int fldce_selftest_wait(int64_t limit_ns, int32_t* status, void* stream) {
    if (status == nullptr) return FLDCE_ERR_INVALID_ARG;
    DeviceInfo dev;
    if (int s = check_device(&dev)) return s;
    const uint64_t lim = (uint64_t)std::min<int64_t>(std::max<int64_t>(limit_ns, 1000), 2000000000);
    k_selftest_wait<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(lim, status);
    return cudaGetLastError() == cudaSuccess ? FLDCE_OK : FLDCE_ERR_CUDA;
}

int fldce_profile_begin(fldce_handle h, int max_calls) {
    if (h == nullptr || max_calls <= 0) return FLDCE_ERR_INVALID_ARG;
    const int64_t chunks = cdiv(h->cfg.max_N, h->chunk);
    const size_t need = (size_t)max_calls * (size_t)(5 + 7 * chunks);
    while (h->ev.size() < need) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return FLDCE_ERR_CUDA;
        h->ev.push_back(e);
    }
    h->ev_kind.assign(h->ev.size(), PK_GAP);
    h->ev_used = 0;
    h->prof_on = true;
    return FLDCE_OK;
}

int fldce_profile_end(fldce_handle h, double* ms, int32_t* launches) {
    if (h == nullptr) return FLDCE_ERR_INVALID_ARG;
    double acc[FLDCE_PROF_KINDS] = {};
    int32_t cnt[FLDCE_PROF_KINDS] = {};
    h->prof_on = false;
    if (h->ev_used > 0 && cudaEventSynchronize(h->ev[h->ev_used - 1]) != cudaSuccess)
        return FLDCE_ERR_CUDA;
    for (size_t i = 1; i < h->ev_used; ++i) {
        const int k = h->ev_kind[i];
        if (k < 0) continue;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, h->ev[i - 1], h->ev[i]) != cudaSuccess) return FLDCE_ERR_CUDA;
        acc[k] += t;
        cnt[k] += 1;
    }
    for (int k = 0; k < FLDCE_PROF_KINDS; ++k) {
        if (ms != nullptr) ms[k] = acc[k];
        if (launches != nullptr) launches[k] = cnt[k];
    }
    h->ev_used = 0;
    return FLDCE_OK;
}

const char* fldce_profile_kind_name(int kind) {
    static const char* names[FLDCE_PROF_KINDS] = {"count_targets", "lse_sweep", "merge",
                                                  "g_sweep", "dh_gemm", "dw_gemm", "finish",
                                                  "convert", "db_colsum"};
    return (kind >= 0 && kind < FLDCE_PROF_KINDS) ? names[kind] : nullptr;
}

int fldce_destroy(fldce_handle h) {
    if (h != nullptr) {
        for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
    }
    delete h;
    return FLDCE_OK;
}

const char* fldce_strerror(int status) {
    switch (status) {
        case FLDCE_OK: return "ok";
        case FLDCE_ERR_INVALID_ARG: return "invalid argument";
        case FLDCE_ERR_UNSUPPORTED: return "unsupported configuration (dtype, flags or D % 8 != 0)";
        case FLDCE_ERR_WORKSPACE: return "workspace too small or not 256-byte aligned";
        case FLDCE_ERR_CUDA: return "CUDA runtime error or failed launch";
        case FLDCE_ERR_DEVICE: return "current device is not a compute capability 10.x GPU";
        case FLDCE_ERR_ALIGN: return "device pointer not 16-byte aligned";
        case FLDCE_ERR_TOO_LARGE:
            return "problem needs more scratch than the 64 MiB static buffer of "
                   "fldce_fwd_bwd_noalloc (use a smaller chunk_N, FLDCE_FLAG_DW_FP32, or "
                   "fldce_fwd_bwd with a workspace)";
        default: return "unknown status";
    }
}

int fldce_version(void) { return kVersion; }

}  // extern "C"
