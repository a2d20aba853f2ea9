// kernels.cuh -- epilogues of the tcgen05 GEMM, the per-row kernels, and the
// fp32 CUDA-core path of the fused linear diffusion cross-entropy.
//
// Notation (the page "fused_linear_diffusion_cross_entropy.py"): acc = <H[n], W[v]>
// is the raw fp32 accumulator, z = s * acc the logit, c = s * log2(e), so that
// t = acc * c = z * log2(e) lives in the base-2 domain where the hardware
// exponential ex2 works.  Running statistics are kept in that domain:
// m2 = max t, l = sum 2^(t - m2), and lse = (m2 + log2 l) * ln 2.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "umma_gemm.cuh"

namespace fldce {

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 lanes per instruction (sm_100 f32x2 arithmetic), each rounded to
// nearest exactly as the scalar operation would be.
__device__ __forceinline__ void mul2(float& x, float& y, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(x), "=f"(y) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void add2(float& x, float& y, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(x), "=f"(y) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void fma2(float& x, float& y, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(x), "=f"(y) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// max(a, b, c) in one instruction (sm_100 three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// The 32 bias values of columns [c0, c0 + 32) (0 past V), added to the raw
// accumulator before the logit scale: z = s (<H, W_v> + b_v), as the page's
// F.linear(x, weight, bias) followed by the scale.
__device__ __forceinline__ void load_bias32(const __nv_bfloat16* bias, int64_t c0, int64_t V,
                                            float (&b)[32]) {
    if (c0 + 32 <= V) {
        const uint4* q = reinterpret_cast<const uint4*>(bias + c0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint4 w = __ldg(q + k);
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
                b[8 * k + 2 * e] = f.x;
                b[8 * k + 2 * e + 1] = f.y;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) b[i] = (c0 + i < V) ? __bfloat162float(bias[c0 + i]) : 0.f;
    }
}

// Walk the NCH 32-column chunks of this thread's accumulator row with the
// next chunk's TMEM load in flight while the current one is processed;
// `f(r, j)` sees chunk j.  The accumulator is released to the MMA warp as
// soon as the last chunk has landed in registers.
template <int NCH, class F>
__device__ __forceinline__ void for_each_chunk(const AccRow& acc, F&& f) {
    static_assert(NCH % 2 == 0, "chunks come in pairs");
    uint32_t ra[32], rb[32];
    acc.load(0, ra);
#pragma unroll 1
    for (int j = 0; j < NCH; j += 2) {
        acc.issue(j + 1, rb);
        f(ra, j);
        acc.wait(rb);
        if (j + 2 < NCH) acc.issue(j + 2, ra); else acc.release();
        f(rb, j + 1);
        if (j + 2 < NCH) acc.wait(ra);
    }
}

// ======================================================================
// Epilogue 1 (sweep 1): per-row partial logsumexp of one 256-wide vocab tile.
// logsumexp_fwd_kernel keeps one (max, log-sum-exp) per row and vocab block;
// here each (row, vocab tile) keeps (m2, l) plus, when asked, the sum of the
// raw logits (label smoothing), the tile argmax, and the target logit when
// the target falls in the tile.  Columns >= V (TMA zero fill) are excluded.
// ======================================================================
struct LseEpi {
    struct Params {
        float c;                 // s * log2(e)
        float s;                 // logit scale
        int64_t V;
        int rows;                // tokens in this chunk
        int ld_part;             // row stride of the partial arrays (chunk capacity)
        const int64_t* target;   // chunk's targets
        float2* part_ml;         // [n_vt][ld_part] (m2, l)
        float* part_sz;          // [n_vt][ld_part] sum of acc, or null
        int32_t* part_am;        // [n_vt][ld_part] argmax column, or null
        float* zy;               // [ld_part] target logit z[n, y_n] log2(e)
        const __nv_bfloat16* bias;   // [V] or null
        int64_t v0;              // first vocabulary id of this shard (0 unsharded)
    };

    template <class Cfg>
    static __device__ __forceinline__ void run(const Params& p, const TileCtx& t,
                                               const AccRow& acc, Stager&) {
        const int m = t.row0 + t.row;
        const int64_t n0 = t.col0;
        const int nt = (int)(n0 / Cfg::BN);
        const bool live = m < (t.rows_dyn >= 0 ? t.rows_dyn : p.rows);
        int yrel = -1;
        if (live) {
            const int64_t y = p.target[m] - p.v0;      // shard-local column
            if (y >= n0 && y < n0 + Cfg::BN && y < p.V) yrel = (int)(y - n0);
        }
        const int ncols = (int)((p.V - n0) < Cfg::BN ? (p.V - n0) : Cfg::BN);
        const bool want_am = p.part_am != nullptr, want_sz = p.part_sz != nullptr;
        float mx = -CUDART_INF_F, l = 0.f, sz = 0.f, zyv = 0.f, amv = -CUDART_INF_F;
        int am = 0;
        static_assert(Cfg::NSUB == 1, "one 256-column MMA per vocabulary tile");
        for_each_chunk<Cfg::NCHUNK>(acc, [&](const uint32_t (&rin)[32], int j) {
            uint32_t r[32];
            if (p.bias != nullptr) {
                float b[32];
                load_bias32(p.bias, n0 + 32 * j, p.V, b);
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(rin[i]) + b[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = rin[i];
            }
            float tv[32];
#pragma unroll
            for (int i = 0; i < 32; i += 2)
                mul2(tv[i], tv[i + 1], __uint_as_float(r[i]), __uint_as_float(r[i + 1]), p.c, p.c);
            if (32 * j + 32 > ncols) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (32 * j + i >= ncols) tv[i] = -CUDART_INF_F;
            }
            float cm0 = fmaxf(tv[0], tv[1]), cm1 = fmaxf(tv[2], tv[3]);
#pragma unroll
            for (int i = 4; i < 32; i += 4) {
                cm0 = fmax3(cm0, tv[i], tv[i + 1]);
                cm1 = fmax3(cm1, tv[i + 2], tv[i + 3]);
            }
            const float nm = fmax3(mx, cm0, cm1);
            if (want_am) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (tv[i] > amv) { amv = tv[i]; am = 32 * j + i; }
            }
            if (want_sz) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    if (32 * j + i < ncols) a0 += __uint_as_float(r[i]);
                    if (32 * j + i + 1 < ncols) a1 += __uint_as_float(r[i + 1]);
                }
                sz += a0 + a1;
            }
            if ((unsigned)(yrel - 32 * j) < 32u) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i == yrel - 32 * j) zyv = __uint_as_float(r[i]);
            }
            float e0 = 0.f, e1 = 0.f, e2 = 0.f, e3 = 0.f;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float d0, d1, d2, d3;
                add2(d0, d1, tv[i], tv[i + 1], -nm, -nm);
                add2(d2, d3, tv[i + 2], tv[i + 3], -nm, -nm);
                add2(e0, e1, e0, e1, ex2(d0), ex2(d1));
                add2(e2, e3, e2, e3, ex2(d2), ex2(d3));
            }
            l = l * ex2(mx - nm) + ((e0 + e1) + (e2 + e3));
            mx = nm;
        });
        if (live) {
            const size_t o = (size_t)nt * p.ld_part + m;
            p.part_ml[o] = make_float2(mx, l);
            if (want_sz) p.part_sz[o] = sz;
            if (want_am) p.part_am[o] = (int32_t)(n0 + am);
            if (yrel >= 0) p.zy[m] = zyv * p.c;    // base 2, rounded like the maxima
        }
    }
};

// Pack 16 fp32 values of r (from r[off]) as bf16 into two 16-byte chunks.
__device__ __forceinline__ void pack16(const float* v, uint4& a, uint4& b) {
    a.x = pack_bf16x2(v[0], v[1]);
    a.y = pack_bf16x2(v[2], v[3]);
    a.z = pack_bf16x2(v[4], v[5]);
    a.w = pack_bf16x2(v[6], v[7]);
    b.x = pack_bf16x2(v[8], v[9]);
    b.y = pack_bf16x2(v[10], v[11]);
    b.z = pack_bf16x2(v[12], v[13]);
    b.w = pack_bf16x2(v[14], v[15]);
}

// Stage 32 bf16 values (chunk j of the row) into half of the 128-byte row
// segment; chunk pairs (2 jj, 2 jj + 1) form one 64-column store box.
__device__ __forceinline__ void stage_bf16_half(Stager& st, int j, const float (&v)[32]) {
    uint4 a, b, c, d;
    pack16(v, a, b);
    pack16(v + 16, c, d);
    const int base = (j & 1) * 4;
    st.put(base + 0, a);
    st.put(base + 1, b);
    st.put(base + 2, c);
    st.put(base + 3, d);
}

// ======================================================================
// Epilogue 2 (sweep 2): the gradient of the logits, rounded once to bf16.
// cross_entropy_kernel steps 5-6 and the backward's grad_out:
//   G = gcoef * (2^(t - lse2) - eps/V) - gcoef * (1 - eps) [v = y],
//   gcoef = g s / (p T), exactly 0 for ignored tokens and columns >= V.
// G leaves through the stager in 32-row x 64-column boxes (TMA store; the
// store map's extent clips rows past the chunk and columns past V).
// ======================================================================
struct GEpi {
    struct Params {
        CUtensorMap gmap;        // G [rows, V] bf16, box 64 x 32, 128B swizzle
        float c;
        int64_t V;
        int rows;
        const float* lse2;       // [chunk] lse in base-2 units
        const float* gcoef;      // [chunk]
        const int32_t* ycol;     // [chunk] validated target or -1
        float eps_over_V;
        float one_minus_eps;
        const __nv_bfloat16* bias;   // [V] or null
    };

    // What one thread needs for its row of a vocabulary tile starting at n0.
    struct Row {
        float gc, L2, base, tcorr;
        int yrel, ncols;
    };

    template <int BN>
    static __device__ __forceinline__ Row row_setup(const Params& p, int m, int rows_dyn,
                                                    int64_t n0) {
        Row w;
        w.gc = 0.f;
        w.L2 = 0.f;
        w.yrel = -1;
        if (m < (rows_dyn >= 0 ? rows_dyn : p.rows)) {
            w.gc = p.gcoef[m];
            if (w.gc != 0.f) {
                w.L2 = p.lse2[m];
                const int y = p.ycol[m];
                if (y >= n0 && y < n0 + BN) w.yrel = (int)(y - n0);
            }
        }
        w.base = w.gc * p.eps_over_V;
        w.tcorr = w.gc * p.one_minus_eps;
        w.ncols = (int)((p.V - n0) < BN ? (p.V - n0) : BN);
        return w;
    }

    // G of columns [n0 + 32 j, n0 + 32 j + 32) of the row from its raw
    // accumulator values r (bias added first when there is one).
    static __device__ __forceinline__ void chunk(const Params& p, const Row& w,
                                                 const uint32_t (&r)[32], int64_t n0, int j,
                                                 float (&g)[32]) {
        const float gc = w.gc, L2 = w.L2, base = w.base;
        if (p.bias != nullptr) {
            float b[32];
            load_bias32(p.bias, n0 + 32 * j, p.V, b);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                float a0, a1, t0, t1;
                add2(a0, a1, __uint_as_float(r[i]), __uint_as_float(r[i + 1]), b[i], b[i + 1]);
                fma2(t0, t1, a0, a1, p.c, p.c, -L2, -L2);
                fma2(g[i], g[i + 1], gc, gc, ex2(t0), ex2(t1), -base, -base);
            }
            if (gc == 0.f) {
#pragma unroll
                for (int i = 0; i < 32; ++i) g[i] = 0.f;
            }
        } else if (gc != 0.f) {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                float t0, t1;
                fma2(t0, t1, __uint_as_float(r[i]), __uint_as_float(r[i + 1]), p.c, p.c, -L2,
                     -L2);
                fma2(g[i], g[i + 1], gc, gc, ex2(t0), ex2(t1), -base, -base);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] = 0.f;
        }
        if ((unsigned)(w.yrel - 32 * j) < 32u) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (i == w.yrel - 32 * j) g[i] -= w.tcorr;
        }
        if (32 * j + 32 > w.ncols) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (32 * j + i >= w.ncols) g[i] = 0.f;
        }
    }

    template <class Cfg>
    static __device__ __forceinline__ void run(const Params& p, const TileCtx& t,
                                               const AccRow& acc, Stager& st) {
        const int64_t n0 = t.col0;
        const Row w = row_setup<Cfg::BN>(p, t.row0 + t.row, t.rows_dyn, n0);
        static_assert(Cfg::NSUB == 1, "one 256-column MMA per vocabulary tile");
        for_each_chunk<Cfg::NCHUNK>(acc, [&](const uint32_t (&r)[32], int j) {
            float g[32];
            chunk(p, w, r, n0, j, g);
            if ((j & 1) == 0) st.acquire();
            stage_bf16_half(st, j, g);
            if (j & 1) st.flush(&p.gmap, (int)(n0 + 32 * (j - 1)), t.row0 + 32 * t.q, false);
        });
    }
};

// ======================================================================
// Epilogue 3: dH / dW tiles.
//   OUT_BF16: bf16 output, 64-column boxes, TMA store;
//   WS_STORE / WS_ADD: fp32 32-column boxes, TMA store or TMA reduce-add
//   (dW accumulated over token chunks).
// A GEMM split over K (dH over vocabulary ranges) stores split j's tile
// split_rows * j rows further down, so every split owns a partial buffer
// that a later pass sums in a fixed order.
// ======================================================================
enum StoreMode { OUT_BF16 = 0, WS_STORE = 1, WS_ADD = 2 };

struct StoreEpi {
    struct Params {
        CUtensorMap omap;        // bf16 [rows, cols] box 64 x 32, or fp32 box 32 x 32
        int mode;
        int split_rows = 0;      // row offset between K splits' partial buffers
    };

    template <class Cfg>
    static __device__ __forceinline__ void run(const Params& p, const TileCtx& t,
                                               const AccRow& acc, Stager& st) {
        const int64_t n0 = t.col0;
        const int y = t.row0 + t.split * p.split_rows + 32 * t.q;
        const int mode = p.mode;
        for_each_chunk<Cfg::NCHUNK>(acc, [&](const uint32_t (&r)[32], int j) {
            if (mode == OUT_BF16) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
                if ((j & 1) == 0) st.acquire();
                stage_bf16_half(st, j, v);
                if (j & 1) st.flush(&p.omap, (int)(n0 + 32 * (j - 1)), y, false);
            } else {
                st.acquire();
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st.put(c, make_uint4(r[4 * c], r[4 * c + 1], r[4 * c + 2], r[4 * c + 3]));
                st.flush(&p.omap, (int)(n0 + 32 * j), y, mode == WS_ADD);
            }
        });
    }
};

// ======================================================================
// Row kernels shared by both element types.
// ======================================================================
struct Counters {
    int32_t n_valid;   // targets != ignore_index and inside [0, V)
    int32_t n_err;     // targets != ignore_index outside [0, V)
    int32_t dev_err;   // FLDCE_DEV_ERR_* bits raised by kernels
    int32_t n_compact; // compacted tokens (FLDCE_FLAG_SKIP_IGNORED)
};

// Targets are read two at a time as 16-byte vectors (longlong2).  An int64
// array is 8-byte aligned, so at most its first element sits before the
// first 16-byte boundary: that element and an odd last one are read alone.
struct TargetPairs {
    const int64_t* head;       // the element before the first boundary, or null
    const longlong2* pairs;    // 16-byte aligned pairs
    int64_t n_pairs;
    const int64_t* tail;       // a last unpaired element, or null

    __device__ __forceinline__ TargetPairs(const int64_t* t, int64_t N) {
        const int64_t h = (N > 0 && (reinterpret_cast<uintptr_t>(t) & 15u) != 0) ? 1 : 0;
        head = h ? t : nullptr;
        pairs = reinterpret_cast<const longlong2*>(t + h);
        n_pairs = (N - h) / 2;
        tail = ((N - h) & 1) ? t + N - 1 : nullptr;
    }
};

// Count the tokens that carry a loss (the page's target.ne(ignore_index).sum(),
// without the host round trip) and the malformed targets.
__global__ void k_count_targets(const int64_t* __restrict__ target, int64_t N, int64_t V,
                                int64_t ignore_index, Counters* cnt) {
    int valid = 0, bad = 0;
    auto take = [&](int64_t y) {
        if (y != ignore_index) {
            if (y >= 0 && y < V) ++valid; else ++bad;
        }
    };
    const TargetPairs tp(target, N);
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    for (int64_t i = tid; i < tp.n_pairs; i += (int64_t)gridDim.x * blockDim.x) {
        const longlong2 v = tp.pairs[i];
        take(v.x);
        take(v.y);
    }
    if (tid == 0) {
        if (tp.head != nullptr) take(*tp.head);
        if (tp.tail != nullptr) take(*tp.tail);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        valid += __shfl_xor_sync(0xffffffffu, valid, o);
        bad += __shfl_xor_sync(0xffffffffu, bad, o);
    }
    if ((threadIdx.x & 31) == 0) {
        if (valid) atomicAdd(&cnt->n_valid, valid);
        if (bad) atomicAdd(&cnt->n_err, bad);
    }
}

// Stable compaction of the tokens that carry a loss (one block): idx lists
// their positions in increasing order, pos maps a position to its compacted
// row (or -1), *count = how many.  Skipping the rest changes no result: an
// ignored token's loss is 0, its dH row is 0 and it adds nothing to dW.
__global__ void k_compact_valid(const int64_t* __restrict__ target, int64_t N, int64_t V,
                                int64_t ignore_index, int32_t* __restrict__ idx,
                                int32_t* __restrict__ pos, int32_t* count) {
    __shared__ int warp_tot[32];
    const int T = blockDim.x;
    // even segments, so that on a 16-byte aligned array every segment starts
    // on a pair boundary and is read as longlong2 vectors
    int64_t seg = (N + T - 1) / T;
    seg += seg & 1;
    const bool vec = (reinterpret_cast<uintptr_t>(target) & 15u) == 0;
    const int64_t a = min(N, threadIdx.x * seg);
    const int64_t b = min(N, a + seg);
    auto ok = [&](int64_t y) { return y != ignore_index && y >= 0 && y < V; };
    // the targets of positions i and i + 1 (the second only when i + 1 < b)
    auto pair_at = [&](int64_t i, int64_t& y0, int64_t& y1) {
        if (vec && i + 1 < b) {
            const longlong2 v = *reinterpret_cast<const longlong2*>(target + i);
            y0 = v.x;
            y1 = v.y;
        } else {
            y0 = target[i];
            y1 = i + 1 < b ? target[i + 1] : ignore_index;
        }
    };
    int c = 0;
    for (int64_t i = a; i < b; i += 2) {
        int64_t y0, y1;
        pair_at(i, y0, y1);
        c += (ok(y0) ? 1 : 0) + (i + 1 < b && ok(y1) ? 1 : 0);
    }
    // exclusive scan of c over the block
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[w] = incl;
    __syncthreads();
    if (w == 0) {
        int v = lane < (T >> 5) ? warp_tot[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += t;
        }
        warp_tot[lane] = v;    // inclusive totals per warp
    }
    __syncthreads();
    int off = incl - c + (w > 0 ? warp_tot[w - 1] : 0);
    for (int64_t i = a; i < b; i += 2) {
        int64_t y[2];
        pair_at(i, y[0], y[1]);
        for (int k = 0; k < 2 && i + k < b; ++k) {
            if (ok(y[k])) {
                idx[off] = (int32_t)(i + k);
                pos[i + k] = off++;
            } else {
                pos[i + k] = -1;
            }
        }
    }
    if (threadIdx.x == T - 1) *count = off;
}

// Gather the compacted rows: Hc[i] = H[idx[i]], yc, pc.  The 256 rows after
// the count are zero-filled: a chunk's last GEMM tile may read up to 255
// rows past it, and zeros (not stale workspace bits) keep them out of dW.
__global__ void k_gather_rows(const __nv_bfloat16* __restrict__ H, const int64_t* __restrict__ y,
                              const float* __restrict__ p, const int32_t* __restrict__ idx,
                              const int32_t* count, int64_t N, int64_t D,
                              __nv_bfloat16* __restrict__ Hc, int64_t* __restrict__ yc,
                              float* __restrict__ pc) {
    const int n = *count;
    const int64_t lim = min(N, (int64_t)n + 256);
    const int64_t per_row = D / 8;                 // 16-byte vectors per row
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < lim * per_row;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / per_row, c = e - i * per_row;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (i < n) v = reinterpret_cast<const uint4*>(H + (int64_t)idx[i] * D)[c];
        reinterpret_cast<uint4*>(Hc + i * D)[c] = v;
        if (c == 0) {
            yc[i] = i < n ? y[idx[i]] : (int64_t)-1;
            pc[i] = i < n ? (p != nullptr ? p[idx[i]] : 1.f) : 1.f;
        }
    }
}

// Scatter back: dH[i] = dHc[pos[i]] (zero row for skipped tokens), and the
// per-token outputs (loss 0, lse NaN, argmax -1 for skipped tokens).
__global__ void k_scatter_rows(const int32_t* __restrict__ pos, int64_t N, int64_t D,
                               const __nv_bfloat16* __restrict__ dHc, __nv_bfloat16* __restrict__ dH,
                               const float* __restrict__ loss_c, float* loss_out,
                               const float* __restrict__ lse_c, float* lse_out,
                               const int32_t* __restrict__ am_c, int32_t* am_out) {
    const int64_t per_row = D / 8;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < N * per_row;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / per_row, c = e - i * per_row;
        const int32_t q = pos[i];
        if (dH != nullptr) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (q >= 0) v = reinterpret_cast<const uint4*>(dHc + (int64_t)q * D)[c];
            reinterpret_cast<uint4*>(dH + i * D)[c] = v;
        }
        if (c == 0) {
            if (loss_out != nullptr) loss_out[i] = q >= 0 ? loss_c[q] : 0.f;
            if (lse_out != nullptr) lse_out[i] = q >= 0 ? lse_c[q] : CUDART_NAN_F;
            if (am_out != nullptr) am_out[i] = q >= 0 ? am_c[q] : -1;
        }
    }
}

// When no token carries a loss, the dW GEMM has no K rows and writes nothing:
// zero its destination instead (a no-op otherwise).
__global__ void k_zero_if_none(const int32_t* count, void* dst, int64_t bytes16) {
    if (*count != 0) return;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < bytes16;
         i += (int64_t)gridDim.x * blockDim.x)
        reinterpret_cast<uint4*>(dst)[i] = make_uint4(0, 0, 0, 0);
}

// The valid count alone, for fldce_count_valid (count zeroed by the caller).
__global__ void k_count_valid_only(const int64_t* __restrict__ target, int64_t N, int64_t V,
                                   int64_t ignore_index, int32_t* count) {
    int valid = 0;
    auto take = [&](int64_t y) { valid += (y != ignore_index && y >= 0 && y < V) ? 1 : 0; };
    const TargetPairs tp(target, N);
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    for (int64_t i = tid; i < tp.n_pairs; i += (int64_t)gridDim.x * blockDim.x) {
        const longlong2 v = tp.pairs[i];
        take(v.x);
        take(v.y);
    }
    if (tid == 0) {
        if (tp.head != nullptr) take(*tp.head);
        if (tp.tail != nullptr) take(*tp.tail);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) valid += __shfl_xor_sync(0xffffffffu, valid, o);
    if ((threadIdx.x & 31) == 0 && valid) atomicAdd(count, valid);
}

enum MergeMode { MERGE_LOCAL = 0, MERGE_EMIT_STATS = 1, MERGE_GATHERED = 2 };

struct MergeParams {
    int mode;                 // MergeMode
    int64_t v0, Vtot;         // shard offset and total vocabulary (0, V unsharded)
    float* stats_out;         // MERGE_EMIT_STATS: [.][8] rows for this chunk
    const float* all_stats;   // MERGE_GATHERED: [n_shards][stats_N][8]
    int n_shards;
    int64_t stats_N;          // tokens per shard's stats block
    int64_t stats_row0;       // first token of this chunk
    int rows;                 // tokens in this chunk (with dyn_count: the capacity)
    const int32_t* dyn_count; // compacted-token count, or null
    int dyn_base;             // first compacted row of this chunk
    int ld_part;              // partial row stride
    int n_vt;                 // vocab tiles
    int64_t V;
    int64_t ignore_index;
    float s, eps, total, grad_out;
    const int64_t* target;    // chunk's targets
    const float* p_mask;      // chunk's p_mask or null
    const float2* part_ml;
    const float* part_sz;     // null when eps == 0
    const int32_t* part_am;   // null when argmax is not wanted
    const float* zy;
    const Counters* cnt;
    const int32_t* count_dev; // job-wide valid count supplied by the caller, or null
    float* loss_tok;          // chunk's per-token loss
    float* lse_out;           // chunk's lse output or null
    int32_t* am_out;          // chunk's argmax output or null
    float* row_lse2;          // [chunk] for sweep 2 (null in forward-only mode)
    float* row_gcoef;
    int32_t* row_y;
    // 1 when target, p_mask and every per-token output above start on a
    // 16-byte boundary: groups of four rows then move as 128-bit vectors
    int vec;
};

// What the merge writes for one token.
struct MergedRow {
    float loss, lse, lse2, gcoef;
    int32_t am, y;            // argmax; validated shard-local target or -1
};

// Threads per row of the split-V merge: each takes every kMergeSub-th vocab
// tile in one online pass; the kMergeSub partial (max, sum) pairs of a row are
// then combined with shuffles in a fixed order (deterministic).
constexpr int kMergeSub = 8;

// The per-token outputs of row m from its merged statistics (base-2 maximum
// M2 and sum L, best vocabulary tile, sum of raw logits): the loss of
// cross_entropy_kernel step 4 with the label-smoothing block, and the
// gradient coefficient of steps 5-6.  y and pm are the row's target and
// p_mask (pm is read only for a token that carries a loss).
__device__ __forceinline__ MergedRow merge_finish_row(const MergeParams& p, int m, float M2,
                                                      float L, int kbest, float szs, int64_t y,
                                                      float pm) {
    const int64_t gm = p.stats_row0 + m;
    const bool valid = (y != p.ignore_index) && y >= 0 && y < p.Vtot;
    const bool local_y = valid && y - p.v0 >= 0 && y - p.v0 < p.V;
    float zyv = 0.f, szv = 0.f;
    int32_t am = -1;
    if (p.mode != MERGE_GATHERED) {
        if (local_y) zyv = p.zy[m];
        szv = p.s * szs;
        if (p.part_am != nullptr) am = p.part_am[(size_t)kbest * p.ld_part + m] + (int32_t)p.v0;
    } else {
        // every shard's statistics, merged in shard order (split softmax:
        // lse = M + log2 sum_r l_r 2^(m_r - M); the target logit and the
        // logit sums add over shards; ties go to the lowest shard)
        int rbest = 0;
        for (int r = 0; r < p.n_shards; ++r) {
            const float v = p.all_stats[((size_t)r * p.stats_N + gm) * 8];
            if (v > M2) { M2 = v; rbest = r; }
        }
        for (int r = 0; r < p.n_shards; ++r) {
            const float* st = p.all_stats + ((size_t)r * p.stats_N + gm) * 8;
            L += st[1] * exp2f(st[0] - M2);
            zyv += st[2];
            szv += st[3];
        }
        am = __float_as_int(p.all_stats[((size_t)rbest * p.stats_N + gm) * 8 + 4]);
    }
    MergedRow o;
    o.lse2 = M2 + log2f(L);
    o.lse = o.lse2 * 0.69314718055994530942f;
    o.am = am;
    o.loss = 0.f;
    o.gcoef = 0.f;
    if (valid) {
        const float T = p.total > 0.f ? p.total
                        : (float)(p.count_dev != nullptr ? *p.count_dev : p.cnt->n_valid);
        const float coef = 1.f / (pm * T);
        // lse - z_y taken in base 2, where both carry the same rounding of
        // acc * s * log2(e) (exactly 0 when the target is the only column)
        float ce = (o.lse2 - zyv) * 0.69314718055994530942f;
        if (p.eps > 0.f) ce = (1.f - p.eps) * ce + p.eps * (o.lse - szv / (float)p.Vtot);
        o.loss = ce * coef;
        o.gcoef = p.grad_out * p.s * coef;
    }
    o.y = local_y ? (int32_t)(y - p.v0) : -1;
    return o;
}

// Split-V merge: lse = M + log sum_k l_k 2^(m_k - M) (logsumexp_fwd's second
// logsumexp; the tensor-parallel tutorial's sum of per-shard denominators),
// then the per-token loss (cross_entropy_kernel step 4 and the
// label-smoothing block) and the per-token gradient coefficient.
//
// A warp covers four consecutive rows (8 lanes each).  Where the four rows
// are all live and the pointers allow it, the warp reads their targets as two
// longlong2 and their p_mask as one float4, and writes each per-token output
// of the four rows as one 128-bit store, a different lane per output;
// otherwise the first lane of each row reads and writes its row alone.
__global__ void __launch_bounds__(256) k_merge_rows(MergeParams p) {
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const int m = tid / kMergeSub;
    const int g = tid % kMergeSub;
    const int live_rows = p.dyn_count != nullptr
                              ? max(0, min(p.rows, *p.dyn_count - p.dyn_base)) : p.rows;
    const bool live = m < live_rows;
    const bool dead_dyn = m < p.rows && !live;
    float M2 = -CUDART_INF_F, L = 0.f, szs = 0.f;
    int kbest = 0x7fffffff;
    if (live && p.mode != MERGE_GATHERED) {
        for (int k = g; k < p.n_vt; k += kMergeSub) {
            const float2 ml = p.part_ml[(size_t)k * p.ld_part + m];
            if (ml.x > M2) {
                L = L * exp2f(M2 - ml.x) + ml.y;
                M2 = ml.x;
                kbest = k;
            } else {
                L += ml.y * exp2f(ml.x - M2);
            }
            if (p.part_sz != nullptr) szs += p.part_sz[(size_t)k * p.ld_part + m];
        }
    }
    // combine the kMergeSub lanes of the row (all lanes take part)
#pragma unroll
    for (int o = 1; o < kMergeSub; o <<= 1) {
        const float Mo = __shfl_xor_sync(0xffffffffu, M2, o);
        const float Lo = __shfl_xor_sync(0xffffffffu, L, o);
        const int ko = __shfl_xor_sync(0xffffffffu, kbest, o);
        const float so = __shfl_xor_sync(0xffffffffu, szs, o);
        const float Mn = fmaxf(M2, Mo);
        const float a = (M2 == -CUDART_INF_F) ? 0.f : L * exp2f(M2 - Mn);
        const float b = (Mo == -CUDART_INF_F) ? 0.f : Lo * exp2f(Mo - Mn);
        kbest = (Mo > M2 || (Mo == M2 && ko < kbest)) ? ko : kbest;
        L = a + b;
        M2 = Mn;
        szs += so;
    }

    // the same for every lane of the warp: its four rows are all live
    const int m0 = m & ~3;
    const bool vec = p.vec != 0 && p.mode != MERGE_EMIT_STATS && m0 + 3 < live_rows;
    if (vec) {
        const uint32_t full = 0xffffffffu;
        const int r = lane >> 3;                 // this lane's row within the four
        longlong2 tq = make_longlong2(0, 0);
        float4 pq = make_float4(1.f, 1.f, 1.f, 1.f);
        if (lane == 1 || lane == 2) tq = reinterpret_cast<const longlong2*>(p.target + m0)[lane - 1];
        if (lane == 0 && p.p_mask != nullptr) pq = *reinterpret_cast<const float4*>(p.p_mask + m0);
        // rows 0, 1 come from lane 1's pair, rows 2, 3 from lane 2's
        const long long t0 = __shfl_sync(full, tq.x, 1), t1 = __shfl_sync(full, tq.y, 1);
        const long long t2 = __shfl_sync(full, tq.x, 2), t3 = __shfl_sync(full, tq.y, 2);
        const float q0 = __shfl_sync(full, pq.x, 0), q1 = __shfl_sync(full, pq.y, 0);
        const float q2 = __shfl_sync(full, pq.z, 0), q3 = __shfl_sync(full, pq.w, 0);
        const int64_t y = r == 0 ? t0 : (r == 1 ? t1 : (r == 2 ? t2 : t3));
        const float pm = r == 0 ? q0 : (r == 1 ? q1 : (r == 2 ? q2 : q3));
        const MergedRow o = merge_finish_row(p, m, M2, L, kbest, szs, y, pm);
        auto g4f = [&](float v) {
            return make_float4(__shfl_sync(full, v, 0), __shfl_sync(full, v, 8),
                               __shfl_sync(full, v, 16), __shfl_sync(full, v, 24));
        };
        auto g4i = [&](int32_t v) {
            return make_int4(__shfl_sync(full, v, 0), __shfl_sync(full, v, 8),
                             __shfl_sync(full, v, 16), __shfl_sync(full, v, 24));
        };
        const float4 loss4 = g4f(o.loss), lse4 = g4f(o.lse);
        const float4 l24 = g4f(o.lse2), gc4 = g4f(o.gcoef);
        const int4 am4 = g4i(o.am), y4 = g4i(o.y);
        if (lane == 0) *reinterpret_cast<float4*>(p.loss_tok + m0) = loss4;
        if (lane == 1 && p.lse_out != nullptr) *reinterpret_cast<float4*>(p.lse_out + m0) = lse4;
        if (lane == 2 && p.am_out != nullptr) *reinterpret_cast<int4*>(p.am_out + m0) = am4;
        if (p.row_lse2 != nullptr) {
            if (lane == 3) *reinterpret_cast<float4*>(p.row_lse2 + m0) = l24;
            if (lane == 4) *reinterpret_cast<float4*>(p.row_gcoef + m0) = gc4;
            if (lane == 5) *reinterpret_cast<int4*>(p.row_y + m0) = y4;
        }
        return;
    }

    if (g != 0 || m >= p.rows) return;
    if (dead_dyn) {
        // past the compacted tokens: no loss, zero gradient row
        p.loss_tok[m] = 0.f;
        if (p.row_lse2 != nullptr) {
            p.row_lse2[m] = 0.f;
            p.row_gcoef[m] = 0.f;
            p.row_y[m] = -1;
        }
        return;
    }
    const int64_t y = p.target[m];
    const bool valid = (y != p.ignore_index) && y >= 0 && y < p.Vtot;
    const float pm = (valid && p.p_mask != nullptr) ? p.p_mask[m] : 1.f;
    if (p.mode == MERGE_EMIT_STATS) {
        // this shard's statistics of the token: 32 bytes, two 128-bit stores
        const bool local_y = valid && y - p.v0 >= 0 && y - p.v0 < p.V;
        const int32_t am = p.part_am != nullptr
                               ? p.part_am[(size_t)kbest * p.ld_part + m] + (int32_t)p.v0 : -1;
        float4* o = reinterpret_cast<float4*>(p.stats_out + (size_t)(p.stats_row0 + m) * 8);
        o[0] = make_float4(M2, L, local_y ? p.zy[m] : 0.f, p.s * szs);
        o[1] = make_float4(__int_as_float(am), 0.f, 0.f, 0.f);
        return;
    }
    const MergedRow o = merge_finish_row(p, m, M2, L, kbest, szs, y, pm);
    p.loss_tok[m] = o.loss;
    if (p.lse_out != nullptr) p.lse_out[m] = o.lse;
    if (p.am_out != nullptr) p.am_out[m] = o.am;
    if (p.row_lse2 != nullptr) {
        p.row_lse2[m] = o.lse2;
        p.row_gcoef[m] = o.gcoef;
        p.row_y[m] = o.y;
    }
}

// loss = sum_n loss[n] in a fixed order (one block, fp64 partials), so the
// scalar is bit-reproducible run to run; also publishes the malformed-target
// count and the device error bits (a timed-out wait) in err_count[0..1].
// The per-token losses are read as float4 from the first 16-byte boundary
// on; the up to three elements before it and the ragged end are added by
// thread 0.
__global__ void k_finish(const float* __restrict__ loss_tok, int64_t N, const Counters* cnt,
                         float* loss, int32_t* err_count) {
    __shared__ double red[1024];
    const uintptr_t mis = reinterpret_cast<uintptr_t>(loss_tok) & 15u;
    const int64_t h = min(N, mis != 0 ? (int64_t)((16u - mis) / 4u) : (int64_t)0);
    const int64_t n4 = (N - h) / 4;
    const float4* q = reinterpret_cast<const float4*>(loss_tok + h);
    double acc = 0.0;
    for (int64_t i = threadIdx.x; i < n4; i += blockDim.x) {
        const float4 v = q[i];
        acc += ((double)v.x + (double)v.y) + ((double)v.z + (double)v.w);
    }
    if (threadIdx.x == 0) {
        for (int64_t i = 0; i < h; ++i) acc += (double)loss_tok[i];
        for (int64_t i = h + 4 * n4; i < N; ++i) acc += (double)loss_tok[i];
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        *loss = (float)red[0];
        if (err_count != nullptr) {
            err_count[0] = cnt->n_err;
            err_count[1] = cnt->dev_err;
        }
    }
}

// fp32 -> bf16 (round to nearest even), 8 elements per thread and step;
// with add, dst = bf16(dst + src) (an accumulated gradient, rounded once).
__global__ void k_f32_to_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                              int64_t n8, int add) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 a = reinterpret_cast<const float4*>(src)[2 * i];
        float4 b = reinterpret_cast<const float4*>(src)[2 * i + 1];
        if (add) {
            const uint4 o = reinterpret_cast<const uint4*>(dst)[i];
            const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.x));
            const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.y));
            const float2 o2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.z));
            const float2 o3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.w));
            a.x += o0.x; a.y += o0.y; a.z += o1.x; a.w += o1.y;
            b.x += o2.x; b.y += o2.y; b.z += o3.x; b.w += o3.y;
        }
        uint4 w;
        w.x = pack_bf16x2(a.x, a.y);
        w.y = pack_bf16x2(a.z, a.w);
        w.z = pack_bf16x2(b.x, b.y);
        w.w = pack_bf16x2(b.z, b.w);
        reinterpret_cast<uint4*>(dst)[i] = w;
    }
}

// out[i] = sum_j part[j * stride + i], j = 0 .. k-1 in that order (the K
// splits of one GEMM), so the result does not depend on which split
// finished first.  n8 = elements / 8.
template <class OutT>
__global__ void k_sum_splits(const float* __restrict__ part, int64_t stride, int k,
                             OutT* __restrict__ out, int64_t n8) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 a = reinterpret_cast<const float4*>(part)[2 * i];
        float4 b = reinterpret_cast<const float4*>(part)[2 * i + 1];
        for (int j = 1; j < k; ++j) {
            const float4* q = reinterpret_cast<const float4*>(part + j * stride);
            const float4 c = q[2 * i], d = q[2 * i + 1];
            a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
            b.x += d.x; b.y += d.y; b.z += d.z; b.w += d.w;
        }
        if constexpr (sizeof(OutT) == 2) {
            uint4 w;
            w.x = pack_bf16x2(a.x, a.y);
            w.y = pack_bf16x2(a.z, a.w);
            w.z = pack_bf16x2(b.x, b.y);
            w.w = pack_bf16x2(b.z, b.w);
            reinterpret_cast<uint4*>(out)[i] = w;
        } else {
            reinterpret_cast<float4*>(out)[2 * i] = a;
            reinterpret_cast<float4*>(out)[2 * i + 1] = b;
        }
    }
}

// One CTA waits, bounded, on an mbarrier that never completes its phase.
__global__ void k_selftest_wait(uint64_t limit_ns, int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool done = mbar_wait_bounded(smem_u32(&bar), 0u, limit_ns);
    __syncthreads();
    if (threadIdx.x == 0) *status = done ? 0 : FLDCE_DEV_ERR_TIMEOUT;
}

// x *= *g in place, 8 elements per thread and step; nothing to do when *g == 1.
template <class T>
__global__ void k_scale(T* __restrict__ x, int64_t n, const float* __restrict__ g) {
    const float gv = *g;
    if (gv == 1.f) return;
    const int64_t n8 = n / 8;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
         i += (int64_t)gridDim.x * blockDim.x) {
        if constexpr (sizeof(T) == 2) {
            uint4 w = reinterpret_cast<uint4*>(x)[i];
            uint32_t* u = &w.x;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u[k]);
                const float2 f = __bfloat1622float2(v);
                u[k] = pack_bf16x2(f.x * gv, f.y * gv);
            }
            reinterpret_cast<uint4*>(x)[i] = w;
        } else {
            float4 a = reinterpret_cast<float4*>(x)[2 * i];
            float4 b = reinterpret_cast<float4*>(x)[2 * i + 1];
            a.x *= gv; a.y *= gv; a.z *= gv; a.w *= gv;
            b.x *= gv; b.y *= gv; b.z *= gv; b.w *= gv;
            reinterpret_cast<float4*>(x)[2 * i] = a;
            reinterpret_cast<float4*>(x)[2 * i + 1] = b;
        }
    }
    // the tail (n % 8 elements), one thread
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int64_t i = n8 * 8; i < n; ++i) {
            if constexpr (sizeof(T) == 2) {
                x[i] = __float2bfloat16_rn(__bfloat162float(x[i]) * gv);
            } else {
                x[i] = x[i] * gv;
            }
        }
    }
}

// db: column sums of G (the page's db += dlogits.sum(0)) in a fixed order.
// Pass 1: each thread sums two adjacent columns over one segment of rows.
template <class T>
__global__ void k_colsum_partial(const T* __restrict__ G, int64_t ldg, int rows, int64_t V,
                                 int seg_rows, float* __restrict__ part,
                                 const int32_t* dyn_count, int dyn_base) {
    const int64_t v = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (v >= V) return;
    if (dyn_count != nullptr) rows = max(0, min(rows, *dyn_count - dyn_base));
    const int r0 = blockIdx.y * seg_rows;
    const int r1 = min(rows, r0 + seg_rows);
    float a0 = 0.f, a1 = 0.f;
    for (int r = r0; r < r1; ++r) {
        const T* row = G + (size_t)r * ldg + v;
        if constexpr (sizeof(T) == 2) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row));
            a0 += f.x;
            a1 += f.y;
        } else {
            a0 += row[0];
            a1 += row[1];
        }
    }
    part[(size_t)blockIdx.y * V + v] = a0;
    if (v + 1 < V) part[(size_t)blockIdx.y * V + v + 1] = a1;
}

// Pass 2: db_acc[v] (=, or +=) sum of the segment partials, in segment order.
__global__ void k_colsum_final(const float* __restrict__ part, int nseg, int64_t V,
                               float* __restrict__ acc, int add) {
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= V) return;
    float s = 0.f;
    for (int k = 0; k < nseg; ++k) s += part[(size_t)k * V + v];
    acc[v] = add ? acc[v] + s : s;
}

// fp32 -> bf16 or fp32 copy, one element per thread (short vectors, any n);
// with add, dst += src (rounded once to the output type).
__global__ void k_cast_out(const float* __restrict__ src, void* dst, int64_t n, int to_bf16,
                           int add) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    if (to_bf16) {
        __nv_bfloat16* d = static_cast<__nv_bfloat16*>(dst);
        d[i] = __float2bfloat16_rn(add ? src[i] + __bfloat162float(d[i]) : src[i]);
    } else {
        float* d = static_cast<float*>(dst);
        d[i] = add ? src[i] + d[i] : src[i];
    }
}

// ======================================================================
// fp32 CUDA-core path: a 64x64-tile SIMT GEMM whose tile is staged in shared
// memory and handed to an epilogue.  Used for the fp32 element type, where
// the tensor cores' tf32 would not meet fp32 accuracy.
// ======================================================================
constexpr int kSimtTile = 64;

struct SimtLse {
    LseEpi::Params p;
    const float* bias;        // [V] fp32 or null
    __device__ void operator()(float (*C)[kSimtTile + 1], int m0, int64_t n0, int nt) const {
        const int r = threadIdx.x;
        if (r >= kSimtTile) return;
        const int m = m0 + r;
        if (m >= p.rows) return;
        const int ncols = (int)((p.V - n0) < kSimtTile ? (p.V - n0) : kSimtTile);
        if (bias != nullptr)
            for (int i = 0; i < ncols; ++i) C[r][i] += bias[n0 + i];
        float mx = -CUDART_INF_F, sz = 0.f;
        int am = 0;
        for (int i = 0; i < ncols; ++i) {
            const float t = C[r][i] * p.c;
            if (t > mx) { mx = t; am = i; }
            sz += C[r][i];
        }
        float l = 0.f;
        for (int i = 0; i < ncols; ++i) l += exp2f(C[r][i] * p.c - mx);
        const size_t o = (size_t)nt * p.ld_part + m;
        p.part_ml[o] = make_float2(mx, l);
        if (p.part_sz != nullptr) p.part_sz[o] = sz;
        if (p.part_am != nullptr) p.part_am[o] = (int32_t)(n0 + am);
        const int64_t y = p.target[m] - p.v0;
        if (y >= n0 && y < n0 + ncols) p.zy[m] = C[r][y - n0] * p.c;
    }
};

struct SimtG {
    float c;
    int64_t V, ldg;
    int rows;
    const float* lse2;
    const float* gcoef;
    const int32_t* ycol;
    float eps_over_V, one_minus_eps;
    float* G;
    const float* bias;        // [V] fp32 or null
    __device__ void operator()(float (*C)[kSimtTile + 1], int m0, int64_t n0, int) const {
        for (int idx = threadIdx.x; idx < kSimtTile * kSimtTile; idx += blockDim.x) {
            const int r = idx / kSimtTile, i = idx % kSimtTile;
            const int m = m0 + r;
            const int64_t v = n0 + i;
            if (m >= rows || v >= ldg) continue;
            const float gc = gcoef[m];
            float g = 0.f;
            if (gc != 0.f && v < V) {
                const float a = C[r][i] + (bias != nullptr ? bias[v] : 0.f);
                g = gc * exp2f(a * c - lse2[m]) - gc * eps_over_V;
                if (v == ycol[m]) g -= gc * one_minus_eps;
            }
            G[(size_t)m * ldg + v] = g;
        }
    }
};

struct SimtStore {
    int rows;
    int64_t cols, ldo;
    float* out;
    float* ws;
    int mode;
    __device__ void operator()(float (*C)[kSimtTile + 1], int m0, int64_t n0, int) const {
        for (int idx = threadIdx.x; idx < kSimtTile * kSimtTile; idx += blockDim.x) {
            const int r = idx / kSimtTile, i = idx % kSimtTile;
            const int m = m0 + r;
            const int64_t col = n0 + i;
            if (m >= rows || col >= cols) continue;
            const size_t o = (size_t)m * ldo + col;
            float x = C[r][i];
            if (mode >= 2) x += ws[o];
            if (mode == 1 || mode == 2) ws[o] = x; else out[o] = x;
        }
    }
};

// C[m, n] = sum_k A[m*sam + k*sak] * B[n*sbn + k*sbk]
template <class Epi>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(const float* __restrict__ A, int64_t sam, int64_t sak,
                 const float* __restrict__ B, int64_t sbn, int64_t sbk, int M, int64_t N, int K,
                 Epi epi) {
    __shared__ float As[16][kSimtTile + 4];
    __shared__ float Bs[16][kSimtTile + 4];
    __shared__ float Cs[kSimtTile][kSimtTile + 1];
    const int m0 = blockIdx.y * kSimtTile;
    const int64_t n0 = (int64_t)blockIdx.x * kSimtTile;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int e = threadIdx.x; e < 16 * kSimtTile; e += 256) {
            const int mm = e % kSimtTile, kk = e / kSimtTile;
            const int gm = m0 + mm, gk = k0 + kk;
            As[kk][mm] = (gm < M && gk < K) ? A[(int64_t)gm * sam + (int64_t)gk * sak] : 0.f;
            const int64_t gn = n0 + mm;
            Bs[kk][mm] = (gn < N && gk < K) ? B[gn * sbn + (int64_t)gk * sbk] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Cs[ty * 4 + i][tx * 4 + j] = acc[i][j];
    __syncthreads();
    epi(Cs, m0, n0, (int)blockIdx.x);
}

}  // namespace fldce
