/*
 * fldce.h -- C ABI of the fused linear diffusion cross-entropy for B200 (sm_100a).
 *
 * What it computes (the page "fused_linear_diffusion_cross_entropy.py":
 * fused_linear_cross_entropy_forward, cross_entropy_kernel steps 1-6 and
 * fused_linear_cross_entropy_backward).  For hidden states H[N,D], LM-head
 * weight W[V,D], targets y[N], masking probabilities p[N], logit scale s,
 * label smoothing eps, normaliser T and upstream gradient g:
 *
 *   z[n,v]  = s * <H[n], W[v]>                (never written to memory)
 *   lse[n]  = log sum_v exp z[n,v]
 *   CE[n]   = (1-eps)(lse[n] - z[n,y_n]) + eps (lse[n] - mean_v z[n,v])
 *   loss[n] = CE[n] / (p_n T),  loss = sum_n loss[n]     (0 for ignored n)
 *   G[n,v]  = g s (softmax[n,v] - eps/V - (1-eps)[v=y_n]) / (p_n T)
 *   dH = G W,  dW = G^T H
 *
 * A token is ignored when y_n == ignore_index; a target outside [0,V) that
 * is not ignore_index is a caller error: it is counted (err_count) and the
 * token is treated as ignored.  p_mask of an ignored token is never read.
 *
 * Conventions for every entry point:
 *   - Return value: FLDCE_OK (0) or a negative FLDCE_ERR_* code; nothing is
 *     launched when an argument check fails.  fldce_strerror() names a code.
 *   - Pointers named "device" must be device memory of the current CUDA
 *     device; the caller allocates and owns every buffer.  The library never
 *     allocates device memory and never synchronises the host: all work is
 *     enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Layouts are dense row-major.  bf16 is IEEE bfloat16 (stored as
 *     uint16), fp32 is IEEE binary32.  Device pointers of H, W, dH, dW, G
 *     and the workspace must be 16-byte aligned; D must be a multiple of 8.
 *     target must be 8-byte aligned, and p_mask and the per-token outputs
 *     (loss_per_token, lse, argmax) 4-byte aligned (their natural
 *     alignment; FLDCE_ERR_ALIGN otherwise).  Where they are 16-byte aligned
 *     (as every torch allocation is), the per-token kernels move them as
 *     128-bit vectors.
 *   - The handle holds host state only (the configuration); it is not
 *     thread-safe: use one handle per host thread, or serialise calls.
 */
#ifndef FLDCE_H_
#define FLDCE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define FLDCE_OK                    0
#define FLDCE_ERR_INVALID_ARG      -1  /* null/ill-sized argument, N > max_N, ... */
#define FLDCE_ERR_UNSUPPORTED      -2  /* D % 8 != 0, unknown dtype or flag      */
#define FLDCE_ERR_WORKSPACE        -3  /* workspace too small or misaligned       */
#define FLDCE_ERR_CUDA             -4  /* a CUDA runtime call or launch failed    */
#define FLDCE_ERR_DEVICE           -5  /* current device is not compute 10.x      */
#define FLDCE_ERR_ALIGN            -6  /* a device pointer is not 16-byte aligned */
#define FLDCE_ERR_TOO_LARGE        -7  /* needs more scratch than the static buffer */

/* Element types of H, W, dH and (unless FLDCE_FLAG_DW_FP32) dW. */
#define FLDCE_BF16  0   /* tcgen05 tensor-core path, fp32 accumulation        */
#define FLDCE_FP32  1   /* CUDA-core fp32 path (small problems, 1e-5 parity)  */

/* Configuration flags. */
#define FLDCE_FLAG_DW_FP32       0x1u  /* dW (and db) are written as fp32 instead of the dtype */
/* Skip the tokens that carry no loss (ignore_index or out of range): the
 * valid tokens are compacted on the device and only they enter the GEMMs.
 * loss, loss_per_token, dH, dW and db are what they are without the flag
 * (a skipped token's loss is 0, its dH row 0, and it adds nothing to dW);
 * lse is NaN and argmax is -1 for skipped tokens.  The workspace grows by
 * about 2 N D + 24 N bytes.  bf16 only (UNSUPPORTED with FLDCE_FP32). */
#define FLDCE_FLAG_SKIP_IGNORED  0x2u
/* dH is written as fp32 instead of the dtype (e.g. partial dH summed over
 * vocabulary shards).  Not with FLDCE_FLAG_SKIP_IGNORED. */
#define FLDCE_FLAG_DH_FP32       0x4u
/* dW (and db) are accumulated into: dW += G^T H, db += sum_n G[n, :], for
 * gradient accumulation over micro-batches.  The caller initialises them
 * (e.g. to zero) before the first call.  A bf16 dW gets the call's fp32
 * gradient added and is rounded once; an fp32 dW (FLDCE_FLAG_DW_FP32 or the
 * fp32 dtype) takes the chunks' fp32 reduce-adds directly.  N == 0 leaves dW
 * and db as they are.  dH is still overwritten.  The pages always overwrite
 * (their dW is a fresh buffer per call); this flag is an extension. */
#define FLDCE_FLAG_DW_ACCUMULATE 0x8u
/* Sweep 2 fused with the dH GEMM (bf16 only, not with
 * FLDCE_FLAG_SKIP_IGNORED): each 256 x 256 tile of the logit gradient G is
 * formed in shared memory and fed from there, as the A operand, to the dH
 * tensor-core MMAs, whose per-tile fp32 partials are reduce-added into an
 * fp32 dH accumulator in the workspace; G still goes to HBM once, for the
 * dW GEMM.  Same results as without the flag (up to the summation order of
 * dH).  The page runs dx = dlogits @ weight on the gradient it wrote over
 * the logits (fused_linear_cross_entropy_forward's chunk loop); this is the
 * on-chip form of that step.  An alternative design, measured against the
 * default (staged G read back by a separate dH GEMM) and not the default:
 * its fp32 partials move 2 D / 256 times the bytes the staged dH reads
 * back, and it ran about twice as long as sweep 2 + dH on B200. */
#define FLDCE_FLAG_FUSED_DH      0x10u

typedef struct fldce_plan* fldce_handle;

typedef struct {
    int32_t dtype;            /* FLDCE_BF16 or FLDCE_FP32                         */
    uint32_t flags;           /* FLDCE_FLAG_*                                     */
    int64_t D;                /* hidden size, > 0, multiple of 8                  */
    int64_t V;                /* vocabulary size, > 0                             */
    int64_t max_N;            /* largest token count passed to a call, > 0        */
    int64_t chunk_N;          /* tokens per internal chunk; 0 = library's choice  */
    float logit_scale;        /* s (the page's logit_scale), finite and nonzero   */
    float label_smoothing;    /* eps in [0, 1]                                    */
    int64_t ignore_index;     /* the page's ignore_index, usually -100            */
    /* Vocabulary sharding (0, 0 = not sharded).  With vocab_total > 0 this
     * plan's W is rows [vocab_start, vocab_start + V) of a vocabulary of
     * vocab_total entries; targets are global ids; only the fldce_vp_* entry
     * points accept such a plan. */
    int64_t vocab_start;
    int64_t vocab_total;
} fldce_config;

/*
 * fldce_create -- validate `cfg` and build a plan (host memory only).
 *   out             [out] the new handle; unchanged on error.
 *   cfg             [in]  configuration; copied, the caller keeps ownership.
 *   workspace_bytes [out, may be NULL] device workspace needed by a call
 *                   with N = cfg->max_N (calls with smaller N need no more).
 * Errors: INVALID_ARG (null out/cfg, a size <= 0, eps outside [0,1],
 * logit_scale zero or not finite, chunk_N < 0), UNSUPPORTED (dtype, flags,
 * D % 8 != 0).
 */
int fldce_create(fldce_handle* out, const fldce_config* cfg, size_t* workspace_bytes);

/*
 * fldce_workspace_size -- device workspace bytes a call with N tokens needs.
 * Errors: INVALID_ARG (null handle/bytes, N < 0 or N > max_N).
 */
int fldce_workspace_size(fldce_handle h, int64_t N, size_t* bytes);

/*
 * fldce_chunk_size -- tokens per internal chunk the plan uses (the explicit
 * chunk_N, or the library's choice: the largest multiple of 256 tokens whose
 * G buffer stays within 4 GiB, capped at max_N).
 * Errors: INVALID_ARG (null handle or out).
 */
int fldce_chunk_size(fldce_handle h, int64_t* chunk_N);

/*
 * fldce_fwd_bwd -- loss and both gradients in one asynchronous call
 * (the page's FusedLinearCrossEntropyFunction.forward computes the loss and
 * all gradients at once; its backward only multiplies them by grad_out,
 * which here is folded in).
 *
 *   H        [device, in]  [N, D] dtype.
 *   W        [device, in]  [V, D] dtype.
 *   target   [device, in]  [N] int64.
 *   p_mask   [device, in]  [N] fp32, or NULL for p = 1 (ordinary CE).
 *   N        tokens, 0 <= N <= max_N.  N == 0 writes loss = 0 and dW = 0
 *            (leaves dW as it is with FLDCE_FLAG_DW_ACCUMULATE).
 *   total    T > 0 is used as given ('mean' over an explicit normaliser;
 *            'sum' is T = 1); T <= 0 means the count of non-ignored,
 *            in-range targets, computed on the device (no host sync).
 *   grad_out g, the upstream gradient of the scalar loss (1 for a loss that
 *            ends the graph).
 *   loss            [device, out] 1 fp32: sum_n loss[n] (fixed-order sum).
 *   loss_per_token  [device, out, may be NULL] [N] fp32 loss[n].
 *   lse             [device, out, may be NULL] [N] fp32 lse[n] (every row).
 *   argmax          [device, out, may be NULL] [N] int32 lowest v with
 *                   z[n,v] = max_v z[n,v] (every row).
 *   dH       [device, out] [N, D] dtype; overwritten.
 *   dW       [device, out] [V, D] dtype (fp32 with FLDCE_FLAG_DW_FP32);
 *            overwritten, or added to with FLDCE_FLAG_DW_ACCUMULATE.
 *   workspace        [device] scratch of at least fldce_workspace_size(N)
 *                    bytes, 256-byte aligned; contents need no initialisation
 *                    and are undefined afterwards.  Calls that share a
 *                    workspace must be ordered on the GPU (same stream).
 *   workspace_bytes  its size.
 *   err_count [device, out, may be NULL] 2 int32: [0] = number of targets
 *             outside [0, V) that are not ignore_index; [1] = device error
 *             bits, 0 when every kernel completed (1 = a pipeline wait timed
 *             out after 4 s: the results are invalid; the kernel waited,
 *             bounded again, for the work it had issued before freeing its
 *             tensor memory, but a caller should treat the CUDA context as
 *             unreliable after this bit and recreate it).
 *   stream    cudaStream_t to enqueue on.  The call allocates nothing and
 *             never waits on the host, so it may be captured into a CUDA
 *             graph; make one call on the device before capturing (the first
 *             call sets the kernels' shared-memory limits).
 * Errors: INVALID_ARG, ALIGN, WORKSPACE, DEVICE, CUDA (launch failure).
 */
int fldce_fwd_bwd(fldce_handle h,
                  const void* H, const void* W, const int64_t* target,
                  const float* p_mask, int64_t N, float total, float grad_out,
                  float* loss, float* loss_per_token, float* lse, int32_t* argmax,
                  void* dH, void* dW,
                  void* workspace, size_t workspace_bytes,
                  int32_t* err_count, void* stream);

/*
 * fldce_fwd_bwd_noalloc -- fldce_fwd_bwd for callers that cannot allocate
 * device memory.  The paper has no counterpart to this entry point.
 *
 * Some callers have no way to obtain a workspace: a plugin inside a host
 * application that owns every byte of device memory through its own pool
 * and gives plugins no allocator, a supervisor-enforced memory budget that
 * forbids allocations outside that pool, or a thin foreign-function binding
 * that can only pass buffers it already has.  This entry point needs no
 * workspace: its scratch is a static device array of
 * FLDCE_STATIC_SCRATCH_BYTES (64 MiB) inside the library, which every GPU
 * that loads the library holds until the process exits.  The call itself
 * never allocates device memory.
 *
 * Arguments mean what they mean for fldce_fwd_bwd; the caller still
 * provides every input and output buffer.
 *   - Size limit: the call needs fldce_workspace_size(h, N) <=
 *     FLDCE_STATIC_SCRATCH_BYTES, else it returns FLDCE_ERR_TOO_LARGE and
 *     launches nothing.  A smaller chunk_N (the G buffer is chunk_N x V bf16)
 *     and FLDCE_FLAG_DW_FP32 (no fp32 dW accumulator across chunks) make a
 *     problem fit.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (with that device current); make that first call before any
 *     stream capture begins.
 *   - Sharing: every call in the process, on any handle, uses the same
 *     array, which keeps the previous call's contents (each call clears the
 *     counters it needs zeroed).  Calls that overlap on the GPU -- on two
 *     streams, or from two host threads -- race on it: order them on one
 *     stream.
 * Errors: those of fldce_fwd_bwd, and TOO_LARGE.
 */
#define FLDCE_STATIC_SCRATCH_BYTES (64ull << 20)
int fldce_fwd_bwd_noalloc(fldce_handle h,
                          const void* H, const void* W, const int64_t* target,
                          const float* p_mask, int64_t N, float total, float grad_out,
                          float* loss, float* loss_per_token, float* lse, int32_t* argmax,
                          void* dH, void* dW, int32_t* err_count, void* stream);

/*
 * Extended call: every argument of fldce_fwd_bwd in one struct, plus the
 * page's optional bias and a device-side normaliser for data-parallel use.
 * Zero-initialise the struct and set what is needed; fields mean what the
 * same-named arguments of fldce_fwd_bwd mean, and:
 *   bias      [device, in, may be NULL] [V] dtype: z = s (<H[n], W[v]> + b[v])
 *             (the page's F.linear(x, weight, bias) before the scale).
 *   db        [device, out] [V] dtype (fp32 with FLDCE_FLAG_DW_FP32);
 *             required when bias is set: db[v] = sum_n G[n, v] (the page's
 *             db += dlogits.sum(0)), summed in a fixed order (added to
 *             db with FLDCE_FLAG_DW_ACCUMULATE).
 *   count_dev [device, in, may be NULL] 1 int32: when total <= 0, the
 *             normaliser is *count_dev instead of this call's own count --
 *             e.g. the job-wide count of valid tokens, summed over
 *             data-parallel ranks from fldce_count_valid (no host sync).
 *   dw_ready_event [may be NULL] a cudaEvent_t.  When set, the last token
 *             chunk computes dW (and db) before dH, and the event is
 *             recorded on `stream` as soon as dW and db hold their final
 *             values, so a caller can start reducing dW across ranks on
 *             another stream while dH is still being computed.
 */
typedef struct {
    const void* H;
    const void* W;
    const void* bias;
    const int64_t* target;
    const float* p_mask;
    int64_t N;
    float total;
    float grad_out;
    const int32_t* count_dev;
    float* loss;
    float* loss_per_token;
    float* lse;
    int32_t* argmax;
    void* dH;
    void* dW;
    void* db;
    void* workspace;
    size_t workspace_bytes;
    int32_t* err_count;
    void* stream;
    void* dw_ready_event;
} fldce_call;

/* fldce_fwd_bwd_ex -- fldce_fwd_bwd with the fields of `call`.
 * Errors: those of fldce_fwd_bwd (INVALID_ARG also for bias without db). */
int fldce_fwd_bwd_ex(fldce_handle h, const fldce_call* call);

/* fldce_forward_ex -- fldce_forward with the fields of `call` (dH, dW and db
 * are not used). */
int fldce_forward_ex(fldce_handle h, const fldce_call* call);

/*
 * Vocabulary-parallel loss (the tensor-parallel tutorial page, section 4:
 * each shard computes its own softmax denominators, they are combined across
 * shards, and every shard then works on its own columns).  A plan made with
 * vocab_total > 0 covers one shard; every rank holds all N tokens.
 *
 * fldce_vp_stats -- sweep 1 over this shard: for each token n, 8 fp32 at
 *   stats[8 n .. 8 n + 7]: m2 (max of z log2 e over the shard), l (sum of
 *   2^(z log2 e - m2)), z[n, y_n] log2 e if y_n is in the shard else 0, s * sum of
 *   (H W^T + b) over the shard, the shard argmax as int32 bits (global id),
 *   3 unused.  Uses call->H, W, bias, target, N, workspace, stream.
 *   stats [device, out] [N][8] fp32.
 *
 * fldce_vp_fwd_bwd -- everything after the exchange: `all_stats` holds the
 *   n_shards shards' stats ([n_shards][N][8], in vocabulary order: the shard
 *   with the lowest vocab_start first), gathered from every rank.  They are
 *   merged in that fixed order into lse, the loss (identical on every rank),
 *   and G for this shard's columns; then dW and db for this shard, and this
 *   shard's partial dH = G_shard W_shard, which the caller sums over shards.
 *   Fields of `call` as for fldce_fwd_bwd_ex (argmax and lse are global).
 * Errors: those of fldce_fwd_bwd_ex; INVALID_ARG for an unsharded plan.
 */
int fldce_vp_stats(fldce_handle h, const fldce_call* call, float* stats);
int fldce_vp_fwd_bwd(fldce_handle h, const fldce_call* call, const float* all_stats,
                     int32_t n_shards);

/*
 * fldce_count_valid -- *count = number of targets that carry a loss (not
 * ignore_index and inside [0, V)), written on `stream` into device memory.
 * The page's target.ne(ignore_index).sum(), without the host round trip; a
 * data-parallel caller sums it over ranks and passes it as count_dev.
 *   target [device, in] [N] int64;  count [device, out] 1 int32.
 * Errors: INVALID_ARG, DEVICE, CUDA.
 */
int fldce_count_valid(fldce_handle h, const int64_t* target, int64_t N, int32_t* count,
                      void* stream);

/*
 * fldce_forward -- the loss sweep alone, for evaluation: loss, and
 * optionally loss_per_token / lse / argmax, with no gradients (the page's
 * logsumexp_fwd plus cross_entropy_kernel step 4, without steps 5-6).
 * Arguments mean what they mean for fldce_fwd_bwd.  Needs no more
 * workspace than fldce_fwd_bwd.
 */
int fldce_forward(fldce_handle h,
                  const void* H, const void* W, const int64_t* target,
                  const float* p_mask, int64_t N, float total,
                  float* loss, float* loss_per_token, float* lse, int32_t* argmax,
                  void* workspace, size_t workspace_bytes,
                  int32_t* err_count, void* stream);

/*
 * Optional profiling window: per-kernel device time over a window of calls.
 * fldce_profile_begin(h, max_calls) creates CUDA events (no device memory)
 * for the next `max_calls` calls on this handle; each of those calls records
 * an event on its stream after every kernel it launches.  Calls past the
 * window are not recorded.  fldce_profile_end() waits for the recorded events,
 * then fills, per kernel kind k < FLDCE_PROF_KINDS, the summed device time
 * in ms[k] and the number of launches in launches[k] (either may be NULL),
 * and closes the window.  The time of a kernel is the interval between the
 * event before it and the event after it on the same stream.
 * Errors: INVALID_ARG (null handle, max_calls <= 0), CUDA.
 */
#define FLDCE_PROF_KINDS 9
int fldce_profile_begin(fldce_handle h, int max_calls);
int fldce_profile_end(fldce_handle h, double* ms, int32_t* launches);
/* Name of kernel kind k ("lse_sweep", "g_sweep", "dh_gemm", ...), or NULL. */
const char* fldce_profile_kind_name(int kind);

/*
 * fldce_scale -- x[i] *= *g for i < n, in place, on `stream`; the kernel
 * returns without touching x when *g == 1 (the page's
 * fused_linear_cross_entropy_backward / elementwise_mul_kernel: scale the
 * saved gradients by the upstream gradient `do`, skipped when do == 1,
 * decided on the device instead of by a host round trip).
 *   x      [device, in/out] n elements of `dtype` (FLDCE_BF16 or FLDCE_FP32),
 *          16-byte aligned.
 *   g      [device, in] 1 fp32.
 * Errors: INVALID_ARG (null pointers with n > 0, n < 0), UNSUPPORTED (dtype),
 * ALIGN, CUDA.
 */
int fldce_scale(void* x, int64_t n, int32_t dtype, const float* g, void* stream);

/*
 * fldce_selftest_wait -- exercise the time-out path of the pipeline waits.
 * Launches one CTA that waits, with the same bounded wait every GEMM
 * pipeline stage uses, on a shared-memory mbarrier that nothing ever arrives
 * on; after `limit_ns` of global time the wait gives up and *status is set
 * to 1 (the device error bit a timed-out pipeline reports in err_count[1]).
 * The GPU context stays usable.  limit_ns is clamped to [1000, 2e9].
 *   status [device, out] 1 int32.
 * Errors: INVALID_ARG (null status), DEVICE, CUDA.
 */
int fldce_selftest_wait(int64_t limit_ns, int32_t* status, void* stream);

/* fldce_destroy -- free the plan's host memory (and profiling events).
 * NULL is accepted. */
int fldce_destroy(fldce_handle h);

/* fldce_strerror -- static English text for a status code. */
const char* fldce_strerror(int status);

/* fldce_version -- library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fldce_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLDCE_H_ */
