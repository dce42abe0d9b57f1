/*
 * fle.h -- fused fp32 Linear + epilogue on NVIDIA B200 (sm_100a).
 *
 * One call computes  y = x * W^T + b  on the tensor cores and applies one of
 * the epilogues below to each tile while it is still on chip, so only the
 * final result reaches device memory.  The operation and its three epilogues
 * are the ones stated by the three pages this library follows:
 *
 *   Linear            nn.Linear on x [M,K] with weight W [N,K] and bias b [N]
 *                     (page "Kimi-K2.6 l2_p98", problem restatement, step 1;
 *                      page "Kimi-K2.6 l2_p53", task statement, step 1).
 *   (a) FLE_EPI_SCALE_HARDTANH_GELU
 *                     out = GELU(clamp(scale * y, clamp_lo, clamp_hi)), exact
 *                     erf GELU (page "Kimi-K2.6 l2_p53", task statement
 *                     steps 2-4; the pages' constants are 0.5 and [-2, 2]).
 *   (b) FLE_EPI_SWISH_SCALE
 *                     out = y * sigmoid(y) * scale (page "Kimi-K2.6 l2_p59",
 *                     problem analysis; the page's constant is 2.0).
 *   (c) FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX
 *                     AvgPool1d(pool_k, stride pool_stride, no padding, floor
 *                     mode) along each row of y, then GELU, then * scale, then
 *                     the maximum over the pooled row: out [M]
 *                     (page "Kimi-K2.6 l2_p98", problem restatement steps 2-5;
 *                      the page's constants are k = 16 and 2.0).
 *   FLE_EPI_NONE      out = y (the Linear alone).
 *
 * All entry points are plain C: host scalars, and device pointers to fp32
 * data that the caller owns.  Nothing here allocates device memory; scratch
 * (split-K partials; in 3xTF32 the low parts of x) comes from the caller
 * (fle_workspace_size / workspace).
 */
#ifndef FLE_H
#define FLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogue kinds (fle_epilogue_desc.kind). */
typedef enum {
    FLE_EPI_SCALE_HARDTANH_GELU = 0,
    FLE_EPI_SWISH_SCALE = 1,
    FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX = 2,
    FLE_EPI_NONE = 3
} fle_epilogue_kind;

/* Tensor-core precision of the contraction (fle_epilogue_desc.precision).
 * FLE_PREC_3XTF32: each fp32 operand is split into a TF32 high part and a
 *   TF32 low part; three products (hi*hi + hi*lo + lo*hi) are accumulated in
 *   fp32, which is about as accurate as an fp32 FMA dot product.
 * FLE_PREC_TF32: one TF32 product per term (10-bit mantissa inputs, fp32
 *   accumulation); three times less tensor work. */
typedef enum {
    FLE_PREC_3XTF32 = 0,
    FLE_PREC_TF32 = 1
} fle_precision;

/* Options (fle_epilogue_desc.flags, bitwise or; 0 is the pages' problems).
 * FLE_FLAG_GELU_TANH: (a), (c) use GELU in its tanh form,
 *   v/2 * (1 + tanh(sqrt(2/pi) * (v + 0.044715 v^3))), the approximation page
 *   "Kimi-K2.6 l2_p53" writes into its first fused elementwise kernel before
 *   choosing the exact erf form (the default here).
 * FLE_FLAG_FOLD_SCALE: (a) applies the scale as s*acc + s*b in one fused
 *   multiply-add, the pages' idea of folding the constant into the GEMM's
 *   alpha (page "Kimi-K2.6 l2_p53", its cuBLAS alpha/beta discussion).  The
 *   same function; only the fp32 rounding of that step differs.  Ignored by
 *   the other kinds, whose scale comes after a nonlinearity. */
enum {
    FLE_FLAG_GELU_TANH = 1,
    FLE_FLAG_FOLD_SCALE = 2
};

/* Parameters of the epilogue.  Fields that a kind does not use are ignored.
 *   scale              (a), (b), (c): multiplier
 *   clamp_lo, clamp_hi (a): Hardtanh bounds, clamp_lo <= clamp_hi
 *   pool_k, pool_stride(c): window and stride; the library supports
 *                       pool_stride == pool_k with pool_k in {1,2,4,8,16,32}
 *   flags              FLE_FLAG_* options; unknown bits are FLE_ERR_DESC */
typedef struct {
    int32_t kind;
    int32_t precision;
    float scale;
    float clamp_lo;
    float clamp_hi;
    int32_t pool_k;
    int32_t pool_stride;
    int32_t flags;
} fle_epilogue_desc;

/* Status codes. */
enum {
    FLE_OK = 0,
    FLE_ERR_NULL = 1,        /* a required pointer is NULL                   */
    FLE_ERR_SHAPE = 2,       /* negative size, size >= 2^31, M*N >= 2^40, or
                                (c) N < pool_k                               */
    FLE_ERR_ALIGN = 3,       /* x or W not 16-byte aligned, K % 4 != 0, or
                                out / b not 4-byte aligned                   */
    FLE_ERR_DESC = 4,        /* unknown kind/precision/flag, non-finite scale
                                or clamp, clamp_lo > clamp_hi, unsupported pool */
    FLE_ERR_WORKSPACE = 5,   /* workspace smaller than fle_workspace_size_min() */
    FLE_ERR_ARCH = 6,        /* current device is not sm_100 (B200)          */
    FLE_ERR_CUDA = 7,        /* a CUDA runtime/driver call failed            */
    FLE_ERR_TIMEOUT = 8,     /* a device-side bounded wait expired           */
    FLE_ERR_UNSUPPORTED = 9, /* valid arguments the library does not handle */
    FLE_ERR_PROTOCOL = 10    /* a barrier-protocol check failed (only the checking
                                build, -DFLE_CHECK_BARRIERS, makes these checks) */
};

/*
 * fle_forward -- out = epilogue(x * W^T + b), stream-ordered.
 *
 *   x       device, fp32 [M,K] row-major (K contiguous), 16-byte aligned
 *   W       device, fp32 [N,K] row-major (nn.Linear weight layout), 16-byte aligned
 *   b       device, fp32 [N], or NULL for no bias
 *   M,K,N   sizes, each in [0, 2^31); K % 4 == 0 (row pitch must be a
 *           multiple of 16 bytes for the tensor-memory-access engine)
 *   desc    host pointer to the epilogue parameters (read during the call only)
 *   out     device, fp32 [M,N] row-major for (a), (b) and NONE; fp32 [M] for
 *           (c).  Must not overlap x, W, b or the workspace.
 *   workspace, workspace_bytes
 *           device scratch of fle_workspace_size(M,K,N,desc) bytes, or at
 *           least fle_workspace_size_min() bytes (then a plan that fits runs:
 *           in 3xTF32 the low parts of x are computed inside the GEMM instead
 *           of once per call into the workspace), 256-byte aligned (may be
 *           NULL/0 when that size is 0).  Its contents on entry are ignored;
 *           it must not be used by another call that runs concurrently on the
 *           GPU.
 *   stream  a cudaStream_t (NULL = the legacy default stream)
 *
 * Returns FLE_OK once the work is enqueued (no host synchronisation).
 * Argument errors are detected on the host before anything is enqueued and
 * leave out untouched.  A device-side failure (a bounded wait that expired)
 * is recorded in a device status word; read it with fle_device_status().
 * Sizes M == 0, or N == 0 for the elementwise kinds, are valid and enqueue
 * nothing.  K == 0 gives out = epilogue(b) (a Linear with no inputs).
 */
int fle_forward(const float* x, const float* W, const float* b,
                int64_t M, int64_t K, int64_t N,
                const fle_epilogue_desc* desc, float* out,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * fle_pool_weights -- the pooled weights of epilogue (c).
 *
 * AvgPool1d(k, stride k) over the output features commutes with the Linear
 * map: the mean of k consecutive outputs is one output of a Linear whose
 * weight row is the mean of those k weight rows (page "Kimi-K2.6 l2_p98",
 * its derivation of pre-averaged weights and biases, checked there on a
 * 2-feature example).  This writes
 *   W_pooled[j][:] = mean_{t<k} W[j*k + t][:],  b_pooled[j] = mean_{t<k} b[j*k + t]
 * for j < P = N / pool_k (trailing N mod k rows are unused, as the pool
 * ignores them).  Then fle_forward(x, W_pooled, b_pooled, M, K, P, desc with
 * pool_k = pool_stride = 1, out, ...) gives the same out [M] as the
 * unpooled epilogue (c) call, up to rounding, with a GEMM P/N as large.
 * W_pooled can be kept and reused while W is unchanged.
 *
 *   W        device fp32 [N,K], 16-byte aligned, K % 4 == 0
 *   b        device fp32 [N] or NULL (then b_pooled is not written)
 *   pool_k   1, 2, 4, 8, 16 or 32; N >= pool_k
 *   W_pooled device fp32 [P,K], 16-byte aligned, caller-owned
 *   b_pooled device fp32 [P] (required when b is not NULL)
 * Stream-ordered; returns FLE_OK or an argument / CUDA error.
 */
int fle_pool_weights(const float* W, const float* b, int64_t N, int64_t K, int32_t pool_k,
                     float* W_pooled, float* b_pooled, void* stream);

/* Workspace bytes for fle_forward_pooled (pooled weights + the GEMM's own). */
size_t fle_workspace_size_pooled(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* desc);

/*
 * fle_forward_pooled -- epilogue (c) by pooled weights in one call: pools W
 * and b into the workspace (fle_pool_weights), then runs the P/N-times
 * smaller fused GEMM with the GELU, scale and row-max epilogue.  Same
 * arguments and result as fle_forward with desc->kind ==
 * FLE_EPI_AVGPOOL_GELU_SCALE_ROWMAX (FLE_ERR_DESC for other kinds); the
 * workspace must hold fle_workspace_size_pooled() bytes.
 */
int fle_forward_pooled(const float* x, const float* W, const float* b,
                       int64_t M, int64_t K, int64_t N,
                       const fle_epilogue_desc* desc, float* out,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of caller workspace for the fastest plan of these arguments (0 when
 * the plan needs none): split-K partial tiles and arrival counters, and in
 * 3xTF32 the low parts of x (M x K fp32, written by a pre-pass so that the
 * GEMM splits only W; not for M <= 64 or x above 1 GiB).  Returns 0 for
 * invalid arguments too; fle_forward then reports the argument error. */
size_t fle_workspace_size(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* desc);

/* The least workspace fle_forward accepts for these arguments: the plan
 * without x's low parts in memory (equal to fle_workspace_size() in TF32).
 * Same results bit for bit; 3xTF32 runs slower with it. */
size_t fle_workspace_size_min(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* desc);

/* Static text for a status code; never NULL. */
const char* fle_status_string(int status);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: FLE_OK, or FLE_ERR_TIMEOUT if a kernel's bounded wait
 * expired since the last call.  FLE_ERR_CUDA if the synchronisation fails. */
int fle_device_status(void* stream);

/* Describes the launch plan fle_forward would use, as one line of text
 * ("tile=128x256 swap=0 splits=1 grid=148 stages=4 ..."), into buf.
 * Returns FLE_OK or an argument error; does not launch anything. */
int fle_plan_string(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* desc,
                    char* buf, size_t buf_bytes);

/* Introspection of the launch plan; needs no GPU.  Lists the work units that
 * CTA `cta` of the plan for (M,K,N,desc) on a device with num_sms SMs would
 * run, in order, as 12 int32 per unit:
 *   tile, tile_a, tile_b, kb_begin, kb_end, partial, slot,
 *   first_contributor, last_contributor, slot_by_rule, b_begin, b_width
 * (slot .. slot_by_rule are -1 for a tile this CTA computes whole; for a
 * shared tile they are its workspace slot, the range of CTAs that share it,
 * and the slot the finishing CTA will read for this CTA.  b_begin and
 * b_width are the tile's first operand-B row (output column, or output row
 * in the swapped order) and its number of B rows; tile_b is -1 in a plan of
 * mixed tile widths, whose tiles are not on one grid).  Writes at most max_units
 * rows to units (host memory); *n_units receives the total count and *grid
 * (if not NULL) the plan's grid size.  Returns FLE_OK or an argument error. */
int fle_plan_units(int64_t M, int64_t K, int64_t N, const fle_epilogue_desc* desc, int num_sms,
                   int cta, int32_t* units, int max_units, int* n_units, int* grid);

/*
 * fle_forward_noalloc -- fle_forward without a caller workspace.
 *
 * (The pages have no counterpart of this call: it serves callers of this
 * library, not the method.)  Some callers cannot allocate device memory at
 * the point where they run the layer: a serving process that hands each
 * model a fixed slice of HBM up front and forbids later allocations, or a
 * latency-critical loop in which cudaMalloc/cudaFree would synchronise the
 * device and stall every other stream.  This entry point needs no workspace
 * argument and allocates nothing: the scratch that fle_forward takes from
 * `workspace` (stream-K partial tiles and arrival counters; 3xTF32's low
 * parts of x when they fit as well) comes from one static device array of
 * FLE_NOALLOC_SCRATCH_BYTES (40 MiB) inside the library.  Every plan on a
 * 148-SM B200 fits with x's low parts computed inside the GEMM
 * (fle_workspace_size_min: at most about 37 MiB); a plan that would need more
 * is rejected with FLE_ERR_WORKSPACE before anything is enqueued.  The caller still owns and passes x, W, b and out, with the same
 * layout, alignment and error rules as fle_forward.
 *
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture on
 * the device.  Every GPU that loads the library keeps the array for the life
 * of the process.  All calls on a device share the one array, and it keeps
 * whatever the last call left in it; each call clears the counters it needs
 * before use.  Calls whose kernels overlap on the GPU (other streams, other
 * threads) race on the shared scratch and give wrong results: serialise them.
 */
#define FLE_NOALLOC_SCRATCH_BYTES ((size_t)40 << 20)
int fle_forward_noalloc(const float* x, const float* W, const float* b,
                        int64_t M, int64_t K, int64_t N,
                        const fle_epilogue_desc* desc, float* out, void* stream);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int fle_version(void);

/* The SHA-256 (hex) of the sources and build flags this library was compiled
 * from; the Python binding refuses a library whose hash does not match the
 * sources beside it.  Static text, never NULL. */
const char* fle_source_hash(void);

/* Test and diagnostic hooks are declared in fle_testing.h. */

#ifdef __cplusplus
}
#endif

#endif /* FLE_H */
