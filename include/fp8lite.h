/*
 * fp8lite -- per-tensor FP8 quantization with delayed scaling, and the
 * per-tensor-scaled FP8 GEMM of a linear layer, for NVIDIA B200 (sm_100a).
 *
 * The C ABI of the library. Plain pointers and sizes only; the caller owns
 * every buffer (device memory unless stated) and the library allocates
 * nothing per call. All compute calls are asynchronous and stream-ordered on
 * `stream` (a cudaStream_t passed as void*; NULL is the legacy default
 * stream) and do no host synchronisation, so a sequence of them can be
 * captured into a CUDA graph. Arguments are validated on the host BEFORE any
 * launch; a rejected call launches nothing and returns a non-OK status.
 *
 * Method sources (AstrAI FP8 commit logs):
 *  [fp8.py@4dc5e923]  astrai/extension/fp8.py, commit 4dc5e923
 *  [fp8.py@f4c44ebf]  astrai/extension/fp8.py, commit f4c44ebf
 *  [mma@cebdd45d]     tests/extension/test_fp8_mma.py, commit cebdd45d
 *  [gemm@5e76fbd1]    csrc/kernels/fp8/gemm.cuh, commit 5e76fbd1
 * FP8 formats: OCP 8-bit floating point specification (OFP8) rev. 1.0.
 */
#ifndef FP8LITE_H
#define FP8LITE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP8LITE_ABI_VERSION 4

/* Exported entry points (the library is built with hidden visibility). */
#if defined(__GNUC__)
#define FP8LITE_API __attribute__((visibility("default")))
#else
#define FP8LITE_API
#endif

/* FP8 encodings (OFP8): E4M3 = the "FN" variant, max 448, no Inf;
 * E5M2 = IEEE-like, max 57344. The pages use E4M3 for activations and
 * weights and E5M2 for gradients [fp8.py@4dc5e923, bullet on the fp8
 * backward regression test]. */
typedef enum fp8_fmt { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_fmt;

/* GEMM layouts, BLAS-style op tags on row-major storage
 * [gemm@5e76fbd1, bullet on RowMajor/ColMajor operand tags]:
 *   FP8_NT: A [M,K], B [N,K]  C = A * B^T   (forward  y  = x W^T)
 *   FP8_NN: A [M,K], B [K,N]  C = A * B     (backward dX = g W)
 *   FP8_TN: A [K,M], B [K,N]  C = A^T * B   (backward dW = g^T x) */
typedef enum fp8_layout { FP8_NT = 0, FP8_NN = 1, FP8_TN = 2 } fp8_layout;

typedef enum fp8_status {
    FP8_OK = 0,
    FP8_ERR_INVALID_ARG = 1,    /* bad enum, null required pointer, bad size */
    FP8_ERR_ALIGNMENT = 2,      /* base or stride not aligned as documented */
    FP8_ERR_UNSUPPORTED = 3,    /* shape or option this build cannot run */
    FP8_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
    FP8_ERR_DEVICE_TIMEOUT = 5  /* a bounded device wait gave up (GEMM) */
} fp8_status;

/* Delayed-scaling amax history of ONE tensor role (x, W or g of one linear)
 * [fp8.py@4dc5e923, bullets on _ScaleRing and the three rings per linear].
 * Device-resident, caller-allocated (FP8_RING_BYTES, 4-byte aligned).
 *   hist[16]   amax of the last 16 calls (fp32), written at hist[idx]
 *   scale      the scale the NEXT call quantizes with (multiplier into FP8)
 *   idx        next slot of hist, 0..15
 *   amax_bits  in-flight amax accumulator; 0 between calls
 *   ticket     last-block election counter; 0 between calls
 * One ring must not be used by two calls that overlap on the GPU. */
#define FP8_RING_HISTORY 16
typedef struct fp8_ring {
    float hist[FP8_RING_HISTORY];
    float scale;
    uint32_t idx;
    uint32_t amax_bits;
    uint32_t ticket;
} fp8_ring;
#define FP8_RING_BYTES 80

/* Human-readable name of a status (static string). */
FP8LITE_API const char* fp8_status_string(fp8_status s);

/* FP8LITE_ABI_VERSION of the built library. */
FP8LITE_API int fp8_abi_version(void);

/* Reset a ring: hist = 0, idx = 0, scale = init_scale, accumulators 0.
 * init_scale must be finite and > 0 (the plain reading starts at 1.0).
 * Asynchronous on `stream` (one tiny kernel, graph-capturable). */
FP8LITE_API fp8_status fp8_ring_init(fp8_ring* ring, float init_scale, void* stream);

/* Checkpoint: copy the ring to host memory `host` (FP8_RING_BYTES).
 * Synchronises `stream` before returning. */
FP8LITE_API fp8_status fp8_ring_get(const fp8_ring* ring, fp8_ring* host, void* stream);

/* Restore: write the host copy `host` into the device ring (asynchronous,
 * by value, no host sync). idx must be < 16 and scale finite and > 0; the
 * accumulators are reset to 0 whatever `host` holds. */
FP8LITE_API fp8_status fp8_ring_set(fp8_ring* ring, const fp8_ring* host, void* stream);

/* Per-tensor quantization of n bf16 values x -> n FP8 codes out8, with the
 * amax measured on the UNQUANTIZED input [fp8.py@4dc5e923, bullets on the
 * amax bug].
 *
 *   q_i = sat_rne_fmt( fp32(x_i * s) )   (fp32 product, then one FP8
 *   rounding to nearest-even; magnitudes above the format's max saturate)
 *
 * ring != NULL -- delayed scaling, ONE kernel launch: s = ring->scale as it
 *   stood before the call; the last thread block to finish (threadfence +
 *   ticket election) writes amax into hist[idx], advances idx, takes the max
 *   of the window and publishes ring->scale = fmt_max / max when that max is
 *   finite and > 0 (otherwise the scale is kept), then resets the ring's
 *   accumulators [fp8.py@4dc5e923, bullet on the last-block epilogue].
 * ring == NULL -- current ("dynamic") scaling [fp8.py@4dc5e923, bullet on
 *   the dynamic path]: s = fmt_max / amax(x) (1 if amax is 0 or not finite);
 *   one launch for bf16/fp16 tensors of up to 65536 elements (one thread
 *   block holds the whole tensor), otherwise a memset and two launches (amax
 *   pass, quantize pass).
 * fmt_max / m is an IEEE fp32 division; an overflow is clamped to FLT_MAX.
 *
 * x          device, bf16[n], 16-byte aligned
 * n          element count, 0 <= n < 2^40 (n = 0 folds amax 0)
 * out8       device, uint8[n], 16-byte aligned, FP8 codes of `fmt`
 * amax_out   device float: amax(x). Optional (NULL) with a ring; REQUIRED
 *            without one (it is the accumulator of the amax pass)
 * scale_out  device float, REQUIRED: the scale s this call used. A GEMM on
 *            out8 must dequantize with THIS value, not with ring->scale,
 *            which the call has already replaced [fp8.py@f4c44ebf, bullet on
 *            snapshotting sx/sw/sg before the finalize].
 * Errors: FP8_ERR_INVALID_ARG (bad fmt, NULL x/out8/scale_out with n > 0,
 *         NULL amax_out without a ring, n out of range),
 *         FP8_ERR_ALIGNMENT (x or out8 not 16-byte aligned, ring not 4-byte
 *         aligned), FP8_ERR_CUDA (launch failure). */
FP8LITE_API fp8_status fp8_quantize(const void* x, int64_t n, fp8_fmt fmt, fp8_ring* ring,
                        uint8_t* out8, float* amax_out, float* scale_out,
                        void* stream);

/* fp8_quantize for bf16, fp16 or fp32 input, with an optional seeded first
 * call of a ring [fp8.py@f4c44ebf, bullet on the quantize kernel templated
 * on the input type; fp8.py@4dc5e923, bullet on the _ScaleRing objects with
 * their update and seed].
 *
 * dtype  the type of x: FP8_IN_BF16 (x is bf16[n]), FP8_IN_F16 (fp16[n]) or
 *        FP8_IN_F32 (fp32[n]); every input value widens to fp32 exactly, so
 *        the codes are those of the same values given as fp32.
 * flags  0, or FP8_QUANTIZE_SEED_RING with a ring: instead of the ring's
 *        current scale, this call measures amax(x) first, quantizes with
 *        s = fmt_max / amax (1 if amax is 0 or not finite), and folds the amax
 *        into the ring as a delayed call would (hist[idx] = amax, idx + 1, the
 *        window's max publishes the next scale). Seeding a fresh ring (hist
 *        all 0) so makes its next scale fmt_max / amax rather than leaving the
 *        first step at the initial scale. Costs what current scaling costs
 *        (a memset and two launches); amax_out is then REQUIRED (it is the
 *        accumulator).
 * Other arguments, results and errors as fp8_quantize (x 16-byte aligned
 * whatever its type); FP8_ERR_INVALID_ARG also for an unknown dtype or flag,
 * for FP8_QUANTIZE_SEED_RING or FP8_QUANTIZE_DEFER_FOLD without a ring, and
 * for both flags together. */
typedef enum fp8_dtype { FP8_IN_BF16 = 0, FP8_IN_F16 = 1, FP8_IN_F32 = 2 } fp8_dtype;
#define FP8_QUANTIZE_SEED_RING 1u
/* FP8_QUANTIZE_DEFER_FOLD (with a ring, not with SEED): a delayed call that
 * quantizes with ring->scale and leaves this call's amax in the ring's
 * accumulator (amax_bits, as fp32 bits) instead of folding it: the ranks of
 * a data-parallel group all-reduce those 4 bytes with MAX (non-negative fp32
 * bit patterns order like unsigned integers) and then call fp8_rings_fold, so
 * every replica's ring sees the group's amax and stays identical. amax_out
 * (optional) receives this rank's own amax. Until the fold the ring must not
 * be used by another call. */
#define FP8_QUANTIZE_DEFER_FOLD 2u
FP8LITE_API fp8_status fp8_quantize_ex(const void* x, fp8_dtype dtype, int64_t n, fp8_fmt fmt, fp8_ring* ring,
                        uint32_t flags, uint8_t* out8, float* amax_out, float* scale_out,
                        void* stream);

/* Folds the amax accumulated in each of `count` rings (by deferred calls, and
 * all-reduced over a data-parallel group) into its history: hist[idx] = amax,
 * idx + 1, the window's max publishes the next scale (as the last block of a
 * delayed call does), the accumulator is reset. One launch for all rings.
 * rings   device array of `count` consecutive rings (e.g. a layer's x, W and g)
 * count   1 .. 64
 * fmts    host int32[count]: each ring's fp8_fmt (its fmt_max sets the scale)
 * Errors: FP8_ERR_INVALID_ARG (count, NULL, bad fmt), FP8_ERR_ALIGNMENT,
 *         FP8_ERR_CUDA. */
FP8LITE_API fp8_status fp8_rings_fold(fp8_ring* rings, int32_t count, const int32_t* fmts, void* stream);

/* Quantize of a row-major [rows, cols] tensor in either or both orientations
 * [fp8.py@f4c44ebf, bullets on quantize(transposed) / quantize_dual and the
 * QuantLayout enum]: the codes of x (row-major [rows, cols]), of x^T
 * (row-major [cols, rows], i.e. the transposed copy a GEMM that wants a
 * K-major operand reads), or both from one read of the input. Both copies
 * hold the same bytes: out8_t[c * rows + r] == out8[r * cols + c]. The scale,
 * amax, ring update and errors are those of fp8_quantize_ex.
 *
 * layout  FP8_QL_ROW: out8 only (fp8_quantize_ex on the flat tensor);
 *         FP8_QL_COL: out8_t only; FP8_QL_BOTH: both.
 * rows, cols  >= 0, rows * cols < 2^40; multiples of 8 when out8_t is
 *         written (FP8_ERR_ALIGNMENT otherwise).
 * out8    device uint8[rows * cols], 16-byte aligned (ROW, BOTH)
 * out8_t  device uint8[cols * rows], 16-byte aligned (COL, BOTH) */
typedef enum fp8_quant_layout { FP8_QL_ROW = 0, FP8_QL_COL = 1, FP8_QL_BOTH = 2 } fp8_quant_layout;
FP8LITE_API fp8_status fp8_quantize_2d(const void* x, fp8_dtype dtype, int64_t rows, int64_t cols, fp8_fmt fmt,
                        fp8_ring* ring, uint32_t flags, fp8_quant_layout layout, uint8_t* out8,
                        uint8_t* out8_t, float* amax_out, float* scale_out, void* stream);

/* Several delayed-scaling quantizations in ONE launch, e.g. the weights of
 * all layers at the start of a training step, or a layer's x and W.
 * Each job is exactly an fp8_quantize call with a ring (same arguments, same
 * results, its ring finalized by the last of the job's thread blocks); the
 * jobs run concurrently. Jobs must use distinct rings and must not overlap
 * in their outputs; current scaling (no ring) is not offered here.
 * count: 1 .. FP8_QUANTIZE_MAX_JOBS. Errors as fp8_quantize, plus
 * FP8_ERR_INVALID_ARG for a bad count, a NULL ring or a ring used twice. */
#define FP8_QUANTIZE_MAX_JOBS 8
typedef struct fp8_quantize_job {
    const void* x;     /* device input of `dtype` [n], 16-byte aligned */
    int64_t n;         /* 0 <= n < 2^40 */
    int32_t fmt;       /* fp8_fmt */
    int32_t dtype;     /* fp8_dtype of x (0 = bf16: a zero-filled job quantizes bf16) */
    fp8_ring* ring;    /* required */
    uint8_t* out8;     /* device uint8[n], 16-byte aligned */
    float* amax_out;   /* optional */
    float* scale_out;  /* required: the scale this job used */
} fp8_quantize_job;
FP8LITE_API fp8_status fp8_quantize_many(const fp8_quantize_job* jobs, int32_t count, void* stream);
/* fp8_quantize_many with flags: 0, or FP8_QUANTIZE_DEFER_FOLD for every job
 * (each job's amax stays in its ring's accumulator for a data-parallel
 * all-reduce and fp8_rings_fold; see fp8_quantize_ex). */
FP8LITE_API fp8_status fp8_quantize_many_ex(const fp8_quantize_job* jobs, int32_t count, uint32_t flags,
                                            void* stream);

/* Current ("dynamic") scaling of up to FP8_QUANTIZE_MAX_JOBS small tensors in
 * ONE launch, e.g. the two operands of a small GEMM [fp8.py@4dc5e923, bullet
 * on the dynamic path]. Each job is exactly an fp8_quantize_ex call with
 * ring == NULL: s = fmt_max / amax(x) (1 if amax is 0 or not finite), the
 * same codes, amax and scale. One thread block per job holds the whole
 * tensor, so every job must be bf16 or fp16 (dtype) with
 * 0 <= n <= FP8_QUANTIZE_SMALL_MAX elements; ring must be NULL; amax_out is
 * optional, scale_out required; x and out8 16-byte aligned.
 * Errors: FP8_ERR_INVALID_ARG (count, fmt, dtype, a ring given, NULL
 * scale_out, NULL x/out8 with n > 0), FP8_ERR_UNSUPPORTED (an fp32 job or one
 * above FP8_QUANTIZE_SMALL_MAX), FP8_ERR_ALIGNMENT, FP8_ERR_CUDA. */
#define FP8_QUANTIZE_SMALL_MAX 65536
FP8LITE_API fp8_status fp8_quantize_current_many(const fp8_quantize_job* jobs, int32_t count, void* stream);

/* Per-tensor-scaled FP8 GEMM with fused bias and bf16 output
 * [fp8.py@f4c44ebf, bullets on the fused bias and 3-D operands;
 *  mma@cebdd45d, bullet on the bias_scale slot].
 *
 *   out[b,i,j] = bf16_rne( (sum_k op(A_b)[i,k] op(B_b)[k,j]) / (sa*sb) + bias_j )
 *
 * accumulated in fp32 on the tensor cores, the scale and the bias applied in
 * fp32, then ONE rounding to bf16. Short problems (M <= 32 in NT or NN) with a
 * long K may be split along K as a cluster of 2 .. 4 CTAs that add their
 * fp32 partials in split order through shared memory (no workspace); the
 * result is then what fp8_mm_ws gives with that split, and it does not
 * depend on timing. bias_j is bias[j] (bf16) when bias_scale
 * is NULL, dec(bias[j]) / *bias_scale (fp8 codes of bias_fmt) when it is not,
 * 0 when bias is NULL; the bias is broadcast over rows and batches.
 *
 * a8, b8     device FP8 codes of formats fa, fb in `layout` (see fp8_layout),
 *            each 16-byte aligned
 * sa, sb     device floats: the scales the operands were quantized with
 *            (the scale_out of fp8_quantize)
 * M, N, K    >= 1 each. The contiguous dimension of every operand must be a
 *            multiple of 16 elements (TMA row pitch): K for A in NT/NN and
 *            B in NT; N for B in NN/TN; M for A in TN. M and N are otherwise
 *            free (M = 1 and N = 7 are valid).
 * batch      >= 1; stride_a / stride_b / stride_c in ELEMENTS between
 *            consecutive batches; stride_a or stride_b = 0 broadcasts one
 *            matrix to every batch; nonzero operand strides must be multiples
 *            of 16; stride_c >= M*N when batch > 1.
 * bias       NULL, device bf16[N], or device FP8 codes[N] of bias_fmt
 * bias_scale NULL (bf16 bias) or device float (FP8 bias)
 * out        device bf16[batch*stride_c], row-major [M,N] per batch,
 *            4-byte aligned
 * Errors: FP8_ERR_INVALID_ARG, FP8_ERR_ALIGNMENT as listed above,
 *         FP8_ERR_UNSUPPORTED (a size >= 2^31 per matrix dimension),
 *         FP8_ERR_CUDA. A bounded device wait that gives up does not fail
 *         the call; it is reported by fp8_last_device_error. */
FP8LITE_API fp8_status fp8_mm(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb,
                  const float* sa, const float* sb, fp8_layout layout,
                  int64_t M, int64_t N, int64_t K, int64_t batch,
                  int64_t stride_a, int64_t stride_b, int64_t stride_c,
                  const void* bias, const float* bias_scale, fp8_fmt bias_fmt,
                  void* out, void* stream);

/* fp8_mm that can split K over a caller-owned workspace: `split_k` CTAs (or
 * SM pairs) share each output tile's k-blocks, each accumulating its part in
 * fp32; the one that finishes last adds the others' partials in split order
 * and runs the epilogue. The result is the same formula; only the fp32
 * accumulation is grouped differently, so it stays within fp8_mm's accuracy,
 * and it is deterministic: it does not depend on the order in which the
 * splits finish.
 *
 * split_k         0: the library's choice: it splits only short problems
 *                 (M <= 32, NT or NN; they run with swapped operands, so a
 *                 tile is 128 columns of C by 16 or 32 rows and its partial
 *                 is small) with a long K, where its measured cost model
 *                 predicts a gain, and only into a workspace large enough
 *                 (fp8_mm_workspace_size(..., 0) gives those bytes); larger
 *                 problems are not split (on every shape measured on B200 the
 *                 partials' round trip through L2 cost more than the shorter
 *                 main loop saved);
 *                 1: no split; 2 .. 4: exactly that many splits.
 * workspace       NULL: as fp8_mm (split_k 0: a short problem may split as a
 *                 cluster, without a workspace; 1: no split; 2 .. 4 need a
 *                 workspace), else device memory,
 *                 16-byte aligned, of workspace_bytes >=
 *                 fp8_mm_workspace_size(..., split_k) bytes. Its first 4096
 *                 bytes are counters: they must be zero before the first call
 *                 that uses the workspace (e.g. cudaMemsetAsync once after
 *                 allocation), and every completed call leaves them zero
 *                 again, so the workspace can be reused, also inside CUDA
 *                 graphs. The rest holds fp32 partial tiles. The caller owns
 *                 it; two calls that may run at the same time (e.g. on two
 *                 streams) need two workspaces. After FP8_ERR_DEVICE_TIMEOUT
 *                 it must be zeroed again.
 * Other arguments and errors as fp8_mm, plus: FP8_ERR_INVALID_ARG for
 * split_k outside 0..4 or a missing / too small workspace; FP8_ERR_UNSUPPORTED
 * when the problem cannot take that split (fewer k-blocks of 128 than splits
 * need, or more than 512 tile halves); FP8_ERR_ALIGNMENT for a misaligned
 * workspace. */
FP8LITE_API fp8_status fp8_mm_ws(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb,
                  const float* sa, const float* sb, fp8_layout layout,
                  int64_t M, int64_t N, int64_t K, int64_t batch,
                  int64_t stride_a, int64_t stride_b, int64_t stride_c,
                  const void* bias, const float* bias_scale, fp8_fmt bias_fmt,
                  void* out, void* workspace, size_t workspace_bytes, int32_t split_k,
                  void* stream);

/* FP8-in / FP8-out GEMM with delayed output scaling [mma@cebdd45d, bullet on
 * the fp8_mm_prequant_fp8 custom op for FP8-in/FP8-out GEMM; the later
 * fp8.py@f4c44ebf page drops that output for bf16 only, so it is an extra
 * entry point and fp8_mm stays bf16]:
 *
 *   y[b,i,j]   = (sum_k op(A_b)[i,k] op(B_b)[k,j]) / (sa*sb) + bias_j   (fp32,
 *                exactly as fp8_mm computes it before its bf16 rounding)
 *   out8[b,i,j] = sat_rne_out_fmt( fp32(y[b,i,j] * s) ),  s = out_ring->scale
 *                as it stood before the call (reported in *out_scale)
 *
 * out_ring is a delayed-scaling ring for the output: the amax of |y| over all
 * outputs (NaN ignored) is folded into it by the last CTA exactly as a
 * delayed fp8_quantize call folds its input's amax, and reported in
 * *out_amax (optional). The next layer can use out8 with *out_scale as its
 * FP8 operand without a separate quantize pass.
 * All arguments as fp8_mm, except: out8 device uint8[batch*stride_c]
 * (row-major [M,N] codes of out_fmt per batch; stride_c in elements = bytes);
 * out_ring required (4-byte aligned); out_scale required. Never splits K and
 * never swaps operands. Errors as fp8_mm; FP8_ERR_INVALID_ARG also for a bad
 * out_fmt or a NULL out_ring / out_scale. */
FP8LITE_API fp8_status fp8_mm_out8(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb,
                  const float* sa, const float* sb, fp8_layout layout,
                  int64_t M, int64_t N, int64_t K, int64_t batch,
                  int64_t stride_a, int64_t stride_b, int64_t stride_c,
                  const void* bias, const float* bias_scale, fp8_fmt bias_fmt,
                  fp8_fmt out_fmt, fp8_ring* out_ring, uint8_t* out8, float* out_amax, float* out_scale,
                  void* stream);

/* Workspace bytes fp8_mm_ws needs for this problem and split_k on the
 * current device (split_k 0: for the library's own choice): 0 when that call
 * would not split, or for arguments fp8_mm_ws rejects. */
FP8LITE_API size_t fp8_mm_workspace_size(int64_t M, int64_t N, int64_t K, int64_t batch, fp8_layout layout,
                                         int32_t split_k);

/* fp8_mm_ws with split_k = 2 .. 4, for callers that cannot allocate device
 * memory. The pages have no counterpart: it is an addition of this library.
 *
 * Who needs it: code that runs where cudaMalloc is not available or not
 * allowed -- a custom allocator or memory pool that owns every device byte,
 * a plug-in or callback invoked from inside another framework's step, a
 * real-time or embedded caller that may not allocate after start-up. Such a
 * caller has no way to provide fp8_mm_ws's workspace. This entry point
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * Its scratch is a 32 MiB device array of the library (a static device
 * variable): every GPU that loads the library holds it until the process
 * exits. The caller still passes the inputs and the output.
 *
 * Set-up: the first call on a device (with that device current) looks up the
 * array's device address and keeps it; that lookup may load the library's
 * GEMM module, which stream capture does not allow, so make the first call
 * on each device outside any capture.
 * Contents: every call on a device shares the array, which keeps the last
 * call's contents. Each call first clears the array's 4096-byte counter block
 * on `stream` (one cudaMemsetAsync; also after a call whose bounded wait gave
 * up), and the fp32 partial tiles are written before they are read, so no
 * state carries from one call into the next. Calls whose work overlaps on the
 * GPU (two streams, or two host threads, on one device) race on the array and
 * give undefined results: run them in order on one stream.
 * Result: bit for bit what fp8_mm_ws gives with the same split_k.
 * Errors: as fp8_mm_ws; FP8_ERR_INVALID_ARG for split_k outside 2 .. 4;
 * FP8_ERR_UNSUPPORTED when the split needs more scratch than the 32 MiB the
 * library holds (fp8_mm_workspace_size(..., split_k) > 33554432) or the
 * problem cannot take the split; FP8_ERR_CUDA if the address lookup or the
 * clear fails. */
FP8LITE_API fp8_status fp8_mm_splitk_static(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb,
                  const float* sa, const float* sb, fp8_layout layout,
                  int64_t M, int64_t N, int64_t K, int64_t batch,
                  int64_t stride_a, int64_t stride_b, int64_t stride_c,
                  const void* bias, const float* bias_scale, fp8_fmt bias_fmt,
                  void* out, int32_t split_k, void* stream);

/* Several independent fp8_mm problems in ONE launch: their output tiles
 * share one persistent grid, one prologue and one tail. Made for the
 * backward pass of a linear layer, whose dX (NN) and dW (TN) GEMMs both read
 * the gradient's codes and nothing of each other [test_fp8_mma.py@cebdd45d,
 * the dX / dW layout cases]. Each problem computes exactly what fp8_mm
 * computes with batch 1 (out = bf16_rne(acc/(sa*sb) + bias_j), fp32
 * accumulation over K in the same k-block order), so its output equals
 * fp8_mm's bit for bit.
 *
 * problems  HOST array of `count` descriptions (read during the call only)
 * count     1 .. FP8_MM_MAX_GROUP
 * Per problem, the fields mean what fp8_mm's arguments of the same name mean,
 * with batch = 1 and out a contiguous row-major bf16 [M, N]. The outputs
 * must not overlap each other or any operand.
 * Errors: as fp8_mm for any one problem (the first failing check decides),
 *         FP8_ERR_INVALID_ARG for a NULL array or count out of range. */
#define FP8_MM_MAX_GROUP 4
typedef struct fp8_mm_problem {
    const uint8_t* a8;
    const uint8_t* b8;
    const float* sa;
    const float* sb;
    const void* bias;        /* NULL, bf16[N], or FP8 codes[N] of bias_fmt */
    const float* bias_scale; /* NULL (bf16 bias) or device float (FP8 bias) */
    void* out;               /* device bf16[M*N], 4-byte aligned */
    int64_t M, N, K;
    int32_t fmt_a, fmt_b;    /* fp8_fmt values */
    int32_t layout;          /* fp8_layout value */
    int32_t bias_fmt;        /* fp8_fmt value, read only for an FP8 bias */
} fp8_mm_problem;
FP8LITE_API fp8_status fp8_mm_grouped(const fp8_mm_problem* problems, int32_t count, void* stream);

/* Synchronises the current device, then reads and clears the library's
 * device error word: FP8_ERR_DEVICE_TIMEOUT if a GEMM thread block gave up a
 * bounded wait since the last call (its output tile is then undefined),
 * FP8_OK otherwise, FP8_ERR_CUDA if the synchronisation failed.
 * A diagnostic, not a hot-path call: it waits for all work on the device
 * (every stream) and cannot be captured into a CUDA graph. After a timeout,
 * a caller-owned split-K workspace (fp8_mm_ws) must be zeroed again before
 * its next use; fp8_mm_splitk_static clears its own counters every call. */
FP8LITE_API fp8_status fp8_last_device_error(void);

/* Bias gradient of a linear layer: out[j] = bf16_rne( sum_i g[i][j] ), the
 * sum over the rows (tokens, leading dimensions flattened) accumulated in
 * fp32 [fp8.py@f4c44ebf, bullets on the bias column-sum and the 3-D
 * backward]. It is a separate call so that it runs only when the bias needs
 * a gradient, and it reads the bf16 gradient (not its FP8 codes).
 * g    device bf16[rows * cols], row-major, 4-byte aligned
 * out  device bf16[cols], 2-byte aligned
 * rows >= 1, cols >= 1 and even.
 * Errors: FP8_ERR_INVALID_ARG, FP8_ERR_ALIGNMENT (odd cols, misaligned
 *         pointers), FP8_ERR_CUDA. */
FP8LITE_API fp8_status fp8_bias_grad(const void* g, int64_t rows, int64_t cols, void* out, void* stream);

/* Diagnostic of the failure path: launches one tiny kernel whose single
 * thread waits, through the same bounded wait the GEMM uses, on a barrier
 * that nothing arrives at. After limit_us (1 .. 1e6 microseconds) the wait
 * gives up and records a timeout in the device error word, exactly as a stuck
 * GEMM would, and the kernel returns normally (no fault, no trap): the next
 * fp8_last_device_error() reports FP8_ERR_DEVICE_TIMEOUT and clears it.
 * Errors: FP8_ERR_INVALID_ARG (limit out of range), FP8_ERR_CUDA. */
FP8LITE_API fp8_status fp8_selftest_wait_timeout(uint32_t limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8LITE_H */
