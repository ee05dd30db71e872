/*
 * q4.h -- C ABI of libq4: grouped symmetric round-to-nearest (RTN) int4/int8
 * weight quantization and the quantized matmul, on one NVIDIA B200 (sm_100a).
 *
 * The quantization rule is the one of pack()/unpack() on the page
 * "量化推理：INT8/INT4 的体积、困惑度与速度为什么不同步" and of "Huit bits,
 * puis quatre", section "Arrondir":
 *   - flatten the weight tensor row-major and cut it into groups of `group`
 *     consecutive values;
 *   - scale = max|w| / qmax in fp32 (qmax = 7 for int4, 127 for int8); a
 *     scale that comes out as 0 is replaced by 1;
 *   - code = clip(rint(w / scale), -qmax, qmax), the quotient being one IEEE
 *     fp32 division and rint rounding half to even;
 *   - int4: byte t of the payload = (code[2t] + 8) | (code[2t+1] + 8) << 4
 *     (even element in the low nibble); int8: the code's two's-complement byte;
 *   - dequantized weight w' = float(code) * scale (one fp32 multiplication).
 *
 * Conventions for every call:
 *   - Matrices are row-major. A weight matrix W is [rows = N output
 *     channels][cols = K inputs]; activations x are [M][K]; y is [M][N].
 *   - Every pointer argument is a DEVICE pointer (cudaMalloc'd or torch
 *     memory on the current device) owned by the caller; the library
 *     allocates nothing, keeps no pointer after a call returns and holds no
 *     global state.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls only
 *     enqueue work: they return before the GPU finishes. Argument errors are
 *     detected on the host BEFORE anything is enqueued, and nothing is
 *     enqueued when a call returns an error.
 *   - No call falls back to the CPU: a shape a kernel does not cover returns
 *     Q4_ERR_UNSUPPORTED.
 */
#ifndef Q4_H
#define Q4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define Q4_API __attribute__((visibility("default")))
#else
#define Q4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum q4_status {
    Q4_OK = 0,
    Q4_ERR_ARG = 1,         /* a null pointer, bits not 4/8, group < 1, a shape the format cannot hold */
    Q4_ERR_UNSUPPORTED = 2, /* a valid format that this kernel does not cover (see each call) */
    Q4_ERR_CUDA = 3,        /* a CUDA runtime call or a kernel launch failed */
    Q4_ERR_NONFINITE = 4,   /* qpack saw Inf or NaN (reported through its status word) */
    Q4_ERR_WORKSPACE = 5,   /* qgemm workspace null, too small or not 256-byte aligned */
    Q4_ERR_SCRATCH_LIMIT = 6 /* qgemm_noalloc: the problem needs more than
                               Q4_NOALLOC_SCRATCH_BYTES of scratch */
} q4_status;

typedef enum q4_xdtype {
    Q4_X_F32 = 0,  /* x is float32 */
    Q4_X_BF16 = 1  /* x is bfloat16 (raw 16-bit values) */
} q4_xdtype;

/* Bits OR-ed into the optional device status words of qpack and qgemm. */
#define Q4_STATUS_NONFINITE 1u /* qpack: a group holds Inf or NaN */
#define Q4_STATUS_TIMEOUT 2u   /* qgemm: a bounded wait inside a kernel gave up; y is invalid */

/* Library version, MAJOR*10000 + MINOR*100 + PATCH. */
Q4_API int q4_version(void);

/* Human-readable name of a status code (static string, never NULL). */
Q4_API const char *q4_status_str(q4_status s);

/* The CUDA error behind the last Q4_ERR_CUDA returned to this host thread: the
 * failing step, cudaGetErrorName and cudaGetErrorString, or "" if none. The string
 * belongs to the library and stays valid until the next call on this thread. */
Q4_API const char *q4_last_cuda_error(void);

/* Bytes of packed codes for rows*cols weights: rows*cols*bits/8 (pack()'s
 * payload length check on the "量化推理" page). Returns 0 for invalid
 * arguments (negative sizes, bits not 4/8, odd rows*cols with bits = 4). */
Q4_API size_t q4_payload_bytes(int64_t rows, int64_t cols, int bits);

/* Number of fp32 scales: rows*cols/group, one per group. Returns -1 when
 * group < 1 or does not divide rows*cols. */
Q4_API int64_t q4_num_scales(int64_t rows, int64_t cols, int64_t group);

/*
 * qpack -- quantize and pack (pack() on the "量化推理" page; the rule of
 * "Huit bits, puis quatre", section "Arrondir").
 *   w        [rows*cols] fp32, row-major, 16-byte alignment recommended
 *   bits     4 or 8
 *   group    1 <= group, group divides rows*cols; groups run over the
 *            flattened tensor, so a group may span rows (group = rows*cols
 *            gives one scale for the whole tensor)
 *   payload  out, q4_payload_bytes(rows, cols, bits) bytes
 *   scales   out, q4_num_scales(rows, cols, group) floats
 *   status_word  optional (may be NULL) device uint32; the kernels OR
 *            Q4_STATUS_NONFINITE into it when any weight is Inf or NaN (the
 *            outputs are then unspecified for that group). The caller zeroes
 *            it and reads it after synchronizing the stream.
 * Errors: Q4_ERR_ARG (null w/payload/scales, bits, group, odd rows*cols for
 * int4, negative sizes), Q4_ERR_CUDA. rows*cols == 0 enqueues nothing.
 * Results are bit-identical to the definition above for every input.
 */
Q4_API q4_status qpack(const float *w, int64_t rows, int64_t cols, int bits, int64_t group,
                uint8_t *payload, float *scales, uint32_t *status_word, void *stream);

/*
 * qdequant -- decode packed codes to fp32 weights (unpack() on the "量化推理"
 * page): w_out[i] = float(code[i]) * scales[i / group], bit-exact.
 *   payload  [q4_payload_bytes(rows, cols, bits)] bytes from qpack
 *   scales   [q4_num_scales(rows, cols, group)] floats
 *   w_out    out, [rows*cols] fp32
 * Errors: as qpack. rows*cols == 0 enqueues nothing.
 */
Q4_API q4_status qdequant(const uint8_t *payload, const float *scales, int64_t rows, int64_t cols,
                   int bits, int64_t group, float *w_out, void *stream);

/*
 * Workspace bytes that qgemm needs for this problem: the activations converted once
 * into tensor-core fragments (exact bf16 pieces, 3 per fp32 activation, in MMA order;
 * for one row of x, per 128-byte stage either those pieces or exact 40-bit fixed-point
 * digits, 2064 bytes per int4 stage and 1040 per int8 stage). One row of x needs none (0)
 * when each CTA's share of K, at most 4096, is built on chip; so do two to four fp32 rows
 * when, in addition, the plan runs one CTA per SM (N up to 74 x 128 rows, as planned for
 * 148 SMs) and their pieces fit in its shared memory. Groups of whole rows
 * (group a multiple of K) add N floats, rounded up to 256 bytes, at the start: their
 * scales spread to one per row. The any-group path needs none (0). Same arguments as
 * qgemm. Returns 0 for arguments qgemm rejects. Depends only on the arguments, not on
 * the device.
 */
Q4_API size_t q4_qgemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int64_t group,
                                q4_xdtype xt);

/*
 * qgemm -- y[m][n] = sum_k x[m][k] * w'[n][k], w' the dequantized weights,
 * computed from the packed codes without materialising w' (the
 * QuantizedMatmul of "Huit bits, puis quatre", section "Ranger des entiers
 * dans des f32": the same numbers as the product with the dequantized
 * weights, up to the order of the sums).
 *   x        [M][K], fp32 or bf16 per xt, row-major, 16-byte aligned (any
 *            alignment of the element type on the any-group path below)
 *   payload  q4_payload_bytes(N, K, bits) bytes from qpack of an [N][K] matrix,
 *            16-byte aligned (any alignment on the any-group path)
 *   scales   [N*K/group] floats from the same qpack
 *   y        out, [M][N] fp32
 *   workspace  device scratch of at least q4_qgemm_workspace_bytes(...)
 *            bytes, 256-byte aligned, owned by the caller. Its contents need
 *            no initialisation and are meaningless after the call. Two calls
 *            that may run at the same time must not share a workspace.
 *   status_word  optional (may be NULL) device uint32. Every wait inside the
 *            kernels is bounded; if one ever gives up, Q4_STATUS_TIMEOUT is
 *            OR-ed into this word and y must be treated as invalid. The
 *            caller zeroes it and reads it after synchronizing the stream.
 * Paths: M <= 63, or fp32 x at any M: the fused unpack->dequant->GEMV kernel
 * (rows of x in chunks of 16). bf16 x with M >= 64: the tensor-core GEMM.
 * Accuracy: |y - y_exact| <= 1e-5 * sum_k |w'[n][k] x[m][k]| + 1e-6 for every
 * finite x (y_exact = the fp64 sum), however widely the magnitudes of x spread: the
 * codes enter the tensor cores exactly; the activations enter as three exact bf16
 * pieces, or (one row of x, a 128-byte stage whose activations span at most 2^21)
 * as fixed-point digits within 2^-18 of each activation's own magnitude; the sums
 * are fp32. Activations below 2^-110 in magnitude may lose bits below 2^-133.
 * Groups: every group qpack accepts (a divisor of N * K; int4 needs N * K even;
 * else Q4_ERR_ARG). With K % 32 == 0 and a group that divides K in a multiple of 32
 * (per-channel scales are group = K), or a multiple of K (groups of whole rows, down
 * to one scale for the whole matrix, the INT4_TENSOR format of the "量化推理：
 * INT8/INT4 ..." page), the paths above run; groups of whole rows are first spread
 * to one scale per row in the workspace (Q4_QGEMM_WEIGHTS_STATIC has no effect on
 * such calls). Any other group or K (g = 16, g = 48, g = 3K/2 crossing rows at a
 * different offset in every row, odd K) runs on the any-group kernel: no workspace,
 * exact fp32 w' as qdequant gives it, fp32 products and compensated fp32 sums
 * (error <= 2^-20 * sum_k |w'x|); it is bound by its per-weight integer work, not
 * by HBM.
 * On the fused paths N, K <= 2^30 and M <= 1048560 (65535 chunks of 16 rows), else
 * Q4_ERR_UNSUPPORTED. M, N >= 0; M == 0 or N == 0 enqueues nothing.
 * Errors: Q4_ERR_ARG (null pointers, bits, shapes), Q4_ERR_UNSUPPORTED,
 * Q4_ERR_WORKSPACE, Q4_ERR_CUDA.
 */
Q4_API q4_status qgemm(const void *x, q4_xdtype xt, int64_t M, const uint8_t *payload,
                const float *scales, int64_t N, int64_t K, int bits, int64_t group, float *y,
                void *workspace, size_t workspace_bytes, uint32_t *status_word, void *stream);

/* qgemm_ex flags. */
#define Q4_QGEMM_WEIGHTS_STATIC 1u

/*
 * qgemm_ex -- qgemm with option flags (the pages have no counterpart: this is a
 * launch-overlap option for sequences of calls, e.g. the linear layers of one
 * decode step, whose packed weights stay fixed while the sequence runs).
 *   flags  0, or Q4_QGEMM_WEIGHTS_STATIC: payload and scales may be read while
 *          the kernel enqueued before this call on the same stream is still
 *          running (programmatic dependent launch), so that their streaming
 *          overlaps that kernel's tail. The caller promises that the last write
 *          to payload and scales finished before that previous kernel started
 *          (weights packed once and reused qualify; packing them with the call
 *          just before does not). x, y, the workspace and the status word keep
 *          full stream order: every read of x and every write waits until the
 *          previous kernel has finished. Only the fused GEMV path (not the
 *          bf16 M >= 64 tensor-core GEMM) uses the flag; the result is bit-for-bit
 *          the same as without it.
 *   Other arguments, results and errors as qgemm; unknown flag bits are
 *   Q4_ERR_ARG. qgemm(...) is qgemm_ex(..., flags = 0, ...).
 */
Q4_API q4_status qgemm_ex(const void *x, q4_xdtype xt, int64_t M, const uint8_t *payload,
                const float *scales, int64_t N, int64_t K, int bits, int64_t group, float *y,
                void *workspace, size_t workspace_bytes, uint32_t flags, uint32_t *status_word,
                void *stream);

/* Size of the one device scratch buffer that qgemm_noalloc uses (4 MiB). */
#define Q4_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * qgemm_noalloc -- qgemm without a caller workspace and without any device
 * allocation in the call. The pages have no counterpart: this is an interface
 * convenience for callers that must not allocate (e.g. code running under a
 * memory budget fixed up front). The result is the same as qgemm's.
 *   Arguments as qgemm, minus workspace and workspace_bytes.
 *   Scratch: a file-scope device array of Q4_NOALLOC_SCRATCH_BYTES inside
 *            libq4, one per device, created by the CUDA runtime with the
 *            library's module. The first call on each device (with that device
 *            current) looks up its address once and caches it; make that first
 *            call before any stream capture on the device. The cached address
 *            lives as long as the device's primary context: after cudaDeviceReset
 *            (or anything else that destroys it), do not call qgemm_noalloc again
 *            in the same process. Nothing in the
 *            scratch has to start at zero: each call writes every byte it reads.
 *   Limit:   problems with q4_qgemm_workspace_bytes(...) greater than
 *            Q4_NOALLOC_SCRATCH_BYTES are rejected with Q4_ERR_SCRATCH_LIMIT
 *            before anything is enqueued (M <= 16 fits for K up to about 60000).
 *   Concurrency: every call on a device shares the one scratch, so two calls
 *            that may overlap on the GPU (different streams with no ordering
 *            between them) race and give wrong results. Calls on one stream,
 *            or otherwise ordered, are safe.
 * Errors: those of qgemm except Q4_ERR_WORKSPACE, plus Q4_ERR_SCRATCH_LIMIT;
 * Q4_ERR_CUDA also when the scratch address cannot be obtained.
 */
Q4_API q4_status qgemm_noalloc(const void *x, q4_xdtype xt, int64_t M, const uint8_t *payload,
                const float *scales, int64_t N, int64_t K, int bits, int64_t group, float *y,
                uint32_t *status_word, void *stream);

/*
 * ---- Decode stack: every GEMV of a decode step in one persistent kernel ("Huit
 * bits, puis quatre", section "La vitesse": a step made of many short kernels is
 * bound by launches and pipeline fills; the weights pay off once the GEMVs are
 * fused so that they wait on memory). One row of activations per GEMV, the
 * arithmetic and accuracy of qgemm.
 *
 * GEMVs are grouped in levels: the GEMVs of level l may read (as x) what GEMVs of
 * levels < l write (as y), and nothing that GEMVs of level >= l write. Inside one
 * launch, level l starts reading x only once every GEMV of level l - 1 has computed
 * all of y: where x is a 16-byte aligned slice of one level l - 1 GEMV's y, it is read
 * as the sum of the partial sums the kernel keeps for those rows (the very values that
 * GEMV's y receives); any other x is read from memory once the y it overlaps is
 * written. Weights stream continuously across levels. A transformer layer is four
 * levels: q|k|v, o, gate|up, down. Every y is complete when the run ends.
 */
typedef struct q4_stack_gemv {
    const uint8_t *payload;  /* [N][K*bits/8] from qpack of an [N][K] matrix, 16-byte aligned */
    const float *scales;     /* [N*K/group] from the same qpack */
    const void *x;           /* [K] activations, fp32 or bf16 (the stack's xt), 16-byte aligned */
    float *y;                /* [N] output; must not overlap another GEMV's y of the same level */
    int64_t N, K;
    int64_t group;           /* divides K, multiple of 32 (group = K: one scale per row) */
    int32_t level;           /* 0 for the first; each next GEMV has the same level or one more */
    int32_t reserved;        /* 0 */
} q4_stack_gemv;

/* Host-side record of a prepared stack (filled by q4_stack_prepare, read by
 * q4_stack_run; plain bytes, may be copied). */
typedef struct q4_stack_plan {
    uint64_t opaque[32];
} q4_stack_plan;

/* Workspace bytes q4_stack_prepare needs for these GEMVs: the GEMV and level tables
 * (one 2D TMA descriptor per GEMV), two counters per level, each CTA's share of every
 * level, and three buffers for the partial sums of 240-row blocks split between CTAs
 * (each sized for the level that needs most on a 148-SM B200). Returns 0 for
 * arguments q4_stack_prepare rejects. */
Q4_API size_t q4_stack_workspace_bytes(const q4_stack_gemv *gemvs, int32_t count, int bits, q4_xdtype xt);

/*
 * q4_stack_prepare -- validate the GEMVs and write the stack's tables into the
 * workspace, then synchronize `stream` (this call is not for stream capture).
 *   gemvs      HOST array of count GEMVs, in level order
 *   bits       4 or 8, for every GEMV; all GEMVs must map to the same kernel variant
 *              (the same groups per 128-byte tile: e.g. all group = 128, or all
 *              one scale per row)
 *   xt         dtype of every x
 *   workspace  device memory of q4_stack_workspace_bytes(...) bytes, 256-byte
 *              aligned, owned by the caller; it belongs to the plan until the
 *              caller stops running it. The weights, x and y pointers are stored:
 *              they must stay valid, and payload and scales must not change, while
 *              the plan is run.
 *   plan       out
 * Errors: Q4_ERR_ARG (null pointers, bits, sizes, levels out of order, reserved != 0),
 * Q4_ERR_UNSUPPORTED (group not a multiple of 32 dividing K, mixed kernel variants,
 * misaligned payload or x, N or K > 2^30), Q4_ERR_WORKSPACE, Q4_ERR_CUDA.
 */
Q4_API q4_status q4_stack_prepare(const q4_stack_gemv *gemvs, int32_t count, int bits, q4_xdtype xt,
                void *workspace, size_t workspace_bytes, q4_stack_plan *plan, void *stream);

/*
 * q4_stack_run -- one launch of the prepared stack on `stream` (capturable in a CUDA
 * graph). Every y is written; results are deterministic and, per GEMV, within
 * qgemm's accuracy bound for the x it read.
 *   status_word  optional device uint32; Q4_STATUS_TIMEOUT is OR-ed into it if a
 *              bounded wait gave up (every y is then invalid; the workspace stays
 *              usable).
 * Two runs of one plan (or plans sharing a workspace) must not overlap in time.
 * Errors: Q4_ERR_ARG (not a prepared plan), Q4_ERR_CUDA (e.g. the grid cannot be
 * resident at once on this device).
 */
Q4_API q4_status q4_stack_run(const q4_stack_plan *plan, uint32_t *status_word, void *stream);

/*
 * q4_stack_set_wait_limit -- the bound of every wait inside the stack kernel, in
 * nanoseconds (1e9 after q4_stack_prepare). A wait that reaches it gives up: the run
 * then ends without waiting further, ORs Q4_STATUS_TIMEOUT into the status word, and
 * leaves the workspace ready for the next run. A bound shorter than the waits of a
 * working run (microseconds) makes that run give up; a caller that watches for a
 * broken producer upstream may want a bound shorter than the default.
 * Errors: Q4_ERR_ARG (not a prepared plan).
 */
Q4_API q4_status q4_stack_set_wait_limit(q4_stack_plan *plan, uint64_t nanoseconds);

/*
 * ---- GPTQ host quantizer ("Huit bits, puis quatre", section "Arrondir mieux :
 * GPTQ"). Host code, fp64; every pointer below is HOST memory owned by the
 * caller. The result is a payload + scales pair in exactly the format of
 * qpack, read by qdequant and qgemm unchanged: the same codes, chosen so that
 * the layer's output x W'^T moves as little as possible on typical inputs x.
 */

/*
 * q4_gptq_hessian -- H += sum over the rows r of x: x[r]^T x[r], in fp64.
 *   x  [rows][K] fp32 calibration inputs of the layer (row-major)
 *   H  [K][K] fp64, accumulated in place (zero it before the first batch)
 *   threads  worker threads (0 = all hardware threads); each owns rows of H,
 *            so the result does not depend on it
 * Errors: Q4_ERR_ARG (shapes, null), Q4_ERR_NONFINITE (x holds NaN or Inf;
 * H is left untouched).
 */
Q4_API q4_status q4_gptq_hessian(const float *x, int64_t rows, int64_t K, double *H, int threads);

/*
 * q4_gptq_prepare -- U, upper triangular, with (H + damp * mean(diag H) * I)^-1
 * = U^T U. The page adds damp = 0.01. O(K^3), split over threads.
 *   H  [K][K] fp64 (symmetric; the mean of its two triangles is used)
 *   U  [K][K] fp64 out, zeros below the diagonal
 *   threads  worker threads (0 = all hardware threads); U does not depend on it
 * Errors: Q4_ERR_ARG (null, K < 1, damp < 0, mean(diag H) <= 0, or the damped
 * H is not positive definite).
 */
Q4_API q4_status q4_gptq_prepare(const double *H, int64_t K, double damp, double *U, int threads);

/*
 * q4_gptq_quantize -- the payload and scales of W [N][K] (fp32, row-major,
 * groups of `group` consecutive weights along K) by GPTQ: the columns k are
 * quantized in order; the error of column k, (w - code * scale) / U[k][k], is
 * taken off each later column j times U[k][j]; a group's scales are set, by
 * the qpack rule, from the corrected weights when its first column is reached.
 *   U        from q4_gptq_prepare (any upper triangular U with a nonzero
 *            diagonal is accepted; a diagonal U gives exactly qpack's result)
 *   payload  out, q4_payload_bytes(N, K, bits) bytes
 *   scales   out, N * K / group floats
 *   threads  worker threads over rows (0 = all); the result does not depend on it
 * Cost: N * K^2 / 2 multiply-subtracts. Requirements: bits 4 or 8, group
 * divides K, N * K even for int4.
 * Errors: Q4_ERR_ARG, Q4_ERR_NONFINITE (W holds NaN or Inf, or an ill-conditioned U
 * drove a corrected weight outside the fp32 range; outputs untouched).
 */
Q4_API q4_status q4_gptq_quantize(const float *w, int64_t N, int64_t K, const double *U, int bits,
                int64_t group, uint8_t *payload, float *scales, int threads);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H */
