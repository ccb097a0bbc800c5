/*
 * q4.h -- C ABI of libq4: affine 4-bit, group-32, weight-only quantized
 * matmul on NVIDIA B200 (sm_100a).
 *
 * Format (model card "personaplex-edge-q4", section "Release details":
 * "affine Q4, group size 32, BF16 activations"; the packed size it prints,
 * 4.87 GiB for 8,371,408,896 parameters, is 5 bits per weight):
 *
 *   W        [N, K]      bf16, row-major: N outputs ("out"), K inputs ("in").
 *   codes    [N, K/2]    uint8: byte k/2 of row n holds q[n,k] in bits 0..3
 *                        when k is even and q[n,k+1] in bits 4..7.  Each
 *                        16-byte run is one group of 32 codes.
 *   scales   [N, K/32]   bf16, one per group of 32 consecutive k of a row.
 *   biases   [N, K/32]   bf16, likewise.
 *   w_hat[n,k] = scales[n,k/32] * q[n,k] + biases[n,k/32],  q in 0..15.
 *
 * The matmul multiplies by the transposed weight, y = x . w_hat^T, as the
 * Swift/MLX blog "NVIDIA PersonaPlex 7B on Apple Silicon" (section
 * "Depformer: per-step weight switching") calls quantizedMM with
 * transpose: true, groupSize and bits.
 *
 * Conventions for every entry point:
 *  - All pointers are DEVICE pointers, allocated and owned by the caller.
 *    The library allocates no device memory and keeps no pointer after a
 *    call returns.  bf16 values are passed as their 16-bit patterns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronize the host or copy between host
 *    and device.
 *  - Arguments are validated, and every host-side step of the launches
 *    (tensor-map encoding, launch configurations) is done, before anything is
 *    enqueued: a status other than Q4_ERR_CUDA means nothing was enqueued.
 *    Q4_ERR_CUDA from a launch that the CUDA runtime rejected may leave the
 *    earlier launches of the same call enqueued.  q4_last_error() returns a
 *    message for the last non-OK status of the calling thread.
 *  - Every wait inside the kernels is bounded (one second); a kernel that
 *    gives one up writes NaN where it cannot vouch for a result and raises a
 *    device flag that q4_device_status() reports.  Results of work enqueued
 *    since the flag was last clear are invalid while it is set.
 *  - Alignment: W, W_out, codes and x must be 16-byte aligned; scales,
 *    biases and y 2-byte aligned.  Row strides are implied by K (dense).
 *  - Sizes: 0 <= M, N; 32 <= K, K % 32 == 0.  M == 0 or N == 0 is a no-op.
 *    `group` must be 32.  K <= 2^24, N <= 2^40, M <= 2^31.
 *  - Output buffers must not overlap inputs (the one exception: a residual
 *    operand may be the output buffer itself, see q4_matmul_residual).
 *  - Device: compute capability 10.0 (B200, sm_100a) only; any other device
 *    returns Q4_ERR_UNSUPPORTED.
 */
#ifndef Q4_H_
#define Q4_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define Q4_API __attribute__((visibility("default")))
#else
#define Q4_API
#endif

typedef uint16_t q4_bf16;                 /* bf16 bit pattern */
typedef struct CUstream_st* q4_stream_t;  /* same type as cudaStream_t */

typedef enum {
  Q4_OK = 0,
  Q4_ERR_NULL = 1,         /* a required pointer is NULL                      */
  Q4_ERR_SHAPE = 2,        /* negative size, K not a positive multiple of 32  */
  Q4_ERR_ALIGN = 3,        /* pointer misaligned for its role                 */
  Q4_ERR_UNSUPPORTED = 4,  /* group != 32, K too large, or not an sm_100 GPU  */
  Q4_ERR_RANGE = 5,        /* step outside [0, num_steps)                     */
  Q4_ERR_CUDA = 6          /* a CUDA runtime call or a launch failed          */
} q4_status;

/*
 * q4_quantize -- per row n and group g of 32 consecutive k:
 *   mn, mx = min, max of the group;
 *   scale  = bf16(fp32(mx - mn) / 15)   (IEEE fp32 subtraction and division,
 *                                        round to nearest even, then RNE to bf16)
 *   bias   = bf16(mn)                   (exact)
 *   q      = 0 if scale == 0, else clamp(round_half_even((w - bias)/scale), 0, 15),
 *            the quotient taken in IEEE binary64.
 * The pages name the method (model card "personaplex-edge-q4", opening
 * paragraph and "Release details"; GeekNews summary of the Swift port,
 * "Arsitektur model dan konversi": 4-bit quantization in the conversion
 * script) but not its arithmetic; this is the plainest reading of "affine,
 * 4-bit, group 32".  Offline: not on the matmul path.
 * In:  W [N, K] bf16.   Out: codes [N, K/2], scales [N, K/32], biases [N, K/32].
 * Non-finite weights give unspecified codes (not checked on the device).
 */
Q4_API q4_status q4_quantize(const q4_bf16* W, int64_t N, int64_t K, int group,
                      uint8_t* codes, q4_bf16* scales, q4_bf16* biases,
                      q4_stream_t stream);

/*
 * q4_dequantize -- W_out[n,k] = bf16_rne(scale * q + bias), the product and
 * sum taken in IEEE binary64 (exact for every non-degenerate group).  The
 * model card "personaplex-edge-q4" (section "Conversion and weight
 * validation") reconstructs every packed tensor this way to validate it.
 * In: codes [N, K/2], scales, biases [N, K/32].  Out: W_out [N, K] bf16.
 */
Q4_API q4_status q4_dequantize(const uint8_t* codes, const q4_bf16* scales,
                        const q4_bf16* biases, int64_t N, int64_t K, int group,
                        q4_bf16* W_out, q4_stream_t stream);

/*
 * q4_matmul -- y[m,n] = sum_k x[m,k] * w_hat[n,k], accumulated in fp32 and
 * rounded to bf16 (nearest even), with the weights read in packed form and
 * never expanded to bf16 in memory (model card "personaplex-edge-q4",
 * opening paragraph: the packed weights run through a quantized matmul and
 * are not expanded back to BF16).
 * In:  x [M, K] bf16 (row-major), codes [N, K/2], scales, biases [N, K/32].
 * Out: y [M, N] bf16 (row-major).
 * Kernel by problem (the same for a problem alone or batched): M = 1, 2 the
 * CUDA-core GEMV (exact products x * (128 + q) in fp32, the offset removed
 * per group); M = 3..16 with K % 256 == 0 and 16-byte aligned x, codes,
 * scale and bias rows, the group-sum tensor-core kernel (exact sums of
 * (128 + q) * x per group of 32 on the tensor cores, the group's scale and
 * bias applied in fp32; the launch's 128-input steps are spread evenly over
 * the SMs, so a tile may be shared by several CTAs whose fp32 partial sums
 * are added in a fixed order); otherwise M = 3..8 tensor-core weight
 * streaming where its shared and tensor memory hold the problem (16-byte
 * aligned scale and bias rows, segments * M <= 128); otherwise, for M >= 3
 * with K % 256 == 0 and aligned scale rows, tensor-core tiles; otherwise the
 * GEMV on pairs of activation rows.  Every kernel reads each weight byte once
 * per call, except the GEMV on pairs (once per pair).  The streaming and tile
 * kernels feed each weight to the MMA as two bf16 parts hi + lo with
 * |s*q + b - hi - lo| <= ~2^-16 |s*q + b| (two MMAs per K step), so no path
 * rounds w_hat to bf16.  Results are deterministic: the same call gives the
 * same bits.  On the GEMV, the weight-streaming kernel and the tiles a
 * problem's result is also the same alone or in any batch; on the group-sum
 * kernel the fp32 partial sums follow the launch's split over the SMs, so a
 * problem can differ in the last bits between batches (always within the
 * acceptance bound).  A group-sum launch that shares tiles takes a small
 * stream-ordered workspace (cudaMallocAsync / cudaFreeAsync on `stream`:
 * about 2 * SMs * 128 * 2 * M * 4 bytes plus SMs counters, zeroed by a
 * cudaMemsetAsync); an allocation failure is Q4_ERR_CUDA.
 * Launch-order contract: the kernels may be launched with programmatic
 * dependent launch; they read nothing written by an earlier kernel in the
 * stream before that kernel has completed.
 */
Q4_API q4_status q4_matmul(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* codes,
                    const q4_bf16* scales, const q4_bf16* biases, int64_t N,
                    int group, q4_bf16* y, q4_stream_t stream);

/*
 * q4_matmul_step -- the per-step weight slice of a stacked tensor (Swift/MLX
 * blog, section "Depformer: per-step weight switching": one weight tensor of
 * [num_steps * N, K] with scales and biases stacked the same way; step s
 * uses rows [s*N, (s+1)*N) of all three).  Equivalent to q4_matmul on
 * codes + s*N*K/2, scales + s*N*K/32, biases + s*N*K/32.
 * Returns Q4_ERR_RANGE unless 0 <= step < num_steps.
 */
Q4_API q4_status q4_matmul_step(const q4_bf16* x, int64_t M, int64_t K,
                         const uint8_t* codes, const q4_bf16* scales,
                         const q4_bf16* biases, int64_t N, int64_t num_steps,
                         int64_t step, int group, q4_bf16* y, q4_stream_t stream);

/*
 * Output epilogues: a step of the feed-forward block that follows the
 * matmul, fused into it so that the fp32 accumulator is rounded to bf16 once.
 * The pages name the blocks these projections belong to (Swift/MLX blog,
 * section "Reusing the Mimi codec": KV cache, RoPE, SwiGLU and RMSNorm are
 * shared with the earlier ports; GeekNews summary, section "Arsitektur model
 * dan konversi", likewise) and fuse per-step kernel dispatches (Swift/MLX
 * blog, "Performance optimizations"); the fused forms are defined here.
 *   Q4_EPI_NONE      y = acc
 *   Q4_EPI_RESIDUAL  y = bf16(r + acc), r [M, N] bf16 (the residual stream;
 *                    r may be y itself, an in-place update)
 *   Q4_EPI_SWIGLU    y = bf16(silu(acc) * acc_up), silu(z) = z / (1 + e^-z),
 *                    acc the gate projection's and acc_up the up
 *                    projection's fp32 accumulators (weights of the same
 *                    shape), both from one pass in one launch on every
 *                    kernel: silu sees the fp32 gate.
 */
typedef enum { Q4_EPI_NONE = 0, Q4_EPI_RESIDUAL = 1, Q4_EPI_SWIGLU = 2 } q4_epilogue;

/* One problem of q4_matmul_batch: pointers and sizes as for q4_matmul, plus
 * an optional epilogue (all-zero fields mean Q4_EPI_NONE). */
typedef struct {
  const q4_bf16* x;       /* [M, K] activations, 16-byte aligned   */
  const uint8_t* codes;   /* [N, K/2], 16-byte aligned (the gate for SWIGLU) */
  const q4_bf16* scales;  /* [N, K/32]                               */
  const q4_bf16* biases;  /* [N, K/32]                               */
  q4_bf16* y;             /* [M, N] output                           */
  int64_t N;
  int64_t K;
  int32_t epilogue;       /* q4_epilogue                              */
  int32_t reserved;       /* must be 0                                */
  const q4_bf16* r;       /* RESIDUAL: [M, N], 2-byte aligned; else NULL */
  const uint8_t* up_codes;   /* SWIGLU: up projection, as codes/scales/biases */
  const q4_bf16* up_scales;
  const q4_bf16* up_biases;
} q4_matmul_desc;

/*
 * q4_matmul_residual -- y = bf16(r + x . w_hat^T), the sum taken in fp32
 * before the one rounding: the attention output and down projections
 * adding their result to the residual stream.  r [M, N] bf16, 2-byte
 * aligned; r == y updates the stream in place; any other overlap of r and y
 * is an error (Q4_ERR_SHAPE).  Same kernels, alignment and status codes as
 * q4_matmul.
 */
Q4_API q4_status q4_matmul_residual(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* codes,
                                    const q4_bf16* scales, const q4_bf16* biases, int64_t N, int group,
                                    const q4_bf16* r, q4_bf16* y, q4_stream_t stream);

/*
 * q4_matmul_swiglu -- h = bf16(silu(x . w_hat_gate^T) * (x . w_hat_up^T)):
 * the gate and up projections of the SwiGLU MLP and its activation in one
 * call (Q4_EPI_SWIGLU above).  Both weights are [N, K] in the packed format
 * with the same alignment rules as q4_matmul; h [M, N] must not overlap any
 * input.  Kernels as q4_matmul chooses them; every kernel computes the gate
 * and up products in one pass (one launch) and keeps both in fp32 until the
 * single rounding of h.
 */
Q4_API q4_status q4_matmul_swiglu(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* gate_codes,
                                  const q4_bf16* gate_scales, const q4_bf16* gate_biases,
                                  const uint8_t* up_codes, const q4_bf16* up_scales,
                                  const q4_bf16* up_biases, int64_t N, int group, q4_bf16* h,
                                  q4_stream_t stream);

/*
 * q4_matmul_batch -- `count` independent matmuls sharing the number of
 * activation rows M, each computing what q4_matmul computes (on the same
 * kernel; see q4_matmul for the group-sum kernel's summation order), enqueued
 * as few kernel launches as possible: one for up to 256 problems that take
 * the bulk-copy GEMV path (or the weight-streaming path), one for up to 160
 * weights (a SwiGLU problem counts two) with at most 8 distinct activation
 * tensors on the group-sum path, one per problem on the tensor-core tile
 * path and on the GEMV's generic fallback.  The Swift/MLX blog ("Performance optimizations":
 * compiling the temporal transformer fuses its ~450 per-step kernel
 * dispatches) and the ONNX README ("All four variants": CUDA Graph capture)
 * both cut per-call launch overhead; this is that fusion for a whole weight
 * stream (every projection of a decode step) in one launch.
 * `descs` is a HOST array of `count` entries, read before the call returns.
 * The problems run concurrently: no output may overlap any input of any
 * problem in the list (a residual operand may be its own problem's output).
 * Each entry's epilogue applies as in q4_matmul_residual / q4_matmul_swiglu.
 * Validation covers every entry before anything is enqueued; count == 0 is
 * a no-op; count < 0 is Q4_ERR_SHAPE; an unknown epilogue or a nonzero
 * `reserved` is Q4_ERR_UNSUPPORTED.
 */
Q4_API q4_status q4_matmul_batch(const q4_matmul_desc* descs, int count, int64_t M, int group,
                                 q4_stream_t stream);

/*
 * q4_matmul_batch_noalloc -- q4_matmul_batch (same arguments, validation,
 * kernels and results) whose group-sum kernel takes its workspace (arrival
 * counters and fp32 partial sums of shared tiles) from a fixed 16 MiB device
 * array inside libq4 instead of a stream-ordered allocation: the call makes
 * no device allocation.  The pages describe no such entry point; it is an
 * engineering variant of the batch call.
 * Limits: the array is one per device and shared by every call of this entry
 * point on it, so calls that may overlap in time (other streams, other host
 * threads) race on it and must be serialized by the caller; calls in one
 * stream are ordered and safe.  A call that would need more than the array
 * holds (about 2 * SMs * 128 * 2 * M * 4 bytes per group-sum launch, plus
 * counters) returns Q4_ERR_UNSUPPORTED before enqueuing anything.  The first
 * call on a device looks up the array's address (cudaGetSymbolAddress); make
 * it before capturing a stream.  Each call zeroes the counters with
 * cudaMemsetAsync on `stream`.
 */
Q4_API q4_status q4_matmul_batch_noalloc(const q4_matmul_desc* descs, int count, int64_t M, int group,
                                         q4_stream_t stream);

/*
 * q4_matmul_chain -- dependent matmuls: stage s is the next stage_counts[s]
 * descriptors of `descs` (n_stages entries summing to count), and the call
 * computes exactly (bit for bit) what q4_matmul_batch on each stage in turn
 * on `stream` computes.  A stage may read, as x or as a residual operand,
 * what earlier stages write; within a stage the batch rules hold.  This is
 * the shape of a decode step (per layer: q, k, v on the layer input; the
 * attention output adding into the residual stream; gate and up as SwiGLU;
 * down adding into the stream), whose per-step dispatches the Swift/MLX blog
 * ("Performance optimizations") and the ONNX README (CUDA Graph capture)
 * fuse; the pages describe no such entry point, this is an engineering
 * variant of the batch call for a dependent sequence.
 * With one or two activation rows and every problem on the bulk-copy GEMV
 * (K a multiple of 256, 16-byte aligned scale rows), the chain runs as one
 * persistent cooperative launch per up to 256 stages and 256 problems: one
 * CTA per SM takes a share of every stage in turn, streaming the next
 * stages' weights while it waits for the CTAs still finishing a stage (a
 * grid-wide arrival counter per stage, every wait bounded: a wait that gives
 * up raises the q4_device_status flag and the outputs it covers are NaN).
 * It takes a stream-ordered workspace of 4 bytes per stage
 * (cudaMallocAsync, cudaMemsetAsync, cudaFreeAsync on `stream`).  Otherwise
 * each stage is one q4_matmul_batch.  `descs` and `stage_counts` are HOST
 * arrays read before the call returns.  Validation covers every descriptor
 * before anything is enqueued; counts that do not add up, or a negative
 * count, are Q4_ERR_SHAPE.
 */
Q4_API q4_status q4_matmul_chain(const q4_matmul_desc* descs, int count, const int* stage_counts, int n_stages,
                                 int64_t M, int group, q4_stream_t stream);

/*
 * The 8-bit variant: the same affine rule with 255 levels and one byte per
 * code.  The pages compare a "standard 8-bit conversion" of the model with
 * the 4-bit builds (TWX4 comparison page, opening section) and ship an INT8
 * bundle (ONNX README, "All four variants"), without its arithmetic; read
 * plainly it is the 4-bit rule with 255 in place of 15:
 *   scale = bf16(fp32(mx - mn) / 255), bias = bf16(mn),
 *   q = 0 if scale == 0, else clamp(round_half_even((w - bias)/scale), 0, 255)
 * (binary64 quotient).  A bf16 scale is within 2^-8 of fp32(mx - mn)/255, so
 * the maximum lands on code 254 or 255 and the clamp can bind: elements above
 * the top code then reconstruct within one scale step instead of half.
 * Layout: codes [N, K] uint8 (byte k of row n is q[n,k]), 16-byte aligned;
 * scales, biases [N, K/32] bf16.  9 bits per weight.  Same conventions and
 * status codes as the 4-bit calls.
 */
Q4_API q4_status q8_quantize(const q4_bf16* W, int64_t N, int64_t K, int group, uint8_t* codes,
                             q4_bf16* scales, q4_bf16* biases, q4_stream_t stream);

/* W_out [N, K] = bf16(scale * q + bias), the value taken in binary64. */
Q4_API q4_status q8_dequantize(const uint8_t* codes, const q4_bf16* scales, const q4_bf16* biases,
                               int64_t N, int64_t K, int group, q4_bf16* W_out, q4_stream_t stream);

/*
 * y [M, N] = x . w_hat^T with 8-bit codes: fp32 accumulation of exact
 * products (each code an exact fp32, x in fp32), bf16 output.  CUDA-core
 * GEMV for every M (activation rows in pairs; each pair reads the weights
 * once): the 4-bit calls' bulk-copy GEMV with 8-bit rows where K is a
 * multiple of 256 and the scale and bias rows are 16-byte aligned (and K
 * fits one team of lanes: K <= 22528 for one row, 12288 for a pair), a
 * warp-per-row kernel otherwise.  K <= 196608 (Q4_ERR_UNSUPPORTED above).
 */
Q4_API q4_status q8_matmul(const q4_bf16* x, int64_t M, int64_t K, const uint8_t* codes,
                           const q4_bf16* scales, const q4_bf16* biases, int64_t N, int group,
                           q4_bf16* y, q4_stream_t stream);

/*
 * q8_matmul_batch -- independent 8-bit matmuls sharing M: q4_matmul_batch's
 * descriptor array with 8-bit codes ([N, K] bytes) in `codes`, each computed
 * exactly as q8_matmul computes it alone; the problems the bulk-copy GEMV
 * takes share one launch (per activation-row pair size, up to 256 problems),
 * the rest run one q8_matmul launch each.  No epilogue (Q4_ERR_UNSUPPORTED
 * for a nonzero `epilogue` or `reserved`).  Validation covers every entry
 * before anything is enqueued.  The pages describe no such entry point; it
 * is the 4-bit batch call for the 8-bit variant.
 */
Q4_API q4_status q8_matmul_batch(const q4_matmul_desc* descs, int count, int64_t M, int group,
                                 q4_stream_t stream);

/* Message for the calling thread's last non-OK status ("" if none). */
Q4_API const char* q4_last_error(void);

/*
 * Status of the kernels on the current device: bit 0 is set if any libq4
 * kernel gave up a bounded internal wait (a pipeline stage that never
 * arrived within one second, e.g. when the context was preempted for that
 * long).  The kernel then finished without waiting, wrote NaN where it could
 * not vouch for a result, and every result enqueued since the flag was last
 * clear must be treated as invalid.  Synchronizes with the device (it copies
 * the flag to the host); call it after the work to be checked.  clear != 0
 * resets the flag.  Returns the flags, or -1 if the copy failed.
 */
Q4_API int q4_device_status(int clear);

/* Diagnostic: number of kernel launches libq4 has enqueued in this process
 * (counted on the host when each launch is issued; graph replays of captured
 * launches are not counted again). */
Q4_API unsigned long long q4_debug_launch_count(void);

/* Diagnostic: kernel families the matmul dispatch may not choose, as a bit
 * mask (0 = all allowed, the default): Q4_KERNEL_GROUP_SUM (the group-sum
 * tensor-core kernel, 3..16 activation rows), Q4_KERNEL_WEIGHT_STREAM (the
 * weight-streaming tensor-core kernel, 3..8 rows) and Q4_KERNEL_TILES (the
 * tensor-core tiles, 3 or more rows).  A problem none of its allowed
 * tensor-core kernels takes goes to the CUDA-core GEMV, which takes every
 * problem.  For tests that pin a kernel to a problem; process-wide, read at
 * each call (set it while no other thread enqueues).  Returns the previous
 * mask. */
#define Q4_KERNEL_GROUP_SUM 1u
#define Q4_KERNEL_WEIGHT_STREAM 2u
#define Q4_KERNEL_TILES 4u
Q4_API unsigned int q4_debug_disable_kernels(unsigned int mask);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H_ */
