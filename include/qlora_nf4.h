/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) QLoRA NF4 frozen-linear library.
 *
 * The library implements one layer, the QLoRA linear of the QLoRA paper
 * digest (aipaper.cc, "QLoRA: Efficient Finetuning of Quantized LLMs",
 * sec. 4 "full QLoRA equation"):
 *
 *     Y = X * doubleDequant(c1, c2, W_nf4)^T + s * (X * A^T) * B^T
 *
 * in the shapes of the LoRA reproduction blog ("LoRA / QLoRA low-rank update,
 * quantization and memory budget", section "LoRA formula and tensor shapes"):
 * W [N = d_out, K = d_in], A [r, K], B [N, r], X [M, K], Y [M, N], s = alpha/r.
 * Beside it sits the blockwise NF4 quantizer that produces W_nf4 (QLoRA blog
 * note p19e99 sec. 2 "NF4"; digest sec. 4 "NF4" and "double quantization").
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers to caller-owned memory, dense and
 *    row-major.  The library keeps no pointer after a call returns and
 *    allocates no device memory (except qlora_paged_alloc, whose job it is):
 *    temporary storage comes from the caller's workspace, whose size the
 *    matching *_workspace() query gives.
 *  - Work is enqueued asynchronously on `stream` (NULL = legacy default).
 *  - Arguments are validated on the host before anything is launched; a bad
 *    argument returns QLORA_ERR_INVALID_ARG or QLORA_ERR_UNSUPPORTED and
 *    enqueues nothing.  A failed launch returns QLORA_ERR_CUDA.
 *  - Every wait inside a kernel is bounded in time.  A wait that runs out
 *    records QLORA_ERR_TIMEOUT in a per-device status word and the kernel
 *    returns; qlora_get_last_error() reports (and clears) that word.
 *  - bf16 tensors are passed as `const void *` and hold IEEE bfloat16 bits.
 *  - Alignment: bf16 tensors, codes and the workspace must be 16-byte
 *    aligned; fp32 tensors 4-byte aligned (QLORA_ERR_INVALID_ARG otherwise).
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qlora_stream_t; /* same type as cudaStream_t */

typedef enum {
    QLORA_OK = 0,
    QLORA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, small workspace */
    QLORA_ERR_UNSUPPORTED = 2, /* valid but outside this build: blocksize not 64,
                                  128 or 256, K % 64 != 0, N % 8 != 0,
                                  r % 8 != 0, r > 256 */
    QLORA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    QLORA_ERR_TIMEOUT = 4,     /* a bounded in-kernel wait ran out (reported
                                  by qlora_get_last_error only) */
    QLORA_ERR_WORKSPACE = 5,   /* the tensor is larger than the fixed internal
                                  scratch of qlora_nf4_quantize_static */
    QLORA_ERR_BOUNDS = 6       /* debug build (libqlora_nf4_debug.so, compiled
                                  with QLORA_DEBUG) only: a device-side bounds
                                  check of a computed store index failed; the
                                  store was skipped (reported by
                                  qlora_get_last_error only; nothing traps) */
} qlora_status;

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/*
 * A quantized frozen weight W [rows = N, cols = K].
 * Blocks are `blocksize` (64 in the pages) consecutive elements of the
 * row-major flattened tensor (QLoRA tutorial "11.3 QLoRA", section "double
 * quantization": 64 parameters share one constant);
 * nb = ceil(rows*cols / blocksize), nb2 = ceil(nb / 256).
 *   codes          [ceil(rows*cols/2)] bytes.  Element 2i sits in the high
 *                  nibble of byte i, element 2i+1 in the low nibble; the
 *                  nibble is the index (0..15) of the nearest NF4 code.
 *   absmax         [nb] fp32 block absolute maxima; read/written only when
 *                  double_quant == 0.
 *   absmax_q8      [nb] bytes, index k of the 8-bit code (k-127)/127 of the
 *                  centred block constant; used when double_quant == 1.
 *   absmax_scale   [nb2] fp32 second-level constants c1 (one per 256 blocks).
 *   absmax_offset  [1] fp32 mean of all block maxima, subtracted before the
 *                  8-bit quantization.
 * Dequantized weight (digest sec. 4, doubleDequant):
 *   a'  = double_quant ? (t8[q8] * c1) + offset : absmax     (fp32, two roundings)
 *   w'  = bf16_round_nearest_even(nf4[code] * a')
 */
typedef struct {
    int64_t rows;          /* N (d_out) */
    int64_t cols;          /* K (d_in)  */
    int32_t blocksize;     /* 64 (the pages' value), 128 or 256 */
    int32_t double_quant;  /* 0 or 1 */
    uint8_t *codes;
    float *absmax;
    uint8_t *absmax_q8;
    float *absmax_scale;
    float *absmax_offset;
    int32_t code_type;     /* QLORA_CODE_NF4 (0) or QLORA_CODE_FP4 (1) */
    int32_t dq_type;       /* QLORA_DQ_INT8 (0) or QLORA_DQ_FP8 (1) */
} qlora_nf4_weight;

/*
 * Data-type variants (QLoRA paper digest, sec. 6: "Float4 (FP4)" against
 * NFloat4; sec. 4: the double-quantized constants "c2^FP8"):
 *  QLORA_CODE_NF4  the 16 NF4 values above.
 *  QLORA_CODE_FP4  the 16 values of a 4-bit float with 1 sign, 2 exponent
 *                  (bias 1) and 1 mantissa bit (magnitudes 0, 0.5, 1, 1.5, 2,
 *                  3, 4, 6) divided by 6, sorted: index 7 is -0 and index 8
 *                  +0; the nearest-code rule (ties to the lower index) never
 *                  stores 8.
 *  QLORA_DQ_INT8   t8[k] = (k - 127) / 127, k = 0..254 (as above).
 *  QLORA_DQ_FP8    the 253 distinct finite values of the 8-bit float E4M3
 *                  (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 *                  largest 448) divided by 448, sorted; q8 = 0..252.
 * Every entry point accepts every combination, with block sizes 64, 128 and
 * 256 (blocks of consecutive elements of the flattened tensor).  A struct
 * that leaves the two fields 0 is the NF4 / linear 8-bit format.
 */
#define QLORA_CODE_NF4 0
#define QLORA_CODE_FP4 1
#define QLORA_DQ_INT8 0
#define QLORA_DQ_FP8 1

/*
 * Workspace bytes that qlora_nf4_quantize needs for a tensor of rows*cols
 * elements in blocks of `blocksize` (0 when double_quant == 0).  Returns 0
 * for invalid sizes.
 */
size_t qlora_nf4_quantize_workspace(int64_t rows, int64_t cols, int32_t blocksize,
                                    int32_t double_quant);

/*
 * Blockwise NF4 quantization (QLoRA blog note p19e99 sec. 2: rescale each
 * block by its absolute maximum into [-1, 1], store the index of the nearest
 * of 16 normal-quantile codes in 4 bits) followed, when out->double_quant,
 * by double quantization of the block constants to 8 bits (digest sec. 4
 * "double quantization"; blog note sec. 3).
 *   W      device [rows, cols] in `wdtype` (bf16 or fp32), finite values.
 *   out    describes caller-allocated outputs; rows, cols, blocksize,
 *          double_quant and the output pointers must be set.  Any rows*cols
 *          >= 0 is accepted (the last block may be partial; rows*cols == 0
 *          enqueues nothing).
 *   ws     device workspace of at least qlora_nf4_quantize_workspace() bytes
 *          (may be NULL when that is 0).
 * Deterministic: the same input gives bit-identical outputs.
 */
qlora_status qlora_nf4_quantize(const void *W, qlora_dtype wdtype, const qlora_nf4_weight *out,
                                void *ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * Largest rows*cols that qlora_nf4_quantize_static accepts: 2^26 elements
 * (every linear of a LLaMA-7B block; the largest is 11008 x 4096).
 */
#define QLORA_STATIC_QUANTIZE_MAX_ELEMS ((int64_t)1 << 26)

/*
 * The same quantization as qlora_nf4_quantize, with identical outputs, but
 * without a workspace argument and without allocating any device memory.
 * The pages have no counterpart of this call: it exists for callers that
 * cannot hand the library a device buffer, for example a plain C host
 * program or a plug-in of a framework that exposes no scratch allocator, or
 * that must not allocate once they are running under a fixed memory budget.
 *
 * The scratch (fp32 block maxima and fp64 group sums for the double
 * quantization) is a fixed device array inside the library, 4 MiB + 32 KiB,
 * reserved when the library's module is loaded on a device.  Every byte of
 * it that is read is first written by the same call, so nothing is cleared.
 *   - rows*cols above QLORA_STATIC_QUANTIZE_MAX_ELEMS returns
 *     QLORA_ERR_WORKSPACE and enqueues nothing.
 *   - The first call on each device (with that device current) looks up the
 *     scratch address with cudaGetSymbolAddress and keeps it; make that
 *     first call before any stream capture.  After cudaDeviceReset the kept
 *     address is stale: do not call this function again in that process.
 *   - One scratch per device: calls that may overlap on the same device
 *     (different streams without ordering, or several host threads) race on
 *     it and give wrong results.  Order such calls on one stream.
 * Other arguments, errors and determinism as for qlora_nf4_quantize.
 */
qlora_status qlora_nf4_quantize_static(const void *W, qlora_dtype wdtype,
                                       const qlora_nf4_weight *out, qlora_stream_t stream);

/*
 * doubleDequant (digest sec. 4): writes the bf16 weight w' [rows, cols] that
 * the linear layer multiplies with.  `out` is a device bf16 buffer.
 */
qlora_status qlora_nf4_dequantize(const qlora_nf4_weight *w, void *out, qlora_stream_t stream);

/*
 * Workspace bytes of qlora_linear_fwd (bwd == 0) or qlora_linear_bwd
 * (bwd == 1) for M tokens, weight w and rank r.  Returns 0 for invalid sizes.
 */
size_t qlora_linear_workspace(int64_t M, const qlora_nf4_weight *w, int32_t r, int32_t bwd);

/*
 * Forward of the frozen NF4 linear with a LoRA adapter (LoRA reproduction
 * blog, "LoRA formula and tensor shapes": y = x W0^T + (alpha/r) x A^T B^T,
 * with W0 the dequantized NF4 weight of the QLoRA paper notes, "Key design 3"):
 *   Y[m,n] = sum_k X[m,k] w'[n,k] + scale * sum_j U[m,j] B[n,j],
 *   U      = X A^T.
 *   X [M, K] bf16, A [r, K] bf16, B [N, r] bf16, Y [M, N] bf16 (written).
 *   r == 0 disables the adapter (A, B may be NULL).  M >= 0.
 * Products accumulate in fp32; U is rounded to bf16 after scaling by `scale`.
 * Requires K % 64 == 0, N % 8 == 0, r % 8 == 0, r <= 256.
 */
qlora_status qlora_linear_fwd(const void *X, int64_t M, const qlora_nf4_weight *w, const void *A,
                              const void *B, int32_t r, float scale, void *Y, void *ws,
                              size_t ws_bytes, qlora_stream_t stream);

/*
 * Backward of the same layer.  Gradients flow through the dequantized frozen
 * weight into the adapters only (digest sec. 4 steps 4; the reproduction
 * blog's invariant "the frozen weight's gradient is empty"), so there is no
 * dW output.  With G = dY B:
 *   dX = dY w' + scale * G A        [M, K] bf16 (written)
 *   dA = scale * G^T X              [r, K] fp32 (written)
 *   dB = scale * dY^T (X A^T)       [N, r] fp32 (written)
 *   dY [M, N] bf16, X [M, K] bf16.  dX may be NULL to skip it.  With r == 0
 *   only dX is produced.  With M == 0, dA and dB are set to zero.
 * Same shape requirements as qlora_linear_fwd.  Deterministic (no floating
 * point atomics on any output).
 * Streams: all work is ordered on `stream`.  With dX and r > 0 (and the
 * default CTA-pair schedule) the sU, dA and dB GEMMs run on a per-device
 * side stream of the library, beside the dX GEMM; the side stream first waits
 * for `stream` (after the sG GEMM) and `stream` waits for it before the call
 * returns, so to the caller the call is one ordered step on `stream` (also
 * inside a stream capture, once the side stream exists: it is created by the
 * first such call made outside a capture).  The library keeps that stream and
 * two events per device for its lifetime.  Calls from several host threads
 * are serialized on the side stream.  There is one side stream per device,
 * shared by every caller stream: the sU/dA/dB work of backward calls issued
 * on independent streams runs one call after another on it, and each caller
 * stream's join may then also wait for side work of another stream's call
 * (an ordering that costs time, never correctness).
 */
qlora_status qlora_linear_bwd(const void *dY, const void *X, int64_t M, const qlora_nf4_weight *w,
                              const void *A, const void *B, int32_t r, float scale, void *dX,
                              float *dA, float *dB, void *ws, size_t ws_bytes,
                              qlora_stream_t stream);

/*
 * Fused projection: nseg linears that share one input X (q, k and v of an
 * attention block, or gate and up of its MLP), stored as ONE quantized weight
 * w [N = nseg * S, K] whose row segment i (rows i*S .. i*S + S - 1) is linear
 * i, each with its own rank-r adapter (LoRA on every linear layer: QLoRA
 * paper digest sec. 6 results; paper notes, "results").  Per segment i the
 * forward and backward are those of qlora_linear_fwd / qlora_linear_bwd:
 *   Y[:, seg i]  = X w'_i^T + scale (X A_i^T) B_i^T
 *   dX           = sum_i ( dY[:, seg i] w'_i + scale G_i A_i ),  G_i = dY[:, seg i] B_i
 *   dA_i         = scale G_i^T X,   dB_i = scale dY[:, seg i]^T (X A_i^T)
 *   A [nseg*r, K] bf16 (A_i = rows i*r ..), B [N, r] bf16 (B_i = rows of seg i),
 *   dA [nseg*r, K] fp32, dB [N, r] fp32; X [M, K], Y/dY [M, N], dX [M, K] bf16.
 * The adapters' U = X A^T (all segments in one pass over X) and G, the dX
 * GEMM (one reduction over all N rows and all nseg*r adapter columns), dA and
 * dB each run as one launch for the whole projection.
 * Requires 1 <= nseg <= 8, N % nseg == 0, S = N / nseg a multiple of 256 when
 * nseg > 1, nseg * r <= 256, and everything qlora_linear_fwd requires
 * (UNSUPPORTED otherwise; nseg < 1 is INVALID_ARG).  nseg == 1 is exactly
 * qlora_linear_fwd / qlora_linear_bwd.  The workspace query takes the same
 * nseg and r.
 */
size_t qlora_fused_linear_workspace(int64_t M, const qlora_nf4_weight *w, int32_t nseg, int32_t r,
                                    int32_t bwd);
qlora_status qlora_fused_linear_fwd(const void *X, int64_t M, const qlora_nf4_weight *w, int32_t nseg,
                                    const void *A, const void *B, int32_t r, float scale, void *Y,
                                    void *ws, size_t ws_bytes, qlora_stream_t stream);
qlora_status qlora_fused_linear_bwd(const void *dY, const void *X, int64_t M, const qlora_nf4_weight *w,
                                    int32_t nseg, const void *A, const void *B, int32_t r, float scale,
                                    void *dX, float *dA, float *dB, void *ws, size_t ws_bytes,
                                    qlora_stream_t stream);

/*
 * LoRA merge (QLoRA tutorial "11.3 QLoRA", pitfalls: merging the adapter
 * into a 4-bit base adds error, so the base is dequantized first; LoRA
 * reproduction blog, "LoRA formula and tensor shapes": the adapter adds
 * (alpha/r) B A to W0):
 *   W_merged[n,k] = bf16_round_nearest_even( w'[n,k] + scale * sum_j B[n,j] A[j,k] )
 *   w  the quantized frozen weight [N, K] (w' its doubleDequant bf16 values),
 *   A [r, K] bf16, B [N, r] bf16, W_merged [N, K] bf16 (written).
 * The rank-r sum accumulates in fp32 on the tensor cores; the base is added
 * with one fused multiply-add in fp32 and the result rounded once to bf16.
 * Requires K % 64 == 0, N % 8 == 0, 1 <= r <= 256, r % 8 == 0 (UNSUPPORTED
 * otherwise); r < 1 is INVALID_ARG.  Pointers 16-byte aligned.  Async on
 * `stream`; writes only W_merged.  The merged dense weight serves inference
 * without the adapter path (Y = X W_merged^T).
 */
qlora_status qlora_lora_merge(const qlora_nf4_weight *w, const void *A, const void *B, int32_t r,
                              float scale, void *W_merged, qlora_stream_t stream);

/*
 * LoRA unmerge, the inverse of qlora_lora_merge on a dense bf16 weight:
 *   W_out[n,k] = bf16_round_nearest_even( W_merged[n,k] - scale * sum_j B[n,j] A[j,k] )
 * W_merged, W_out [rows, cols] bf16 (W_out written; it may not overlap
 * W_merged), A [r, cols], B [rows, r] bf16.  It gives back the base weight
 * (up to the bf16 rounding of the merge) so that the frozen base and the
 * adapter path can be used apart again.  Same requirements as
 * qlora_lora_merge.
 */
qlora_status qlora_lora_unmerge(const void *W_merged, int64_t rows, int64_t cols, const void *A,
                                const void *B, int32_t r, float scale, void *W_out,
                                qlora_stream_t stream);

/*
 * Optimizer step of the adapters (QLoRA paper digest, sec. 4 steps: Adam
 * updates the LoRA matrices only; the frozen 4-bit weight is never updated).
 * AdamW with decoupled weight decay on n fp32 parameters, with bias
 * correction for step t = cfg->step (t >= 1, counting this step):
 *   g = grad * grad_scale
 *   param <- param * (1 - lr * weight_decay)
 *   m <- beta1 m + (1 - beta1) g;   v <- beta2 v + (1 - beta2) g^2
 *   param <- param - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
 * computed in fp32, element by element.  param, exp_avg (m), exp_avg_sq (v)
 * are updated in place; grad is read; param_bf16 (may be NULL) receives the
 * bf16 round-to-nearest-even copy of the new parameters, for the linear calls.
 * Every adapter of a block can be one flat buffer (the backward's dA and dB
 * written into views of the flat gradient), so one call updates them all.
 * Pointers 16-byte aligned (param_bf16 8-byte).  m and v may be paged memory
 * from qlora_paged_alloc.  Invalid hyper-parameters (step < 1, lr < 0,
 * betas outside [0, 1), eps <= 0, weight_decay < 0): INVALID_ARG.
 */
typedef struct {
    float lr, beta1, beta2, eps, weight_decay, grad_scale;
    int64_t step;
} qlora_adamw_config;

qlora_status qlora_adamw_step(float *param, float *exp_avg, float *exp_avg_sq, const float *grad,
                              void *param_bf16, int64_t n, const qlora_adamw_config *cfg,
                              qlora_stream_t stream);

/*
 * Paged optimizer state (QLoRA blog note sec. 4 and tutorial "11.3 QLoRA",
 * "paged optimizers": optimizer states live in unified memory, so that under
 * a memory spike their pages move to host RAM and come back when the
 * optimizer step touches them).
 * qlora_paged_alloc: the one allocating call of the library: `bytes` of
 *   managed (unified) memory, reachable from the host and every device
 *   through the same pointer; *ptr = NULL for bytes == 0.  The caller owns
 *   it and frees it with qlora_paged_free.  CUDA failure: QLORA_ERR_CUDA.
 * qlora_paged_prefetch: migrates [ptr, ptr + bytes) ahead of use, to host
 *   memory (to_host != 0: page the state out before a memory-heavy phase) or
 *   to the current device (before the optimizer step), ordered on `stream`.
 *   Without a prefetch, pages still migrate on demand when touched.
 */
qlora_status qlora_paged_alloc(size_t bytes, void **ptr);
qlora_status qlora_paged_free(void *ptr);
qlora_status qlora_paged_prefetch(const void *ptr, size_t bytes, int32_t to_host, qlora_stream_t stream);

/*
 * Synchronizes `stream`, then returns (and clears) the device status word of
 * the current device: QLORA_ERR_TIMEOUT if a bounded in-kernel wait ran out
 * since the last call, QLORA_ERR_CUDA if the stream reports an error,
 * QLORA_OK otherwise.
 */
qlora_status qlora_get_last_error(qlora_stream_t stream);

/* Host copy of the 16 NF4 codes this library uses (sorted, index 7 == 0). */
void qlora_nf4_table(float out[16]);

/*
 * Nearest-NF4-code search of the quantizer, exposed so that it can be checked
 * on every fp32 input: codes[i] = index (0..15) of the NF4 code nearest to
 * x[i], exact ties to the lower index.  x and codes are device arrays of n
 * elements (one code per byte).  Test entry point.
 */
qlora_status qlora_nf4_encode(const float *x, int64_t n, uint8_t *codes, qlora_stream_t stream);

/*
 * Nearest-code search of the double quantization, exposed so that it can be
 * checked on every fp32 input: codes[i] = index of the entry of the 8-bit
 * code book dq_type (QLORA_DQ_INT8: 0..254, QLORA_DQ_FP8: 0..252) nearest to
 * y[i] clamped to [-1, 1], exact ties to the lower index.  Device arrays of n
 * elements.  Test entry point.
 */
qlora_status qlora_dq_encode(const float *y, int64_t n, uint8_t *codes, int32_t dq_type,
                             qlora_stream_t stream);

/*
 * Upper bound, in nanoseconds, of every in-kernel wait (default 10 s).
 * Test entry point; 0 restores the default.
 */
void qlora_set_wait_timeout_ns(uint64_t ns);

/*
 * Test modes.  Mode 1 (fault injection for the failure-detection tests) makes
 * the next launches of the tensor-core GEMM skip their producer's loads, so
 * that the consumers' bounded waits run out and QLORA_ERR_TIMEOUT is
 * recorded; no GPU fault is raised, the kernels return normally.  Mode 2
 * runs the forward and dX GEMMs (M > 64) on the single-CTA kernel with the
 * stream-K schedule over 7 CTAs whatever the shape (coverage of the
 * split-tile merge); mode 3 on the single-CTA kernel with one CTA per tile;
 * mode 4 on the CTA-pair kernel with the stream-K schedule over 4 pairs;
 * mode 5 forms the double-quantization offset in its own kernel even for
 * tensors whose 8-bit pass would form it itself; mode 6 runs the backward's
 * dA and dB GEMMs on the caller's stream after the dX GEMM instead of beside
 * it on the library's side stream; mode 7 runs the forward for M <= 32 on the
 * register-fed warp-MMA kernel (code-byte table lookups, block constant on
 * each block's fp32 partial), mode 8 the forward for M <= 16 on the tcgen05
 * small-M kernel.
 * Mode 0: normal (CTA-pair kernel, one pair per tile; in the backward the
 * dA/dB GEMMs beside the dX GEMM on the side stream; M <= 16 on the warp-MMA
 * kernel, 17 <= M <= 64 on the tcgen05 small-M kernel).
 * The mode is process-wide: it changes the kernels of every later call from
 * every thread and stream on every device, until it is set back to 0; it is
 * meant for tests only.  Likewise the environment variable QLORA_SCHEDULE
 * (pair | pairsk | grid | streamk: the schedule of the large-M GEMMs) is read
 * once, at the first large-M call of the process, and applies to all calls.
 */
void qlora_debug_inject(int32_t mode);

/*
 * Measurement hooks (used by the benchmark).
 * qlora_kernel_launches: number of kernels this library has launched in this
 *   process (all devices, all streams).
 * qlora_profile_enable(1) clears the records, creates the event pool (the
 *   first time) and starts recording a CUDA event pair around every launch
 *   of the tracked kernels below, on the stream the kernel is launched on
 *   (not while that stream is being captured into a graph); 0 stops
 *   recording.
 * qlora_profile_read: synchronizes the recorded events and returns, for one
 *   kind, the summed device time (ms) and the number of launches recorded.
 *   Returns QLORA_ERR_INVALID_ARG for an unknown kind.
 */
typedef enum {
    QLORA_KERNEL_QUANTIZE = 0,  /* blockwise NF4 quantizer (first kernel of qlora_nf4_quantize) */
    QLORA_KERNEL_DEQUANTIZE = 1,
    QLORA_KERNEL_FWD_GEMM = 2,  /* forward dequant-GEMM, M > 64 */
    QLORA_KERNEL_DX_GEMM = 3,   /* backward dX dequant-GEMM */
    QLORA_KERNEL_SMALLM_GEMM = 4, /* forward dequant-GEMM, M <= 64 */
    QLORA_KERNEL_LORA_GEMM = 5, /* rank-r LoRA GEMMs (U, G, dA, dB) */
    QLORA_KERNEL_MERGE = 6,     /* LoRA merge / unmerge */
    QLORA_KERNEL_KINDS = 7
} qlora_kernel_kind;

uint64_t qlora_kernel_launches(void);
void qlora_profile_enable(int32_t on);
qlora_status qlora_profile_read(int32_t kind, double *total_ms, int64_t *launches);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
