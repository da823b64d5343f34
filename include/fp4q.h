/*
 * fp4q.h -- C ABI of libfp4q.so: block-wise microscaling FP4 quantization of
 * bf16 tensors on NVIDIA B200 (sm_100a).
 *
 * The operations follow three pages:
 *  "Diagnosing FP4 inference: a layer-wise and block-wise sensitivity
 *   analysis of NVFP4 and MXFP4", technical summary, Methodology (MXFP4: blocks
 *   of 32 E2M1 values sharing an 8-bit exponent; NVFP4: blocks of 16 with a
 *   scale and "max" calibration; weights kept in 16 bits, quantized on the fly
 *   and dequantized for the compute);
 *  "Bridging the Gap Between Promise and Performance for Microscaling FP4
 *   Quantization", technical summary s1-s3 (E8M0 power-of-two scales, E4M3
 *   scales, round-to-nearest, block-wise Hadamard rotations fused with the
 *   quantization and the scale computation);
 *  "Finer is better? Limits of micro-scaling formats in LLMs", Theoretical
 *   framework, Contributions and Results (UE4M3 scales, smallest non-zero
 *   2^-9; UE4M3 under a per-tensor scale; UE5M3; per-block and per-tensor MSE
 *   split into non-max elements, block max and zero-rounded blocks).
 *
 * Conventions shared by every entry point
 *  - Tensors are row-major and contiguous, [rows][cols].  A quantization block
 *    is `block` consecutive elements of one row; a rotation acts on `rot`
 *    consecutive elements of one row.  cols % block == 0 and, if rot > 0,
 *    cols % rot == 0.  rows == 0 or cols == 0 is a valid empty tensor.
 *  - Codes: 4-bit E2M1 nibbles (bit 3 = sign, bits 0-2 = magnitude index of
 *    {0, 0.5, 1, 1.5, 2, 3, 4, 6}); byte j of the code buffer holds element 2j
 *    in its low nibble and element 2j+1 in its high nibble: rows*cols/2 bytes.
 *  - Scales: one byte per block, row-major [rows][cols/block].  E8M0: the
 *    scale is 2^(byte-127).  UE4M3: unsigned E4M3 (bias 7, 0x7F NaN, max 448,
 *    min 2^-9), block scale S = fp32(decode(byte) * G).  UE5M3: unsigned E5M3
 *    (bias 15, 0xFF NaN, max 114688, min 2^-17), S = fp32(decode(byte) * G).
 *  - G is the FP32 per-tensor scale (1 when none is used).
 *  - All pointers except `stream` are DEVICE pointers owned by the caller; the
 *    library allocates no memory.  `stream` is a cudaStream_t passed as void*
 *    (NULL = the legacy default stream).  Every call only enqueues work on
 *    that stream and returns; outputs are valid once the stream reaches it.
 *  - Alignment: bf16 tensors and code buffers 32 bytes; scale and per-block
 *    MSE buffers 16 bytes; gscale 4 bytes; terms and workspace 8 bytes.
 *  - Errors: invalid arguments return a negative fp4q_status before anything
 *    is enqueued.  A failed launch returns FP4Q_ERR_CUDA.  No call but
 *    fp4q_device_fault synchronizes the device.  Inputs must be finite: a block holding NaN or
 *    Inf gets an unspecified scale byte and codes (no fault).
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP4Q_API __attribute__((visibility("default")))
#else
#define FP4Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4Q_OK = 0,
    FP4Q_ERR_NULL = -1,        /* a required pointer is NULL                    */
    FP4Q_ERR_SHAPE = -2,       /* negative size, or cols not a multiple of block/rot */
    FP4Q_ERR_ALIGN = -3,       /* a pointer breaks the alignment rules above    */
    FP4Q_ERR_UNSUPPORTED = -4, /* format / block / rot / mode combination        */
    FP4Q_ERR_CUDA = -5,        /* a CUDA launch or runtime call failed           */
    FP4Q_ERR_WORKSPACE = -6    /* workspace smaller than fp4q_block_mse_workspace_size */
} fp4q_status;

typedef enum {
    FP4Q_SCALE_E8M0 = 0,       /* MXFP4 power-of-two scale                      */
    FP4Q_SCALE_UE4M3 = 1,      /* NVFP4 unsigned E4M3 scale                     */
    FP4Q_SCALE_UE5M3 = 2       /* unsigned E5M3 scale (min 2^-17)               */
} fp4q_scale_fmt;

typedef enum {
    FP4Q_GLOBAL_NONE = 0,      /* G = 1 (always for E8M0; plain UE4M3 / UE5M3)  */
    FP4Q_GLOBAL_COMPUTE = 1,   /* G = amax(|y|)/(6*448) (1 if amax = 0), written to *gscale */
    FP4Q_GLOBAL_GIVEN = 2,     /* G read from *gscale (must be finite and > 0)  */
    FP4Q_GLOBAL_FROM_AMAX = 3  /* gscale[0] holds amax(|y|) on entry (for instance from
                                  fp4q_tensor_amax); G = amax/(6*448) (1 if amax = 0) is
                                  computed by the call and written to gscale[1]         */
} fp4q_global_mode;

typedef enum {
    FP4Q_OUT_BF16 = 0,         /* dequantized values rounded to bf16 (RNE)      */
    FP4Q_OUT_F32 = 1           /* dequantized values as fp32                    */
} fp4q_out_dtype;

/*
 * fp4q_quantize -- rotate (optional), scale and round a bf16 tensor to FP4.
 * ("Bridging the Gap", s3.4: rotation fused with quantization and scale
 * computation; "Diagnosing FP4 inference", Methodology: "max" calibration.)
 *
 *  x       bf16 [rows][cols] input (device).
 *  fmt     fp4q_scale_fmt.  block: power of two in [8, 256].
 *  rot     0 (none) or 16, 32, 128: y = H_rot x / sqrt(rot) per run of rot
 *          elements (Sylvester Hadamard), computed in fp32.
 *  gmode   fp4q_global_mode; must be FP4Q_GLOBAL_NONE for E8M0.
 *  codes   out: rows*cols/2 bytes.  scales: out, rows*cols/block bytes.
 *  gscale  1 float: written in COMPUTE mode, read in GIVEN mode, ignored (may
 *          be NULL) in NONE mode.  FROM_AMAX: 2 floats, the tensor's maximum
 *          |y| in gscale[0] (read) and G in gscale[1] (written); same codes,
 *          scales and G as COMPUTE without a pass over x for the maximum.
 * Per block: m = max |y|; E8M0 S = 2^(floor(log2 m)-2); UE4M3/UE5M3
 * s = nearest code to fp32(m / fp32(6 G)) (ties to even, saturating), S =
 * fp32(decode(s) G).  Each nibble is the E2M1 value nearest to fp32(y / S)
 * (correctly rounded quotient; ties to the even code; saturation at 6; sign
 * kept); a block with S = 0 stores 0x0 nibbles.
 */
FP4Q_API int fp4q_quantize(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                  int gmode, uint8_t* codes, uint8_t* scales, float* gscale, void* stream);

/*
 * fp4q_quantize_search -- fp4q_quantize with MSE-optimised block scales
 * ("Bridging the Gap", s3, MR-GPTQ item 2: scales chosen to minimise the
 * squared reconstruction error rather than by the max rule).  The pages give
 * no procedure; this call tries, per block, the max-rule code s0, then
 * s0+1 .. s0+above, then s0-1 .. s0-below (codes outside the format's finite
 * range skipped: E8M0 0..254, UE4M3 0..0x7E, UE5M3 0..0xFE) and keeps the code
 * of least error; a later candidate wins only with a strictly smaller error,
 * so ties keep the earlier code.  The error of a code is the fp32 sum over the
 * block of d*d, d = fp32(y - v), v = fp32(decode(nibble) S) (0 when S = 0),
 * each term added with one rounding; the sum's order is the kernel's, so a
 * choice between two codes whose errors agree to fp32 rounding may differ from
 * an element-order sum.  The nibbles are those fp4q_quantize computes for the
 * chosen S.  below, above: 0 .. FP4Q_SEARCH_MAX (0, 0 is fp4q_quantize).
 * Other arguments, G handling and errors as for fp4q_quantize;
 * FP4Q_ERR_UNSUPPORTED for a window out of range.
 */
#define FP4Q_SEARCH_MAX 16
FP4Q_API int fp4q_quantize_search(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                                  int gmode, int below, int above, uint8_t* codes, uint8_t* scales,
                                  float* gscale, void* stream);

/*
 * fp4q_quantize_mse_dequantize_batched -- fp4q_quantize_mse_dequantize for
 * `count` tensors of one format, block and rotation (a model layer's
 * projections), in one launch per 8 tensors.  The tensors' tiles are laid end
 * to end and streamed by one kernel, so small tensors cost no launch ramp and
 * tail of their own.  Each tensor keeps its own per-tensor scale, outputs and
 * MSE terms, bit for bit those of the single call ("Finer is better?",
 * Theoretical framework; "Diagnosing FP4 inference", Methodology: quantized
 * on the fly, then dequantized for the compute).
 *  tensors    host array of `count` descriptors, read during the call only;
 *             per tensor the arguments of fp4q_quantize_mse_dequantize, with
 *             the same layouts, alignment and meaning (y required).
 *  fmt, block FP4Q_SCALE_E8M0 with block 32 (MXFP4) or FP4Q_SCALE_UE4M3 with
 *             block 16 (NVFP4); other pairs: FP4Q_ERR_UNSUPPORTED (use the
 *             single call).
 *  rot, gmode as for fp4q_quantize (E8M0: FP4Q_GLOBAL_NONE only).
 *  workspace  device scratch of fp4q_quantize_batch_workspace_size(count)
 *             bytes (8-byte aligned), zero-filled before its first use and
 *             left so by every call: tensor i uses slice i (a completion
 *             counter and per-CTA partials).
 * Every tensor is checked before anything is enqueued; errors as for
 * fp4q_quantize_mse_dequantize, FP4Q_ERR_SHAPE for count < 0 (count = 0 does
 * nothing).
 */
typedef struct fp4q_tensor {
    const void* x;       /* bf16 [rows][cols] (device, 32-byte aligned) */
    int64_t rows, cols;
    uint8_t* codes;      /* rows*cols/2 bytes (32-byte aligned) */
    uint8_t* scales;     /* rows*cols/block bytes (16-byte aligned) */
    float* gscale;       /* per gmode, as fp4q_quantize; NULL for FP4Q_GLOBAL_NONE */
    void* y;             /* bf16 [rows][cols] dequantized values (32-byte aligned) */
    float* block_mse;    /* rows*cols/block floats (16-byte aligned) or NULL */
    double* terms;       /* 4 doubles: total, non-max, max, zero-rounded MSE (8-byte aligned) */
} fp4q_tensor;
FP4Q_API size_t fp4q_quantize_batch_workspace_size(int count);
FP4Q_API int fp4q_quantize_mse_dequantize_batched(int count, const fp4q_tensor* tensors, int fmt, int block,
                                                  int rot, int gmode, void* workspace, size_t ws_bytes,
                                                  void* stream);

/*
 * fp4q_tensor_amax -- amax = max |y| over the whole (optionally rotated)
 * tensor, written as one float.  This is the first half of the per-tensor
 * scale of COMPUTE mode ("Finer is better?", Results: UE4M3 with a dynamic
 * per-tensor scale needs this extra pass).
 */
FP4Q_API int fp4q_tensor_amax(const void* x, int64_t rows, int64_t cols, int rot, float* amax,
                     void* stream);

/*
 * fp4q_tensor_amax_accumulate -- *amax = max(*amax, max |y| over the tensor):
 * the maximum of fp4q_tensor_amax folded into a value already in place, with
 * no clearing pass.  *amax must hold a non-negative float on entry (0, or the
 * maximum of other shards of the same tensor, so that shards quantized with
 * one per-tensor scale share it).  Calls on one slot may run concurrently.
 */
FP4Q_API int fp4q_tensor_amax_accumulate(const void* x, int64_t rows, int64_t cols, int rot, float* amax,
                                         void* stream);

/*
 * fp4q_tensor_amax_batched -- the maxima of `count` tensors in one pass:
 * *amax[i] = max |y| over tensor i (accumulate = 0), or max(*amax[i], that)
 * (accumulate != 0, as fp4q_tensor_amax_accumulate).  All tensors take the
 * same rot.  The host arrays xs, rows, cols and amax (count entries each) are
 * read during the call only; the tensors' tiles are laid end to end and
 * streamed by one kernel launch per 32 tensors, so many small tensors (the
 * projections of a model layer) cost about what one tensor of their total
 * size does.  Slots must be distinct within a call.  Every tensor is checked
 * before anything is enqueued; errors as for fp4q_tensor_amax, and
 * FP4Q_ERR_SHAPE for count < 0 (count = 0 does nothing).
 */
FP4Q_API int fp4q_tensor_amax_batched(int count, const void* const* xs, const int64_t* rows, const int64_t* cols,
                                      int rot, float* const* amax, int accumulate, void* stream);

/*
 * fp4q_global_scale -- *gscale = amax / (6 * 448) (correctly rounded fp32), or
 * 1 when amax = 0: the per-tensor scale of COMPUTE mode from an absolute
 * maximum that is already known (for instance one reduced across several
 * shards of a tensor).  amax and gscale may be the same address.
 * ("Finer is better?", Results: UE4M3 under a per-tensor scale.)
 */
FP4Q_API int fp4q_global_scale(const float* amax, float* gscale, void* stream);

/*
 * fp4q_dequantize -- v = fp32(decode(nibble) * S) ("Diagnosing FP4
 * inference", Methodology: dequantized for the compute).
 *  gscale   NULL means G = 1; otherwise G = *gscale (ignored for E8M0).
 *  rot      0: v in the quantized (rotated) domain; 16/32/128: v is rotated
 *           back, H_rot v / sqrt(rot) (the rotation is its own inverse).
 *  out_dtype  FP4Q_OUT_BF16 (RNE of the fp32 value) or FP4Q_OUT_F32.
 *  y        out: rows*cols values.
 */
FP4Q_API int fp4q_dequantize(const uint8_t* codes, const uint8_t* scales, const float* gscale,
                    int64_t rows, int64_t cols, int fmt, int block, int rot, int out_dtype,
                    void* y, void* stream);

/*
 * fp4q_block_mse -- quantization MSE per block and per tensor with the
 * three-term split of "Finer is better?", Theoretical framework.
 * Recomputes y from x (rotating when rot > 0) and v from codes/scales, then
 *  block_mse[i] = sum_{j in block i} (y_j - v_j)^2 / block   (fp32; may be NULL)
 *  terms[0..3]  = {total, non-max elements, block max, zero-rounded blocks},
 *                 each a sum of squared errors over the tensor divided by
 *                 rows*cols (fp64, device).  A block is zero-rounded when all
 *                 of its dequantized values are 0; the block max is an element
 *                 of largest |y|.
 *  workspace    device scratch of at least fp4q_block_mse_workspace_size()
 *               bytes, 8-byte aligned.  Its first 16 bytes hold the counter
 *               through which the kernel's CTAs find the last one to finish
 *               (which then sums the per-CTA partials): they must be zero
 *               before the first call that uses the workspace, and every
 *               completed call leaves them zero.  Allocate it zero-filled once
 *               and reuse it for tensors of any size (at least as large as
 *               the workspace size each needs); the rest is overwritten by
 *               each call.  Calls that share a workspace must not run at the
 *               same time.
 * The per-tensor sums use a fixed reduction order (deterministic run to run).
 */
FP4Q_API int fp4q_block_mse(const void* x, const uint8_t* codes, const uint8_t* scales,
                   const float* gscale, int64_t rows, int64_t cols, int fmt, int block, int rot,
                   float* block_mse, double* terms, void* workspace, size_t ws_bytes,
                   void* stream);

/*
 * fp4q_quantize_mse -- fp4q_quantize and the MSE of fp4q_block_mse in one pass
 * over x: the errors are measured in the quantizing kernel, from the values
 * and codes it has in registers, so x is read once instead of twice.  Outputs
 * and arguments as for the two calls; block_mse may be NULL.  The block
 * maximum's error is taken against the largest dequantized magnitude of the
 * block (the value the maximum rounds to), the per-block sums are fp32 and the
 * tensor terms fp64 in a fixed order.  workspace: at least
 * fp4q_block_mse_workspace_size() bytes, with the zeroed completion counter
 * described at fp4q_block_mse.  gmode may be FP4Q_GLOBAL_FROM_AMAX as for
 * fp4q_quantize.
 */
FP4Q_API int fp4q_quantize_mse(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                               int gmode, uint8_t* codes, uint8_t* scales, float* gscale,
                               float* block_mse, double* terms, void* workspace, size_t ws_bytes,
                               void* stream);

/*
 * fp4q_quantize_mse_dequantize -- fp4q_quantize_mse that also writes the
 * dequantized tensor: y (bf16 [rows][cols], 32-byte aligned) receives exactly
 * what fp4q_dequantize(codes, scales, G, ..., rot = 0, FP4Q_OUT_BF16) would
 * write (values in the quantized, i.e. rotated, domain), computed from the
 * values the MSE already forms, so the codes are not read back ("Diagnosing
 * FP4 inference", Methodology: quantized on the fly, then dequantized for the
 * compute).  Other arguments, outputs and errors as fp4q_quantize_mse.
 */
FP4Q_API int fp4q_quantize_mse_dequantize(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                                          int gmode, uint8_t* codes, uint8_t* scales, float* gscale, void* y,
                                          float* block_mse, double* terms, void* workspace, size_t ws_bytes,
                                          void* stream);

/* Bytes of device workspace fp4q_block_mse and fp4q_quantize_mse need for this
 * shape (host only; at most 128 KiB + 16): the completion counter and the
 * per-CTA partials. */
FP4Q_API size_t fp4q_block_mse_workspace_size(int64_t rows, int64_t cols, int block);

/*
 * fp4q_outlier_stats -- activation outlier statistics ("Diagnosing FP4
 * inference", Methodology and Results C: the maximum and the 99.9th percentile
 * of a projection's activations, and their ratio).  The pages define neither
 * the percentile nor whether signs count; this call takes magnitudes and the
 * nearest rank:
 *  x          bf16 [rows][cols] = [tokens][channels] (device, 16-byte aligned);
 *             cols a multiple of 8.  Inputs must be finite.
 *  p          quantile in (0, 1], for instance 0.999.
 *  stats      out (device, 2 floats): stats[0] = max |x|; stats[1] = the k-th
 *             smallest |x|, k = ceil(p * rows*cols) evaluated in double and
 *             clamped to [1, rows*cols] (a value present in x).  Both 0 for an
 *             empty tensor.
 *  col_absmax out (device, cols floats) or NULL: the largest |x| of each column.
 *  workspace  device scratch of at least fp4q_outlier_stats_workspace_size()
 *             bytes (8-byte aligned): two histograms over the 2^15 bf16
 *             magnitude patterns, their totals per exponent (256 each) and a
 *             control word, cleared by the call.
 * Results are exact (integer counts over bf16 patterns).  The call zeroes its
 * outputs and the workspace on the stream.  Below 2^22 elements it makes one
 * histogram pass over x.  Larger tensors get three passes:
 *  - a histogram of a sample of rows sets a threshold below the quantile;
 *  - a pass over x counts only the magnitudes at or above the threshold and
 *    takes the channel maxima: a streaming pass that adds each counted
 *    magnitude to the histogram with a global atomic when the sample puts at
 *    most 1/64 of the magnitudes there, else a pass with a shared-memory
 *    histogram per CTA (both are launched; the one not needed returns at
 *    once);
 *  - a further pass, which returns at once unless the rank turned out to lie
 *    below the threshold, counts the rest.
 * Each pass is followed by a single-CTA scan.  Errors: FP4Q_ERR_SHAPE
 * (cols % 8), FP4Q_ERR_UNSUPPORTED (p outside (0, 1]), FP4Q_ERR_NULL,
 * FP4Q_ERR_ALIGN, FP4Q_ERR_WORKSPACE.
 */
#define FP4Q_OUTLIER_WS_BYTES (2 * 32768 * 8 + 2 * 256 * 8 + 16)
FP4Q_API size_t fp4q_outlier_stats_workspace_size(void);
FP4Q_API int fp4q_outlier_stats(const void* x, int64_t rows, int64_t cols, double p, float* stats,
                                float* col_absmax, void* workspace, size_t ws_bytes, void* stream);

/*
 * fp4q_block_mse_noalloc -- fp4q_block_mse without a workspace argument, for
 * callers that cannot allocate device memory (code running where no
 * allocation may happen, or a host that owns no device allocator and
 * would have nowhere to get the workspace from).  The pages have no
 * counterpart: this is an interface convenience, not a step of the method.
 *
 * Same arguments, results and errors as fp4q_block_mse; the per-CTA partials
 * live in a fixed static device buffer of libfp4q.so instead of a caller
 * workspace.  The library allocates nothing (no cudaMalloc, no allocating
 * library routine).
 *  - Limit: the buffer holds 4096 partial slots (128 KiB).  The MSE kernel
 *    never uses more, whatever the tensor size; a launch that would need more
 *    returns FP4Q_ERR_WORKSPACE before anything is enqueued.
 *  - Setup: the first call on each device (with that device current) looks
 *    up the buffer's device address with cudaGetSymbolAddress and caches it.
 *    Make that first call before any stream capture begins on the device.
 *  - The buffer ends with the completion counter of the in-kernel reduction
 *    (see fp4q_block_mse): it is zero when the library is loaded and every
 *    completed call leaves it zero; the partials are overwritten by each call.
 *  - One buffer per device: two calls in flight at the same time on one
 *    device (on different streams, or from different host threads without
 *    ordering) race on it and give wrong terms.  Calls ordered on one stream
 *    are safe.
 */
FP4Q_API int fp4q_block_mse_noalloc(const void* x, const uint8_t* codes, const uint8_t* scales,
                                    const float* gscale, int64_t rows, int64_t cols, int fmt, int block,
                                    int rot, float* block_mse, double* terms, void* stream);

/*
 * Element and scale codecs on their own, one value at a time ("Bridging the
 * Gap", s1; "Finer is better?", Theoretical framework and Contributions).
 * fp4q_e2m1_encode_f32: nibble of the E2M1 value nearest to r[i] (the rule of
 *   fp4q_quantize with S = 1: ties to the even code, saturation at 6, sign
 *   kept), packed like the code buffer (low nibble = even element).
 * fp4q_scale_encode_f32: one scale byte per value.  UE4M3 / UE5M3: the code
 *   nearest to s[i] >= 0 (ties to even, saturating at the largest finite
 *   value).  E8M0: the byte fp4q_quantize stores for a block whose absolute
 *   maximum is s[i] (2^(floor(log2 s) - 2), clamped to 2^-127).
 * Inputs 4-byte aligned; outputs 4-byte aligned.
 */
FP4Q_API int fp4q_e2m1_encode_f32(const float* r, int64_t n, uint8_t* packed, void* stream);
FP4Q_API int fp4q_scale_encode_f32(const float* s, int64_t n, int fmt, uint8_t* codes, void* stream);

/* MSE-optimised per-tensor scale ("Bridging the Gap", s3.2, MR-GPTQ item 2:
 * the global scale optimised together with the group scales).  Candidates
 * G_j = fp32(G0 * (16 + j) / 16) for j in [-below, above] (0 <= below <= 8,
 * 0 <= above <= 15), G0 = amax / 2688 of the (rotated) tensor (1 when it is
 * all zero), tried in the order j = 0, 1, -1, 2, -2, ...; under each, block
 * scales by the max rule; the candidate whose total squared error is
 * strictly smallest is kept, so G0 wins every tie.  Writes G* to gscale[0]
 * (device float) and, if errors != NULL, each candidate's per-tensor MSE to
 * errors[j + below] (device doubles).  The codes for G* are then
 * fp4q_quantize(..., FP4Q_GLOBAL_GIVEN, gscale).  fmt UE4M3 or UE5M3 (E8M0
 * has no per-tensor scale: FP4Q_ERR_UNSUPPORTED); block and rot as
 * fp4q_quantize.  workspace: device, 16-byte aligned, at least
 * fp4q_global_scale_search_workspace_size() bytes, no initial contents
 * required (the call clears what it needs).  One pass over x for the
 * maximum and one for all candidates; enqueued on `stream`. */
FP4Q_API int fp4q_global_scale_search(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot,
                                      int below, int above, float* gscale, double* errors, void* workspace,
                                      size_t ws_bytes, void* stream);
FP4Q_API size_t fp4q_global_scale_search_workspace_size(void);

/* fp4q_quantize with the scale bytes written in the layout the block-scaled
 * tensor-core MMA reads them from (the operand layout of fp4q_gemm), for the
 * two formats that MMA takes: MXFP4 (E8M0, block 32) and NVFP4 (UE4M3, block
 * 16).  "Bridging the Gap", s3.4 and s4: the quantized codes and block scales
 * feed FP4 GEMMs directly.  Codes and G are exactly fp4q_quantize's.
 * Layout of scales_mma (fp4q_mma_scales_size bytes; rows padded to 128, the
 * cols / block scale columns to 4): 512-byte atoms of 128 rows x 4
 * consecutive block scales, atom (r / 128, j / 4) at byte
 * ((r / 128) * ceil(cols / block / 4) + j / 4) * 512; inside an atom, the
 * scale of row r (r % 128 = 32 g + i) and column j is byte i * 16 + g * 4 +
 * j % 4.  Bytes of padding rows and columns are left as they were.  Other
 * formats or block sizes: FP4Q_ERR_UNSUPPORTED.  Other arguments and errors
 * as fp4q_quantize (scales_mma aligned to 16 bytes). */
FP4Q_API int fp4q_quantize_mma(const void* x, int64_t rows, int64_t cols, int fmt, int block, int rot, int gmode,
                               uint8_t* codes, uint8_t* scales_mma, float* gscale, void* stream);

/* The block-scaled FP4 GEMM that consumes two quantized operands ("Bridging
 * the Gap", s3.4 and s4: FP4 GEMMs take the codes and block scales of both
 * operands; "Diagnosing FP4 inference", Methodology: quantized weights feed
 * the compute), on the tensor cores:
 *   y[i][j] = G_A G_B sum_k q_A[i][k] s_A[i][k / b] q_B[j][k] s_B[j][k / b],
 * q the E2M1 value of a code, s the decoded scale byte without the per-tensor
 * scale, b = 16 (fmt UE4M3, NVFP4) or 32 (fmt E8M0, MXFP4).  A is m x k, B is
 * n x k, both as fp4q_quantize_mma writes them: codes [rows][k / 2], scales
 * in the MMA layout (fp4q_mma_scales_size(rows, k, b) bytes).  gscale_a /
 * gscale_b: device pointers to G_A / G_B, or NULL for 1 (must be NULL for
 * E8M0).  y: device fp32 [m][n], row-major, overwritten.  The products are
 * exact and the sum is accumulated in fp32 in the tensor cores, then scaled
 * by fp32(G_A G_B).  k % 64 == 0 (FP4Q_ERR_SHAPE otherwise); m, n >= 0 any;
 * codes and scales 16-byte aligned, y 16-byte aligned.  k == 0 writes zeros.
 * Enqueued on `stream`. */
FP4Q_API int fp4q_gemm(const uint8_t* codes_a, const uint8_t* scales_a, const float* gscale_a, int64_t m,
                       const uint8_t* codes_b, const uint8_t* scales_b, const float* gscale_b, int64_t n,
                       int64_t k, int fmt, float* y, void* stream);

/* Bytes of the block-scaled MMA scale layout for a rows x cols tensor: 512 *
 * ceil(rows / 128) * ceil(cols / block / 4); 0 for an empty tensor. */
FP4Q_API size_t fp4q_mma_scales_size(int64_t rows, int64_t cols, int block);

/* The library's device fault word on the current device, read into
 * *fault_out: 0 normally; 1 once a kernel on the tensor cores (fp4q_gemm)
 * gave up a bounded wait for its copies or matrix-multiply instructions
 * instead of hanging; the outputs of that call are then incomplete.  clear != 0 resets the word to 0
 * after reading it.  The pages have no counterpart: this is the library's own
 * failure report.  Unlike every other entry point this call synchronizes the
 * current device (it reads device memory).  FP4Q_ERR_NULL if fault_out is
 * NULL; FP4Q_ERR_CUDA if the device cannot be read. */
FP4Q_API int fp4q_device_fault(unsigned int* fault_out, int clear);

/* Static text for a status code; never NULL. */
FP4Q_API const char* fp4q_status_string(int status);

/* ABI version of this header (incremented on any signature change). */
FP4Q_API int fp4q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H */
