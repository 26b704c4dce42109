/*
 * qlora.h -- C ABI of the B200 (sm_100a) QLoRA NF4 library.
 *
 * The library implements the data-parallel hot path of QLoRA:
 *   1. the NF4 ("NormalFloat4") codebook,
 *   2. block-wise absmax quantization of a frozen bf16 weight to 4-bit codes,
 *   3. double quantization of the fp32 absmax constants to int8 codes (or,
 *      as the variant the paper compares it with, single-level storage that
 *      keeps the fp32 constants),
 *   4. block-wise dequantization back to bf16,
 *   5. the QLoRA linear layer  Y = X W'^T + s (X A^T) B^T  (W' = dequant(W)),
 *      forward and backward (dX, dA, dB; W stays frozen, no dW),
 *   6. merging weighted LoRA adapters into the base weight,
 *   7. paged AdamW for the LoRA parameters (optimizer state in managed memory
 *      that pages between GPU and CPU).
 *
 * Sources (web pages describing the method; no code is printed on them):
 *   [G]  "Guanaco" (chipfoundryservices.com/topic/guanaco), sections
 *        "Core Architecture & Training" and "Technical Innovations".
 *   [E]  "QLoRA: Efficient Finetuning of Quantized LLMs" (ai-papercheck
 *        errata page), findings quoting the paper's p.4 Section 2 and
 *        p.5 Section 3.
 *   [C]  "QLoRA vs ChatGPT" (unfragile.ai compare page), capability blurbs
 *        1 (NF4, block-wise absmax), 2 (LoRA on a frozen 4-bit base),
 *        3 (double quantization), 4 (paged optimizers), 5 (on-the-fly
 *        block-wise dequantization, gradients only for the LoRA parameters)
 *        and 6 (adapter composition and merging).
 *
 * Conventions for every call below:
 *   - bf16 tensors are passed as void*, row-major and contiguous, with base
 *     addresses aligned to 16 bytes (else QLORA_ERR_ALIGNMENT).
 *   - Device pointers are owned by the caller. The library never allocates,
 *     frees or synchronizes (except qlora_paged_alloc / qlora_paged_free, whose
 *     purpose that is): every kernel is launched asynchronously on the given
 *     stream. Argument, shape and alignment errors are returned before
 *     anything is launched; a launch failure returns QLORA_ERR_CUDA.
 *   - Outputs are overwritten (no accumulation into them).
 *   - Workspace: calls that need scratch device memory take (workspace,
 *     workspace_bytes). With workspace == NULL the call stores the required
 *     size in *workspace_bytes and returns QLORA_OK without launching. With a
 *     non-NULL workspace, *workspace_bytes must hold at least that size
 *     (else QLORA_ERR_WORKSPACE). The workspace base must be 256-byte aligned.
 *     Workspace contents need no initialisation and are not preserved.
 *   - The library keeps no state between calls and may be used from several
 *     host threads at once (on distinct workspaces).
 *   - Inputs must be finite; non-finite weights give unspecified codes.
 *   - s = (float)alpha / (float)r, one fp32 division.
 */
#ifndef QLORA_B200_H
#define QLORA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The stream type is the CUDA runtime's cudaStream_t (NULL = legacy default). */
typedef struct CUstream_st* qlora_stream_t;
/* The event type is the CUDA runtime's cudaEvent_t. */
typedef struct CUevent_st* qlora_event_t;

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size  */
  QLORA_ERR_UNSUPPORTED = 2,   /* block size other than 64, dq_blocksize other
                                  than 256 (or 0 where single-level is allowed),
                                  cols % 64 != 0,
                                  r outside [8, 256] or r % 8 != 0             */
  QLORA_ERR_ALIGNMENT = 3,     /* a pointer is not aligned as required          */
  QLORA_ERR_CUDA = 4,          /* a launch or CUDA runtime call failed          */
  QLORA_ERR_WORKSPACE = 5,     /* the workspace given is smaller than required  */
  QLORA_ERR_DEVICE = 6         /* no sm_100 device is current                   */
} qlora_status;

/* NF4 storage of one frozen weight W [rows, cols] (rows = N = out_features,
 * cols = K = in_features, as in a PyTorch Linear), in one of two kinds.
 *
 *   packed    : rows*cols/2 bytes. Byte i holds code[2i] in its low nibble and
 *               code[2i+1] in its high nibble (elements in row-major order).
 *
 * Double-quantized (dq_blocksize == 256, the QLoRA format; [C] 3):
 *   absmax_q  : nblk = rows*cols/64 int8 codes in [-127, 127], one per block of
 *               64 consecutive weights (a block never crosses a row).
 *   dq_scale  : ngrp = ceil(nblk/256) fp32 scales, one per 256 consecutive
 *               absmax codes (the last group may be shorter).
 *   mean      : one fp32, the mean of all first-level absmax constants.
 *   absmax    : unused (NULL).
 *   A block's decoded constant is m' = fmaf((float)absmax_q[b], dq_scale[b/256],
 *   mean).
 *
 * Single-level (dq_blocksize == 0; "NFloat4" without DQ in the paper's p.8
 * Table 4, quoted on [E]; [C] 3 contrasts it with double quantization):
 *   absmax    : nblk fp32 constants m_b, the block's absmax itself (0.5625
 *               bytes per weight in all, against 0.515869 double-quantized).
 *   absmax_q, dq_scale, mean: unused (NULL).
 *   The block's constant is m' = absmax[b].
 *
 * Either way a block's weights decode to bf16_rn(codebook[code] * m')
 * ([C] 1, 5), and blocksize must be 64. All pointers are device memory owned
 * by the caller; packed and absmax_q must be 16-byte aligned, dq_scale, mean
 * and absmax 4-byte aligned.
 */
typedef struct {
  uint8_t* packed;
  int8_t*  absmax_q;
  float*   dq_scale;
  float*   mean;
  int64_t  rows;
  int64_t  cols;
  int32_t  blocksize;
  int32_t  dq_blocksize;
  float*   absmax;
} qlora_nf4_weight;

/* Human-readable name of a status code (static string). */
const char* qlora_status_string(qlora_status s);

/* qlora_nf4_codebook -- the 16 NF4 values, ascending, as fp32 (host call,
 * synchronous, no device needed).
 *
 * The values are normal quantiles at equally spaced probabilities: 8 positive
 * values Phi^-1(1/2 + (d - 1/2) j/8), j = 1..8, 7 negative values
 * -Phi^-1(1/2 + (d - 1/2) j/7), j = 1..7, and an exact 0, all divided by
 * Phi^-1(d) with d = 1 - (1/30 + 1/32)/2, then rounded to fp32. Index 0 is -1,
 * index 7 is 0, index 15 is +1. ([G] "Technical Innovations": a 4-bit type for
 * normally distributed weights; [E] p.5 Section 3: a discrete zero point and
 * all 2^k values used. The pages print neither the construction nor d; this
 * is the library's stated reading.)
 * Errors: QLORA_ERR_INVALID_ARG if out16 is NULL. */
qlora_status qlora_nf4_codebook(float out16[16]);

/* 4-bit data types. NF4 is the QLoRA type ([G] "Technical Innovations", [C] 1);
 * FP4 is the 4-bit float the paper compares it with (the errata page [E],
 * findings on the paper's p.8 Table 4: NFloat4 against Float4; the pages print
 * no FP4 format). Reading taken for FP4: 1 sign, 2 exponent and 1 mantissa
 * bit, magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} divided by 6 (range [-1, 1]),
 * ascending; its two encodings of zero are one value, kept once, so indices
 * 0..14 hold the 15 distinct values and index 15 repeats +1 (the nearest code
 * takes the lower index on a tie, so no weight is ever coded 15). */
typedef enum {
  QLORA_DTYPE_NF4 = 0,
  QLORA_DTYPE_FP4 = 1
} qlora_dtype;

/* qlora_codebook -- the 16 values of a 4-bit data type, ascending, fp32 (host
 * call). QLORA_DTYPE_NF4 gives qlora_nf4_codebook's values.
 * Errors: INVALID_ARG (NULL out16), UNSUPPORTED (unknown dtype). */
qlora_status qlora_codebook(qlora_dtype dtype, float out16[16]);

/* qlora_nf4_storage_bytes -- sizes of the four arrays of qlora_nf4_weight for
 * a [rows, cols] weight (host call). out[0..3] = bytes of packed, absmax_q,
 * dq_scale, mean. Errors: QLORA_ERR_INVALID_ARG (NULL out, negative sizes),
 * QLORA_ERR_UNSUPPORTED (cols % 64 != 0). */
qlora_status qlora_nf4_storage_bytes(int64_t rows, int64_t cols, size_t out[4]);

/* qlora_nf4_single_storage_bytes -- sizes of the arrays of a single-level
 * qlora_nf4_weight (host call): out[0] = bytes of packed, out[1] = bytes of
 * absmax. Errors: as qlora_nf4_storage_bytes. */
qlora_status qlora_nf4_single_storage_bytes(int64_t rows, int64_t cols, size_t out[2]);

/* qlora_quantize_nf4 -- single-level quantization: the level-1 step of
 * qlora_quantize_nf4_dq alone. Per block b of 64 weights: m_b = max |w|, stored
 * in q->absmax[b]; the codes are those qlora_quantize_nf4_dq writes (bit for
 * bit: level 1 does not depend on level 2). q->dq_blocksize must be 0 (else
 * QLORA_ERR_UNSUPPORTED). No workspace. rows == 0 writes nothing.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA, DEVICE. */
qlora_status qlora_quantize_nf4(const void* W_bf16, const qlora_nf4_weight* q, qlora_stream_t stream);

/* qlora_quantize_nf4_dq -- quantize a frozen bf16 weight W [rows, cols] into
 * q's arrays ([C] 1: block-wise absmax quantization; [C] 3 and [G] "Core
 * Architecture & Training": the absmax constants are quantized again to 8 bit
 * with their own scales).
 *
 *   Level 1, per block b of 64 weights: m_b = max |w| (exact); if m_b == 0 all
 *   codes are 7, else v = fp32(w / m_b) (IEEE division) and the code is the
 *   index of the nearest codebook value, ties to the lower index.
 *   Level 2: mu = fp32(fp64(S) / nblk) with S the exact sum of all m_b;
 *   c_b = fp32(m_b - mu); per group of 256: s_g = max |c_b|,
 *   dq_scale_g = fp32(s_g / 127), absmax_q_b = clamp(rint_even(fp32(c_b /
 *   dq_scale_g)), -127, 127); a group with s_g == 0 stores scale 0, codes 0.
 *
 * W_bf16: device, [rows, cols] bf16, 16-byte aligned. q: host struct whose
 * pointers and sizes describe caller-owned device arrays (q->rows, q->cols
 * must equal the weight's shape; q->dq_blocksize must be 256). rows == 0
 * returns QLORA_OK and writes nothing. The result does not depend on launch configuration (the mean uses
 * an exact integer accumulation).
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, DEVICE. */
qlora_status qlora_quantize_nf4_dq(const void* W_bf16, const qlora_nf4_weight* q,
                                   void* workspace, size_t* workspace_bytes,
                                   qlora_stream_t stream);

/* qlora_quantize_nf4_dq_noalloc -- the same quantization as qlora_quantize_nf4_dq
 * (identical outputs), for callers that cannot allocate device memory or supply
 * a workspace: serving runtimes whose device memory is fully planned at start-up
 * and forbid allocation afterwards, or hosts where cudaMalloc's implicit device
 * synchronization is not acceptable. The paper has no counterpart; this is a
 * convenience of this library.
 *
 * The call allocates nothing. Its scratch (about 16 MiB) is a fixed array in the
 * library's device memory that every GPU loading the library keeps until the
 * process exits; the weight may have at most 2^22 blocks of 64 (268,435,456
 * weights), larger weights return QLORA_ERR_UNSUPPORTED before any launch. The
 * first call on a device looks up that array's device address (one
 * cudaGetSymbolAddress with the device current); make that first call before
 * any stream capture. A failed lookup is not kept: that call returns
 * QLORA_ERR_CUDA and the next one tries again. The address is kept for the
 * life of the process, so after cudaDeviceReset on a device this call must not
 * be used on it again. All calls share the array, so calls that overlap on the
 * GPU race: order them on one stream. Other arguments, alignment rules and
 * errors are those of qlora_quantize_nf4_dq. */
qlora_status qlora_quantize_nf4_dq_noalloc(const void* W_bf16, const qlora_nf4_weight* q,
                                           qlora_stream_t stream);

/* qlora_quantize_nf4_dq_shard_begin / qlora_quantize_nf4_dq_shard_end --
 * qlora_quantize_nf4_dq of one weight W [total_rows, cols] whose rows are
 * split over several callers (e.g. one row shard per GPU of a data-parallel
 * job), with outputs bit-identical to quantizing W at once ([C] 1 and 3, [G]
 * "Core Architecture & Training"). Level 1 is local to each 64-weight block;
 * level 2 couples the shards only through the mean mu of all constants, which
 * is exchanged as an exact integer sum.
 *
 * Each shard covers rows [row_offset, row_offset + q->rows) of W; q describes
 * that shard's storage (q->rows rows, its own packed codes, absmax_q of
 * q->rows*cols/64 codes, dq_scale of ceil(q->rows*cols/16384) groups, one mean).
 * A shard starts on a 256-constant group boundary ((row_offset*cols) % 16384
 * == 0) and every shard but the last (row_offset + q->rows < total_rows) also
 * ends on one; else QLORA_ERR_INVALID_ARG. The groups of the shards are then
 * the groups of W, and their concatenated outputs equal W's. W may hold at
 * most 2^56 weights (else QLORA_ERR_UNSUPPORTED).
 *
 * begin: level 1 of the shard's rows W_bf16 [q->rows, cols] (device): the codes
 *   into q->packed, the fp32 constants m_b into the workspace, and the exact
 *   sum of those constants into bin_totals (device, 256 uint64, 8-byte
 *   aligned, overwritten): each m_b is an 8-bit significand sig times
 *   2^(E - 134) with E = max(exponent field, 1), and bin_totals[E] is the sum of
 *   the significands of the bin. The workspace follows the library's
 *   convention (NULL: size query), except that its contents must be kept
 *   unchanged until the matching end call.
 * Between the calls the caller adds bin_totals over all shards, element-wise as
 *   integers (e.g. an all-reduce SUM of 256 uint64, or of int64: the totals stay
 *   below 2^58). Any order gives the same exact totals.
 * end: mu = fp32(fp64(S) / (total_rows*cols/64)) from the summed totals, stored
 *   in *q->mean (the same value on every shard), then the int8 codes and group
 *   scales of this shard's constants, as qlora_quantize_nf4_dq computes them.
 *   workspace / workspace_bytes: the begin call's workspace and its size.
 * Both calls are asynchronous on `stream`; an empty shard (q->rows == 0) writes
 * zero totals in begin and nothing in end.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, DEVICE. */
qlora_status qlora_quantize_nf4_dq_shard_begin(const void* W_bf16, const qlora_nf4_weight* q,
                                               int64_t row_offset, int64_t total_rows,
                                               uint64_t* bin_totals, void* workspace,
                                               size_t* workspace_bytes, qlora_stream_t stream);
qlora_status qlora_quantize_nf4_dq_shard_end(const qlora_nf4_weight* q, int64_t row_offset,
                                             int64_t total_rows, const uint64_t* bin_totals,
                                             const void* workspace, size_t workspace_bytes,
                                             qlora_stream_t stream);

/* qlora_quantize_4bit -- block-wise absmax quantization with the codebook of
 * `dtype`: the computation of qlora_quantize_nf4_dq (q->dq_blocksize == 256,
 * double-quantized constants) or of qlora_quantize_nf4 (q->dq_blocksize == 0,
 * fp32 constants), with codebook[code] taken from qlora_codebook(dtype). The
 * nearest code ties to the lower index, as for NF4. Workspace as in
 * qlora_quantize_nf4_dq; single-level storage uses none of it (a size query
 * returns 256, and any non-NULL workspace is accepted and left untouched).
 * Errors: those of the two calls, and UNSUPPORTED for an unknown dtype. */
qlora_status qlora_quantize_4bit(const void* W_bf16, const qlora_nf4_weight* q, qlora_dtype dtype,
                                 void* workspace, size_t* workspace_bytes, qlora_stream_t stream);

/* qlora_dequantize_4bit -- qlora_dequantize_nf4 with the codebook of `dtype`:
 * w' = bf16_rn(fp32(codebook[code] * m'_b)) for either storage kind.
 * Errors: those of qlora_dequantize_nf4, and UNSUPPORTED for an unknown dtype. */
qlora_status qlora_dequantize_4bit(const qlora_nf4_weight* q, qlora_dtype dtype, void* out_bf16,
                                   qlora_stream_t stream);

/* qlora_dequantize_nf4 -- decode q (either storage kind) to a bf16 matrix
 * out_bf16 [rows, cols] (device, 16-byte aligned): w' = bf16_rn(fp32(
 * codebook[code] * m'_b)) with the block constant m'_b of the storage kind
 * ([C] 5: block-wise dequantization). Bit-identical to the dequantization used
 * inside qlora_linear_fwd/bwd and qlora_merge_lora.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA, DEVICE. */
qlora_status qlora_dequantize_nf4(const qlora_nf4_weight* q, void* out_bf16, qlora_stream_t stream);

/* qlora_dequantize_nf4_dq -- the same call as qlora_dequantize_nf4 (kept under
 * the name of the double-quantized format; it accepts both kinds). */
qlora_status qlora_dequantize_nf4_dq(const qlora_nf4_weight* q, void* out_bf16,
                                     qlora_stream_t stream);

/* qlora_linear_fwd -- Y = X W'^T + s (X A^T) B^T  ([C] 2 and 5).
 *
 *   q      : the frozen weight (either storage kind), W' = dequant(q) is
 *            [N, K] = [q->rows, q->cols].
 *   X      : device bf16 [M, K].        A : device bf16 [r, K].
 *   B      : device bf16 [N, r].        Y : device bf16 [M, N] (output).
 *   T_save : device fp32 [M, r] or NULL; when given, receives T = X A^T
 *            (fp32 accumulation) for reuse by qlora_linear_bwd.
 *   M >= 0 (M == 0: nothing is launched); 8 <= r <= 256, r % 8 == 0.
 * M <= 16 runs the decode kernels (weight-bandwidth bound, codes decoded in
 * registers); larger M runs the tcgen05 tensor-core kernels.
 * Accuracy: relative Frobenius error against an fp64 evaluation with the same
 * bf16 inputs and the same W' is about 1e-3 (the bf16 rounding of Y).
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, DEVICE. */
qlora_status qlora_linear_fwd(const qlora_nf4_weight* q, const void* X, int64_t M,
                              const void* A, const void* B, int32_t r, float alpha,
                              void* Y, float* T_save,
                              void* workspace, size_t* workspace_bytes,
                              qlora_stream_t stream);

/* qlora_linear_bwd -- gradients of qlora_linear_fwd with W frozen ([C] 5:
 * gradients only for the LoRA parameters; [E] p.4 Section 2: the input
 * gradients are produced too):
 *   dX = dY W' + s (dY B) A          [M, K] bf16 (skipped when dX == NULL)
 *   dA = s (dY B)^T X                [r, K] bf16
 *   dB = s dY^T (X A^T)              [N, r] bf16
 * dY: device bf16 [M, N]. T_saved: device fp32 [M, r] from qlora_linear_fwd,
 * or NULL to recompute X A^T. M == 0 writes zeros to dA and dB.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, DEVICE. */
qlora_status qlora_linear_bwd(const qlora_nf4_weight* q, const void* X, int64_t M,
                              const void* A, const void* B, int32_t r, float alpha,
                              const void* dY, const float* T_saved,
                              void* dX, void* dA, void* dB,
                              void* workspace, size_t* workspace_bytes,
                              qlora_stream_t stream);

/* qlora_linear_bwd_f32 -- qlora_linear_bwd with dA [r, K] and dB [N, r] written
 * in fp32 (16-byte aligned) instead of bf16, i.e. before their rounding to bf16.
 * For data-parallel training: the gradients of the ranks' token shards are
 * summed in fp32 and rounded once, so the sum keeps the accuracy of a
 * single-GPU backward. dX (when not NULL) is bf16 as in qlora_linear_bwd.
 * Errors: as qlora_linear_bwd. */
qlora_status qlora_linear_bwd_f32(const qlora_nf4_weight* q, const void* X, int64_t M,
                                  const void* A, const void* B, int32_t r, float alpha,
                                  const void* dY, const float* T_saved,
                                  void* dX, float* dA, float* dB,
                                  void* workspace, size_t* workspace_bytes,
                                  qlora_stream_t stream);

/* qlora_linear_bwd_dp -- the backward of one rank's token shard in data-parallel
 * training ([C] 5: gradients are computed only for the LoRA parameters, so the
 * ranks exchange only r (K + N) values per linear). The same gradients as
 * qlora_linear_bwd_f32, laid out for the exchange and ordered so that it can
 * overlap the dX GEMM:
 *   grads       : device fp32 [r*K + N*r], 16-byte aligned: dA [r, K] row-major
 *                 followed by dB [N, r] row-major, both before any rounding.
 *   grads_ready : a cudaEvent_t or NULL. When given, it is recorded on `stream`
 *                 as soon as `grads` is complete, before the kernels of dX are
 *                 launched, so that another stream can wait on it and sum
 *                 `grads` over the ranks (e.g. an NCCL all-reduce) while dX is
 *                 computed. Round the sums with qlora_round_bf16.
 * dX (bf16 [M, K], or NULL), the other arguments and the errors are those of
 * qlora_linear_bwd. */
qlora_status qlora_linear_bwd_dp(const qlora_nf4_weight* q, const void* X, int64_t M,
                                 const void* A, const void* B, int32_t r, float alpha,
                                 const void* dY, const float* T_saved, void* dX, float* grads,
                                 qlora_event_t grads_ready, void* workspace, size_t* workspace_bytes,
                                 qlora_stream_t stream);

/* qlora_round_bf16 -- dst[i] = bf16_rn(src[i]) (nearest, ties to even) for
 * 0 <= i < n: the one rounding that qlora_linear_bwd applies to its fp32
 * gradients, applied by a data-parallel step to the sums over its ranks
 * ([C] 5). src: device fp32 [n], 4-byte aligned; dst_bf16: device bf16 [n],
 * 2-byte aligned (16- and 8-byte alignment take a vector path). n == 0 launches
 * nothing. Asynchronous on `stream`.
 * Errors: INVALID_ARG (n < 0, NULL pointers with n > 0), ALIGNMENT, CUDA, DEVICE. */
qlora_status qlora_round_bf16(const float* src, void* dst_bf16, int64_t n, qlora_stream_t stream);

/* One LoRA adapter of a merge: A [r, cols] and B [rows, r] (device bf16,
 * 16-byte aligned, row-major), 8 <= r <= 256 with r % 8 == 0, scale
 * s = (float)alpha / (float)r, composition weight w. */
typedef struct {
  const void* A;
  const void* B;
  int32_t r;
  float alpha;
  float weight;
} qlora_lora_adapter;

/* qlora_merge_lora -- merge weighted adapters into the frozen base ([C] 6:
 * adapters trained on one quantized base are composed with weights and merged
 * into the base weights to give a standalone checkpoint):
 *   W_out = bf16_rn( W' + sum_a c_a (B_a A_a) ),  c_a = fp32(w_a * s_a),
 * evaluated in fp64 in a fixed order (for each element: start from W', then for
 * a = 0, 1, ...: P = sum over j = 0 .. r_a - 1 of B_a[n, j] A_a[j, k] added in
 * that order, y = y + c_a * P), rounded once to bf16 (nearest, ties to even).
 *   q         : the base weight (either storage kind), W' = dequant(q), [rows, cols].
 *   adapters  : host array of n_adapters entries (read before returning);
 *               0 <= n_adapters <= 8 (0 writes W' itself).
 *   W_out     : device bf16 [rows, cols] (16-byte aligned), overwritten.
 * The merged weight can be re-quantized with qlora_quantize_nf4_dq.
 * Errors: INVALID_ARG, UNSUPPORTED (r out of range, more than 8 adapters),
 * ALIGNMENT, CUDA, DEVICE. */
qlora_status qlora_merge_lora(const qlora_nf4_weight* q, const qlora_lora_adapter* adapters,
                              int32_t n_adapters, void* W_out, qlora_stream_t stream);

/* qlora_linear_fwd_multi -- several LoRA adapters applied at once to the same
 * frozen weight without merging them ([C] 6: adapters trained on one quantized
 * base are composed with weights):
 *   Y = X W'^T + sum_a c_a (X A_a^T) B_a^T,   c_a = fp32(w_a * s_a),
 * s_a = (float)alpha_a / (float)r_a and w_a the adapter's composition weight
 * (the c_a of qlora_merge_lora, so that the result matches applying the merged
 * weight up to the final bf16 rounding). The adapters are passed concatenated
 * along the rank (qlora_pack_adapters builds the three arrays):
 *   A_cat     : device bf16 [r_total, K], the A_a one after another.
 *   B_cat     : device bf16 [N, r_total], the B_a side by side.
 *   col_scale : device fp32 [r_total], c_a of the adapter of each rank column.
 * 8 <= r_total <= 256, r_total % 8 == 0. Each rank column of T = X A_cat^T is
 * multiplied by its scale as T is formed (fp32), then the LoRA term is added as
 * in qlora_linear_fwd (which this equals for one adapter with c = s, up to where
 * the scale is applied). X, M, Y, workspace and errors as in qlora_linear_fwd
 * (no T is saved: this is the inference path). */
qlora_status qlora_linear_fwd_multi(const qlora_nf4_weight* q, const void* X, int64_t M,
                                    const void* A_cat, const void* B_cat, int32_t r_total,
                                    const float* col_scale, void* Y, void* workspace,
                                    size_t* workspace_bytes, qlora_stream_t stream);

/* qlora_pack_adapters -- build the concatenated operands of
 * qlora_linear_fwd_multi from n_adapters adapters (host array, read before the
 * call returns; 1 <= n_adapters <= 8, each r_a in [8, 256] with r_a % 8 == 0,
 * sum r_a <= 256) of a [rows, cols] weight: A_cat [sum r_a, cols] and B_cat
 * [rows, sum r_a] (device bf16, 16-byte aligned, caller-owned) and col_scale
 * [sum r_a] (device fp32) = fp32(weight_a * alpha_a / r_a) per column. One
 * asynchronous copy kernel on `stream`; do it once per adapter set.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA, DEVICE. */
qlora_status qlora_pack_adapters(const qlora_lora_adapter* adapters, int32_t n_adapters, int64_t rows,
                                 int64_t cols, void* A_cat, void* B_cat, float* col_scale,
                                 qlora_stream_t stream);

/* qlora_paged_alloc -- allocate `bytes` of paged memory for optimizer state
 * ([C] 4: a unified pool that pages between GPU and CPU memory, so the state
 * need not be pre-allocated in device memory; [G] "Core Architecture &
 * Training": paged optimizers). The memory is CUDA managed memory whose
 * preferred location is GPU `device`: its pages live in that GPU's memory while
 * it has room, move to host memory under memory pressure and move back when a
 * kernel touches them. Unlike every other call, this one allocates; free with
 * qlora_paged_free. *out receives the pointer (NULL on error). Contents are
 * uninitialized.
 * Errors: INVALID_ARG (NULL out, bytes == 0, no such device), CUDA. */
qlora_status qlora_paged_alloc(size_t bytes, int32_t device, void** out);

/* qlora_paged_free -- free memory from qlora_paged_alloc (NULL is a no-op). The
 * caller orders it after every kernel that uses the memory. Errors: CUDA. */
qlora_status qlora_paged_free(void* p);

/* qlora_paged_prefetch -- move [p, p + bytes) of paged memory asynchronously on
 * `stream` to GPU `device`, or to host memory with device == -1: to device
 * before the optimizer step, back to the host after it when device memory is
 * needed for something else. The data are unchanged.
 * Errors: INVALID_ARG (NULL p, device < -1 or no such device), CUDA. */
qlora_status qlora_paged_prefetch(const void* p, size_t bytes, int32_t device, qlora_stream_t stream);

/* qlora_adamw_step -- one AdamW update (decoupled weight decay) of n
 * parameters held as flat buffers (lay out every LoRA A and B of a model
 * contiguously to update them with one call). Step t >= 1:
 *   p <- p * (1 - lr * weight_decay)
 *   m <- beta1 * m + (1 - beta1) * g
 *   v <- beta2 * v + (1 - beta2) * g^2
 *   p <- p - (lr / (1 - beta1^t)) * m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
 * with the bias corrections computed in double precision on the host and the
 * rest in fp32 on the device. (The pages name the paged optimizer but print no
 * formula; this is the usual AdamW with 32-bit state, the library's reading.)
 *   param      : device fp32 [n] master parameters, updated in place (16-byte aligned).
 *   param_bf16 : device bf16 [n] or NULL; receives bf16_rn(p) for the next
 *                forward (8-byte aligned).
 *   grad_bf16  : device bf16 [n] gradients, e.g. dA and dB of qlora_linear_bwd
 *                (8-byte aligned).
 *   exp_avg, exp_avg_sq : fp32 [n] first and second moments (16-byte aligned),
 *                zero before the first step; device or paged memory.
 * Errors: INVALID_ARG (n < 0, step < 1, beta outside [0, 1), eps <= 0, lr < 0,
 * weight_decay < 0, NULL pointers when n > 0), ALIGNMENT, CUDA, DEVICE. */
qlora_status qlora_adamw_step(float* param, void* param_bf16, const void* grad_bf16, float* exp_avg,
                              float* exp_avg_sq, int64_t n, float lr, float beta1, float beta2, float eps,
                              float weight_decay, int64_t step, qlora_stream_t stream);

/* qlora_device_error -- read and clear the library's device-side error word on
 * the current device (synchronizes the stream). Kernels whose waits on
 * asynchronous copies exceed a time bound set this word and return early
 * instead of hanging; 0 means no such event. *code receives the word.
 * Errors: INVALID_ARG (NULL code), CUDA. */
qlora_status qlora_device_error(int32_t* code, qlora_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* QLORA_B200_H */
