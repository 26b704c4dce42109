// Double quantization of one weight that is split by rows over several callers
// (e.g. one row shard per GPU), with a result bit-identical to quantizing the
// whole weight at once ("QLoRA vs ChatGPT", capability 5: block-wise absmax
// quantization; "Guanaco", "Core Architecture & Training": double quantization
// of the constants, mean-centred, int8 codes per 256 constants).
//
// The only quantity that couples the shards is the mean of all block constants.
// The first call of a shard stores its codes and fp32 constants and writes the
// exact sum of its constants as 256 uint64 exponent-bin totals (each constant is
// an 8-bit significand times a power of two, so the sum is a sum of integers per
// exponent). Integer totals added over the shards, in any order, give the
// whole tensor's exact sum. The second call forms the mean from the summed
// totals and codes this shard's constants in its own 256-constant groups;
// shards therefore start on a group boundary.
#include "qlora.h"

#include "common.cuh"
#include "kernels.h"

namespace {

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t x) { return (x + 255) / 256 * 256; }

// Argument checks shared by both calls (no device access).
qlora_status check_shard(const qlora_nf4_weight* q, int64_t row_offset, int64_t total_rows) {
  if (!q) return QLORA_ERR_INVALID_ARG;
  if (q->rows < 0 || q->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (q->blocksize != 64 || q->dq_blocksize != 256 || q->cols % 64) return QLORA_ERR_UNSUPPORTED;
  if (q->cols > (int64_t(1) << 31) || total_rows > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  if (row_offset < 0 || total_rows < 0 || q->rows > total_rows - row_offset) return QLORA_ERR_INVALID_ARG;
  // at most 2^56 weights in W: every summed bin total stays below 2^58
  if (total_rows * q->cols > (int64_t(1) << 56)) return QLORA_ERR_UNSUPPORTED;
  // 256 constants span 16384 weights: a shard starts on a group boundary, and
  // every shard but the last ends on one
  if ((row_offset * q->cols) % 16384 != 0) return QLORA_ERR_INVALID_ARG;
  if (row_offset + q->rows < total_rows && (q->rows * q->cols) % 16384 != 0) return QLORA_ERR_INVALID_ARG;
  if (q->rows > 0) {
    if (!q->packed || !q->absmax_q || !q->dq_scale || !q->mean) return QLORA_ERR_INVALID_ARG;
    if (!is_aligned(q->packed, 16) || !is_aligned(q->absmax_q, 16) || !is_aligned(q->dq_scale, 4) ||
        !is_aligned(q->mean, 4))
      return QLORA_ERR_ALIGNMENT;
  }
  return QLORA_OK;
}

qlora_status sm_count(int* sms) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return major == 10 ? QLORA_OK : QLORA_ERR_DEVICE;
}

}  // namespace

extern "C" {

qlora_status qlora_quantize_nf4_dq_shard_begin(const void* W_bf16, const qlora_nf4_weight* q, int64_t row_offset,
                                               int64_t total_rows, uint64_t* bin_totals, void* workspace,
                                               size_t* workspace_bytes, qlora_stream_t stream) {
  qlora_status st = check_shard(q, row_offset, total_rows);
  if (st != QLORA_OK) return st;
  const int64_t nblk = q->rows * q->cols / 64;
  const size_t need = round_up(static_cast<size_t>(nblk) * sizeof(float));
  if (!workspace_bytes) return QLORA_ERR_INVALID_ARG;
  if (!workspace) {  // size query
    *workspace_bytes = need;
    return QLORA_OK;
  }
  if (*workspace_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!is_aligned(workspace, 256)) return QLORA_ERR_ALIGNMENT;
  if (!bin_totals) return QLORA_ERR_INVALID_ARG;
  if (!is_aligned(bin_totals, 8)) return QLORA_ERR_ALIGNMENT;
  if (nblk > 0 && !W_bf16) return QLORA_ERR_INVALID_ARG;
  if (W_bf16 && !is_aligned(W_bf16, 16)) return QLORA_ERR_ALIGNMENT;
  int sms = 0;
  if ((st = sm_count(&sms)) != QLORA_OK) return st;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  unsigned long long* totals = reinterpret_cast<unsigned long long*>(bin_totals);
  if (nblk == 0)  // an empty shard adds nothing to the sum
    return cudaMemsetAsync(totals, 0, qlora::kQuantScratchBytes, cs) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  const cudaError_t e = qlora::launch_quantize_first(W_bf16, nblk, q->packed, static_cast<float*>(workspace),
                                                     totals, sms, cs);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_quantize_nf4_dq_shard_end(const qlora_nf4_weight* q, int64_t row_offset, int64_t total_rows,
                                             const uint64_t* bin_totals, const void* workspace,
                                             size_t workspace_bytes, qlora_stream_t stream) {
  qlora_status st = check_shard(q, row_offset, total_rows);
  if (st != QLORA_OK) return st;
  const int64_t nblk = q->rows * q->cols / 64;
  const int64_t nblk_all = total_rows * q->cols / 64;
  if (nblk == 0) return QLORA_OK;
  if (!workspace) return QLORA_ERR_INVALID_ARG;
  if (workspace_bytes < round_up(static_cast<size_t>(nblk) * sizeof(float))) return QLORA_ERR_WORKSPACE;
  if (!is_aligned(workspace, 256)) return QLORA_ERR_ALIGNMENT;
  if (!bin_totals) return QLORA_ERR_INVALID_ARG;
  if (!is_aligned(bin_totals, 8)) return QLORA_ERR_ALIGNMENT;
  int sms = 0;
  if ((st = sm_count(&sms)) != QLORA_OK) return st;
  const cudaError_t e = qlora::launch_quantize_second(
      static_cast<const float*>(workspace), nblk, reinterpret_cast<const unsigned long long*>(bin_totals), nblk_all,
      q->absmax_q, q->dq_scale, q->mean, sms, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // extern "C"
