// qlora_quantize_nf4_dq_noalloc: the quantize + double-quant call for callers
// that cannot allocate device memory or hand the library a workspace. Examples
// are serving runtimes whose device memory is fully planned at start-up and
// forbid allocation afterwards, and hosts where cudaMalloc's implicit device
// synchronization would stall other work.
//
// The scratch the quantize kernels need (the exponent-bin totals of the exact
// sum of the constants, and one fp32 absmax per 64-weight block) lives in a
// file-scope device array of a fixed size. Every GPU that loads this code holds that array until the process
// exits. All calls share it, so calls that overlap on the GPU (different
// streams, or different host threads on one device) race and must be ordered by
// the caller. Every region is fully written by a kernel of the call before
// another kernel of the call reads it.
#include <mutex>

#include "qlora.h"
#include "common.cuh"
#include "host_tables.h"
#include "kernels.h"

namespace {

// At most 2^22 blocks of 64 weights (268,435,456 weights, e.g. any single
// Llama-65B linear weight): 2 KiB of bin totals + 16 MiB of
// absmax per device.
constexpr int64_t kNoAllocMaxBlocks = int64_t(1) << 22;
constexpr size_t kBinsBytes = (qlora::kQuantScratchBytes + 255) / 256 * 256;
constexpr size_t kScratchBytes = kBinsBytes + static_cast<size_t>(kNoAllocMaxBlocks) * sizeof(float);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

struct DeviceScratch {
  std::mutex mu;
  void* ptr = nullptr;  // set once the lookup has succeeded
};

DeviceScratch g_scratch[kMaxDevices];

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so its device address is looked
// up with that device current. Only a successful lookup is kept: a call that
// fails (for instance the first call made inside a stream capture) returns
// QLORA_ERR_CUDA and the next call on that device tries again.
qlora_status scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_DEVICE;
  DeviceScratch& d = g_scratch[dev];
  std::lock_guard<std::mutex> lock(d.mu);
  if (!d.ptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();  // do not leave the failure for the caller's next error check
      return QLORA_ERR_CUDA;
    }
    d.ptr = p;
  }
  *out = d.ptr;
  return QLORA_OK;
}

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" qlora_status qlora_quantize_nf4_dq_noalloc(const void* W_bf16, const qlora_nf4_weight* q,
                                                      qlora_stream_t stream) {
  if (!q) return QLORA_ERR_INVALID_ARG;
  if (q->rows < 0 || q->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (q->blocksize != 64 || q->dq_blocksize != 256 || q->cols % 64) return QLORA_ERR_UNSUPPORTED;
  if (q->rows > (int64_t(1) << 31) || q->cols > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  const int64_t numel = q->rows * q->cols;
  const int64_t nblk = numel / 64;
  if (nblk > kNoAllocMaxBlocks) return QLORA_ERR_UNSUPPORTED;  // larger than the fixed scratch
  if (numel == 0) return QLORA_OK;
  if (!W_bf16 || !q->packed || !q->absmax_q || !q->dq_scale || !q->mean) return QLORA_ERR_INVALID_ARG;
  if (!is_aligned(W_bf16, 16) || !is_aligned(q->packed, 16) || !is_aligned(q->absmax_q, 16) ||
      !is_aligned(q->dq_scale, 4) || !is_aligned(q->mean, 4))
    return QLORA_ERR_ALIGNMENT;
  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (major != 10) return QLORA_ERR_DEVICE;
  void* scratch = nullptr;
  qlora_status st = scratch_on_current_device(&scratch);
  if (st != QLORA_OK) return st;
  char* base = static_cast<char*>(scratch);
  cudaError_t e = qlora::launch_quantize(W_bf16, numel, q->packed, q->absmax_q, q->dq_scale, q->mean,
                                         reinterpret_cast<float*>(base + kBinsBytes),
                                         base, sms,
                                         reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}
