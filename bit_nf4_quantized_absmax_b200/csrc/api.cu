// C ABI entry points (include/qlora.h): argument checks, workspace layout and
// kernel dispatch. Nothing here allocates, frees or synchronizes, except
// qlora_device_error, which reads the device error word.
#include "qlora.h"

#include <cstring>

#include "common.cuh"
#include "host_tables.h"
#include "kernels.h"

namespace qlora {
__device__ int32_t g_device_error = 0;
}  // namespace qlora

namespace {

using namespace qlora;

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DeviceInfo {
  int num_sms;
};

qlora_status device_info(DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (major != 10) return QLORA_ERR_DEVICE;
  info->num_sms = sms;
  return QLORA_OK;
}

qlora_status check_weight(const qlora_nf4_weight* q, bool need_rows) {
  if (!q) return QLORA_ERR_INVALID_ARG;
  if (q->rows < 0 || q->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (q->blocksize != 64 || q->dq_blocksize != 256) return QLORA_ERR_UNSUPPORTED;
  if (q->cols % 64) return QLORA_ERR_UNSUPPORTED;
  if (q->rows > (int64_t(1) << 31) || q->cols > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  if (need_rows && q->rows == 0) return QLORA_ERR_INVALID_ARG;
  if (q->rows > 0) {
    if (!q->packed || !q->absmax_q || !q->dq_scale || !q->mean) return QLORA_ERR_INVALID_ARG;
    if (!aligned(q->packed, 16) || !aligned(q->absmax_q, 16) || !aligned(q->dq_scale, 4) || !aligned(q->mean, 4))
      return QLORA_ERR_ALIGNMENT;
  }
  return QLORA_OK;
}

qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// Workspace query / check shared by every call that needs scratch.
// Returns QLORA_OK with *launch == false for a pure size query.
qlora_status workspace_check(void* ws, size_t* ws_bytes, size_t need, bool* launch) {
  if (!ws_bytes) return QLORA_ERR_INVALID_ARG;
  if (!ws) {
    *ws_bytes = need;
    *launch = false;
    return QLORA_OK;
  }
  if (*ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, kAlign)) return QLORA_ERR_ALIGNMENT;
  *launch = true;
  return QLORA_OK;
}

}  // namespace

extern "C" {

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
    case QLORA_ERR_UNSUPPORTED: return "QLORA_ERR_UNSUPPORTED";
    case QLORA_ERR_ALIGNMENT: return "QLORA_ERR_ALIGNMENT";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE";
    case QLORA_ERR_DEVICE: return "QLORA_ERR_DEVICE";
  }
  return "QLORA_ERR_UNKNOWN";
}

qlora_status qlora_nf4_codebook(float out16[16]) {
  if (!out16) return QLORA_ERR_INVALID_ARG;
  std::memcpy(out16, quant_tables().codebook, sizeof(float) * 16);
  return QLORA_OK;
}

qlora_status qlora_nf4_storage_bytes(int64_t rows, int64_t cols, size_t out[4]) {
  if (!out || rows < 0 || cols < 0) return QLORA_ERR_INVALID_ARG;
  if (cols % 64) return QLORA_ERR_UNSUPPORTED;
  const int64_t numel = rows * cols;
  const int64_t nblk = numel / 64;
  out[0] = static_cast<size_t>(numel / 2);
  out[1] = static_cast<size_t>(nblk);
  out[2] = static_cast<size_t>((nblk + 255) / 256) * sizeof(float);
  out[3] = sizeof(float);
  return QLORA_OK;
}

qlora_status qlora_quantize_nf4_dq(const void* W_bf16, const qlora_nf4_weight* q, void* workspace,
                                   size_t* workspace_bytes, qlora_stream_t stream) {
  qlora_status st = check_weight(q, false);
  if (st != QLORA_OK) return st;
  if (!W_bf16 && q->rows > 0) return QLORA_ERR_INVALID_ARG;
  if (W_bf16 && !aligned(W_bf16, 16)) return QLORA_ERR_ALIGNMENT;
  const int64_t numel = q->rows * q->cols;
  const int64_t nblk = numel / 64;
  const size_t off_absmax = align_up(kQuantBinWords * sizeof(unsigned long long));
  const size_t need = off_absmax + align_up(static_cast<size_t>(nblk) * sizeof(float));
  bool launch = false;
  st = workspace_check(workspace, workspace_bytes, need, &launch);
  if (st != QLORA_OK || !launch || numel == 0) return st;
  DeviceInfo di;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  char* ws = static_cast<char*>(workspace);
  return cuda_status(launch_quantize(W_bf16, numel, q->packed, q->absmax_q, q->dq_scale, q->mean,
                                     reinterpret_cast<float*>(ws + off_absmax),
                                     reinterpret_cast<unsigned long long*>(ws), di.num_sms,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status qlora_dequantize_nf4_dq(const qlora_nf4_weight* q, void* out_bf16, qlora_stream_t stream) {
  qlora_status st = check_weight(q, false);
  if (st != QLORA_OK) return st;
  const int64_t numel = q->rows * q->cols;
  if (numel == 0) return QLORA_OK;
  if (!out_bf16) return QLORA_ERR_INVALID_ARG;
  if (!aligned(out_bf16, 16)) return QLORA_ERR_ALIGNMENT;
  DeviceInfo di;
  if ((st = device_info(&di)) != QLORA_OK) return st;
  return cuda_status(launch_dequantize(q->packed, q->absmax_q, q->dq_scale, q->mean, out_bf16, numel,
                                       quant_tables().codebook, di.num_sms,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

qlora_status qlora_linear_fwd(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A,
                              const void* B, int32_t r, float alpha, void* Y, float* T_save, void* workspace,
                              size_t* workspace_bytes, qlora_stream_t stream) {
  (void)q; (void)X; (void)M; (void)A; (void)B; (void)r; (void)alpha; (void)Y; (void)T_save;
  (void)workspace; (void)workspace_bytes; (void)stream;
  return QLORA_ERR_UNSUPPORTED;
}

qlora_status qlora_linear_bwd(const qlora_nf4_weight* q, const void* X, int64_t M, const void* A,
                              const void* B, int32_t r, float alpha, const void* dY, const float* T_saved,
                              void* dX, void* dA, void* dB, void* workspace, size_t* workspace_bytes,
                              qlora_stream_t stream) {
  (void)q; (void)X; (void)M; (void)A; (void)B; (void)r; (void)alpha; (void)dY; (void)T_saved;
  (void)dX; (void)dA; (void)dB; (void)workspace; (void)workspace_bytes; (void)stream;
  return QLORA_ERR_UNSUPPORTED;
}

qlora_status qlora_device_error(int32_t* code, qlora_stream_t stream) {
  if (!code) return QLORA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return QLORA_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, qlora::g_device_error, sizeof(v)) != cudaSuccess) return QLORA_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbol(qlora::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return QLORA_ERR_CUDA;
  *code = v;
  return QLORA_OK;
}

}  // extern "C"
