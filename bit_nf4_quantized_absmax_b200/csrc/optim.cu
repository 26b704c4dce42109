// Paged AdamW for the LoRA parameters ("QLoRA vs ChatGPT", capability 4: the
// optimizer state lives in a unified memory pool that pages between GPU and CPU
// memory, so it need not be pre-allocated on the device; "Guanaco", "Core
// Architecture & Training": paged optimizers).
//
// Paged memory is CUDA managed memory with the owning GPU as its preferred
// location: pages live in device memory while they fit, migrate to host memory
// under pressure and fault back on access. qlora_paged_prefetch moves a range
// ahead of use (before the optimizer step) or back to the host (after it).
//
// k_adamw: one element-wise update over flat fp32 buffers (master parameters,
// first and second moments) with bf16 gradients, AdamW with decoupled weight
// decay, four elements per thread and iteration (16-byte state accesses).
#include "qlora.h"

#include <cmath>

#include "common.cuh"

namespace qlora {
namespace {

struct AdamWArgs {
  float decay;         // 1 - lr * weight_decay
  float beta1, beta2;
  float one_m_beta1;   // 1 - beta1
  float one_m_beta2;   // 1 - beta2
  float step_size;     // lr / (1 - beta1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - beta2^t)
  float eps;
};

__device__ __forceinline__ void adamw_one(float& p, float& m, float& v, float g, const AdamWArgs& a) {
  p = p * a.decay;
  m = __fmaf_rn(a.beta1, m, a.one_m_beta1 * g);
  v = __fmaf_rn(a.beta2, v, a.one_m_beta2 * (g * g));
  const float denom = __fmaf_rn(sqrtf(v), a.inv_sqrt_bc2, a.eps);
  p = p - a.step_size * (m / denom);
}

__global__ void __launch_bounds__(256)
k_adamw(float* __restrict__ p, __nv_bfloat16* __restrict__ p_bf16, const __nv_bfloat16* __restrict__ g,
        float* __restrict__ m, float* __restrict__ v, int64_t n, const AdamWArgs a) {
  pdl_enter();
  const int64_t n4 = n / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 pv = reinterpret_cast<float4*>(p)[i];
    float4 mv = reinterpret_cast<float4*>(m)[i];
    float4 vv = reinterpret_cast<float4*>(v)[i];
    const uint2 gw = reinterpret_cast<const uint2*>(g)[i];
    adamw_one(pv.x, mv.x, vv.x, bf16lo_to_f32(gw.x), a);
    adamw_one(pv.y, mv.y, vv.y, bf16hi_to_f32(gw.x), a);
    adamw_one(pv.z, mv.z, vv.z, bf16lo_to_f32(gw.y), a);
    adamw_one(pv.w, mv.w, vv.w, bf16hi_to_f32(gw.y), a);
    reinterpret_cast<float4*>(p)[i] = pv;
    reinterpret_cast<float4*>(m)[i] = mv;
    reinterpret_cast<float4*>(v)[i] = vv;
    if (p_bf16) reinterpret_cast<uint2*>(p_bf16)[i] = make_uint2(pack_bf16x2(pv.x, pv.y), pack_bf16x2(pv.z, pv.w));
  }
  // the last n % 4 elements
  const int64_t t = n4 * 4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < n) {
    float pv = p[t], mv = m[t], vv = v[t];
    adamw_one(pv, mv, vv, __bfloat162float(g[t]), a);
    p[t] = pv;
    m[t] = mv;
    v[t] = vv;
    if (p_bf16) p_bf16[t] = __float2bfloat16_rn(pv);
  }
}

bool is_aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace
}  // namespace qlora

extern "C" {

qlora_status qlora_paged_alloc(size_t bytes, int32_t device, void** out) {
  if (!out || bytes == 0) return QLORA_ERR_INVALID_ARG;
  *out = nullptr;
  int n_dev = 0;
  if (cudaGetDeviceCount(&n_dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (device < 0 || device >= n_dev) return QLORA_ERR_INVALID_ARG;
  void* p = nullptr;
  if (cudaMallocManaged(&p, bytes, cudaMemAttachGlobal) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemAdvise(p, bytes, cudaMemAdviseSetPreferredLocation, device) != cudaSuccess ||
      cudaMemAdvise(p, bytes, cudaMemAdviseSetAccessedBy, device) != cudaSuccess) {
    cudaFree(p);
    return QLORA_ERR_CUDA;
  }
  *out = p;
  return QLORA_OK;
}

qlora_status qlora_paged_free(void* p) {
  if (!p) return QLORA_OK;
  return cudaFree(p) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_paged_prefetch(const void* p, size_t bytes, int32_t device, qlora_stream_t stream) {
  if (!p) return QLORA_ERR_INVALID_ARG;
  if (bytes == 0) return QLORA_OK;
  int n_dev = 0;
  if (cudaGetDeviceCount(&n_dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (device < -1 || device >= n_dev) return QLORA_ERR_INVALID_ARG;
  const int dst = device == -1 ? cudaCpuDeviceId : device;
  return cudaMemPrefetchAsync(p, bytes, dst, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

qlora_status qlora_adamw_step(float* param, void* param_bf16, const void* grad_bf16, float* exp_avg,
                              float* exp_avg_sq, int64_t n, float lr, float beta1, float beta2, float eps,
                              float weight_decay, int64_t step, qlora_stream_t stream) {
  using namespace qlora;
  if (n < 0 || step < 1) return QLORA_ERR_INVALID_ARG;
  if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps > 0.0f) || !(lr >= 0.0f) ||
      !(weight_decay >= 0.0f))
    return QLORA_ERR_INVALID_ARG;
  if (n == 0) return QLORA_OK;
  if (!param || !grad_bf16 || !exp_avg || !exp_avg_sq) return QLORA_ERR_INVALID_ARG;
  if (!is_aligned(param, 16) || !is_aligned(exp_avg, 16) || !is_aligned(exp_avg_sq, 16) ||
      !is_aligned(grad_bf16, 8) || (param_bf16 && !is_aligned(param_bf16, 8)))
    return QLORA_ERR_ALIGNMENT;
  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (major != 10) return QLORA_ERR_DEVICE;
  // bias corrections in double precision on the host, then rounded once to fp32
  const double bc1 = 1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step));
  AdamWArgs a;
  a.decay = static_cast<float>(1.0 - static_cast<double>(lr) * static_cast<double>(weight_decay));
  a.beta1 = beta1;
  a.beta2 = beta2;
  a.one_m_beta1 = static_cast<float>(1.0 - static_cast<double>(beta1));
  a.one_m_beta2 = static_cast<float>(1.0 - static_cast<double>(beta2));
  a.step_size = static_cast<float>(static_cast<double>(lr) / bc1);
  a.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
  a.eps = eps;
  const int64_t n4 = n / 4;
  int64_t grid = (n4 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const cudaError_t e = launch_pdl(k_adamw, dim3(static_cast<unsigned>(grid)), dim3(256), 0,
                                   reinterpret_cast<cudaStream_t>(stream), param,
                                   static_cast<__nv_bfloat16*>(param_bf16),
                                   static_cast<const __nv_bfloat16*>(grad_bf16), exp_avg, exp_avg_sq, n, a);
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // extern "C"
