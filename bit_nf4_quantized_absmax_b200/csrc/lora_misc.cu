// Small element-wise kernels around the LoRA gradient contractions
// ("QLoRA vs ChatGPT", capability 5: gradients only for the LoRA parameters).
//
//   k_lora_finish sums the split partials of T = X A^T or U = dY B in a fixed
//                 order and writes fp32, s * (.) in bf16, and the bf16 split
//                 hi = bf16(v), lo = bf16(v - hi) ([M, rpad], zero padding) that
//                 lets a bf16 tensor-core contraction keep ~16 significant bits;
//                 the same launch can split a saved fp32 T the same way.
//   k_grad_reduce out = s * sum_p P[p] over the split partials, in a fixed
//                 order, optionally transposed ([R, rpad] -> [r, R]), written
//                 as bf16 or (for a later cross-rank sum) as fp32.
//   k_zero_bf16   zero fill (gradients of an empty batch).
#include "common.cuh"
#include "kernels.h"
#include "lora_finish.cuh"

namespace qlora {
namespace {


// Sum the split partials P[p][m][j] (fixed order) and emit the LoRA operands:
// f32[m][j] (j < r, optional), s_bf16 = bf16(s v), hi = bf16(v), lo = bf16(v - hi)
// for j < rpad (zero columns stay zero). Two adjacent columns per thread.
__global__ void k_lora_finish(const __grid_constant__ LoraFinishJob job) {
  pdl_enter();
  lora_finish_range(job, static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x,
                    static_cast<int64_t>(gridDim.x) * blockDim.x);
}

// out = bf16(s * sum_p P[p]) for a [R, rpad] partial stack (rows R, the first r
// columns kept). A CTA owns a 32-row x 64-column tile: coalesced float2 reads of
// every split (fixed order), then either direct row-major writes ([R, r]) or a
// transpose through shared memory so that the [r, R] writes are coalesced too.
template <typename OutT>
__device__ __forceinline__ OutT to_out(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ float to_out<float>(float v) { return v; }

// One CTA per 16 rows x 64 columns; thread (ty, tx) sums the split partials of
// row ty, columns 4 tx .. 4 tx + 3 (float4 loads), with the loads of four
// splits in flight at a time; the sum runs over p = 0, 1, ... in order.
template <typename OutT>
__global__ void __launch_bounds__(256)
k_grad_reduce(const float* __restrict__ P, int splits, int64_t R, int rpad, int r, float s, int transpose,
              OutT* __restrict__ out) {
  pdl_enter();
  __shared__ float tile[64][17];
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 16;
  const int col0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 15;   // column quad within the tile
  const int ty = threadIdx.x >> 4;   // row within the tile
  const int64_t pstride = R * rpad / 4;  // float4 elements per split
  const int64_t row = row0 + ty;
  float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (row < R) {
    const float4* src = reinterpret_cast<const float4*>(P + row * rpad + col0) + tx;
    int p = 0;
    for (; p + 4 <= splits; p += 4) {
      float4 q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = __ldcs(src + (p + i) * pstride);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v.x += q[i].x; v.y += q[i].y; v.z += q[i].z; v.w += q[i].w;
      }
    }
    for (; p < splits; ++p) {
      const float4 q = __ldcs(src + p * pstride);
      v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
    }
  }
  const int c = 4 * tx;
  if (!transpose) {
    if (row < R) {
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (col0 + c + i < r) out[row * r + col0 + c + i] = to_out<OutT>(s * vv[i]);
    }
    return;
  }
  tile[c][ty] = v.x;
  tile[c + 1][ty] = v.y;
  tile[c + 2][ty] = v.z;
  tile[c + 3][ty] = v.w;
  __syncthreads();
  // out[j][row]: 16 consecutive rows per column j
  for (int idx = threadIdx.x; idx < 64 * 16; idx += blockDim.x) {
    const int j = col0 + (idx >> 4);
    const int64_t rr = row0 + (idx & 15);
    if (j < r && rr < R) out[static_cast<int64_t>(j) * R + rr] = to_out<OutT>(s * tile[idx >> 4][idx & 15]);
  }
}

__global__ void k_zero_bf16(__nv_bfloat16* __restrict__ p, int64_t n) {
  pdl_enter();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = __float2bfloat16_rn(0.0f);
}

int grid_for(int64_t n, int num_sms) {
  int64_t g = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace


cudaError_t launch_lora_finish(const float* P, int splits, int64_t M, int r, int rpad, float s, float* f32,
                               void* s_bf16, void* hi, void* lo, int num_sms, cudaStream_t stream,
                               const float* t_src, void* t_hi, void* t_lo) {
  LoraFinishJob job;
  job.P = P;
  job.splits = splits;
  job.M = M;
  job.r = r;
  job.rpad = rpad;
  job.s = s;
  job.f32 = f32;
  job.s_bf16 = s_bf16;
  job.hi = hi;
  job.lo = lo;
  job.t_src = t_src;
  job.t_hi = t_hi;
  job.t_lo = t_lo;
  return launch_pdl(k_lora_finish, dim3(grid_for(M * rpad / 2, num_sms)), dim3(256), 0, stream, job);
}

cudaError_t launch_grad_reduce(const float* P, int splits, int64_t R, int rpad, int r, float s, bool transpose,
                               void* out, bool out_f32, int num_sms, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((R + 15) / 16), static_cast<unsigned>(rpad / 64));
  if (out_f32)
    return launch_pdl(k_grad_reduce<float>, grid, dim3(256), 0, stream, P, splits, R, rpad, r, s, transpose ? 1 : 0,
                      static_cast<float*>(out));
  return launch_pdl(k_grad_reduce<__nv_bfloat16>, grid, dim3(256), 0, stream, P, splits, R, rpad, r, s,
                    transpose ? 1 : 0, static_cast<__nv_bfloat16*>(out));
}

cudaError_t launch_zero_bf16(void* p, int64_t n, int num_sms, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  return launch_pdl(k_zero_bf16, dim3(grid_for(n, num_sms)), dim3(256), 0, stream, static_cast<__nv_bfloat16*>(p),
                    n);
}

}  // namespace qlora
