// Small element-wise kernels around the LoRA gradient contractions
// ("QLoRA vs ChatGPT", capability 5: gradients only for the LoRA parameters).
//
//   k_split_hilo  T fp32 [M, r] -> T_hi = bf16(T), T_lo = bf16(T - T_hi),
//                 both [M, rpad] with zero padding, so that a bf16 tensor-core
//                 contraction with (T_hi + T_lo) keeps ~16 significant bits.
//   k_grad_reduce out = s * sum_p P[p] over the split partials, in a fixed
//                 order, optionally transposed ([R, rpad] -> [r, R]), written
//                 as bf16 or (for a later cross-rank sum) as fp32.
//   k_zero_bf16   zero fill (gradients of an empty batch).
//   k_round_bf16  fp32 -> bf16 (nearest, ties to even), e.g. the LoRA gradients
//                 of a data-parallel step once the ranks' fp32 sums are in.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

__global__ void k_split_hilo(const float* __restrict__ T, int64_t M, int r, int rpad, __nv_bfloat16* __restrict__ hi,
                             __nv_bfloat16* __restrict__ lo) {
  pdl_enter();
  const int64_t n = M * rpad;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / rpad;
    const int j = static_cast<int>(i % rpad);
    const float v = j < r ? T[m * r + j] : 0.0f;
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// Sum the split partials P[p][m][j] (fixed order) and emit the LoRA operands:
// f32[m][j] (j < r, optional), s_bf16 = bf16(s v), hi = bf16(v), lo = bf16(v - hi)
// for j < rpad (zero columns stay zero). Two adjacent columns per thread.
__global__ void k_lora_finish(const float* __restrict__ P, int splits, int64_t M, int r, int rpad, float s,
                              float* __restrict__ f32, __nv_bfloat16* __restrict__ s_bf16,
                              __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo,
                              const float* __restrict__ col_scale) {
  pdl_enter();
  const int64_t n2 = M * rpad / 2;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n2;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = 2 * i;
    const int64_t m = e / rpad;
    const int j = static_cast<int>(e % rpad);
    float2 v = make_float2(0.0f, 0.0f);
    // unrolled so that the loads of several splits are in flight together; the
    // additions still run in split order
#pragma unroll 8
    for (int p = 0; p < splits; ++p) {
      const float2 pv = __ldcg(reinterpret_cast<const float2*>(P + (static_cast<int64_t>(p) * M) * rpad) + i);
      v.x += pv.x;
      v.y += pv.y;
    }
    if (f32) {
      if (j < r) f32[m * r + j] = v.x;
      if (j + 1 < r) f32[m * r + j + 1] = v.y;
    }
    if (s_bf16) {  // one scale, or one per rank column (several adapters; zero padding columns stay zero)
      const float s0 = col_scale ? (j < r ? col_scale[j] : 0.0f) : s;
      const float s1 = col_scale ? (j + 1 < r ? col_scale[j + 1] : 0.0f) : s;
      reinterpret_cast<uint32_t*>(s_bf16)[i] = pack_bf16x2(s0 * v.x, s1 * v.y);
    }
    if (hi) {
      const uint32_t h = pack_bf16x2(v.x, v.y);
      reinterpret_cast<uint32_t*>(hi)[i] = h;
      reinterpret_cast<uint32_t*>(lo)[i] = pack_bf16x2(v.x - bf16lo_to_f32(h), v.y - bf16hi_to_f32(h));
    }
  }
}

// out = bf16(s * sum_p P[p]) for a [R, rpad] partial stack (rows R, the first r
// columns kept). A CTA owns a 32-row x 64-column tile: coalesced float2 reads of
// every split (fixed order), then either direct row-major writes ([R, r]) or a
// transpose through shared memory so that the [r, R] writes are coalesced too.
// One CTA per 32 rows x 64 columns; thread (ty, tx) sums the split partials of
// rows ty and ty + 16, columns 4 tx .. 4 tx + 3 (float4 loads), with the loads
// of four splits in flight at a time; the sum runs over p = 0, 1, ... in order.
template <typename OutT>
__device__ __forceinline__ OutT to_out(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ float to_out<float>(float v) { return v; }

template <typename OutT>
__global__ void __launch_bounds__(256)
k_grad_reduce(const float* __restrict__ P, int splits, int64_t R, int rpad, int r, float s, int transpose,
              OutT* __restrict__ out) {
  pdl_enter();
  __shared__ float tile[64][33];
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int col0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 15;   // column quad within the tile
  const int ty = threadIdx.x >> 4;   // 16 row lanes
  const int64_t pstride = R * rpad / 4;  // float4 elements per split
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int rr = ty + 16 * h;
    const int64_t row = row0 + rr;
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
    } else {
      tile[c][rr] = v.x;
      tile[c + 1][rr] = v.y;
      tile[c + 2][rr] = v.z;
      tile[c + 3][rr] = v.w;
    }
  }
  if (!transpose) return;
  __syncthreads();
  // out[j][row]: 32 consecutive rows per column j, one warp per column
  const int wx = threadIdx.x & 31, wy = threadIdx.x >> 5;
  for (int cc = wy; cc < 64; cc += 8) {
    const int j = col0 + cc;
    const int64_t row = row0 + wx;
    if (j < r && row < R) out[static_cast<int64_t>(j) * R + row] = to_out<OutT>(s * tile[cc][wx]);
  }
}

__global__ void k_zero_bf16(__nv_bfloat16* __restrict__ p, int64_t n) {
  pdl_enter();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = __float2bfloat16_rn(0.0f);
}

// Four elements per thread and step (16-byte loads, 8-byte stores) when both
// pointers allow it; the tail and unaligned buffers go element by element.
__global__ void k_round_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n, int vec) {
  pdl_enter();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  int64_t done = 0;
  if (vec) {
    const int64_t n4 = n / 4;
    for (int64_t i = t0; i < n4; i += stride) {
      const float4 v = reinterpret_cast<const float4*>(src)[i];
      reinterpret_cast<uint2*>(dst)[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
    done = 4 * n4;
  }
  for (int64_t i = done + t0; i < n; i += stride) dst[i] = __float2bfloat16_rn(src[i]);
}

// Several adapters side by side along r: A_cat rows are the A_a rows one
// adapter after another, B_cat [N, rt] holds B_a in columns off_a .. off_a + r_a,
// and col_scale[j] = c_a of column j. Plain copies (two bytes per element).
struct PackArgs {
  const __nv_bfloat16* A[kMaxMergeAdapters];
  const __nv_bfloat16* B[kMaxMergeAdapters];
  int r[kMaxMergeAdapters];
  int off[kMaxMergeAdapters];
  float c[kMaxMergeAdapters];
  int n, rt;
};

__global__ void k_pack_adapters(const __grid_constant__ PackArgs a, int64_t N, int64_t K,
                                __nv_bfloat16* __restrict__ A_cat, __nv_bfloat16* __restrict__ B_cat,
                                float* __restrict__ col_scale) {
  pdl_enter();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t na = static_cast<int64_t>(a.rt) * K;
  const int64_t nb = N * a.rt;
  for (int64_t i = t0; i < na + nb + a.rt; i += stride) {
    if (i < na) {  // A_cat[j, k]: row j of the adapter that holds rank j
      const int j = static_cast<int>(i / K);
      int ad = 0;
      while (ad + 1 < a.n && j >= a.off[ad + 1]) ++ad;
      A_cat[i] = a.A[ad][static_cast<int64_t>(j - a.off[ad]) * K + (i - static_cast<int64_t>(j) * K)];
    } else if (i < na + nb) {  // B_cat[n, j]
      const int64_t e = i - na;
      const int64_t n = e / a.rt;
      const int j = static_cast<int>(e - n * a.rt);
      int ad = 0;
      while (ad + 1 < a.n && j >= a.off[ad + 1]) ++ad;
      B_cat[e] = a.B[ad][n * a.r[ad] + (j - a.off[ad])];
    } else {
      const int j = static_cast<int>(i - na - nb);
      int ad = 0;
      while (ad + 1 < a.n && j >= a.off[ad + 1]) ++ad;
      col_scale[j] = a.c[ad];
    }
  }
}

int grid_for(int64_t n, int num_sms) {
  int64_t g = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_split_hilo(const float* T, int64_t M, int r, int rpad, void* hi, void* lo, int num_sms,
                              cudaStream_t stream) {
  return launch_pdl(k_split_hilo, dim3(grid_for(M * rpad, num_sms)), dim3(256), 0, stream, T, M, r, rpad,
                    static_cast<__nv_bfloat16*>(hi), static_cast<__nv_bfloat16*>(lo));
}

cudaError_t launch_lora_finish(const float* P, int splits, int64_t M, int r, int rpad, float s, float* f32,
                               void* s_bf16, void* hi, void* lo, int num_sms, cudaStream_t stream,
                               const float* col_scale) {
  return launch_pdl(k_lora_finish, dim3(grid_for(M * rpad / 2, num_sms)), dim3(256), 0, stream, P, splits, M, r,
                    rpad, s, f32, static_cast<__nv_bfloat16*>(s_bf16), static_cast<__nv_bfloat16*>(hi),
                    static_cast<__nv_bfloat16*>(lo), col_scale);
}

cudaError_t launch_pack_adapters(const MergeAdapter* adapters, int n_adapters, int64_t N, int64_t K, void* A_cat,
                                 void* B_cat, float* col_scale, int num_sms, cudaStream_t stream) {
  PackArgs a{};
  int off = 0;
  for (int i = 0; i < n_adapters; ++i) {
    a.A[i] = static_cast<const __nv_bfloat16*>(adapters[i].A);
    a.B[i] = static_cast<const __nv_bfloat16*>(adapters[i].B);
    a.r[i] = adapters[i].r;
    a.c[i] = adapters[i].c;
    a.off[i] = off;
    off += adapters[i].r;
  }
  a.n = n_adapters;
  a.rt = off;
  const int64_t work = static_cast<int64_t>(off) * (K + N) + off;
  return launch_pdl(k_pack_adapters, dim3(grid_for(work, num_sms)), dim3(256), 0, stream, a, N, K,
                    static_cast<__nv_bfloat16*>(A_cat), static_cast<__nv_bfloat16*>(B_cat), col_scale);
}

cudaError_t launch_grad_reduce(const float* P, int splits, int64_t R, int rpad, int r, float s, bool transpose,
                               void* out, bool out_f32, int num_sms, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((R + 31) / 32), static_cast<unsigned>(rpad / 64));
  if (out_f32)
    return launch_pdl(k_grad_reduce<float>, grid, dim3(256), 0, stream, P, splits, R, rpad, r, s, transpose ? 1 : 0,
                      static_cast<float*>(out));
  return launch_pdl(k_grad_reduce<__nv_bfloat16>, grid, dim3(256), 0, stream, P, splits, R, rpad, r, s,
                    transpose ? 1 : 0, static_cast<__nv_bfloat16*>(out));
}

cudaError_t launch_round_bf16(const float* src, void* dst, int64_t n, int num_sms, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const int vec = ((reinterpret_cast<uintptr_t>(src) & 15u) == 0 && (reinterpret_cast<uintptr_t>(dst) & 7u) == 0) ? 1 : 0;
  return launch_pdl(k_round_bf16, dim3(grid_for(vec ? (n + 3) / 4 : n, num_sms)), dim3(256), 0, stream, src,
                    static_cast<__nv_bfloat16*>(dst), n, vec);
}

cudaError_t launch_zero_bf16(void* p, int64_t n, int num_sms, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  return launch_pdl(k_zero_bf16, dim3(grid_for(n, num_sms)), dim3(256), 0, stream, static_cast<__nv_bfloat16*>(p),
                    n);
}

}  // namespace qlora
