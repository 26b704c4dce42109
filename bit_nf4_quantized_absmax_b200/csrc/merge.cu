// Merging weighted LoRA adapters into the frozen base ("QLoRA vs ChatGPT",
// capability 6: adapters trained on one quantized base are composed with
// weights, w1 * adapter1 + w2 * adapter2, and merged into the base weights).
//
//   y = W'[n, k]                          (k_dequant writes W' into the output first)
//   for each adapter a in order:
//     P = sum_{j < r_a} B_a[n, j] A_a[j, k]       fp64, j in increasing order
//     y = y + c_a * P                              fp64 (multiply, then add), c_a = fp32(w_a * s_a)
//   out[n, k] = bf16_rn(y)                 one rounding from fp64
//
// Each bf16 x bf16 product is exact in fp64, so the fused multiply-adds of the
// sum round exactly as additions of the exact products; the result is a fixed
// function of the inputs. 64 x 64 outputs per CTA, 4 x 4 per thread; adapter
// chunks of 32 ranks staged in shared memory as fp64.
#include "common.cuh"
#include "kernels.h"

namespace qlora {
namespace {

constexpr int kMT = 64;  // output tile (rows and columns)
constexpr int kMJ = 32;  // ranks per shared-memory chunk

struct MergeArgs {
  const __nv_bfloat16* A[kMaxMergeAdapters];
  const __nv_bfloat16* B[kMaxMergeAdapters];
  int r[kMaxMergeAdapters];
  float c[kMaxMergeAdapters];
  int n;
};

// fp64 -> bf16 bits, round to nearest even in one step: truncate to fp32, set the
// lowest bit when that was inexact (round to odd, 16 bits more than bf16 keeps),
// then round the fp32 value to bf16 (Boldo and Melquiond, "Emulation of FMA and
// correctly rounded sums: proved algorithms using rounding to odd", 2008).
__device__ __forceinline__ unsigned short f64_to_bf16_bits(double y) {
  float f = __double2float_rz(y);
  if (static_cast<double>(f) != y) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__global__ void __launch_bounds__(256)
k_merge(__nv_bfloat16* __restrict__ W, int64_t N, int64_t K, const __grid_constant__ MergeArgs ma) {
  __shared__ double As[kMJ][kMT + 1];  // [rank][column]
  __shared__ double Bs[kMT][kMJ + 1];  // [row][rank]
  pdl_enter();  // W' comes from the preceding dequant kernel
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kMT, k0 = static_cast<int64_t>(blockIdx.x) * kMT;
  double y[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = n0 + 4 * ty + i;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t k = k0 + tx + 16 * c;
      y[i][c] = (n < N && k < K) ? static_cast<double>(__bfloat162float(W[n * K + k])) : 0.0;
    }
  }
  for (int a = 0; a < ma.n; ++a) {
    const int r = ma.r[a];
    const __nv_bfloat16* __restrict__ A = ma.A[a];
    const __nv_bfloat16* __restrict__ B = ma.B[a];
    double P[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) P[i][c] = 0.0;
    for (int j0 = 0; j0 < r; j0 += kMJ) {
      __syncthreads();  // the previous chunk has been read
      for (int e = threadIdx.x; e < kMJ * kMT; e += blockDim.x) {
        const int jj = e / kMT, kk = e % kMT;
        const int64_t j = j0 + jj, k = k0 + kk;
        As[jj][kk] = (j < r && k < K) ? static_cast<double>(__bfloat162float(A[j * K + k])) : 0.0;
        const int nn = e / kMJ, jb = e % kMJ;
        const int64_t n = n0 + nn, j2 = j0 + jb;
        Bs[nn][jb] = (n < N && j2 < r) ? static_cast<double>(__bfloat162float(B[n * r + j2])) : 0.0;
      }
      __syncthreads();
      const int jn = min(kMJ, r - j0);
      for (int jj = 0; jj < jn; ++jj) {
        double bv[4], av[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) bv[i] = Bs[4 * ty + i][jj];
#pragma unroll
        for (int c = 0; c < 4; ++c) av[c] = As[jj][tx + 16 * c];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) P[i][c] = __fma_rn(bv[i], av[c], P[i][c]);
      }
    }
    const double cc = static_cast<double>(ma.c[a]);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) y[i][c] = __dadd_rn(y[i][c], __dmul_rn(cc, P[i][c]));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = n0 + 4 * ty + i;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t k = k0 + tx + 16 * c;
      if (n < N && k < K) W[n * K + k] = __ushort_as_bfloat16(f64_to_bf16_bits(y[i][c]));
    }
  }
}

}  // namespace

cudaError_t launch_merge(const Nf4View& w, const MergeAdapter* adapters, int n_adapters, void* out,
                         const float codebook[16], int num_sms, cudaStream_t stream) {
  if (n_adapters < 0 || n_adapters > kMaxMergeAdapters) return cudaErrorInvalidValue;
  cudaError_t e = launch_dequantize(w, out, codebook, num_sms, stream);
  if (e != cudaSuccess || n_adapters == 0) return e;
  MergeArgs ma{};
  ma.n = n_adapters;
  for (int a = 0; a < n_adapters; ++a) {
    ma.A[a] = static_cast<const __nv_bfloat16*>(adapters[a].A);
    ma.B[a] = static_cast<const __nv_bfloat16*>(adapters[a].B);
    ma.r[a] = adapters[a].r;
    ma.c[a] = adapters[a].c;
  }
  const int64_t gx = (w.K + kMT - 1) / kMT, gy = (w.N + kMT - 1) / kMT;
  if (gy > 65535) return cudaErrorInvalidValue;
  return launch_pdl(k_merge, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), dim3(256), 0, stream,
                    static_cast<__nv_bfloat16*>(out), w.N, w.K, ma);
}

}  // namespace qlora
