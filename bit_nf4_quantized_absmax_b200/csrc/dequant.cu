// Block-wise dequantization of NF4 storage to bf16 ("QLoRA vs ChatGPT",
// capability 5: weights are dequantized block by block).
//
// One thread decodes 32 weights (half a 64-weight block): it forms the block
// constant (m' = fmaf(q_b, dq_scale_g, mean) for double-quantized storage, the
// stored fp32 m_b for single-level storage), builds the block's 16-entry bf16
// table and decodes its 16 packed bytes with byte permutes.
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace qlora {
namespace {

constexpr int kDeqUnroll = 4;

template <bool V8>
__device__ __forceinline__ void dequant_unit(const uint4 nib, int64_t u, float mp, uint4* __restrict__ out,
                                             const Nf4Codebook& cb) {
  const Nf4Lut t = make_nf4_lut(cb, mp);
  uint32_t o[2][8];
  nf4_lookup8(t, nib.x, o[0] + 0);
  nf4_lookup8(t, nib.y, o[0] + 4);
  nf4_lookup8(t, nib.z, o[1] + 0);
  nf4_lookup8(t, nib.w, o[1] + 4);
  uint4* dst = out + u * 4;
  if (V8) {  // two full 32-byte sectors per thread
    st_global_cs_v8(dst, o[0]);
    st_global_cs_v8(dst + 2, o[1]);
  } else {
    __stcs(dst + 0, make_uint4(o[0][0], o[0][1], o[0][2], o[0][3]));
    __stcs(dst + 1, make_uint4(o[0][4], o[0][5], o[0][6], o[0][7]));
    __stcs(dst + 2, make_uint4(o[1][0], o[1][1], o[1][2], o[1][3]));
    __stcs(dst + 3, make_uint4(o[1][4], o[1][5], o[1][6], o[1][7]));
  }
}

// Grid-stride over 32-weight units; each thread keeps kDeqUnroll 16-byte
// loads in flight before decoding them.
template <bool V8, bool SINGLE>
__global__ void __launch_bounds__(256)
k_dequant(const uint4* __restrict__ packed, const int8_t* __restrict__ absmax_q,
          const float* __restrict__ dq_scale, const float* __restrict__ mean, const float* __restrict__ absmax,
          uint4* __restrict__ out, int64_t n_units, const __grid_constant__ Nf4Codebook cb) {
  pdl_enter();
  const float mu = SINGLE ? 0.0f : *mean;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t u0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u0 < n_units;
       u0 += stride * kDeqUnroll) {
    // issue every load of the iteration (codes and block constants) before any use
    uint4 nib[kDeqUnroll];
    int qv[kDeqUnroll];
    float sc[kDeqUnroll];
#pragma unroll
    for (int i = 0; i < kDeqUnroll; ++i) {
      const int64_t u = u0 + i * stride;
      const bool ok = u < n_units;
      nib[i] = ok ? __ldcs(packed + u) : make_uint4(0, 0, 0, 0);
      if (SINGLE) {
        qv[i] = 0;
        sc[i] = ok ? __ldg(absmax + (u >> 1)) : 0.0f;
      } else {
        qv[i] = ok ? static_cast<int>(__ldg(absmax_q + (u >> 1))) : 0;
        sc[i] = ok ? __ldg(dq_scale + (u >> 9)) : 0.0f;
      }
    }
#pragma unroll
    for (int i = 0; i < kDeqUnroll; ++i) {
      const int64_t u = u0 + i * stride;
      if (u < n_units)
        dequant_unit<V8>(nib[i], u, SINGLE ? sc[i] : __fmaf_rn(static_cast<float>(qv[i]), sc[i], mu), out, cb);
    }
  }
}

}  // namespace

cudaError_t launch_dequantize(const Nf4View& w, void* out, const float codebook[16], int num_sms,
                              cudaStream_t stream) {
  Nf4Codebook cb;
  for (int i = 0; i < 16; ++i) cb.c[i] = codebook[i];
  const int64_t n_units = w.N * w.K / 32;
  int64_t want = (n_units + 256 * kDeqUnroll - 1) / (256 * kDeqUnroll);
  int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int grid = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
  const bool v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
  const bool single = w.absmax != nullptr;
  auto kern = single ? (v8 ? k_dequant<true, true> : k_dequant<false, true>)
                     : (v8 ? k_dequant<true, false> : k_dequant<false, false>);
  return launch_pdl(kern, dim3(grid), dim3(256), 0, stream, reinterpret_cast<const uint4*>(w.packed), w.absmax_q,
                    w.dq_scale, w.mean, w.absmax, reinterpret_cast<uint4*>(out), n_units, cb);
}

}  // namespace qlora
