// Block-wise NF4 quantization with absmax scaling and double quantization of
// the absmax constants ("QLoRA vs ChatGPT", capabilities 1 and 3; "Guanaco",
// "Core Architecture & Training").
//
// Three launches:
//   k_quant_zero   clears the 256 exponent bins and the CTA ticket.
//   k_quant_pass1  streams W once: per 64-weight block the absmax (8-lane
//                  shuffle reduction over 16-byte loads), the exact quotient
//                  v = w / m, the nearest code (one lookup in a 32-bin table + one compare),
//                  4-bit packing; it also accumulates the exact sum of the
//                  absmax constants as integer significand sums per exponent.
//                  The last CTA to finish turns that sum into the mean.
//   k_dq_quantize  one warp per 256 constants: centre on the mean, group
//                  absmax, int8 codes with round-to-nearest-even.
#include "common.cuh"
#include "host_tables.h"
#include "kernels.h"

namespace qlora {

struct QuantBinTable {
  BinEntry bins[kBins];
};

namespace {

constexpr int kPass1Threads = 256;
constexpr int kPass1Unroll = 4;

__global__ void k_quant_zero(unsigned long long* bins) {
  pdl_enter();
  const int i = threadIdx.x;
  if (i < kQuantBinWords) bins[i] = 0ull;
}

// Exact fp64 value of sum_E hist[E] * 2^(E - 134) (E = biased exponent, the
// significand sums are integers): the sum is formed in a 320-bit fixed-point
// integer with unit 2^-133 (five 64-bit limbs kept in registers), then rounded
// once to fp64 (nearest, ties to even).
__device__ double exact_sum_to_double(const unsigned long long* hist) {
  unsigned long long L[5] = {0, 0, 0, 0, 0};
  for (int E = 1; E < 256; ++E) {
    const unsigned long long x = hist[E];
    if (!x) continue;
    const int pos = E - 1;  // bit position of x's lsb
    const int li = pos >> 6, off = pos & 63;
    const unsigned long long lo = x << off;
    const unsigned long long hi = off ? (x >> (64 - off)) : 0ull;
    unsigned long long carry = 0ull;
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const unsigned long long add = (k == li) ? lo : ((k == li + 1) ? hi : 0ull);
      const unsigned long long s1 = L[k] + add;
      const unsigned long long c1 = s1 < L[k] ? 1ull : 0ull;
      const unsigned long long s2 = s1 + carry;
      const unsigned long long c2 = s2 < s1 ? 1ull : 0ull;
      L[k] = s2;
      carry = c1 + c2;
    }
  }
  // highest set bit
  int top = -1;
#pragma unroll
  for (int k = 0; k < 5; ++k)
    if (L[k]) top = k * 64 + 63 - __clzll(static_cast<long long>(L[k]));
  if (top < 0) return 0.0;
  if (top < 53) return ldexp(static_cast<double>(L[0]), -133);
  // 53-bit significand = bits [top-52, top]; guard = bit top-53; sticky = below
  const int sh = top - 52;  // >= 1
  const int w = sh >> 6, b = sh & 63;
  unsigned long long lo_w = 0ull, hi_w = 0ull;
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    if (k == w) lo_w = L[k];
    if (k == w + 1) hi_w = L[k];
  }
  unsigned long long mant = b ? ((lo_w >> b) | (hi_w << (64 - b))) : lo_w;
  mant &= (1ull << 53) - 1ull;
  const int g = sh - 1;
  const int gw = g >> 6, gb = g & 63;
  unsigned long long gword = 0ull;
  bool sticky = false;
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    if (k == gw) {
      gword = L[k];
      sticky = sticky || ((L[k] & ((1ull << gb) - 1ull)) != 0ull);
    }
    if (k < gw) sticky = sticky || (L[k] != 0ull);
  }
  const unsigned long long guard = (gword >> gb) & 1ull;
  if (guard && (sticky || (mant & 1ull))) mant += 1ull;
  int exp2 = sh - 133;
  if (mant == (1ull << 53)) {
    mant >>= 1;
    exp2 += 1;
  }
  return ldexp(static_cast<double>(mant), exp2);
}

__device__ __forceinline__ void quant_item(const uint4 d, bool valid, int lane, int64_t item,
                                           uint32_t* __restrict__ packed, float* __restrict__ absmax,
                                           const uint2* __restrict__ s_bins,
                                           unsigned int* __restrict__ s_hist) {
  float w[8];
  w[0] = bf16lo_to_f32(d.x); w[1] = bf16hi_to_f32(d.x);
  w[2] = bf16lo_to_f32(d.y); w[3] = bf16hi_to_f32(d.y);
  w[4] = bf16lo_to_f32(d.z); w[5] = bf16hi_to_f32(d.z);
  w[6] = bf16lo_to_f32(d.w); w[7] = bf16hi_to_f32(d.w);
  float a = fabsf(w[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) a = fmaxf(a, fabsf(w[i]));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
  if (!valid) return;
  const float m = a;  // block absmax (exact)
  if ((lane & 7) == 0) {
    absmax[item >> 3] = m;
    if (m > 0.0f) {
      const uint32_t u = __float_as_uint(m);
      const uint32_t e = u >> 23;
      const uint32_t mant7 = (u >> 16) & 0x7Fu;
      const uint32_t sig = e ? (mant7 | 0x80u) : mant7;
      const uint32_t E = e ? e : 1u;
      atomicAdd(&s_hist[E], sig);
    }
  }
  uint32_t word;
  if (m == 0.0f) {
    word = 0x77777777u;  // an all-zero block: every code is the exact zero
  } else {
    // Keep 1/m normal: scale w and m by a power of two (exact for bf16 values;
    // only weights whose quotient is below 2^-126 can lose bits, and those map
    // to the zero code either way).
    float ms = m;
    if (m < 5.421010862e-20f || m > 1.8446744e19f) {     // outside [2^-64, 2^64]: rare
      const float sc = m < 5.421010862e-20f ? 1.8446744e19f : 5.421010862e-20f;
      ms = m * sc;
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] *= sc;
    }
    const float r = __frcp_rn(ms);
    const unsigned char* bins = reinterpret_cast<const unsigned char*>(s_bins);
    word = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // v = RN(w / m): q0 = RN(w * RN(1/m)) is within one ulp, the remainder
      // w - q0 m is exact, and one correction step rounds correctly (Markstein).
      const float q0 = __fmul_rn(w[i], r);
      const float res = __fmaf_rn(q0, -ms, w[i]);
      const float v = __fmaf_rn(res, r, q0);
      // bin: low byte of RN(v * 127 + 1.5 * 2^23 + 128); entry = (T_j, j + 1)
      const float x = __fmaf_rn(v, kBinMul, kBinAdd);
      const uint2 e = *reinterpret_cast<const uint2*>(bins + (__float_as_uint(x) & 0xF8u));
      // code = j + (v >= T_j) = (j + 1) - [v < T_j]; RN(v - T_j) has the sign of
      // v - T_j and is +0 when they are equal
      const float d = __fsub_rn(v, __uint_as_float(e.x));
      const uint32_t c = e.y - __umulhi(__float_as_uint(d), 2u);
      word += c * (1u << (4 * i));
    }
  }
  packed[item] = word;
}

__global__ void __launch_bounds__(kPass1Threads)
k_quant_pass1(const uint4* __restrict__ W, int64_t n_items, uint32_t* __restrict__ packed,
              float* __restrict__ absmax, unsigned long long* __restrict__ gbins, float* __restrict__ mean_out,
              int64_t nblk, const __grid_constant__ QuantBinTable tab) {
  __shared__ uint2 s_bins[kBins];
  __shared__ unsigned int s_hist[256];          // per-CTA significand sums (native 32-bit atomics)
  __shared__ unsigned long long s_tot[256];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  if (tid < kBins) s_bins[tid] = make_uint2(__float_as_uint(tab.bins[tid].threshold), tab.bins[tid].j + 1u);
  s_hist[tid] = 0u;
  __syncthreads();
  pdl_enter();

  const int64_t stride = static_cast<int64_t>(gridDim.x) * kPass1Threads;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kPass1Threads + tid; base - tid < n_items;
       base += stride * kPass1Unroll) {
    uint4 d[kPass1Unroll];
#pragma unroll
    for (int u = 0; u < kPass1Unroll; ++u) {
      const int64_t it = base + u * stride;
      d[u] = (it < n_items) ? __ldcs(W + it) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPass1Unroll; ++u) {
      const int64_t it = base + u * stride;
      quant_item(d[u], it < n_items, lane, it, packed, absmax, s_bins, s_hist);
    }
  }
  __syncthreads();
  if (s_hist[tid]) atomicAdd(&gbins[tid], static_cast<unsigned long long>(s_hist[tid]));
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned long long t = atomicAdd(&gbins[256], 1ull);
    s_last = (t == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    s_tot[tid] = atomicAdd(&gbins[tid], 0ull);  // coherent read of the final bins
    __syncthreads();
    if (tid == 0) {
      const double S = exact_sum_to_double(s_tot);
      const double mu = __ddiv_rn(S, static_cast<double>(nblk));
      *mean_out = __double2float_rn(mu);
    }
  }
}

__global__ void __launch_bounds__(256)
k_dq_quantize(const float* __restrict__ absmax, int64_t nblk, const float* __restrict__ mean,
              int8_t* __restrict__ q, float* __restrict__ dq_scale, int64_t ngrp) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (g >= ngrp) return;  // whole warp leaves together
  const float mu = *mean;
  const int64_t i0 = g * 256 + lane * 8;
  float c[8];
  bool ok[8];
  if (i0 + 8 <= nblk) {
    const float4 a = *reinterpret_cast<const float4*>(absmax + i0);
    const float4 b = *reinterpret_cast<const float4*>(absmax + i0 + 4);
    const float mm[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) { c[j] = __fsub_rn(mm[j], mu); ok[j] = true; }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ok[j] = (i0 + j) < nblk;
      c[j] = ok[j] ? __fsub_rn(absmax[i0 + j], mu) : 0.0f;
    }
  }
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) s = fmaxf(s, fabsf(c[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, o));
  const float sc = __fdiv_rn(s, 127.0f);
  int8_t qq[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    int v = 0;
    if (s > 0.0f) {
      v = __float2int_rn(__fdiv_rn(c[j], sc));
      v = max(-127, min(127, v));
    }
    qq[j] = static_cast<int8_t>(v);
  }
  if (i0 + 8 <= nblk) {
    uint2 pk;
    pk.x = (uint32_t)(uint8_t)qq[0] | ((uint32_t)(uint8_t)qq[1] << 8) | ((uint32_t)(uint8_t)qq[2] << 16) |
           ((uint32_t)(uint8_t)qq[3] << 24);
    pk.y = (uint32_t)(uint8_t)qq[4] | ((uint32_t)(uint8_t)qq[5] << 8) | ((uint32_t)(uint8_t)qq[6] << 16) |
           ((uint32_t)(uint8_t)qq[7] << 24);
    *reinterpret_cast<uint2*>(q + i0) = pk;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (ok[j]) q[i0 + j] = qq[j];
  }
  if (lane == 0) dq_scale[g] = sc;
}

}  // namespace

cudaError_t launch_quantize(const void* W, int64_t numel, uint8_t* packed, int8_t* absmax_q, float* dq_scale,
                            float* mean, float* absmax_scratch, unsigned long long* bins, int num_sms,
                            cudaStream_t stream) {
  const QuantTables& tabs = quant_tables();
  QuantBinTable tab;
  for (int i = 0; i < kBins; ++i) tab.bins[i] = tabs.bins[i];
  const int64_t n_items = numel / 8;
  const int64_t nblk = numel / 64;
  const int64_t ngrp = (nblk + 255) / 256;

  cudaError_t e = launch_pdl(k_quant_zero, dim3(1), dim3(320), 0, stream, bins);
  if (e != cudaSuccess) return e;
  int64_t want = (n_items + kPass1Threads * kPass1Unroll - 1) / (kPass1Threads * kPass1Unroll);
  int64_t cap = static_cast<int64_t>(num_sms) * 8;
  int64_t g = want < cap ? (want > 0 ? want : 1) : cap;
  // A CTA sums at most 2^24 significands of 8 bits, so its 32-bit bins cannot overflow.
  const int64_t min_grid = (nblk + (int64_t(1) << 24) - 1) >> 24;
  if (g < min_grid) g = min_grid;
  const int grid = static_cast<int>(g);
  e = launch_pdl(k_quant_pass1, dim3(grid), dim3(kPass1Threads), 0, stream, reinterpret_cast<const uint4*>(W),
                 n_items, reinterpret_cast<uint32_t*>(packed), absmax_scratch, bins, mean, nblk, tab);
  if (e != cudaSuccess) return e;
  const int dq_grid = static_cast<int>((ngrp + 7) / 8);
  return launch_pdl(k_dq_quantize, dim3(dq_grid), dim3(256), 0, stream, static_cast<const float*>(absmax_scratch),
                    nblk, static_cast<const float*>(mean), absmax_q, dq_scale, ngrp);
}

}  // namespace qlora
