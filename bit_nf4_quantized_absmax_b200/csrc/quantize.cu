// Block-wise NF4 quantization with absmax scaling and double quantization of
// the absmax constants ("QLoRA vs ChatGPT", capabilities 1 and 3; "Guanaco",
// "Core Architecture & Training").
//
// Three launches (the first alone gives single-level storage):
//   k_quant_pass1  streams W once, four lanes per 64-weight block (one 32-byte
//                  load each, 1 KB contiguous per warp instruction): the absmax
//                  (packed 16-bit max of the magnitude bits), stored as fp32,
//                  the exact quotient v = w / m, the nearest code (one lookup in
//                  a 33-bin table + one compare), 4-bit packing.
//   k_quant_sums   the exact sum of the absmax constants, as integer sums of
//                  their 8-bit significands per exponent (order-independent),
//                  eight loads in flight per thread and two running bins in
//                  registers per thread.
//   k_dq_quantize  every CTA forms the mean from the 256 bin totals (the
//                  320-bit sum added across one warp), then one warp per 256
//                  constants at a time: centre on the mean, group absmax, int8
//                  codes with round-to-nearest-even. One wave of the CTAs
//                  resident at once.
#include "common.cuh"
#include "host_tables.h"
#include "kernels.h"

namespace qlora {

struct QuantBinTable {
  BinEntry bins[kBins];
};

namespace {

constexpr int kPass1Threads = 256;

// Exact sums of the absmax constants: each constant m = sig * 2^(E - 134)
// (E the biased exponent, sig its 8-bit significand) is counted as the integer
// sig in exponent bin E. The total sum_E bins[E] * 2^(E - 134) is formed in a
// 320-bit fixed-point integer with unit 2^-133 (five 64-bit limbs kept in
// registers), then rounded once to fp64 (nearest, ties to even).
__device__ __forceinline__ void acc_bin(unsigned long long (&L)[5], unsigned long long x, int E) {
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

__device__ double limbs_to_double(const unsigned long long (&L)[5]) {
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

// Codes of 16 weights of a block given m (possibly scaled by a power of two
// together with the weights) and r = RN(1/m); out[k] packs weights 8k..8k+7.
template <bool SCALED>
__device__ __forceinline__ void encode16(const uint32_t (&d)[8], float ms, float r, float wsc,
                                         const unsigned char* bins, uint32_t (&out)[2]) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint32_t word = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t bits = d[4 * k + (i >> 1)];
      float w = __uint_as_float((i & 1) ? (bits & 0xFFFF0000u) : (bits << 16));
      if (SCALED) w = __fmul_rn(w, wsc);
      // v = RN(w / m): q0 = RN(w * RN(1/m)) is within one ulp, the remainder
      // w - q0 m is exact, and one correction step rounds correctly (Markstein).
      const float q0 = __fmul_rn(w, r);
      const float res = __fmaf_rn(q0, -ms, w);
      const float v = __fmaf_rn(res, r, q0);
      // bin: low byte of RN(v * 63.5 + 1.5 * 2^23 + 64); entry = (T_j, j + 1)
      const float x = __fmaf_rn(v, kBinMul, kBinAdd);
      const uint2 e = *reinterpret_cast<const uint2*>(bins + ((__float_as_uint(x) & 0xFCu) << 1));
      // code = j + (v >= T_j) = (j + 1) - [v < T_j]; RN(v - T_j) has the sign of
      // v - T_j and is +0 when they are equal
      const float dv = __fsub_rn(v, __uint_as_float(e.x));
      const uint32_t c = e.y - __umulhi(__float_as_uint(dv), 2u);
      word += c * (1u << (4 * i));
    }
    out[k] = word;
  }
}

// Fast path of encode16: the bin and the comparison from v' = RN(w * r) with
// r = rcp.approx(m) (at most 1 ulp from 1/m), instead of the exact quotient
// v = RN(w / m). For |w| <= m, |v' - w/m| <= 2^-23 + 2^-24 and |v - w/m| <=
// 2^-24, so |v' - v| < 2^-22 and v' lies in [-1 - 2^-22, 1 + 2^-22]: the bin of
// v' is a valid entry (|round(v' * 63.5)| <= 64), and the code from v' is the
// nearest code of v whenever |v' - T| >= 2^-21 for the threshold T it is
// compared with (v and v' are then on the same side of T; the rule counts the
// thresholds at or below its input, and checks every fp32 input). Returns true
// if some weight was within 2^-21 of its threshold; the caller then codes the
// 16 weights again through the exact quotient.
constexpr float kNearEps = 4.76837158203125e-07f;  // 2^-21

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Paired fp32 arithmetic (one instruction for two IEEE single-precision
// operations, each rounded to nearest even, no flush of subnormals).
__device__ __forceinline__ void mul2_rn(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  asm("{.reg .b64 a, b, r; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5}; mul.rn.f32x2 r, a, b; mov.b64 {%0, %1}, r;}"
      : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fma2_rn(float a0, float a1, float b0, float b1, float c0, float c1, float& r0,
                                        float& r1) {
  asm("{.reg .b64 a, b, c, r; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5}; mov.b64 c, {%6, %7};"
      " fma.rn.f32x2 r, a, b, c; mov.b64 {%0, %1}, r;}"
      : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void sub2_rn(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  asm("{.reg .b64 a, b, r; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5}; sub.rn.f32x2 r, a, b; mov.b64 {%0, %1}, r;}"
      : "=f"(r0), "=f"(r1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// The fast path reads the bin table as two arrays of 4-byte entries, the
// thresholds T_j and the codes j + 1 (byte offset of bin b: 4 b, the low byte
// of x's pattern with its two low bits cleared), so each lookup of a warp
// touches each bank once. The two weights of one bf16 pair go through the
// quotient, the bin and the comparison together as one paired operation each.
__device__ __forceinline__ bool encode16_fast(const uint32_t (&d)[8], float r, const unsigned char* tbin,
                                              const unsigned char* cbin, uint32_t (&out)[2]) {
  bool near = false;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint32_t word = 0u;
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // weights 8k + 2q (low half of the pair) and 8k + 2q + 1
      const uint32_t bits = d[4 * k + q];
      float v0, v1, x0, x1, dv0, dv1;
      mul2_rn(__uint_as_float(bits << 16), __uint_as_float(bits & 0xFFFF0000u), r, r, v0, v1);
      fma2_rn(v0, v1, kBinMul, kBinMul, kBinAdd, kBinAdd, x0, x1);
      const uint32_t o0 = __float_as_uint(x0) & 0xFCu, o1 = __float_as_uint(x1) & 0xFCu;
      const float T0 = *reinterpret_cast<const float*>(tbin + o0);
      const float T1 = *reinterpret_cast<const float*>(tbin + o1);
      const uint32_t c0 = *reinterpret_cast<const uint32_t*>(cbin + o0);
      const uint32_t c1 = *reinterpret_cast<const uint32_t*>(cbin + o1);
      sub2_rn(v0, v1, T0, T1, dv0, dv1);
      near = near || (fabsf(dv0) < kNearEps) || (fabsf(dv1) < kNearEps);
      // code = j + (v >= T_j) = (j + 1) - [v < T_j]; RN(v - T_j) has the sign of
      // v - T_j and is +0 when they are equal
      word += (c0 - __umulhi(__float_as_uint(dv0), 2u)) * (1u << (8 * q));
      word += (c1 - __umulhi(__float_as_uint(dv1), 2u)) * (1u << (8 * q + 4));
    }
    out[k] = word;
  }
  return near;
}

// The exact path for the rare group of 16 weights where the fast path came
// within 2^-21 of a threshold; kept out of line so the common path keeps few
// registers.
__device__ __noinline__ uint2 encode16_exact(const uint4* __restrict__ src, bool v8, float m,
                                             const unsigned char* bins) {
  uint32_t d[8];
  if (v8) {
    ld_global_cs_v8(src, d);
  } else {
    const uint4 a = __ldcs(src), b = __ldcs(src + 1);
    d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w; d[4] = b.x; d[5] = b.y; d[6] = b.z; d[7] = b.w;
  }
  uint32_t out[2];
  encode16<false>(d, m, __frcp_rn(m), 1.0f, bins, out);
  return make_uint2(out[0], out[1]);
}

__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Four lanes per 64-weight block (16 weights each, one 32-byte load): a warp
// reads 1 KB of contiguous weights per load instruction, and every lane of a
// warp runs the same iterations (the block's four lanes share its absmax
// through two shuffles).
template <bool V8>
__device__ __forceinline__ void pass1_loop(const uint4* __restrict__ W, int64_t nblk, uint32_t* __restrict__ packed,
                                           float* __restrict__ absmax, const unsigned char* bins,
                                           const unsigned char* tbin, const unsigned char* cbin) {
  const int lane = threadIdx.x & 31;
  const int qtr = lane & 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (kPass1Threads / 4);
  int64_t blk = (static_cast<int64_t>(blockIdx.x) * kPass1Threads + threadIdx.x) >> 2;
  for (; blk - (lane >> 2) < nblk; blk += stride) {
    const bool valid = blk < nblk;
    uint32_t d[8];
    if (valid) {
      const uint4* src = W + blk * 8 + qtr * 2;
      if (V8) {
        ld_global_cs_v8(src, d);
      } else {
        const uint4 a = __ldcs(src), b = __ldcs(src + 1);
        d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w; d[4] = b.x; d[5] = b.y; d[6] = b.z; d[7] = b.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = 0u;
    }
    // absmax: packed max of |w| (the sign bits of the result are dropped), then
    // the two halves as unsigned 15-bit magnitude fields (for finite bf16, |w|
    // orders as that field)
    uint32_t mx = absmax_bf16x2(d[0], d[1]);
#pragma unroll
    for (int i = 2; i < 8; ++i) mx = absmax_bf16x2(mx, d[i]);
    mx &= 0x7FFF7FFFu;
    mx = max(mx & 0xFFFFu, mx >> 16);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m = __uint_as_float(mx << 16);  // block absmax (exact)
    if (valid) {
      if (qtr == 0) absmax[blk] = m;
      uint32_t out[2];
      if (m == 0.0f) {
        out[0] = out[1] = 0x77777777u;  // an all-zero block: every code is the exact zero
      } else {
        // Keep 1/m normal: scale w and m by a power of two (exact for bf16 values;
        // only weights whose quotient is below 2^-126 can lose bits, and those map
        // to the zero code either way).
        const bool rare = m < 5.421010862e-20f || m > 1.8446744e19f;  // outside [2^-64, 2^64]
        if (!rare) {
          if (encode16_fast(d, rcp_approx(m), tbin, cbin, out)) {  // rare: reload and code exactly
            const uint2 o = encode16_exact(W + blk * 8 + qtr * 2, V8, m, bins);
            out[0] = o.x;
            out[1] = o.y;
          }
        } else {
          const float wsc = m < 5.421010862e-20f ? 1.8446744e19f : 5.421010862e-20f;
          const float ms = m * wsc;
          encode16<true>(d, ms, __frcp_rn(ms), wsc, bins, out);
        }
      }
      *reinterpret_cast<uint2*>(packed + blk * 8 + qtr * 2) = make_uint2(out[0], out[1]);
    }
  }
}

// zero_totals (double-quantized storage only): the 256 bin totals that
// k_quant_sums adds into, cleared here by CTA 0 before that kernel starts.
__global__ void __launch_bounds__(kPass1Threads, 8)
k_quant_pass1(const uint4* __restrict__ W, bool v8, uint32_t* __restrict__ packed,
              float* __restrict__ absmax, unsigned long long* __restrict__ zero_totals, int64_t nblk,
              const __grid_constant__ QuantBinTable tab) {
  __shared__ uint2 s_bins[kBins];
  __shared__ uint32_t s_tbin[kBins], s_cbin[kBins];
  const int tid = threadIdx.x;
  if (tid < kBins) {
    s_bins[tid] = make_uint2(__float_as_uint(tab.bins[tid].threshold), tab.bins[tid].j + 1u);
    s_tbin[tid] = __float_as_uint(tab.bins[tid].threshold);
    s_cbin[tid] = tab.bins[tid].j + 1u;
  }
  __syncthreads();
  pdl_enter();
  if (zero_totals && blockIdx.x == 0) zero_totals[tid] = 0ull;  // kPass1Threads == 256 bins

  const unsigned char* bins = reinterpret_cast<const unsigned char*>(s_bins);
  const unsigned char* tbin = reinterpret_cast<const unsigned char*>(s_tbin);
  const unsigned char* cbin = reinterpret_cast<const unsigned char*>(s_cbin);
  if (v8)
    pass1_loop<true>(W, nblk, packed, absmax, bins, tbin, cbin);
  else
    pass1_loop<false>(W, nblk, packed, absmax, bins, tbin, cbin);
}

// totals[e] += the 8-bit significands of the constants with exponent bin e (a
// constant m = sig * 2^(E - 134), E = max(exponent field, 1)). Each CTA takes a
// contiguous chunk of at most 2^24 constants, so its 32-bit shared bins cannot
// overflow. A thread loads eight constants at a time (all eight loads issued
// before any is used) and adds each significand into one of two running bins
// held in registers; the constants of one weight span few binades, so the
// shared bins see an atomic only for a third exponent in a thread's share and
// once per running bin at the end; then one 64-bit global atomic per nonzero
// bin. Integer additions in any order give the same totals.
constexpr int kSumsUnroll = 8;
constexpr int kSumsChunk = kSumsUnroll * 256;  // constants per CTA per loop trip

__global__ void __launch_bounds__(256)
k_quant_sums(const float* __restrict__ absmax, int64_t nblk, int64_t per_cta,
             unsigned long long* __restrict__ totals) {
  __shared__ unsigned int s_hist[256];
  s_hist[threadIdx.x] = 0u;
  __syncthreads();
  pdl_enter();
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * per_cta;
  const int64_t b1 = b0 + per_cta < nblk ? b0 + per_cta : nblk;
  uint32_t ea = 0u, eb = 0u, sa = 0u, sb = 0u;  // running bins (bin 0 = none: E >= 1)
  for (int64_t base = b0; base < b1; base += kSumsChunk) {
    float v[kSumsUnroll];
#pragma unroll
    for (int k = 0; k < kSumsUnroll; ++k) {
      const int64_t i = base + threadIdx.x + k * 256;
      v[k] = i < b1 ? __ldg(absmax + i) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < kSumsUnroll; ++k) {
      const uint32_t u = __float_as_uint(v[k]);
      const uint32_t e = u >> 23;
      const uint32_t E = e ? e : 1u;
      const uint32_t sig = ((u >> 16) & 0x7Fu) | (e ? 0x80u : 0u);
      if (sig == 0u) continue;  // a zero constant adds nothing
      if (E == ea) {
        sa += sig;
      } else if (E == eb) {
        sb += sig;
      } else if (ea == 0u) {
        ea = E;
        sa = sig;
      } else if (eb == 0u) {
        eb = E;
        sb = sig;
      } else {
        atomicAdd(&s_hist[E], sig);
      }
    }
  }
  if (sa) atomicAdd(&s_hist[ea], sa);
  if (sb) atomicAdd(&s_hist[eb], sb);
  __syncthreads();
  const unsigned int v = s_hist[threadIdx.x];
  if (v) atomicAdd(&totals[threadIdx.x], static_cast<unsigned long long>(v));
}

// mu = fp32(RN_fp64(S) / nblk) from the exact bin totals, formed by warp 0 of
// the CTA: lane l adds bins l, l + 32, ..., l + 224 into a 320-bit partial sum,
// the partial sums are added across the warp (integer additions with carries,
// so any order gives the same bits), and lane 0 rounds the total once. CTA 0
// also stores it. nblk counts every constant the totals cover (the whole tensor
// when this call only codes one shard of its constants).
__device__ float mean_from_bins(const unsigned long long* __restrict__ totals, int64_t nblk, float* mean_out,
                                bool store) {
  __shared__ float s_mu;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    unsigned long long L[5] = {0, 0, 0, 0, 0};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const unsigned long long x = __ldcg(totals + 32 * k + lane);  // the atomics' results, from L2
      if (x) acc_bin(L, x, 32 * k + lane);  // bin 0 is always empty
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      unsigned long long carry = 0ull;
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        const unsigned long long y = __shfl_down_sync(0xffffffffu, L[j], o);
        const unsigned long long s1 = L[j] + y;
        const unsigned long long c1 = s1 < y ? 1ull : 0ull;
        const unsigned long long s2 = s1 + carry;
        const unsigned long long c2 = s2 < s1 ? 1ull : 0ull;
        L[j] = s2;
        carry = c1 + c2;
      }
    }
    if (lane == 0) {
      const double S = limbs_to_double(L);
      const float mu = __double2float_rn(__ddiv_rn(S, static_cast<double>(nblk)));
      s_mu = mu;
      if (store) *mean_out = mu;
    }
  }
  __syncthreads();
  return s_mu;
}

__global__ void __launch_bounds__(256)
k_dq_quantize(const float* __restrict__ absmax, int64_t nblk, const unsigned long long* __restrict__ totals,
              int64_t nblk_mean, float* __restrict__ mean_out, int8_t* __restrict__ q, float* __restrict__ dq_scale,
              int64_t ngrp) {
  pdl_enter();
  // the mean, formed in every CTA from the bin totals (for a row shard, after
  // the totals of all shards were added), stored by CTA 0
  const float mu = mean_from_bins(totals, nblk_mean, mean_out, blockIdx.x == 0);
  const int lane = threadIdx.x & 31;
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); g < ngrp; g += gstride) {
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
}

// Persistent grid of pass 1: exactly the CTAs that are resident at once (four
// lanes per 64-weight block), so no SM idles through a partial last wave.
int pass1_grid(int64_t nblk, int num_sms) {
  static std::atomic<int> per_sm_cache{0};  // the same on every B200; racing writers store equal values
  int per_sm = per_sm_cache.load(std::memory_order_relaxed);
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_pass1, kPass1Threads, 0) != cudaSuccess ||
        per_sm < 1)
      per_sm = 4;
    per_sm_cache.store(per_sm, std::memory_order_relaxed);
  }
  const int64_t want = (nblk * 4 + kPass1Threads - 1) / kPass1Threads;
  const int64_t cap = static_cast<int64_t>(num_sms) * per_sm;
  const int64_t g = want < cap ? (want > 0 ? want : 1) : cap;
  return static_cast<int>(g);
}

cudaError_t launch_pass1(const void* W, int64_t nblk, uint8_t* packed, float* absmax, unsigned long long* zero_totals,
                         int num_sms, cudaStream_t stream, int dtype) {
  const QuantTables& tabs = quant_tables(dtype);
  QuantBinTable tab;
  for (int i = 0; i < kBins; ++i) tab.bins[i] = tabs.bins[i];
  const bool v8 = ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(packed)) & 31u) == 0;
  return launch_pdl(k_quant_pass1, dim3(pass1_grid(nblk, num_sms)), dim3(kPass1Threads), 0, stream,
                    reinterpret_cast<const uint4*>(W), v8, reinterpret_cast<uint32_t*>(packed), absmax, zero_totals,
                    nblk, tab);
}

}  // namespace

cudaError_t launch_quantize_first(const void* W, int64_t nblk, uint8_t* packed, float* absmax_scratch,
                                  unsigned long long* totals, int num_sms, cudaStream_t stream, int dtype) {
  cudaError_t e = launch_pass1(W, nblk, packed, absmax_scratch, totals, num_sms, stream, dtype);
  if (e != cudaSuccess) return e;
  // chunks of at least one loop trip of a CTA and at most 4 CTAs per SM, at
  // most 2^24 constants each
  int64_t g = (nblk + kSumsChunk - 1) / kSumsChunk;
  if (g > 4 * num_sms) g = 4 * num_sms;
  const int64_t min_g = (nblk + (int64_t(1) << 24) - 1) >> 24;
  if (g < min_g) g = min_g;
  if (g < 1) g = 1;
  if (g > 0x7fffffff) return cudaErrorInvalidValue;
  const int64_t per_cta = (nblk + g - 1) / g;
  return launch_pdl(k_quant_sums, dim3(static_cast<unsigned>(g)), dim3(256), 0, stream,
                    static_cast<const float*>(absmax_scratch), nblk, per_cta, totals);
}

cudaError_t launch_quantize_second(const float* absmax_scratch, int64_t nblk, const unsigned long long* totals,
                                   int64_t nblk_mean, int8_t* absmax_q, float* dq_scale, float* mean,
                                   int num_sms, cudaStream_t stream) {
  const int64_t ngrp = (nblk + 255) / 256;
  // one wave of the CTAs resident at once, so that the mean is formed once per
  // resident CTA; the warps loop over the groups
  static std::atomic<int> per_sm_cache{0};  // the same on every B200; racing writers store equal values
  int per_sm = per_sm_cache.load(std::memory_order_relaxed);
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_dq_quantize, 256, 0) != cudaSuccess || per_sm < 1)
      per_sm = 4;
    per_sm_cache.store(per_sm, std::memory_order_relaxed);
  }
  int64_t dq_grid = (ngrp + 7) / 8;
  const int64_t cap = static_cast<int64_t>(per_sm) * num_sms;
  if (dq_grid > cap) dq_grid = cap;
  if (dq_grid > 0x7fffffff) return cudaErrorInvalidValue;
  return launch_pdl(k_dq_quantize, dim3(static_cast<unsigned>(dq_grid)), dim3(256), 0, stream, absmax_scratch,
                    nblk, totals, nblk_mean, mean, absmax_q, dq_scale, ngrp);
}

cudaError_t launch_quantize(const void* W, int64_t numel, uint8_t* packed, int8_t* absmax_q, float* dq_scale,
                            float* mean, float* absmax_scratch, void* totals_scratch, int num_sms,
                            cudaStream_t stream, int dtype) {
  const int64_t nblk = numel / 64;
  unsigned long long* totals = static_cast<unsigned long long*>(totals_scratch);
  // (Forming the mean once, in the CTA of k_quant_sums that adds the last
  // totals, measured slower than forming it in every CTA of k_dq_quantize:
  // 43.6 against 41.9 us for 11008x4096, its ticket and the mean's store and
  // load add round trips to the critical path.)
  cudaError_t e = launch_quantize_first(W, nblk, packed, absmax_scratch, totals, num_sms, stream, dtype);
  if (e != cudaSuccess) return e;
  return launch_quantize_second(absmax_scratch, nblk, totals, nblk, absmax_q, dq_scale, mean, num_sms, stream);
}

cudaError_t launch_quantize_single(const void* W, int64_t numel, uint8_t* packed, float* absmax, int num_sms,
                                   cudaStream_t stream, int dtype) {
  return launch_pass1(W, numel / 64, packed, absmax, nullptr, num_sms, stream, dtype);
}

}  // namespace qlora
