// Tile helpers shared by the two decode-shaped forward kernels (decode.cu,
// decode_res.cu): the LoRA term of a 16-row tile on the tensor cores and the
// store of the tile's Y. Lane (g, t) of a warp holds rows tile * 16 + g and
// + 8, tokens 8 m + 2 t and + 1 (the mma.sync m16n8k16 accumulator layout).
#pragma once

#include "common.cuh"

namespace qlora {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// acc[m][i] = fmaf(s, l, acc[m][i]) with l = (T B^T) for this lane's rows and
// tokens: rows of B [N, r] (bf16) are the A operand, T^T [r, M] (fp32, split into
// bf16 hi + lo) the B operand. Ranks go in chunks of 64 (32 for two token
// groups, to bound the registers) with every load of a chunk issued before its
// MMAs (one round trip to L2 per chunk). A step covers ranks j0 .. j0 + 15;
// since r % 8 == 0 its upper half is either wholly inside [0, r) or wholly
// outside (and then zero). T is read through L2 (__ldcg): the LoRA-down kernel
// wrote it.
template <int MT>
__device__ __forceinline__ void lora_tile_accumulate(float (&acc)[MT][4], int64_t tile, int lane, const float* T,
                                                     const __nv_bfloat16* Bl, int r, float s, int M, int64_t N) {
  const int g = lane >> 2, t = lane & 3;
  const int64_t na = tile * 16 + g, nb = na + 8;
  float l[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m) l[m][0] = l[m][1] = l[m][2] = l[m][3] = 0.0f;
  constexpr int kSteps = MT == 1 ? 4 : 2;  // 16-rank steps per chunk
  for (int c0 = 0; c0 < r; c0 += 16 * kSteps) {
    uint32_t bv[kSteps][4];
    float tv[kSteps][MT][4];
#pragma unroll
    for (int q = 0; q < kSteps; ++q) {
      const int j0 = c0 + 16 * q;
      const bool lo_in = j0 < r, hi_in = j0 + 8 < r;
      const __nv_bfloat16* Ba = Bl + na * r + j0 + 2 * t;
      const __nv_bfloat16* Bb = Bl + nb * r + j0 + 2 * t;
      bv[q][0] = na < N && lo_in ? *reinterpret_cast<const uint32_t*>(Ba) : 0u;
      bv[q][1] = nb < N && lo_in ? *reinterpret_cast<const uint32_t*>(Bb) : 0u;
      bv[q][2] = na < N && hi_in ? *reinterpret_cast<const uint32_t*>(Ba + 8) : 0u;
      bv[q][3] = nb < N && hi_in ? *reinterpret_cast<const uint32_t*>(Bb + 8) : 0u;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int tok = g + 8 * m;
        const float* tp = T + static_cast<int64_t>(tok) * r + j0 + 2 * t;
        const bool tin = tok < M;
        tv[q][m][0] = tin && lo_in ? __ldcg(tp) : 0.0f;
        tv[q][m][1] = tin && lo_in ? __ldcg(tp + 1) : 0.0f;
        tv[q][m][2] = tin && hi_in ? __ldcg(tp + 8) : 0.0f;
        tv[q][m][3] = tin && hi_in ? __ldcg(tp + 9) : 0.0f;
      }
    }
#pragma unroll
    for (int q = 0; q < kSteps; ++q) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        uint32_t hi[2], lo[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t x = pack_bf16x2(tv[q][m][2 * h], tv[q][m][2 * h + 1]);
          hi[h] = x;
          lo[h] = pack_bf16x2(tv[q][m][2 * h] - bf16lo_to_f32(x), tv[q][m][2 * h + 1] - bf16hi_to_f32(x));
        }
        mma_bf16_16816(l[m], bv[q][0], bv[q][1], bv[q][2], bv[q][3], hi[0], hi[1]);
        mma_bf16_16816(l[m], bv[q][0], bv[q][1], bv[q][2], bv[q][3], lo[0], lo[1]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[m][i] = __fmaf_rn(s, l[m][i], acc[m][i]);
}

// Y of this lane's rows and tokens, rounded to bf16 (tokens >= M and rows >= N
// are not stored).
template <int MT>
__device__ __forceinline__ void store_tile_y(const float (&y)[MT][4], int64_t tile, int lane, __nv_bfloat16* Y,
                                             int M, int64_t N) {
  const int g = lane >> 2, t = lane & 3;
  const int64_t na = tile * 16 + g, nb = na + 8;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const int tok0 = 8 * m + 2 * t, tok1 = tok0 + 1;
    if (na < N) {
      if (tok0 < M) Y[static_cast<int64_t>(tok0) * N + na] = __float2bfloat16_rn(y[m][0]);
      if (tok1 < M) Y[static_cast<int64_t>(tok1) * N + na] = __float2bfloat16_rn(y[m][1]);
    }
    if (nb < N) {
      if (tok0 < M) Y[static_cast<int64_t>(tok0) * N + nb] = __float2bfloat16_rn(y[m][2]);
      if (tok1 < M) Y[static_cast<int64_t>(tok1) * N + nb] = __float2bfloat16_rn(y[m][3]);
    }
  }
}

// floor(a / b) for 0 <= a < 2^53 and 1 <= b < 2^31 through one fp64 division:
// the correctly rounded quotient lies within (a / b) 2^-53 of a / b, while a
// non-integer a / b is at least 1 / b from the integers on either side, so the
// floor of the rounded quotient is exact whenever a / b < 2^21.
__device__ __forceinline__ int64_t floor_div_small(int64_t a, int64_t b) {
  return static_cast<int64_t>(floor(__ddiv_rn(static_cast<double>(a), static_cast<double>(b))));
}

}  // namespace qlora
