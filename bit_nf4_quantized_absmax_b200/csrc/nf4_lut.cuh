// In-register NF4 decode: a per-block table of the 16 bf16 values
// bf16_rn(codebook[i] * m') and a byte-permute lookup that turns four 4-bit
// codes into two bf16x2 words. Shared by the dequant kernel and by every GEMM
// that decodes weights on the fly, so all of them produce the same bits.
#pragma once

#include "common.cuh"

namespace qlora {

struct Nf4Codebook {
  float c[16];
};

// Byte tables: lo[k] holds the low bytes of entries 4k..4k+3, hi[k] their high bytes.
struct Nf4Lut {
  uint32_t lo[4];
  uint32_t hi[4];
};

// Entry i = bf16_rn(fp32(c[i] * m)), one rounding per step as the format defines.
__device__ __forceinline__ Nf4Lut make_nf4_lut(const Nf4Codebook& cb, float m) {
  uint32_t pair[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    pair[i] = pack_bf16x2(__fmul_rn(cb.c[2 * i], m), __fmul_rn(cb.c[2 * i + 1], m));
  }
  Nf4Lut t;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t.lo[k] = prmt(pair[2 * k], pair[2 * k + 1], 0x6420);
    t.hi[k] = prmt(pair[2 * k], pair[2 * k + 1], 0x7531);
  }
  return t;
}

// Decode the four codes held in nibbles 0..3 of `w` (element k in nibble k).
// out01 = {e0 (low half), e1 (high half)}, out23 = {e2, e3}.
__device__ __forceinline__ void nf4_lookup4(const Nf4Lut& t, uint32_t w, uint32_t& out01, uint32_t& out23) {
  const uint32_t s = w & 0x7777u;                                   // entry index within a half table
  const uint32_t s2 = ((w >> 1) & 0x4444u) | 0x3210u;              // which half: bit 3 of each code
  const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], s), prmt(t.lo[2], t.lo[3], s), s2);
  const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], s), prmt(t.hi[2], t.hi[3], s), s2);
  out01 = prmt(lo, hi, 0x5140);
  out23 = prmt(lo, hi, 0x7362);
}

// Decode 8 codes (one packed 32-bit word, element k in nibble k) to 4 bf16x2.
__device__ __forceinline__ void nf4_lookup8(const Nf4Lut& t, uint32_t w, uint32_t out[4]) {
  nf4_lookup4(t, w, out[0], out[1]);
  nf4_lookup4(t, w >> 16, out[2], out[3]);
}

}  // namespace qlora
