// The element loop of a LoRA finish job (kernels.h: LoraFinishJob), shared by
// its own kernel (lora_misc.cu) and the dequant kernel that can carry it.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace qlora {

// Element pairs i = start, start + stride, ... of the [M, rpad] outputs.
__device__ __forceinline__ void lora_finish_range(const LoraFinishJob& j, int64_t start, int64_t stride) {
  const int64_t n2 = j.M * j.rpad / 2;
  for (int64_t i = start; i < n2; i += stride) {
    const int64_t e = 2 * i;
    const int64_t m = e / j.rpad;
    const int c = static_cast<int>(e % j.rpad);
    float2 v = make_float2(0.0f, 0.0f);
    for (int p = 0; p < j.splits; ++p) {  // fixed order
      const float2 pv = reinterpret_cast<const float2*>(j.P + (static_cast<int64_t>(p) * j.M) * j.rpad)[i];
      v.x += pv.x;
      v.y += pv.y;
    }
    if (j.f32) {
      if (c < j.r) j.f32[m * j.r + c] = v.x;
      if (c + 1 < j.r) j.f32[m * j.r + c + 1] = v.y;
    }
    if (j.s_bf16) reinterpret_cast<uint32_t*>(j.s_bf16)[i] = pack_bf16x2(j.s * v.x, j.s * v.y);
    if (j.hi) {
      const uint32_t h = pack_bf16x2(v.x, v.y);
      reinterpret_cast<uint32_t*>(j.hi)[i] = h;
      reinterpret_cast<uint32_t*>(j.lo)[i] = pack_bf16x2(v.x - bf16lo_to_f32(h), v.y - bf16hi_to_f32(h));
    }
    if (j.t_src) {
      const float t0 = c < j.r ? j.t_src[m * j.r + c] : 0.0f;
      const float t1 = c + 1 < j.r ? j.t_src[m * j.r + c + 1] : 0.0f;
      const uint32_t h = pack_bf16x2(t0, t1);
      reinterpret_cast<uint32_t*>(j.t_hi)[i] = h;
      reinterpret_cast<uint32_t*>(j.t_lo)[i] = pack_bf16x2(t0 - bf16lo_to_f32(h), t1 - bf16hi_to_f32(h));
    }
  }
}

}  // namespace qlora
