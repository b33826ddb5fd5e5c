// swa_codec.cuh -- the FP8 SWA row codec shared by the append kernel and the SWA replay, so that a
// replayed ring slot is byte-identical to the slot an append of the same row writes.
//
// Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, FP4 KV Cache paragraph: the SWA
// KV stays in FP8. Reading: one fp32 scale per token, s = amax / 448 (a correctly rounded fp32
// quotient); element = E4M3 round-to-nearest-even, saturating, of the fp32 quotient x / s; all
// elements 0 when s == 0.
#pragma once

#include "common.cuh"

namespace csa2 {

// One token row held by a whole warp: lane l holds channels 16 l .. 16 l + 15 in v. Returns the
// token's scale and the lane's 16 E4M3 bytes (channel 16 l + i in byte i of e). Warp-collective.
__device__ __forceinline__ float swa_quantize_row_lane(const float (&v)[16], uint32_t (&e)[4]) {
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(v[k]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  const float s = __fdiv_rn(amax, 448.0f);
  e[0] = e[1] = e[2] = e[3] = 0u;
  if (s > 0.0f) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t two = cvt_e4m3x2(__fdiv_rn(v[2 * k], s), __fdiv_rn(v[2 * k + 1], s));
      e[k >> 1] |= two << (16 * (k & 1));
    }
  }
  return s;
}

}  // namespace csa2
