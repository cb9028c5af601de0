// NVFP4 group quantizer used by the activation kernel, the unfused baseline and the weight
// packing step. Per 16 consecutive elements along K ("Nunchaku Lite in Diffusers",
// quantization_config: nvfp4, group_size 16):
//   amax  = max |v_i|
//   scale = e4m3_rn_satfinite(fp32(amax / d)),   d = fp32(6 s), s the fp32 tensor scale
//   code_i = 0 when scale == 0, else e2m1_rn_satfinite(fp32(v_i / fp32(scale * s)))
// Division is the correctly rounded fp32 quotient.
#pragma once

#include "common.cuh"

namespace svdq {

// Quantizes v[0..15]; writes the 16 codes as two 32-bit words (element i of the group in
// bits [4(i % 8), 4(i % 8) + 4) of word i / 8) and returns the e4m3 scale code.
__device__ __forceinline__ uint32_t nvfp4_group16(const float *v, float s, float d, uint32_t &w0,
                                                  uint32_t &w1) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sc = e4m3_code(__fdiv_rn(amax, d));
  const float sg = e4m3_value(sc);
  if (sg == 0.0f) {
    w0 = 0u;
    w1 = 0u;
    return sc;
  }
  const float eff = __fmul_rn(sg, s);
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], eff);
  w0 = e2m1x8(q);
  w1 = e2m1x8(q + 8);
  return sc;
}

}  // namespace svdq
