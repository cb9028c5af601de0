// NVFP4 group quantizer used by the activation kernel, the unfused baseline and the weight
// packing step. Per 16 consecutive elements along K ("Nunchaku Lite in Diffusers",
// quantization_config: nvfp4, group_size 16):
//   amax  = max |v_i|
//   scale = e4m3_rn_satfinite(fp32(amax / d)),   d = fp32(6 s), s the fp32 tensor scale
//   code_i = 0 when scale == 0, else e2m1_rn_satfinite(fp32(v_i / fp32(scale * s)))
// Division means the correctly rounded fp32 quotient.
//
// The element quotients are computed as q_i = v_i * rcp(eff) with the hardware's approximate
// reciprocal (at most 1 ulp off), so |q_i - v_i / eff| < 2^-21.5 |v_i / eff|, and the correctly
// rounded quotient f_i lies within the same bound. Their e2m1 codes can differ only if an e2m1
// rounding threshold (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) lies between q_i and f_i or equals
// f_i. Every threshold has at most two leading significand bits set, so it suffices to flag
// any |q_i| >= 0.2 within 16 ulps (>= 2^-20 relative) of a value whose low 21 significand bits
// are zero; a flagged group is redone with correctly rounded divisions. Values below 0.2 code
// as zero either way.
#pragma once

#include "common.cuh"

namespace svdq {

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// 1 when |q| may sit within 2^-20 of an e2m1 rounding threshold, else 0.
__device__ __forceinline__ uint32_t near_e2m1_threshold(float q) {
  const uint32_t u = __float_as_uint(q) & 0x7FFFFFFFu;
  return static_cast<uint32_t>(u >= 0x3E4CCCCDu) & static_cast<uint32_t>(((u + 16u) & 0x1FFFFFu) <= 32u);
}

__device__ __forceinline__ float absmax16(const float *v) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(v[i]), fabsf(v[i + 8]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = fmaxf(m[i], m[i + 4]);
  return fmaxf(fmaxf(m[0], m[2]), fmaxf(m[1], m[3]));
}

// Quantizes v[0..15]; writes the 16 codes as two 32-bit words (element i of the group in
// bits [4(i % 8), 4(i % 8) + 4) of word i / 8) and returns the e4m3 scale code.
__device__ __forceinline__ uint32_t nvfp4_group16(const float *v, float s, float d, uint32_t &w0,
                                                  uint32_t &w1) {
  const float amax = absmax16(v);
  const uint32_t sc = e4m3_code(__fdiv_rn(amax, d));
  const float sg = e4m3_value(sc);
  if (sg == 0.0f) {
    w0 = 0u;
    w1 = 0u;
    return sc;
  }
  const float eff = __fmul_rn(sg, s);
  const float r = rcp_approx(eff);
  float q[16];
  uint32_t flag = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    q[i] = __fmul_rn(v[i], r);
    flag |= near_e2m1_threshold(q[i]);
  }
  if (flag) {
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], eff);
  }
  w0 = e2m1x8(q);
  w1 = e2m1x8(q + 8);
  return sc;
}

}  // namespace svdq
