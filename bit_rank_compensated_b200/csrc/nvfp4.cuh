// NVFP4 group quantizer used by the activation kernel, the unfused baseline and the weight
// packing step. Per 16 consecutive elements along K ("Nunchaku Lite in Diffusers",
// quantization_config: nvfp4, group_size 16):
//   amax  = max |v_i|
//   scale = e4m3_rn_satfinite(fp32(amax / d)),   d = fp32(6 s), s the fp32 tensor scale
//   code_i = 0 when scale == 0, else e2m1_rn_satfinite(fp32(v_i / fp32(scale * s)))
// Division means the correctly rounded fp32 quotient.
//
// Both divisions go through a reciprocal: q = x * r with r = rcp.approx(y) (at most 1 ulp from
// 1/y) satisfies |q - x/y| < 2^-21.5 |x/y|, and so does the correctly rounded quotient f. The
// code (e4m3 or e2m1, both monotone in the value) of any number in [q (1 - 2^-20), q (1 + 2^-20)]
// is therefore the code of f whenever the codes of the two ends agree; when they differ the
// group is recomputed with correctly rounded divisions (a rare case: the quotient is within
// 2^-20 of a rounding threshold).
#pragma once

#include "common.cuh"

namespace svdq {

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Packed pair of fp32 values in one 64-bit register.
struct f2 {
  uint64_t v;
};

__device__ __forceinline__ f2 mk2(float lo, float hi) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void un2(f2 a, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a.v));
}
// Element-wise a * b, each product rounded to nearest (two fp32 multiplies in one instruction).
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(a.v), "l"(b.v));
  return r;
}

// Low and high ends of the bracket around a quotient q: q (1 -/+ 2^-20).
constexpr float kBracketLo = 1.0f - 9.5367431640625e-07f;  // 1 - 2^-20
constexpr float kBracketHi = 1.0f + 9.5367431640625e-07f;  // 1 + 2^-20

__device__ __forceinline__ float absmax16(const float *v) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(v[i]), fabsf(v[i + 8]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = fmaxf(m[i], m[i + 4]);
  return fmaxf(fmaxf(m[0], m[2]), fmaxf(m[1], m[3]));
}

// e4m3 code of fp32(amax / d) for amax >= 0, d > 0, with inv_d = rcp.approx(d).
__device__ __forceinline__ uint32_t scale_code(float amax, float d, float inv_d) {
  const float q = __fmul_rn(amax, inv_d);
  uint16_t both;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(both) : "f"(__fmul_rn(q, kBracketHi)), "f"(__fmul_rn(q, kBracketLo)));
  const uint32_t lo = both & 0xFFu, hi = both >> 8;
  return lo == hi ? lo : e4m3_code(__fdiv_rn(amax, d));
}

// Quantizes v[0..15] in two phases so that callers can interleave several groups: the first
// phase has no branches; the second, needed only when the first reports `exact` (the bracket
// ends disagree for some element, which is rare), recomputes the codes with correctly rounded
// divisions. Codes: element i of the group in bits [4(i % 8), 4(i % 8) + 4) of word i / 8.
struct Group16 {
  uint32_t w0, w1, sc;
  float eff;    // sg * s
  bool exact;   // the codes must be recomputed by nvfp4_group16_exact
};

__device__ __forceinline__ Group16 nvfp4_group16_fast(const float *v, float s, float d, float inv_d) {
  Group16 g;
  const float amax = absmax16(v);
  g.sc = scale_code(amax, d, inv_d);
  const float sg = e4m3_value(g.sc);
  g.eff = __fmul_rn(sg, s);
  const float r = rcp_approx(g.eff);  // +inf when sg == 0; the codes are then forced to zero
  const f2 r2 = mk2(r, r), blo = mk2(kBracketLo, kBracketLo), bhi = mk2(kBracketHi, kBracketHi);
  float lo[16], hi[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const f2 q = mul2(mk2(v[i], v[i + 1]), r2);
    un2(mul2(q, blo), lo[i], lo[i + 1]);
    un2(mul2(q, bhi), hi[i], hi[i + 1]);
  }
  const uint32_t l0 = e2m1x8(lo), l1 = e2m1x8(lo + 8);
  const uint32_t h0 = e2m1x8(hi), h1 = e2m1x8(hi + 8);
  const bool zero = sg == 0.0f;
  g.w0 = zero ? 0u : l0;
  g.w1 = zero ? 0u : l1;
  g.exact = !zero && ((l0 != h0) | (l1 != h1));
  return g;
}

__device__ __forceinline__ void nvfp4_group16_exact(const float *v, Group16 &g) {
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], g.eff);
  g.w0 = e2m1x8(q);
  g.w1 = e2m1x8(q + 8);
}

// Both phases; writes the codes to w0, w1 and returns the e4m3 scale code.
__device__ __forceinline__ uint32_t nvfp4_group16(const float *v, float s, float d, float inv_d, uint32_t &w0,
                                                  uint32_t &w1) {
  Group16 g = nvfp4_group16_fast(v, s, d, inv_d);
  if (g.exact) nvfp4_group16_exact(v, g);
  w0 = g.w0;
  w1 = g.w1;
  return g.sc;
}

}  // namespace svdq
