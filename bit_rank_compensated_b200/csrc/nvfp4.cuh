// NVFP4 group quantizer used by the activation kernel, the unfused baseline and the weight
// packing step. Per 16 consecutive elements along K ("Nunchaku Lite in Diffusers",
// quantization_config: nvfp4, group_size 16):
//   amax  = max |v_i|
//   scale = e4m3_rn_satfinite(fp32(amax / d)),   d = fp32(6 s), s the fp32 tensor scale
//   code_i = 0 when scale == 0, else e2m1_rn_satfinite(fp32(v_i / fp32(scale * s)))
// Division means the correctly rounded fp32 quotient.
//
// Both divisions go through a reciprocal r = rcp.approx(y), at most 1 ulp (relative 2^-23) from
// 1/y. For the scale: q = x * r satisfies |q - x/y| < 2^-21.5 |x/y|, and so does the correctly
// rounded quotient f, so the e4m3 code (monotone in the value) of any number in
// [q (1 - 2^-20), q (1 + 2^-20)] is the code of f whenever the codes of the two ends agree.
// For the element codes the bracket is moved onto the reciprocal: with r_lo = RN(r (1 - 2^-20))
// and r_hi = RN(r (1 + 2^-20)), r_lo < (1 - 2^-21)/y and r_hi > (1 + 2^-21)/y, hence
// |RN(x r_lo)| < |x/y| (1 - 2^-22) < |f| < |x/y| (1 + 2^-22) < |RN(x r_hi)|, and the e2m1 code of f
// is the common code of the two products whenever they agree. When the ends disagree the group
// is recomputed with correctly rounded divisions (a rare case: the quotient is within 2^-20 of
// a rounding threshold).
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

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float absmax16(const float *v) {
  float m[6];
#pragma unroll
  for (int i = 0; i < 5; ++i) m[i] = max3(fabsf(v[3 * i]), fabsf(v[3 * i + 1]), fabsf(v[3 * i + 2]));
  m[5] = fabsf(v[15]);
  return fmaxf(max3(m[0], m[1], m[2]), max3(m[3], m[4], m[5]));
}

// e4m3 code of the correctly rounded quotient fp32(amax / d). Kept out of line: it is needed only
// when the bracket ends disagree, and an inlined division gets evaluated on every group.
static __device__ __noinline__ uint32_t e4m3_code_of_quotient(float amax, float d) {
  return e4m3_code(__fdiv_rn(amax, d));
}

// e4m3 code of fp32(amax / d) for amax >= 0, d > 0, with inv_d = rcp.approx(d).
__device__ __forceinline__ uint32_t scale_code(float amax, float d, float inv_d) {
  const float q = __fmul_rn(amax, inv_d);
  uint16_t both;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(both) : "f"(__fmul_rn(q, kBracketHi)), "f"(__fmul_rn(q, kBracketLo)));
  const uint32_t lo = both & 0xFFu, hi = both >> 8;
  return lo == hi ? lo : e4m3_code_of_quotient(amax, d);
}

// Quantizes v[0..15] in two phases so that callers can interleave several groups: the first
// phase has no branches; the second, needed only when the first reports `exact` (the bracket
// ends disagree for some element, which is rare), recomputes the codes with correctly rounded
// divisions. Codes: element i of the group in bits [4(i % 8), 4(i % 8) + 4) of word i / 8.
struct Group16 {
  uint32_t w0, w1, sc;
  uint32_t d0, d1;  // raw codes of the two bracket ends XORed: non-zero nibbles mark undecided elements
  float eff;        // sg * s
  bool exact;       // some element is undecided: its code needs the correctly rounded quotient
};

__device__ __forceinline__ Group16 nvfp4_group16_fast(const float *v, float s, float d, float inv_d) {
  Group16 g;
  const float amax = absmax16(v);
  g.sc = scale_code(amax, d, inv_d);
  const float sg = e4m3_value(g.sc);
  g.eff = __fmul_rn(sg, s);
  const float r = rcp_approx(g.eff);  // +inf when sg == 0; the codes are then forced to zero
  const float rl = __fmul_rn(r, kBracketLo), rh = __fmul_rn(r, kBracketHi);
  const f2 rl2 = mk2(rl, rl), rh2 = mk2(rh, rh);
  float lo[16], hi[16];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const f2 p = mk2(v[2 * e], v[2 * e + 1]);
    un2(mul2(p, rl2), lo[2 * e], lo[2 * e + 1]);
    un2(mul2(p, rh2), hi[2 * e], hi[2 * e + 1]);
  }
  // Both ends carry the sign of v, so their raw codes agree exactly when the magnitudes do.
  const uint32_t l0 = e2m1x8_raw(lo), l1 = e2m1x8_raw(lo + 8);
  const uint32_t h0 = e2m1x8_raw(hi), h1 = e2m1x8_raw(hi + 8);
  const bool zero = sg == 0.0f;
  g.w0 = zero ? 0u : e2m1_clear_neg_zero(l0);
  g.w1 = zero ? 0u : e2m1_clear_neg_zero(l1);
  g.d0 = l0 ^ h0;
  g.d1 = l1 ^ h1;
  g.exact = !zero && ((g.d0 | g.d1) != 0u);
  return g;
}

// e2m1 code (4 bits) of one fp32 value, -0 encoded as +0.
__device__ __forceinline__ uint32_t e2m1_code1(float q) {
  uint16_t b;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}" : "=h"(b) : "f"(0.0f), "f"(q));
  const uint32_t c = b & 0xFu;
  return (c & 7u) ? c : 0u;
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
