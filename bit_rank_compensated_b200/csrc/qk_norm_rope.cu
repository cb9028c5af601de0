// Unfused output stage of the fused QKV projection: per-head RMS normalization and rotary
// embedding applied to a bf16 Y = [Q | K | V] that a plain projection has already written.
//
// "Nunchaku Lite in Diffusers", section on quantized models with structural rewrites: the
// default path normalizes Q and K (norm_q, norm_k) and applies the rotary embedding as separate
// steps after the projection; the engine's operator fuses them into the projection (K2's QKNR
// output stage). This kernel is that separate step, kept as the comparison point: it reads the
// Q and K sections back from HBM (already rounded to bf16) and writes them again.
//
// One warp per token: lane l holds columns 4l .. 4l + 3 (two rotation pairs) of every Q and K
// head of the token. The token's (cos, sin) row (16 bytes per lane) and the two weight vectors
// are loaded once and reused for all 2 x heads heads; each head is an 8-byte load per lane
// (256 coalesced bytes per warp), a warp-wide sum of squares and an 8-byte store, eight heads in
// flight at a time.
#include "common.cuh"
#include "internal.h"

namespace svdq {
namespace {

constexpr int kHeadDim = 128;
constexpr int kUnroll = 8;

__global__ void __launch_bounds__(256) qk_norm_rope_kernel(uint16_t *Y, int M, int heads, const float *norm_q,
                                                           const float *norm_k, const float *rope, float eps) {
  const int m = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  const int N = 3 * heads * kHeadDim;
  uint16_t *yrow = Y + static_cast<size_t>(m) * N + 4 * lane;
  const float4 cs = *reinterpret_cast<const float4 *>(rope + static_cast<size_t>(m) * kHeadDim + 4 * lane);
  const float4 wq = *reinterpret_cast<const float4 *>(norm_q + 4 * lane);
  const float4 wk = *reinterpret_cast<const float4 *>(norm_k + 4 * lane);
  const int nh = 2 * heads;  // Q heads then K heads
  for (int h0 = 0; h0 < nh; h0 += kUnroll) {
    uint2 raw[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j)
      if (h0 + j < nh) raw[j] = *reinterpret_cast<const uint2 *>(yrow + static_cast<size_t>(h0 + j) * kHeadDim);
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      if (h0 + j >= nh) break;
      const float4 w = (h0 + j) >= heads ? wk : wq;
      const float v[4] = {bf16_lo(raw[j].x), bf16_hi(raw[j].x), bf16_lo(raw[j].y), bf16_hi(raw[j].y)};
      float ss = fmaf(v[0], v[0], v[1] * v[1]) + fmaf(v[2], v[2], v[3] * v[3]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = __frsqrt_rn(__fadd_rn(__fmul_rn(ss, 1.0f / kHeadDim), eps));
      const float u0 = __fmul_rn(__fmul_rn(v[0], inv), w.x), u1 = __fmul_rn(__fmul_rn(v[1], inv), w.y);
      const float u2 = __fmul_rn(__fmul_rn(v[2], inv), w.z), u3 = __fmul_rn(__fmul_rn(v[3], inv), w.w);
      const uint32_t p0 = pack_bf16x2(fmaf(u0, cs.x, -__fmul_rn(u1, cs.y)), fmaf(u1, cs.x, __fmul_rn(u0, cs.y)));
      const uint32_t p1 = pack_bf16x2(fmaf(u2, cs.z, -__fmul_rn(u3, cs.w)), fmaf(u3, cs.z, __fmul_rn(u2, cs.w)));
      *reinterpret_cast<uint2 *>(yrow + static_cast<size_t>(h0 + j) * kHeadDim) = make_uint2(p0, p1);
    }
  }
}

}  // namespace

cudaError_t launch_qk_norm_rope(uint16_t *Y, int M, int heads, const float *norm_q, const float *norm_k,
                                const float *rope, float eps, cudaStream_t st) {
  const long blocks = (static_cast<long>(M) * 32 + 255) / 256;
  qk_norm_rope_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(Y, M, heads, norm_q, norm_k, rope, eps);
  return cudaGetLastError();
}

}  // namespace svdq
