// Unfused output stage of the fused QKV projection: per-head RMS normalization and rotary
// embedding applied to a bf16 Y = [Q | K | V] that a plain projection has already written.
//
// "Nunchaku Lite in Diffusers", section on quantized models with structural rewrites: the
// default path normalizes Q and K (norm_q, norm_k) and applies the rotary embedding as separate
// steps after the projection; the engine's operator fuses them into the projection (K2's QKNR
// output stage). This kernel is that separate step, kept as the comparison point: it reads the
// Q and K sections back from HBM (already rounded to bf16) and writes them again.
//
// One warp per (token, head) of the Q and K sections; lane l holds columns 4l .. 4l + 3 (two
// rotation pairs): an 8-byte load, a warp-wide sum of squares, 16 bytes of the (cos, sin) table,
// an 8-byte store. The warps of a block take consecutive heads of one token.
#include "common.cuh"
#include "internal.h"

namespace svdq {
namespace {

constexpr int kHeadDim = 128;

__global__ void __launch_bounds__(256) qk_norm_rope_kernel(uint16_t *Y, int M, int heads, const float *norm_q,
                                                           const float *norm_k, const float *rope, float eps) {
  const int warp = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int per_token = 2 * heads;  // Q heads then K heads
  if (warp >= M * per_token) return;
  const int m = warp / per_token;
  const int hk = warp % per_token;  // head index across Q and K
  const int sec = hk >= heads ? 1 : 0;
  const int N = 3 * heads * kHeadDim;
  uint16_t *yp = Y + static_cast<size_t>(m) * N + static_cast<size_t>(hk) * kHeadDim + 4 * lane;
  const uint2 raw = *reinterpret_cast<const uint2 *>(yp);
  float v[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
  float ss = fmaf(v[0], v[0], v[1] * v[1]) + fmaf(v[2], v[2], v[3] * v[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = __frsqrt_rn(__fadd_rn(__fmul_rn(ss, 1.0f / kHeadDim), eps));
  const float4 w = *reinterpret_cast<const float4 *>((sec ? norm_k : norm_q) + 4 * lane);
  const float4 cs = *reinterpret_cast<const float4 *>(rope + static_cast<size_t>(m) * kHeadDim + 4 * lane);
  const float u0 = __fmul_rn(__fmul_rn(v[0], inv), w.x), u1 = __fmul_rn(__fmul_rn(v[1], inv), w.y);
  const float u2 = __fmul_rn(__fmul_rn(v[2], inv), w.z), u3 = __fmul_rn(__fmul_rn(v[3], inv), w.w);
  const uint32_t p0 = pack_bf16x2(fmaf(u0, cs.x, -__fmul_rn(u1, cs.y)), fmaf(u1, cs.x, __fmul_rn(u0, cs.y)));
  const uint32_t p1 = pack_bf16x2(fmaf(u2, cs.z, -__fmul_rn(u3, cs.w)), fmaf(u3, cs.z, __fmul_rn(u2, cs.w)));
  *reinterpret_cast<uint2 *>(yp) = make_uint2(p0, p1);
}

}  // namespace

cudaError_t launch_qk_norm_rope(uint16_t *Y, int M, int heads, const float *norm_q, const float *norm_k,
                                const float *rope, float eps, cudaStream_t st) {
  const long warps = static_cast<long>(M) * 2 * heads;
  const long blocks = (warps * 32 + 255) / 256;
  qk_norm_rope_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(Y, M, heads, norm_q, norm_k, rope, eps);
  return cudaGetLastError();
}

}  // namespace svdq
