// awq_w4a16: 4-bit weights (groups of 64 input channels with an fp16 scale and a zero point)
// times 16-bit activations, for the adaptive-normalization / modulation projections.
//
// "Nunchaku Lite in Diffusers": the engine's second kernel family serves FLUX's
// adaLN_modulation layers, which are memory-bound and sensitive to precision; the page's
// quantization_config fixes int4 and group_size 64. Storage (reading of the page):
//   wq      N x K/2 bytes, element 2i of a row in the low nibble of byte i;
//   scales  N x K/64 fp16;   zeros  N x K/64 bytes (0 .. 15);
//   W_hat[n, k] = (q[n, k] - z[n, k / 64]) * s[n, k / 64].
//
// The product is a GEMV for the few tokens a modulation layer sees (M <= 8), bound by reading the
// 4-bit weights once. The GEMV streams them from a tile layout (svdq_awq_pack_weights, once per
// layer) in which a lane's 16 bytes are its operand-A registers of an m16n8k16 bf16 tensor-core
// MMA for four k-steps, so each 512-byte tile feeds four warp-wide MMAs after one LOP3 per pair of
// codes (the nibble ORed into the bit pattern of 128.0 gives the exact bf16 integer 128 + q). The
// tokens are operand B (staged once per block in fragment order); the products (128 + q) x are
// exact and summed in fp32, and the scale and zero point enter once per group of 64:
//   sum_k (q_k - z) s x_k = s (sum_k (128 + q_k) x_k - (128 + z) sum_k x_k).
// The output is rounded to bf16 once.
#include "common.cuh"
#include "internal.h"

#include <cuda_fp16.h>

namespace svdq {
namespace {

constexpr int kAwqGroup = 64;

// One thread per group of 64: round-to-nearest int4 with a zero point, decided in fp32.
__global__ void awq_quantize_kernel(const float *W, int N, int K, uint8_t *wq, uint16_t *scales, uint8_t *zeros) {
  const long gid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int gpr = K / kAwqGroup;
  if (gid >= static_cast<long>(N) * gpr) return;
  const int n = static_cast<int>(gid / gpr), g = static_cast<int>(gid % gpr);
  const float4 *src = reinterpret_cast<const float4 *>(W + static_cast<size_t>(n) * K + g * kAwqGroup);
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll 4
  for (int i = 0; i < kAwqGroup / 4; ++i) {
    const float4 v = src[i];
    mx = fmaxf(fmaxf(mx, v.x), fmaxf(fmaxf(v.y, v.z), v.w));
    mn = fminf(fminf(mn, v.x), fminf(fminf(v.y, v.z), v.w));
  }
  float range = __fsub_rn(mx, mn);
  if (range < 1e-5f) range = 1e-5f;
  const __half sh = __float2half_rn(__fdiv_rn(range, 15.0f));
  const float s = __half2float(sh);
  const float z = fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.0f), 15.0f);
  uint32_t words[8];
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    uint32_t acc = 0;
#pragma unroll
    for (int e = 0; e < 8; e += 4) {
      const float4 v = src[2 * w + e / 4];
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float q = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(vv[i], s)), z), 0.0f), 15.0f);
        acc |= static_cast<uint32_t>(q) << (4 * (e + i));
      }
    }
    words[w] = acc;
  }
  uint4 *dst = reinterpret_cast<uint4 *>(wq + static_cast<size_t>(n) * (K / 2) + g * (kAwqGroup / 2));
  dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
  dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
  scales[gid] = __half_as_ushort(sh);
  zeros[gid] = static_cast<uint8_t>(z);
}

// Weight tiles for the tensor-core GEMV. Rows are taken 16 at a time (row block rb, rows 16 rb ..
// 16 rb + 15, rows >= N zero) and K 64 at a time (group G); a tile is 512 bytes at offset
// (rb K/64 + G) 512, and lane L = 4 g + t of a warp reads its bytes 16 L .. 16 L + 15 as four
// 32-bit words, word s for the tile's k-step s (16 k each). Nibble j = 4 h + i of word s (bits
// 4 j .. 4 j + 3) holds
//     q[16 rb + g + 8 (i & 1)][64 G + 16 s + 2 t + 8 (i >> 1) + h],
// which is the operand-A fragment of an m16n8k16 bf16 MMA (register i: rows g / g + 8, columns
// 2 t, 2 t + 1 / 2 t + 8, 2 t + 9), the two halves of register i coming from nibbles i and i + 4.
// The per-(row, group) scale and zero point travel beside it: for each (rb, G) 64 bytes, lane
// group g's 8 bytes = {fp16 s of row g, fp16 s of row g + 8, z of row g, z of row g + 8, 0, 0}.
__global__ void awq_pack_kernel(const uint8_t *wq, const uint16_t *scales, const uint8_t *zeros, int N, int K,
                                uint8_t *wt, uint8_t *szt) {
  const int gpr = K / kAwqGroup;
  const long tiles = static_cast<long>((N + 15) / 16) * gpr;
  const long tid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= tiles * 32) return;
  const long tile = tid >> 5;
  const int L = static_cast<int>(tid & 31), g = L >> 2, t = L & 3;
  const int rb = static_cast<int>(tile / gpr), G = static_cast<int>(tile % gpr);
  auto code = [&](int row, int k) -> uint32_t {
    if (row >= N) return 0u;
    const uint8_t b = wq[static_cast<size_t>(row) * (K / 2) + k / 2];
    return (k & 1) ? (b >> 4) : (b & 0xFu);
  };
  uint32_t words[4];
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = j & 3, h = j >> 2;
      w |= code(16 * rb + g + 8 * (i & 1), 64 * G + 16 * st + 2 * t + 8 * (i >> 1) + h) << (4 * j);
    }
    words[st] = w;
  }
  *reinterpret_cast<uint4 *>(wt + static_cast<size_t>(tile) * 512 + 16 * L) =
      make_uint4(words[0], words[1], words[2], words[3]);
  if (t == 0) {
    const int r0 = 16 * rb + g, r1 = r0 + 8;
    const uint16_t s0 = r0 < N ? scales[static_cast<size_t>(r0) * gpr + G] : 0, s1 = r1 < N ? scales[static_cast<size_t>(r1) * gpr + G] : 0;
    const uint8_t z0 = r0 < N ? zeros[static_cast<size_t>(r0) * gpr + G] : 0, z1 = r1 < N ? zeros[static_cast<size_t>(r1) * gpr + G] : 0;
    *reinterpret_cast<uint2 *>(szt + static_cast<size_t>(tile) * 64 + 8 * g) =
        make_uint2(static_cast<uint32_t>(s0) | (static_cast<uint32_t>(s1) << 16), z0 | (static_cast<uint32_t>(z1) << 8));
  }
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Tensor-core GEMV, bound by reading the 4-bit weights once. What keeps it at the memory's
// rate is the number of bytes in flight per SM: every lane streams its own share of the tiles
// into shared memory with cp.async (16 bytes of codes per lane per tile, plus the tile's 64 bytes
// of scales and zero points from four lanes), up to 16 tiles ahead per warp, with no register held
// per tile in flight (one CTA of 16 warps per SM: ~147 KiB in flight). Each lane's 16 bytes of a
// tile are exactly its operand-A registers, so a warp only waits for its own copies.
// Per tile: an m16n8k16 bf16 MMA per k-step with the 16 weight rows of the row block as operand A
// (each code q turned into the exact bf16 integer 128 + q in registers, one LOP3 per pair) and up
// to 8 tokens as operand B (the bf16 activations, staged once per CTA in fragment order); the
// products are exact and summed in fp32, and the scale and zero point are applied per group:
// acc += s D_G - s (128 + z) sum_G(x). (Summing 128 + q instead of q costs about 2^-23 x 143 / 8 of
// the group's sum in rounding, ~2e-5 relative.)
// Work: ks consecutive warps of a CTA (ks = 1, 2, 4 or 8) share a row block, warp slice
// j = warp % ks taking groups j gps .. (j + 1) gps - 1 (gps = K/64 / ks); the slices' partial sums
// meet in shared memory (double-buffered by unit parity, one named barrier per unit) and slice 0
// adds them in slice order and writes Y. The grid is persistent: a warp group takes row blocks
// rb0, rb0 + stride, ... and each warp streams its tiles in order, across row blocks.
constexpr int kMaxWarps = 16;
constexpr uint32_t kTileSlot = 576; // 512 bytes of codes + 64 of scales and zero points

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int DEPTH>
__global__ void __launch_bounds__(kMaxWarps * 32) awq_gemv_mma_kernel(const uint16_t *X, int M, const uint8_t *wt,
                                                                      const uint8_t *szt, const float *bias, int N,
                                                                      int K, int ks, uint16_t *Y) {
  extern __shared__ __align__(16) uint32_t smem_w[];
  const int nwarps = blockDim.x >> 5;
  const int gpr = K / kAwqGroup;
  uint32_t *xb = smem_w;                                       // gpr x 32 lanes x 8 words (bf16 pairs)
  float *sxg = reinterpret_cast<float *>(smem_w + gpr * 256);  // gpr x 8 tokens
  float *red = sxg + gpr * 8;                                  // 2 x nwarps x 32 lanes x 4 partial sums
  uint8_t *rings = reinterpret_cast<uint8_t *>(red + 2 * nwarps * 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int row_blocks = (N + 15) / 16;
  const int slice = warp % ks, gps = gpr / ks, g0 = slice * gps;
  const int stride = gridDim.x * (nwarps / ks);  // row blocks per round of the grid
  const int rb0 = blockIdx.x * (nwarps / ks) + warp / ks;
  const int units = rb0 < row_blocks ? (row_blocks - 1 - rb0) / stride + 1 : 0;
  const int items = units * gps;

  // this warp's ring: tile (row block rb0 + i / gps stride, group g0 + i % gps) goes to slot i % DEPTH
  const uint32_t ring = smem_u32(rings) + static_cast<uint32_t>(warp) * DEPTH * kTileSlot;
  uint32_t pf_tile = static_cast<uint32_t>(rb0) * gpr + g0;  // tiles fit 32 bits (N K / 1024 < 2^32)
  const uint32_t wrap = static_cast<uint32_t>(stride) * gpr - gps;
  int pf_G = 0, pf_i = 0;
  auto issue = [&](int slot) {
    if (pf_i < items) {
      const uint32_t dst = ring + static_cast<uint32_t>(slot) * kTileSlot;
      cp_async16(dst + lane * 16, wt + static_cast<size_t>(pf_tile) * 512 + lane * 16);
      if (lane < 4) cp_async16(dst + 512 + lane * 16, szt + static_cast<size_t>(pf_tile) * 64 + lane * 16);
      ++pf_tile;
      if (++pf_G == gps) {
        pf_G = 0;
        pf_tile += wrap;
      }
      ++pf_i;
    }
    cp_async_commit();  // one group per tile (empty past the end), so wait_group counts tiles
  };
#pragma unroll
  for (int p = 0; p < DEPTH; ++p) issue(p);

  // Stage X in fragment order: pair w (k = 2 w) of token m goes to word (G 32 + 4 m + t) 8 + 2 s + u
  // with k = 64 G + 16 s + 8 u + 2 t. Every thread reads consecutive pairs of the M real tokens
  // (coalesced). Lane L's operand-B registers belong to token L / 4, so the lanes of tokens M .. 7
  // take zeros in registers and their slots are never written or read.
  const int kw = K / 2;
  auto xb_index = [&](int m, int w) {
    const int e = (2 * w) & 63;
    return (((2 * w) >> 6) * 32 + 4 * m + ((e & 7) >> 1)) * 8 + 2 * (e >> 4) + ((e >> 3) & 1);
  };
  for (int m = 0; m < M; ++m) {
#pragma unroll 4
    for (int w = threadIdx.x; w < kw; w += blockDim.x)
      xb[xb_index(m, w)] = __ldg(reinterpret_cast<const uint32_t *>(X + static_cast<size_t>(m) * K) + w);
  }
  __syncthreads();
  // sums of x over each group, per token, from the staged pairs (lanes 4 m .. 4 m + 3, all words)
  for (int i = threadIdx.x; i < gpr * 8; i += blockDim.x) {
    const int G = i >> 3, m = i & 7;  // tokens M .. 7: zero sums
    float sum = 0.0f;
    if (m < M) {
      const uint4 *w4 = reinterpret_cast<const uint4 *>(xb + (G * 32 + 4 * m) * 8);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 w = w4[j];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) sum += __uint_as_float(ws[e] << 16) + __uint_as_float(ws[e] & 0xFFFF0000u);
      }
    }
    sxg[i] = sum;
  }
  __syncthreads();

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int rb = rb0, G = g0, unit = 0;
  for (int i = 0; i < items; ++i) {
    const int slot = i % DEPTH;
    // this lane's copies of tile i are complete (one group per tile, DEPTH - 1 younger ones may
    // still be in flight); the warp then sees every lane's (the scale bytes come from lanes 0..3)
    cp_async_wait<DEPTH - 1>();
    __syncwarp();
    const uint32_t sl = ring + static_cast<uint32_t>(slot) * kTileSlot;
    const uint4 c = ld_shared_u32x4(sl + lane * 16);
    const uint32_t zz0 = ld_shared_u32(sl + 512 + g * 8);
    const uint32_t zz1 = ld_shared_u32(sl + 512 + g * 8 + 4);
    __syncwarp();  // every lane has read the slot before it is refilled
    issue(slot);   // the tile DEPTH ahead
    uint4 xa = make_uint4(0u, 0u, 0u, 0u), xc = xa;
    if (g < M) {
      xa = *reinterpret_cast<const uint4 *>(xb + (G * 32 + lane) * 8);
      xc = *reinterpret_cast<const uint4 *>(xb + (G * 32 + lane) * 8 + 4);
    }
    const uint32_t bx[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int st = 0; st < 4; ++st) {
      uint32_t a[4];
      // (128 + q_lo, 128 + q_hi) as a bf16 pair (exact): the 128 joins the zero point below
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = ((cw[st] >> (4 * r)) & 0x000F000Fu) | 0x43004300u;
      mma_bf16_16816(d, a, bx[2 * st], bx[2 * st + 1]);
    }
    const float s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(zz0 & 0xFFFFu)));
    const float s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(zz0 >> 16)));
    // D = sum (128 + q) x, so acc += s D - s (128 + z) sum x (s (128 + z) is exact in fp32)
    const float sz0 = s0 * static_cast<float>(128u + (zz1 & 0xFFu));
    const float sz1 = s1 * static_cast<float>(128u + ((zz1 >> 8) & 0xFFu));
    const float2 sx = *reinterpret_cast<const float2 *>(sxg + G * 8 + 2 * t);
    acc[0] = fmaf(-sz0, sx.x, fmaf(s0, d[0], acc[0]));
    acc[1] = fmaf(-sz0, sx.y, fmaf(s0, d[1], acc[1]));
    acc[2] = fmaf(-sz1, sx.x, fmaf(s1, d[2], acc[2]));
    acc[3] = fmaf(-sz1, sx.y, fmaf(s1, d[3], acc[3]));
    if (++G == g0 + gps) {
      // this warp's slice of the row block is done: meet the other slices, slice 0 writes
      float *mine = red + ((unit & 1) * nwarps + warp) * 128 + lane * 4;
      if (ks > 1) {
        *reinterpret_cast<float4 *>(mine) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        asm volatile("bar.sync %0, %1;" ::"r"(1 + warp / ks), "r"(32 * ks) : "memory");
      }
      if (slice == 0) {
        float v[4] = {acc[0], acc[1], acc[2], acc[3]};
        for (int j = 1; j < ks; ++j) {
          const float4 o = *reinterpret_cast<const float4 *>(mine + j * 128);
          v[0] += o.x;
          v[1] += o.y;
          v[2] += o.z;
          v[3] += o.w;
        }
        // rows 16 rb + g (v 0, 1) and + 8 (v 2, 3); tokens 2 t, 2 t + 1
        const int r0 = 16 * rb + g, r1 = r0 + 8, m0 = 2 * t, m1 = m0 + 1;
        const float b0 = (bias && r0 < N) ? bias[r0] : 0.0f, b1 = (bias && r1 < N) ? bias[r1] : 0.0f;
        auto put = [&](int m, int r, float x) {
          if (m < M && r < N) Y[static_cast<size_t>(m) * N + r] = static_cast<uint16_t>(pack_bf16x2(x, 0.0f) & 0xFFFFu);
        };
        put(m0, r0, v[0] + b0);
        put(m1, r0, v[1] + b0);
        put(m0, r1, v[2] + b1);
        put(m1, r1, v[3] + b1);
      }
      acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
      G = g0;
      rb += stride;
      ++unit;
    }
  }
  cp_async_wait<0>();  // no copy in flight when the CTA exits
}

}  // namespace

// Launch shape of the GEMV for K: warps per CTA (16, or 8 where 16 warps' rings do not fit beside
// the staged activations) and tiles in flight per warp (DEPTH: 16, 8, 4 or 2); 0 when K is too
// large for two tiles per warp.
constexpr size_t kSmemLimit = 227 * 1024;
size_t awq_fixed_smem(int K, int warps) {
  return static_cast<size_t>(K / kAwqGroup) * (1024 + 32) + 2u * warps * 512u;
}
void awq_shape(int K, int *warps, int *depth) {
  *warps = 0;
  *depth = 0;
  for (int w : {16, 8}) {
    for (int d : {16, 8, 4, 2}) {
      if (awq_fixed_smem(K, w) + static_cast<size_t>(w) * d * kTileSlot <= kSmemLimit) {
        *warps = w;
        *depth = d;
        return;
      }
    }
  }
}
constexpr int kMaxK = 12288;  // the documented limit (8 warps with 4 tiles in flight each fit up to it)
size_t awq_smem_bytes(int, int K) {
  int w, d;
  awq_shape(K, &w, &d);
  if (w == 0 || K > kMaxK) return kSmemLimit + 1;  // too large: the caller rejects the shape
  return awq_fixed_smem(K, w) + static_cast<size_t>(w) * d * kTileSlot;
}

namespace {

// Warps per row block: enough (ks = K/64 / groups per warp) that a grid of resident blocks has
// row blocks x ks warps of work, with ks dividing the groups of a row.
int pick_ks(int gpr, int row_blocks, int slots, int warps) {
  int ks = 1;
  while (ks < warps && ks < 8 && gpr % (2 * ks) == 0 &&
         static_cast<long>(row_blocks) * ks < static_cast<long>(slots) * warps * 2)
    ks *= 2;
  return ks;
}

template <int DEPTH>
cudaError_t launch_gemv_depth(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias,
                              int N, int K, uint16_t *Y, int warps, cudaStream_t st) {
  const size_t smem = awq_smem_bytes(M, K);
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(awq_gemv_mma_kernel<DEPTH>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, awq_gemv_mma_kernel<DEPTH>, warps * 32, smem) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || per_sm <= 0)
    return cudaErrorLaunchOutOfResources;
  const int slots = per_sm * sms;  // persistent grid: the blocks resident at once
  const int row_blocks = (N + 15) / 16;
  const int ks = pick_ks(K / kAwqGroup, row_blocks, slots, warps);
  const int need = (row_blocks * ks + warps - 1) / warps;
  const int blocks = need < slots ? need : slots;
  awq_gemv_mma_kernel<DEPTH><<<blocks, warps * 32, smem, st>>>(X, M, wt, szt, bias, N, K, ks, Y);
  return cudaGetLastError();
}

cudaError_t launch_gemv(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias, int N,
                        int K, uint16_t *Y, cudaStream_t st) {
  int warps, depth;
  awq_shape(K, &warps, &depth);
  switch (depth) {
    case 16: return launch_gemv_depth<16>(X, M, wt, szt, bias, N, K, Y, warps, st);
    case 8: return launch_gemv_depth<8>(X, M, wt, szt, bias, N, K, Y, warps, st);
    case 4: return launch_gemv_depth<4>(X, M, wt, szt, bias, N, K, Y, warps, st);
    case 2: return launch_gemv_depth<2>(X, M, wt, szt, bias, N, K, Y, warps, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

int awq_max_tokens() { return 8; }
size_t awq_packed_weight_bytes(int N, int K) { return static_cast<size_t>((N + 15) / 16) * 16 * (K / 2); }
size_t awq_packed_sz_bytes(int N, int K) { return static_cast<size_t>((N + 15) / 16) * (K / kAwqGroup) * 64; }

cudaError_t launch_awq_quantize(const float *W, int N, int K, uint8_t *wq, uint16_t *scales, uint8_t *zeros,
                                cudaStream_t st) {
  const long groups = static_cast<long>(N) * (K / kAwqGroup);
  const int threads = 128;
  awq_quantize_kernel<<<static_cast<unsigned>((groups + threads - 1) / threads), threads, 0, st>>>(W, N, K, wq, scales,
                                                                                                    zeros);
  return cudaGetLastError();
}

cudaError_t launch_awq_pack(const uint8_t *wq, const uint16_t *scales, const uint8_t *zeros, int N, int K, uint8_t *wt,
                            uint8_t *szt, cudaStream_t st) {
  const long threads_total = static_cast<long>((N + 15) / 16) * (K / kAwqGroup) * 32;
  awq_pack_kernel<<<static_cast<unsigned>((threads_total + 255) / 256), 256, 0, st>>>(wq, scales, zeros, N, K, wt, szt);
  return cudaGetLastError();
}

cudaError_t launch_awq_gemv(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias, int N,
                            int K, uint16_t *Y, uint32_t *, cudaStream_t st) {
  return launch_gemv(X, M, wt, szt, bias, N, K, Y, st);
}

}  // namespace svdq
