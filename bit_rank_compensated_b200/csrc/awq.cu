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

// Streaming tensor-core GEMV. The work is bound by reading the 4-bit weights once, so it is
// organised around keeping enough bytes in flight: one warp per CTA streams the CTA's tiles with
// bulk copies (cp.async.bulk) into a ring of shared-memory slots, each slot a run of up to 16
// consecutive groups of one row block (16 x 512 bytes of codes, 16 x 64 bytes of scales and zero
// points, contiguous in the packed layout), up to 12 slots (108 KiB) ahead; no registers are held
// per tile in flight.
// The 16 consumer warps take one group each of every run (warp w: group 16 j + w of run j of the
// row block): an m16n8k16 bf16 MMA per k-step with the 16 weight rows of the row block as operand
// A (each code q turned into the exact bf16 integer 128 + q, one LOP3 per pair) and up to 8 tokens
// as operand B (the bf16 activations, staged once per CTA in fragment order); the products are
// exact and summed in fp32, and the scale and zero point enter once per group:
// acc += s D_G - s (128 + z) sum_G(x). At the end of a row block the 16 warps' sums meet in shared
// memory and warp 0 adds them in warp order (deterministic) and writes Y. Row blocks are dealt to
// the CTAs round-robin (persistent grid, one CTA per SM at the benchmarked shapes).
constexpr int kCW = 16;                               // consumer warps
constexpr int kRunG = 16;                             // groups per run (slot)
constexpr uint32_t kSlotBytes = kRunG * (512 + 64);   // 9 KiB
constexpr int kMaxSlots = 12;
constexpr uint32_t kRedBytes = kCW * 32 * 4 * 4;      // the warps' partial sums of a row block

__global__ void __launch_bounds__((kCW + 1) * 32, 1)
    awq_gemv_stream_kernel(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias, int N,
                           int K, int nslots, uint16_t *Y, uint32_t *err) {
  extern __shared__ __align__(16) uint32_t smem_w[];
  const int gpr = K / kAwqGroup;
  uint32_t *xb = smem_w;                                       // gpr x 32 lanes x 8 words (bf16 pairs)
  float *sxg = reinterpret_cast<float *>(smem_w + gpr * 256);  // gpr x 8 tokens
  float *red = sxg + gpr * 8;                                  // kCW warps x 32 lanes x 4 partial sums
  uint8_t *ring = reinterpret_cast<uint8_t *>(red) + kRedBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring + static_cast<size_t>(nslots) * kSlotBytes);
  const uint32_t bar_full = smem_u32(bars), bar_empty = bar_full + 8 * nslots;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int row_blocks = (N + 15) / 16;
  const int runs_per_rb = (gpr + kRunG - 1) / kRunG;
  const int my_rbs = blockIdx.x < row_blocks ? (row_blocks - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;
  const int runs = my_rbs * runs_per_rb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nslots; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, kCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int c = 0; c < runs; ++c) {
        const int s = c % nslots;
        if (c >= nslots && !mbar_wait(bar_empty + 8 * s, ((c / nslots) - 1) & 1, err, KID_AWQ, 1)) break;
        const int rb = static_cast<int>(blockIdx.x) + (c / runs_per_rb) * static_cast<int>(gridDim.x);
        const int G0 = (c % runs_per_rb) * kRunG;
        const int ng = min(kRunG, gpr - G0);
        const size_t tile0 = static_cast<size_t>(rb) * gpr + G0;
        const uint32_t dst = smem_u32(ring + static_cast<size_t>(s) * kSlotBytes);
        mbar_arrive_expect_tx(bar_full + 8 * s, static_cast<uint32_t>(ng) * (512u + 64u));
        bulk_load(dst, wt + tile0 * 512, static_cast<uint32_t>(ng) * 512u, bar_full + 8 * s);
        bulk_load(dst + kRunG * 512u, szt + tile0 * 64, static_cast<uint32_t>(ng) * 64u, bar_full + 8 * s);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers (512 threads)
  // Stage X in fragment order: pair w (k = 2 w) of token m goes to word (G 32 + 4 m + t) 8 + 2 s + u
  // with k = 64 G + 16 s + 8 u + 2 t. Consecutive threads read consecutive pairs of the M real
  // tokens (coalesced); the slots of tokens M .. 7 are zero.
  const int ct = threadIdx.x, nct = kCW * 32;
  const int kw = K / 2;
  auto xb_index = [&](int m, int w) {
    const int e = (2 * w) & 63;
    return (((2 * w) >> 6) * 32 + 4 * m + ((e & 7) >> 1)) * 8 + 2 * (e >> 4) + ((e >> 3) & 1);
  };
  for (int m = 0; m < 8; ++m) {
    if (m < M) {
#pragma unroll 4
      for (int w = ct; w < kw; w += nct)
        xb[xb_index(m, w)] = __ldg(reinterpret_cast<const uint32_t *>(X + static_cast<size_t>(m) * K) + w);
    } else {
      for (int w = ct; w < kw; w += nct) xb[xb_index(m, w)] = 0u;
    }
  }
  named_bar_sync(1, nct);
  // sums of x over each group, per token, from the staged pairs (lanes 4 m .. 4 m + 3, all words)
  for (int i = ct; i < gpr * 8; i += nct) {
    const int G = i >> 3, m = i & 7;
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
  named_bar_sync(1, nct);

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  bool ok = true;
  for (int c = 0; c < runs; ++c) {
    const int s = c % nslots;
    const int j = c % runs_per_rb;
    const int G = j * kRunG + warp;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_parked(bar_full + 8 * s, (c / nslots) & 1, err, KID_AWQ, 2));
    if (ok && G < gpr) {
      const uint8_t *slot = ring + static_cast<size_t>(s) * kSlotBytes;
      const uint4 cq = ld_shared_u32x4(smem_u32(slot + warp * 512 + lane * 16));
      const uint32_t zz0 = ld_shared_u32(smem_u32(slot + kRunG * 512 + warp * 64 + g * 8));
      const uint32_t zz1 = ld_shared_u32(smem_u32(slot + kRunG * 512 + warp * 64 + g * 8 + 4));
      const uint4 xa = *reinterpret_cast<const uint4 *>(xb + (G * 32 + lane) * 8);
      const uint4 xc = *reinterpret_cast<const uint4 *>(xb + (G * 32 + lane) * 8 + 4);
      const uint32_t bx[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
      const uint32_t cw[4] = {cq.x, cq.y, cq.z, cq.w};
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
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);  // also after a failed wait: the producer's waits stay bounded
    if (j == runs_per_rb - 1) {
      // the row block is done: the warps' sums meet, warp 0 adds them in warp order and writes Y
      *reinterpret_cast<float4 *>(red + (warp * 32 + lane) * 4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      named_bar_sync(1, nct);
      if (warp == 0) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        for (int w = 0; w < kCW; ++w) {
          const float4 o = *reinterpret_cast<const float4 *>(red + (w * 32 + lane) * 4);
          v[0] += o.x;
          v[1] += o.y;
          v[2] += o.z;
          v[3] += o.w;
        }
        // rows 16 rb + g (v 0, 1) and + 8 (v 2, 3); tokens 2 t, 2 t + 1
        const int rb = static_cast<int>(blockIdx.x) + (c / runs_per_rb) * static_cast<int>(gridDim.x);
        const int r0 = 16 * rb + g, r1 = r0 + 8, m0 = 2 * t, m1 = m0 + 1;
        const float b0 = (bias && r0 < N) ? bias[r0] : 0.0f, b1 = (bias && r1 < N) ? bias[r1] : 0.0f;
        auto put = [&](int m, int r, float x) {
          if (ok && m < M && r < N) Y[static_cast<size_t>(m) * N + r] = static_cast<uint16_t>(pack_bf16x2(x, 0.0f) & 0xFFFFu);
        };
        put(m0, r0, v[0] + b0);
        put(m1, r0, v[1] + b0);
        put(m0, r1, v[2] + b1);
        put(m1, r1, v[3] + b1);
      }
      named_bar_sync(1, nct);  // red is free again
      acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
    }
  }
  // After a wait that gave up, the CTA still must not exit with bulk copies in flight into its
  // shared memory: wait (bounded) for the slots' last phases.
  if (!ok && warp == 0) {
    for (int c = runs > nslots ? runs - nslots : 0; c < runs; ++c)
      mbar_wait(bar_full + 8 * (c % nslots), (c / nslots) & 1, nullptr, KID_AWQ, 3);
  }
}

}  // namespace

size_t awq_smem_bytes(int M, int K);
int awq_slots(int K);

namespace {

cudaError_t launch_gemv_stream(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias,
                               int N, int K, uint16_t *Y, uint32_t *err, cudaStream_t st) {
  const size_t smem = awq_smem_bytes(M, K);
  const int nslots = awq_slots(K);
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(awq_gemv_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, awq_gemv_stream_kernel, (kCW + 1) * 32, smem) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || per_sm <= 0)
    return cudaErrorLaunchOutOfResources;
  const int row_blocks = (N + 15) / 16;
  const int slots = per_sm * sms;
  const int blocks = row_blocks < slots ? row_blocks : slots;
  awq_gemv_stream_kernel<<<blocks, (kCW + 1) * 32, smem, st>>>(X, M, wt, szt, bias, N, K, nslots, Y, err);
  return cudaGetLastError();
}

}  // namespace

int awq_max_tokens() { return 8; }
// Shared memory of the GEMV: staged activations (K/64 groups x 1 KiB of bf16 pairs), group sums (8
// tokens x 4 bytes per group), the warps' partial sums, the ring of weight runs (as many slots as
// fit, 12 at most, at least 2) and its barriers. The same for every token count up to 8.
constexpr size_t kSmemLimit = 227 * 1024;
size_t awq_fixed_smem(int K) { return static_cast<size_t>(K / kAwqGroup) * (1024 + 32) + kRedBytes; }
int awq_slots(int K) {
  const size_t fixed = awq_fixed_smem(K);
  if (fixed >= kSmemLimit) return 0;
  size_t n = (kSmemLimit - fixed) / (kSlotBytes + 16);
  return static_cast<int>(n > static_cast<size_t>(kMaxSlots) ? kMaxSlots : n);
}
constexpr int kMaxK = 12288;  // the documented limit (at least two slots fit up to it)
size_t awq_smem_bytes(int, int K) {
  const int n = awq_slots(K);
  if (n < 2 || K > kMaxK) return kSmemLimit + 1;  // too large: the caller rejects the shape
  return awq_fixed_smem(K) + static_cast<size_t>(n) * (kSlotBytes + 16);
}
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
                            int K, uint16_t *Y, uint32_t *err, cudaStream_t st) {
  return launch_gemv_stream(X, M, wt, szt, bias, N, K, Y, err, st);
}

}  // namespace svdq
