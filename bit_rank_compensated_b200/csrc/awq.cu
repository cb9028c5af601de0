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
// group g's 8 bytes = {fp16 s of row g, fp16 s of row g + 8, fp16 128 + z of row g, fp16 128 + z of
// row g + 8} (128 + z is an exact fp16 integer; the GEMV needs it in that form).
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
    const int z0 = r0 < N ? zeros[static_cast<size_t>(r0) * gpr + G] : 0, z1 = r1 < N ? zeros[static_cast<size_t>(r1) * gpr + G] : 0;
    const uint32_t c0 = __half_as_ushort(__int2half_rn(128 + z0)), c1 = __half_as_ushort(__int2half_rn(128 + z1));
    *reinterpret_cast<uint2 *>(szt + static_cast<size_t>(tile) * 64 + 8 * g) =
        make_uint2(static_cast<uint32_t>(s0) | (static_cast<uint32_t>(s1) << 16), c0 | (c1 << 16));
  }
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Tensor-core GEMV, bound by reading the 4-bit weights once. Every warp streams its own tiles
// into a ring of shared-memory slots with bulk copies (the copy engine: one copy of a step's codes
// and one of its side bytes, completing on the slot's mbarrier), up to 16 tiles ahead, with no
// register held per tile in flight (one CTA of 16 warps per SM: ~147 KiB in flight; the loop finds
// every step already landed). Each lane's 16 bytes of a tile are exactly its operand-A registers.
// Per tile: an m16n8k16 bf16 MMA per k-step with the 16 weight rows of the row block as operand A
// (each code q turned into the exact bf16 integer 128 + q in registers, one LOP3 per pair) and up
// to 8 tokens as operand B (the bf16 activations, staged once per CTA in fragment order, zeros in
// the slots of tokens M .. 7 so that every lane loads its registers unconditionally); the products
// are exact and summed in fp32, and the scale and zero point are applied per group:
// acc += s (D_G - (128 + z) sum_G(x)). (Summing 128 + q instead of q costs about 2^-23 x 143 / 8 of
// the group's sum in rounding, ~2e-5 relative.)
// Work: ks consecutive warps of a CTA (ks = 1, 2, 4 or 8) share a row block, warp slice
// j = warp % ks taking groups j gps .. (j + 1) gps - 1 (gps = K/64 / ks); the slices' partial sums
// meet in shared memory (double-buffered by unit parity, one named barrier per unit) and slice 0
// adds them in slice order and writes Y. The grid is persistent: a warp group takes row blocks
// rb0, rb0 + stride, ... and each warp streams its tiles in order, across row blocks.
// A step takes GS consecutive groups of a unit (GS = 1, 2 or 4 dividing gps; their tiles are
// adjacent in memory) with one wait, one pair of copies and one ring slot of GS tiles, so that the
// loop's bookkeeping is shared.
// Every wait is bounded (about two seconds); a warp that gives up records the error, waits (again
// bounded) for the copies it still has in flight and leaves.
constexpr int kMaxWarps = 16;
constexpr uint32_t kTileSlot = 576; // 512 bytes of codes + 64 of scales and zero points

// Shared-memory loads of the main loop with the state space explicit; volatile keeps them after the
// slot's mbarrier wait, with no memory clobber so that the compiler may still schedule the other
// loads around them.
constexpr int kMaxSlots = 16;  // mbarriers reserved per warp
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ float2 lds64f(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ float half_lo(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<uint16_t>(w & 0xFFFFu)));
}
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half(static_cast<uint16_t>(w >> 16))); }

template <int SLOTS, int GS>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) awq_gemv_mma_kernel(const uint16_t *X, int M, const uint8_t *wt,
                                                                      const uint8_t *szt, const float *bias, int N,
                                                                      int K, int ks, uint16_t *Y, uint32_t *err) {
  // a ring slot: the codes of GS tiles (512 bytes each), then their side bytes (64 each)
  constexpr uint32_t kSlot = GS * kTileSlot;
  extern __shared__ __align__(16) uint32_t smem_w[];
  const int nwarps = blockDim.x >> 5;
  const int gpr = K / kAwqGroup;
  uint32_t *xb = smem_w;                                       // gpr x 32 lanes x 8 words (bf16 pairs)
  float *sxg = reinterpret_cast<float *>(smem_w + gpr * 256);  // gpr x 8 tokens
  float *red = sxg + gpr * 8;                                  // 2 x nwarps x 32 lanes x 4 partial sums
  uint64_t *bars = reinterpret_cast<uint64_t *>(red + 2 * nwarps * 128);  // nwarps x kMaxSlots
  uint8_t *rings = reinterpret_cast<uint8_t *>(bars + nwarps * kMaxSlots);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int row_blocks = (N + 15) / 16;
  const int slice = warp % ks, gps = gpr / ks, g0 = slice * gps, steps = gps / GS;
  const int stride = gridDim.x * (nwarps / ks);  // row blocks per round of the grid
  const int rb0 = blockIdx.x * (nwarps / ks) + warp / ks;
  const int units = rb0 < row_blocks ? (row_blocks - 1 - rb0) / stride + 1 : 0;

  // this warp's ring of SLOTS slots: the step consumed next sits in slot `sl` (mbarrier `bar`,
  // phase parity `ph`), and the copies that refill it (the step SLOTS ahead) go to the same slot
  // once every lane has read it
  const uint32_t ring = smem_u32(rings) + static_cast<uint32_t>(warp) * SLOTS * kSlot;
  const uint32_t ring_end = ring + SLOTS * kSlot;
  const uint32_t bar0 = smem_u32(bars + warp * kMaxSlots);
  // Word i of X (row-major, M x K/2 bf16 pairs) is word i % (K/2) of token i / (K/2); a thread
  // holds up to kXFirst of its words in registers across the rest of the ring's prologue.
  constexpr int kXFirst = 4;
  const int kw = K / 2, xwords = M * kw;
  const uint32_t *Xw = reinterpret_cast<const uint32_t *>(X);
  if (lane == 0) {
    for (int i = 0; i < SLOTS; ++i) mbar_init(bar0 + 8 * i, 1);
    fence_mbar_init();
  }
  __syncwarp();
  uint32_t sl = ring, bar = bar0, ph = 0;
  const size_t first = static_cast<size_t>(rb0) * gpr + g0;
  const size_t skip = static_cast<size_t>(stride) * gpr - gps;  // tiles between two units of this warp
  const uint8_t *pf_w = wt + first * 512;
  const uint8_t *pf_s = szt + first * 64;
  int pf_step = 0, pf_left = units * steps;
  // the refill of slot `sl` (by lane 0), then the ring position moves on
  auto issue = [&]() {
    if (pf_left > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, GS * kTileSlot);
        bulk_load(sl, pf_w, GS * 512, bar);
        bulk_load(sl + GS * 512, pf_s, GS * 64, bar);
      }
      pf_w += GS * 512;
      pf_s += GS * 64;
      if (++pf_step == steps) {
        pf_step = 0;
        pf_w += skip * 512;
        pf_s += skip * 64;
      }
      --pf_left;
    }
    if (sl + kSlot == ring_end) {
      sl = ring;
      bar = bar0;
      ph ^= 1u;
    } else {
      sl += kSlot;
      bar += 8;
    }
  };
  // Prologue. The launch may overlap the tail of the previous kernel of the stream (programmatic
  // dependent launch): the first step of the ring is requested before the dependency wait, since
  // the packed weights are a layer's constants, complete before that kernel began (the interface
  // requires it); the activations, which that kernel may produce, only after the wait. They are
  // requested before the rest of the ring: ~150 KiB of weight copies per SM queued ahead of them
  // in the memory system delayed them by about 3 us.
  issue();
  grid_dep_wait();
  grid_dep_launch();
  uint32_t xfirst[kXFirst];
#pragma unroll
  for (int j = 0; j < kXFirst; ++j) {
    const int i = threadIdx.x + j * blockDim.x;
    xfirst[j] = i < xwords ? __ldg(Xw + i) : 0u;
  }
#pragma unroll 1
  for (int p = 1; p < SLOTS; ++p) issue();
  ph = 0;  // the prologue wrapped the ring once; the first pass waits for every slot's first phase

  // Stage X in fragment order: pair w (k = 2 w) of token m goes to word (G 32 + 4 m + t) 8 + 2 s + u
  // with k = 64 G + 16 s + 8 u + 2 t (coalesced reads of the M real tokens); the slots of tokens
  // M .. 7 (lanes 4 M .. 31 of every group) are written with zeros.
  auto xb_index = [&](int i) {
    const int m = i / kw, w = i - m * kw, e = (2 * w) & 63;
    return (((2 * w) >> 6) * 32 + 4 * m + ((e & 7) >> 1)) * 8 + 2 * (e >> 4) + ((e >> 3) & 1);
  };
#pragma unroll
  for (int j = 0; j < kXFirst; ++j) {
    const int i = threadIdx.x + j * blockDim.x;
    if (i < xwords) xb[xb_index(i)] = xfirst[j];
  }
#pragma unroll 4
  for (int i = threadIdx.x + kXFirst * blockDim.x; i < xwords; i += blockDim.x) xb[xb_index(i)] = __ldg(Xw + i);
  for (int i = threadIdx.x; i < gpr * 64; i += blockDim.x)  // 16-byte quarter i: lane (i / 2) % 32
    if (((i >> 1) & 31) >= 4 * M) reinterpret_cast<uint4 *>(xb)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < gpr * 8; i += blockDim.x)   // group i / 8, token i % 8
    if ((i & 7) >= M) sxg[i] = 0.0f;
  __syncthreads();
  // sums of x over each group, per token, from the staged pairs (lanes 4 m .. 4 m + 3, all words)
  for (int i = threadIdx.x; i < gpr * M; i += blockDim.x) {
    const int m = i / gpr, G = i - m * gpr;
    const uint4 *w4 = reinterpret_cast<const uint4 *>(xb + (G * 32 + 4 * m) * 8);
    float sum = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 w = w4[j];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) sum += __uint_as_float(ws[e] << 16) + __uint_as_float(ws[e] & 0xFFFF0000u);
    }
    sxg[G * 8 + m] = sum;
  }
  __syncthreads();

  const uint32_t xg0 = smem_u32(xb + (g0 * 32 + lane) * 8);
  const uint32_t sx0 = smem_u32(sxg + g0 * 8 + 2 * t);
  int rb = rb0, consumed = 0;
  bool ok = true;
  for (int u = 0; u < units; ++u, rb += stride) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t xg = xg0, sxp = sx0;
    for (int j = 0; j < steps && ok; ++j, xg += GS * 1024, sxp += GS * 32) {
      // the step's copies have landed
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar, ph, err, KID_AWQ, 1))) {
        ok = false;
        break;
      }
      ++consumed;
      uint4 c[GS];
      uint2 sz[GS];
#pragma unroll
      for (int tt = 0; tt < GS; ++tt) {
        c[tt] = lds128(sl + tt * 512 + lane * 16);
        sz[tt] = lds64(sl + GS * 512 + tt * 64 + g * 8);
      }
      // every lane's reads of the slot are done and ordered before the copy engine refills it
      fence_proxy_async_smem();
      __syncwarp();
      issue();  // the step SLOTS ahead, into this slot; advances sl, bar, ph
#pragma unroll
      for (int tt = 0; tt < GS; ++tt) {
        const uint4 xa = lds128(xg + tt * 1024);
        const uint4 xc = lds128(xg + tt * 1024 + 16);
        const uint32_t bx[8] = {xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w};
        const uint32_t cw[4] = {c[tt].x, c[tt].y, c[tt].z, c[tt].w};
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          uint32_t a[4];
          // (128 + q_lo, 128 + q_hi) as a bf16 pair (exact): the 128 joins the zero point below
#pragma unroll
          for (int r = 0; r < 4; ++r) a[r] = ((cw[st] >> (4 * r)) & 0x000F000Fu) | 0x43004300u;
          mma_bf16_16816(d, a, bx[2 * st], bx[2 * st + 1]);
        }
        // D = sum (128 + q) x, so acc += s (D - (128 + z) sum x)
        const float s0 = half_lo(sz[tt].x), s1 = half_hi(sz[tt].x), c0 = half_lo(sz[tt].y), c1 = half_hi(sz[tt].y);
        const float2 sx = lds64f(sxp + tt * 32);
        acc[0] = fmaf(s0, fmaf(-c0, sx.x, d[0]), acc[0]);
        acc[1] = fmaf(s0, fmaf(-c0, sx.y, d[1]), acc[1]);
        acc[2] = fmaf(s1, fmaf(-c1, sx.x, d[2]), acc[2]);
        acc[3] = fmaf(s1, fmaf(-c1, sx.y, d[3]), acc[3]);
      }
    }
    // this warp's slice of the row block is done: meet the other slices, slice 0 writes (a warp
    // that lost a wait still takes part in the named barriers of its remaining units, so that the
    // other slices never wait for it there)
    float *mine = red + ((u & 1) * nwarps + warp) * 128 + lane * 4;
    if (ks > 1) {
      *reinterpret_cast<float4 *>(mine) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      asm volatile("bar.sync %0, %1;" ::"r"(1 + warp / ks), "r"(32 * ks) : "memory");
    }
    if (slice == 0 && ok) {
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
  }
  if (!ok) {
    // a lost wait: the copies issued and not consumed (the slots from `sl` on) must land before
    // the CTA's shared memory is released
    const int issued = units * steps - pf_left;
    for (int i = consumed; i < issued; ++i) {
      mbar_wait(bar, ph, nullptr, KID_AWQ, 2);
      if (sl + kSlot == ring_end) {
        sl = ring;
        bar = bar0;
        ph ^= 1u;
      } else {
        sl += kSlot;
        bar += 8;
      }
    }
  }
}

}  // namespace

// Launch shape of the GEMV for K: warps per CTA (16, or 8 where 16 warps' rings do not fit beside
// the staged activations) and tiles in flight per warp (16, 8, 4 or 2); 0 when K is too large for
// two tiles per warp.
constexpr size_t kSmemLimit = 227 * 1024;
size_t awq_fixed_smem(int K, int warps) {
  return static_cast<size_t>(K / kAwqGroup) * (1024 + 32) + 2u * warps * 512u + static_cast<size_t>(warps) * kMaxSlots * 8u;
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

int groups_per_step(int gps, int depth) {
  for (int gs : {4, 2})
    if (gps % gs == 0 && depth >= 2 * gs) return gs;
  return 1;
}

// Warps per row block (ks, dividing the groups of a row) and groups per step: the launch that
// needs the fewest rounds of tile work per warp group, where a round of ks warps costs the groups
// of its slice, and a step's fixed bookkeeping is counted as ~2/3 of a group's work.
void pick_split(int gpr, int row_blocks, int slots, int warps, int depth, int *ks_out, int *gs_out) {
  double best = 0.0;
  *ks_out = 1;
  *gs_out = groups_per_step(gpr, depth);
  for (int ks = 1; ks <= 8 && ks <= warps && gpr % ks == 0; ks *= 2) {
    const int gps = gpr / ks, gs = groups_per_step(gps, depth);
    const long groups_at_once = static_cast<long>(slots) * (warps / ks);
    const long rounds = (row_blocks + groups_at_once - 1) / groups_at_once;
    const double cost = static_cast<double>(rounds) * gps * (1.0 + 0.67 / gs);
    if (ks == 1 || cost < best) {
      best = cost;
      *ks_out = ks;
      *gs_out = gs;
    }
  }
}

template <int SLOTS, int GS>
cudaError_t launch_gemv_shape(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias,
                              int N, int K, uint16_t *Y, int warps, int ks, uint32_t *err, cudaStream_t st) {
  const size_t smem = awq_smem_bytes(M, K);
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(awq_gemv_mma_kernel<SLOTS, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return cudaErrorInvalidValue;
  const int row_blocks = (N + 15) / 16;
  const int need = (row_blocks * ks + warps - 1) / warps;
  const int blocks = need < sms ? need : sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks, 1, 1);
  cfg.blockDim = dim3(warps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, awq_gemv_mma_kernel<SLOTS, GS>, X, M, wt, szt, bias, N, K, ks, Y, err);
}

cudaError_t launch_gemv(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias, int N,
                        int K, uint16_t *Y, uint32_t *err, cudaStream_t st) {
  int warps, depth, dev = 0, sms = 0;
  awq_shape(K, &warps, &depth);
  if (warps == 0) return cudaErrorInvalidValue;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  int ks, gs;
  // one CTA per SM (the rings take most of the shared memory)
  pick_split(K / kAwqGroup, (N + 15) / 16, sms, warps, depth, &ks, &gs);
  const int slots = depth / gs;  // tiles in flight per warp stay `depth`
#define AWQ_SHAPE(S, G)                                                                   \
  if (slots == S && gs == G) return launch_gemv_shape<S, G>(X, M, wt, szt, bias, N, K, Y, warps, ks, err, st);
  AWQ_SHAPE(16, 1) AWQ_SHAPE(8, 1) AWQ_SHAPE(4, 1) AWQ_SHAPE(2, 1)
  AWQ_SHAPE(8, 2) AWQ_SHAPE(4, 2) AWQ_SHAPE(2, 2)
  AWQ_SHAPE(4, 4) AWQ_SHAPE(2, 4)
#undef AWQ_SHAPE
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
                            int K, uint16_t *Y, uint32_t *err, cudaStream_t st) {
  return launch_gemv(X, M, wt, szt, bias, N, K, Y, err, st);
}

}  // namespace svdq
