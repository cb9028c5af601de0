// K2: block-scaled NVFP4 tensor-core GEMM whose output stage adds the low-rank up-projection
// and the bias and writes bf16 once.
//
// "Svdq Int4 Flux.1 Canny Dev" model card, "Nunchaku 引擎設計" (a)/(b): the up-projection and
// the 4-bit GEMM produce the same output, so one kernel serves both and the 16-bit output is
// written once.
//
// Persistent kernel, one CTA per SM, output tiles of 128 x 256 (rows of X x rows of W).
// Per tile the k-loop is a sequence of pipeline steps through a 3-stage shared-memory ring:
//   - rank / kc low-rank steps, kc = min(rank, 32): the hi and lo planes of lora_act
//     (128 x kc bf16 each) and an L2t tile (256 x kc bf16); bf16 tcgen05 MMAs (K = 16 each),
//     hi and lo against the same L2t tile;
//   - K / 256 4-bit steps: xq tile (128 rows x 128 bytes) and wq tile (256 x 128 bytes), both
//     with 128B swizzle; four kind::mxf4nvf4 MMAs (K = 64 each).
// All steps accumulate into one fp32 accumulator in tensor memory (128 lanes x 256 columns).
// lora_act arrives pre-divided by alpha = s_x s_w, so the output stage computes
// Y = bf16(alpha * acc + bias) for every element.
//
// Scale factors reach tensor memory without the tensor-memory copy unit: four warps (one per
// 32-lane sub-partition) read each step's 512-byte scale blocks from global memory (L2) and
// write them with tcgen05.st in the replicated layout the block-scaled MMA reads (lane i of
// every sub-partition holds rows i, i+32, i+64, i+96 of a block, one 32-bit column each).
//
// Warp roles (320 threads): warp 0 TMA producer; warp 1 tensor-memory owner and MMA issuer;
// warps 2..5 scale-factor writers; warps 6..9 output stage (warp w reaches lanes 32 (w % 4)..).
// The output stage drains the accumulator into a swizzled bf16 tile in shared memory, releases
// it to the MMA warp, and writes the tile with TMA stores (which clip the M / N edges).
#include "common.cuh"
#include "internal.h"

namespace svdq {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int STAGES = 3;
constexpr uint32_t A_BYTES = 128u * 128u;
constexpr uint32_t B_BYTES = 256u * 128u;
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KiB
constexpr uint32_t DATA_BYTES = STAGES * STAGE_BYTES;
constexpr uint32_t YST_BYTES = BM * BN * 2;          // bf16 output staging (4 boxes of 128 x 64)
constexpr uint32_t BIAS_BYTES = BN * 4;
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM = DATA_BYTES + YST_BYTES + BIAS_BYTES + BAR_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 256;  // scale columns follow the accumulator
constexpr uint32_t SF_COLS = 48;   // per stage: 4 k-blocks x (4 SFA + 8 SFB) columns
constexpr int THREADS = 320;

struct GArgs {
  const uint8_t *xs;
  const uint8_t *ws;
  const float *bias;
  uint16_t *Y;
  int M, N, K;
  int Mt, Nt;
  float alpha;
  uint32_t *err;
};

template <int RANK, bool FP4, bool ADD_Y>
__global__ void __launch_bounds__(THREADS, 1)
    k2_gemm_w4a4_lora_up(const __grid_constant__ CUtensorMap tm_xq, const __grid_constant__ CUtensorMap tm_wq,
                         const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_l2,
                         const __grid_constant__ CUtensorMap tm_y, GArgs a) {
  // Low-rank steps: kc columns of lora_act (hi and lo planes) and of L2t per step.
  constexpr int KC = RANK == 0 ? 32 : (RANK < 32 ? RANK : 32);
  constexpr int N_LORA = RANK == 0 ? 0 : RANK / KC;
  constexpr uint32_t LORA_ROW = KC * 2;  // bytes per row of a low-rank tile
  constexpr uint32_t LORA_SWZ = LORA_ROW == 64 ? 4u : 6u;
  constexpr uint32_t LORA_A_BYTES = 128u * LORA_ROW;
  constexpr uint32_t LORA_B_BYTES = 256u * LORA_ROW;
  constexpr uint32_t LORA_LO_OFF = 8192u;  // lo plane inside the A slot

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ystage = smem + DATA_BYTES;
  float *bias_s = reinterpret_cast<float *>(smem + DATA_BYTES + YST_BYTES);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + DATA_BYTES + YST_BYTES + BIAS_BYTES);
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_sffull = bar_empty + 8 * STAGES;
  const uint32_t bar_accfull = bar_sffull + 8 * STAGES;
  const uint32_t bar_accempty = bar_accfull + 8;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 3 * STAGES + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kblocks = a.K / 64;
  const int n_kt = FP4 ? (kblocks + 3) / 4 : 0;
  const int total = N_LORA + n_kt;
  const int tiles = a.Mt * a.Nt;

  auto a_tile = [&](int s) { return smem + s * STAGE_BYTES; };
  auto b_tile = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
      mbar_init(bar_sffull + 8 * s, 128);
    }
    mbar_init(bar_accfull, 1);
    mbar_init(bar_accempty, 128);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      if (FP4) {
        tma_prefetch_desc(&tm_xq);
        tma_prefetch_desc(&tm_wq);
      }
      if (RANK) {
        tma_prefetch_desc(&tm_la);
        tma_prefetch_desc(&tm_l2);
      }
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int mt = tile % a.Mt;
        const int nt = tile / a.Mt;
        for (int j = 0; j < total; ++j, ++it) {
          const int s = it % STAGES;
          if (it >= STAGES && !mbar_wait(bar_empty + 8 * s, ((it / STAGES) - 1) & 1, a.err, KID_GEMM, 1)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar_full + 8 * s;
          if (j < N_LORA) {
            mbar_arrive_expect_tx(fb, 2 * LORA_A_BYTES + LORA_B_BYTES);
            tma_load_2d(smem_u32(a_tile(s)), &tm_la, j * KC, mt * BM, fb);
            tma_load_2d(smem_u32(a_tile(s)) + LORA_LO_OFF, &tm_la, RANK + j * KC, mt * BM, fb);
            tma_load_2d(smem_u32(b_tile(s)), &tm_l2, j * KC, nt * BN, fb);
          } else {
            const int kt = j - N_LORA;
            mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
            tma_load_2d(smem_u32(a_tile(s)), &tm_xq, kt * 128, mt * BM, fb);
            tma_load_2d(smem_u32(b_tile(s)), &tm_wq, kt * 128, nt * BN, fb);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kind::mxf4nvf4: A, B e2m1 (bits 7-9, 10-12 = 1), K-major, N = 256 (bits 17-22),
      // scale type ue4m3 (bit 23 = 0), M = 128 (bits 24-28), scale ids 0, K = 64.
      const uint32_t idesc_fp4 = (1u << 7) | (1u << 10) | ((uint32_t(BN) >> 3) << 17) | ((uint32_t(BM) >> 4) << 24);
      // kind::f16: D fp32, A, B bf16, N = 256, M = 128.
      const uint32_t idesc_bf16 =
          (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t(BN) >> 3) << 17) | ((uint32_t(BM) >> 4) << 24);
      uint32_t it = 0;
      uint32_t tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tcount) {
        if (tcount > 0 && !mbar_wait(bar_accempty, (tcount - 1) & 1, a.err, KID_GEMM, 2)) break;
        tc_fence_after();
        for (int j = 0; j < total; ++j, ++it) {
          const int s = it % STAGES;
          const uint32_t par = (it / STAGES) & 1;
          if (!mbar_wait(bar_full + 8 * s, par, a.err, KID_GEMM, 3)) {
            ok = false;
            break;
          }
          if (j < N_LORA) {
            tc_fence_after();
            const uint64_t ad = umma_desc(smem_u32(a_tile(s)), 16, 8 * LORA_ROW, LORA_SWZ);
            const uint64_t ald = umma_desc(smem_u32(a_tile(s)) + LORA_LO_OFF, 16, 8 * LORA_ROW, LORA_SWZ);
            const uint64_t bd = umma_desc(smem_u32(b_tile(s)), 16, 8 * LORA_ROW, LORA_SWZ);
#pragma unroll
            for (int k = 0; k < KC / 16; ++k) {
              mma_bf16(tbase, ad + 2u * k, bd + 2u * k, idesc_bf16, (j | k) != 0 ? 1u : 0u);
              mma_bf16(tbase, ald + 2u * k, bd + 2u * k, idesc_bf16, 1u);
            }
          } else {
            if (!mbar_wait(bar_sffull + 8 * s, par, a.err, KID_GEMM, 5)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int kt = j - N_LORA;
            const int kbv = min(4, kblocks - 4 * kt);
            const uint32_t tsf = tbase + SF_COL0 + SF_COLS * s;
            const uint64_t ad = umma_desc(smem_u32(a_tile(s)), 16, 1024, 2);
            const uint64_t bd = umma_desc(smem_u32(b_tile(s)), 16, 1024, 2);
            for (int kb = 0; kb < kbv; ++kb)
              mma_nvfp4(tbase, ad + 2u * kb, bd + 2u * kb, idesc_fp4, tsf + 4 * kb, tsf + 16 + 8 * kb,
                        (j | kb) != 0 ? 1u : 0u);
          }
          tc_commit(bar_empty + 8 * s);
        }
        if (!ok) break;
        tc_commit(bar_accfull);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ scale-factor writers
    // Lane i of the warp for sub-partition q writes TMEM lane 32 q + i: per k-block the 16-byte
    // line i of the activation block (4 columns) and of the two weight blocks (8 columns).
    // The loads for step t + 1 are issued before step t is stored (two register sets).
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int my_tiles = tiles > static_cast<int>(blockIdx.x) ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int nsteps = my_tiles * total;
    auto load = [&](int step, uint32_t(&sa)[16], uint32_t(&sb)[32]) {
      const int j = step % total;
      if (j < N_LORA) return;
      const int tile = blockIdx.x + (step / total) * gridDim.x;
      const int mt = tile % a.Mt, nt = tile / a.Mt;
      const int kt = j - N_LORA;
      const int kbv = min(4, kblocks - 4 * kt);
      const uint8_t *xs_t = a.xs + (static_cast<size_t>(mt) * kblocks + 4 * kt) * 512 + lane * 16;
      const uint8_t *ws0 = a.ws + (static_cast<size_t>(2 * nt) * kblocks + 4 * kt) * 512 + lane * 16;
      const uint8_t *ws1 = ws0 + static_cast<size_t>(kblocks) * 512;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        uint4 va = make_uint4(0, 0, 0, 0), v0 = va, v1 = va;
        if (kb < kbv) {
          va = __ldg(reinterpret_cast<const uint4 *>(xs_t + kb * 512));
          v0 = __ldg(reinterpret_cast<const uint4 *>(ws0 + kb * 512));
          v1 = __ldg(reinterpret_cast<const uint4 *>(ws1 + kb * 512));
        }
        sa[4 * kb + 0] = va.x; sa[4 * kb + 1] = va.y; sa[4 * kb + 2] = va.z; sa[4 * kb + 3] = va.w;
        sb[8 * kb + 0] = v0.x; sb[8 * kb + 1] = v0.y; sb[8 * kb + 2] = v0.z; sb[8 * kb + 3] = v0.w;
        sb[8 * kb + 4] = v1.x; sb[8 * kb + 5] = v1.y; sb[8 * kb + 6] = v1.z; sb[8 * kb + 7] = v1.w;
      }
    };
    auto put = [&](int step, const uint32_t(&sa)[16], const uint32_t(&sb)[32]) -> bool {
      const int s = step % STAGES;
      if (step >= STAGES && !mbar_wait(bar_empty + 8 * s, ((step / STAGES) - 1) & 1, a.err, KID_GEMM, 6))
        return false;
      if (step % total >= N_LORA) {
        const uint32_t tsf = tbase + lane_base + SF_COL0 + SF_COLS * s;
        tmem_st16(tsf, sa);
        tmem_st32(tsf + 16, sb);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar_sffull + 8 * s);
      return true;
    };
    uint32_t sa0[16], sb0[32], sa1[16], sb1[32];
    if (nsteps > 0) load(0, sa0, sb0);
    for (int step = 0; step < nsteps; step += 2) {
      if (step + 1 < nsteps) load(step + 1, sa1, sb1);
      if (!put(step, sa0, sb0)) break;
      if (step + 1 >= nsteps) break;
      if (step + 2 < nsteps) load(step + 2, sa0, sb0);
      if (!put(step + 1, sa1, sb1)) break;
    }
  } else {
    // ------------------------------------------------------------ output stage
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int et = threadIdx.x - 192;  // 0..127
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tcount) {
      const int mt = tile % a.Mt;
      const int nt = tile / a.Mt;
      const int n0 = nt * BN;
      const int m = mt * BM + row;
      const uint32_t taddr = tbase + (static_cast<uint32_t>(quad * 32) << 16);
      if constexpr (!ADD_Y) {
        // previous tile: bias reads done (barrier) and its TMA stores finished reading ystage
        if (et == 0) bulk_wait_read0();
        named_bar_sync(1, 128);
#pragma unroll
        for (int e = et; e < BN; e += 128) bias_s[e] = (a.bias && n0 + e < a.N) ? __ldg(a.bias + n0 + e) : 0.0f;
        named_bar_sync(1, 128);
        if (!mbar_wait(bar_accfull, tcount & 1, a.err, KID_GEMM, 4)) break;
        tc_fence_after();
        // 4 boxes of 64 columns; row r of a box holds 128 bytes with 16-byte chunk c at c ^ (r % 8)
#pragma unroll 1
        for (int box = 0; box < BN / 64; ++box) {
          uint32_t r[64];
          tmem_ld32(taddr + box * 64, *reinterpret_cast<uint32_t(*)[32]>(r));
          tmem_ld32(taddr + box * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
          tmem_wait_ld();
          uint8_t *rowp = ystage + box * (BM * 128) + row * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {  // 16-byte chunk ch = columns 8 ch .. 8 ch + 7 of the box
            uint32_t p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = box * 64 + ch * 8 + 2 * e;
              p[e] = pack_bf16x2(fmaf(a.alpha, __uint_as_float(r[ch * 8 + 2 * e]), bias_s[c]),
                                 fmaf(a.alpha, __uint_as_float(r[ch * 8 + 2 * e + 1]), bias_s[c + 1]));
            }
            *reinterpret_cast<uint4 *>(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(p[0], p[1], p[2], p[3]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar_accempty);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (et == 0) {
          for (int box = 0; box < BN / 64; ++box)
            if (n0 + 64 * box < a.N) tma_store_2d(&tm_y, smem_u32(ystage + box * (BM * 128)), n0 + 64 * box, mt * BM);
          bulk_commit();
        }
      } else {
        if (!mbar_wait(bar_accfull, tcount & 1, a.err, KID_GEMM, 4)) break;
        tc_fence_after();
        // Unfused up-projection: Y = bf16(Y + alpha * acc), one 32-column chunk at a time.
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_wait_ld();
          if (c == BN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar_accempty);
          }
          const int n = n0 + c * 32;
          if (n >= a.N || m >= a.M) continue;
          uint16_t *yrow = a.Y + static_cast<size_t>(m) * a.N + n;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (n + 8 * q >= a.N) break;
            const uint4 old = *reinterpret_cast<const uint4 *>(yrow + 8 * q);
            const uint32_t w[4] = {old.x, old.y, old.z, old.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o[e] = pack_bf16x2(fmaf(a.alpha, __uint_as_float(r[8 * q + 2 * e]), bf16_lo(w[e])),
                                 fmaf(a.alpha, __uint_as_float(r[8 * q + 2 * e + 1]), bf16_hi(w[e])));
            *reinterpret_cast<uint4 *>(yrow + 8 * q) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
    if (!ADD_Y && et == 0) bulk_wait0();  // stores complete before the CTA exits
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
}

template <int RANK, bool FP4, bool ADD_Y>
cudaError_t launch_t(const GemmLaunch &g) {
  auto kern = k2_gemm_w4a4_lora_up<RANK, FP4, ADD_Y>;
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  GArgs a{g.xs, g.ws, g.bias, g.Y, g.M, g.N, g.K, (g.M + BM - 1) / BM, (g.N + BN - 1) / BN, g.alpha, g.err};
  const int tiles = a.Mt * a.Nt;
  const int grid = tiles < g.num_sms ? tiles : g.num_sms;
  kern<<<grid, THREADS, SMEM, g.stream>>>(g.tm_xq, g.tm_wq, g.tm_la, g.tm_l2, g.tm_y, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch &g) {
  if (g.fp4 && !g.add_y) {
    switch (g.rank) {
      case 0: return launch_t<0, true, false>(g);
      case 16: return launch_t<16, true, false>(g);
      case 32: return launch_t<32, true, false>(g);
      case 64: return launch_t<64, true, false>(g);
      case 128: return launch_t<128, true, false>(g);
    }
  } else if (!g.fp4 && g.add_y) {
    switch (g.rank) {
      case 16: return launch_t<16, false, true>(g);
      case 32: return launch_t<32, false, true>(g);
      case 64: return launch_t<64, false, true>(g);
      case 128: return launch_t<128, false, true>(g);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace svdq
