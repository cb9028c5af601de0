// K1: smoothing + NVFP4 activation quantization + low-rank down-projection in one read of X.
//
// "Svdq Int4 Flux.1 Canny Dev" model card, "Nunchaku 引擎設計" (b): the down-projection and
// the quantizer consume the same input, so one kernel serves both. The smoothing is folded
// into the stored factor (L1s = diag(lambda)^-1 L1, prepared offline), so the tensor cores
// read the bf16 X tile exactly as TMA delivered it and only the quantizer computes
// X_hat = fp32(X * inv_lambda).
//
// Work decomposition: a CTA owns a tile of kQuantRows (64) rows and a contiguous range of
// 64-column chunks of K, taken four chunks (32 KB of X) per pipeline stage. The row tiles cover
// the activation scale buffer's padded rows (a multiple of 128), so the padding scales are
// written as zero. The CTAs that share a row tile form a thread-block cluster along K (sized
// so that the grid fits the GPU in one wave; 64-row tiles let two-CTA clusters fill it for
// the common shapes, which clusters of three or four cannot); their fp32 partial
// down-projections are summed through distributed shared memory in cluster-rank order, so
// the result is deterministic and nothing goes through global scratch memory.
//
// The down-projection is stored pre-divided by alpha = s_x s_w as an unevaluated sum of two
// bf16 values (hi + lo), so the fp32 result reaches K2 without a 16-bit rounding.
//
// Warp roles (576 threads, 704 where the reduction has warps of its own):
//   warp 0       TMA producer: per chunk of a stage the X tile (rows x 64 bf16, 128B swizzle),
//                the L1s tile (rank x 64 bf16, 128B swizzle) and the chunk's inv_lambda values.
//   warp 1       owns the tensor-memory accumulator (rows x rank fp32) and issues the bf16
//                tcgen05 MMAs (M = rows)  acc += X chunk * L1s chunk  straight from the X tile.
//   warps 2..17  quantizers. With W = rows / 16 warps per chunk, warp 2 + W u + t handles chunk
//                u of the stage, rows 16t .. 16t + 15; lane l takes the 16-column group l / 8 of
//                rows 16t + l % 8 and 16t + 8 + l % 8.
//                Each quarter-warp reads eight consecutive rows of one group (conflict-free
//                under the 128B swizzle) and one broadcast copy of the group's 16 inv_lambda
//                values, which serve both of the lane's rows.
//   warps 18..21 (ranks up to 64) split-K reduction: one warp per tensor-memory quadrant reads
//                its accumulator rows once the last MMAs are committed, sends the partials of
//                rows another CTA owns with st.async, sums its own rows and stores lora_act,
//                while the quantizers are still on their last stages.
#include "common.cuh"
#include "internal.h"
#include "nvfp4.cuh"

namespace svdq {
namespace {

template <int RANK, bool QUANT>
struct QCfg {
  static constexpr int ROWS = kQuantRows;
  static constexpr int QWARPS = 16;
  static constexpr int WARPS_PER_CHUNK = ROWS / 16;
  static constexpr int SUB = QWARPS / WARPS_PER_CHUNK;  // 64-column chunks per stage
  static constexpr uint32_t X_BYTES = ROWS * 128u;  // per chunk
  static constexpr uint32_t L1_BYTES = RANK * 128u;
  static constexpr uint32_t IL_BYTES = QUANT ? 64u * 4u : 0u;
  // stage: X[SUB] | L1s[SUB] | inv_lambda[SUB x 64]
  static constexpr uint32_t STAGE_BYTES = (SUB * (X_BYTES + L1_BYTES + IL_BYTES) + 1023u) & ~1023u;
  static constexpr uint32_t STAGE_BUDGET = 200u * 1024u;
  static constexpr int STAGES = (STAGE_BUDGET / STAGE_BYTES) > 6 ? 6 : static_cast<int>(STAGE_BUDGET / STAGE_BYTES);
  // split-K slots: nsplit x ceil(ROWS / nsplit) <= ROWS + 7 rows of RANK fp32, row stride RANK + 4
  // (16-byte accesses spread over banks)
  static constexpr uint32_t RED_STRIDE = RANK + 4;
  static constexpr uint32_t RED_BYTES = RED_STRIDE * (ROWS + 8) * 4u;
  static constexpr uint32_t BAR_BYTES = 256;
  // Where the split-K slots fit beside the stages, they get a region of their own and four more
  // warps (one per tensor-memory quadrant) reduce as soon as the accumulator is complete, while
  // the quantizers finish their last stages; otherwise (rank 128) the slots reuse the stage
  // memory once it is idle and the quantizer warps reduce.
  static constexpr uint32_t STAGE_TOTAL = STAGES * STAGE_BYTES;
  static constexpr bool RED_SEPARATE = RANK > 0 && STAGE_TOTAL + RED_BYTES + BAR_BYTES + 1024u <= 232448u;
  static constexpr int RED_WARPS = RED_SEPARATE ? 4 : 0;
  static constexpr int RED_WARP0 = 2 + QWARPS;
  static constexpr int THREADS = 64 + 32 * QWARPS + 32 * RED_WARPS;
  static constexpr uint32_t RED_OFF = RED_SEPARATE ? STAGE_TOTAL : 0u;
  static constexpr uint32_t DATA_BYTES =
      RED_SEPARATE ? STAGE_TOTAL + RED_BYTES : (STAGE_TOTAL > RED_BYTES ? STAGE_TOTAL : RED_BYTES);
  static constexpr uint32_t SMEM = DATA_BYTES + BAR_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = RANK <= 32 ? 32u : static_cast<uint32_t>(RANK);
  // arrivals that free a stage: one per quantizer warp, one MMA commit
  static constexpr uint32_t EMPTY_COUNT = (QUANT ? QWARPS : 0) + (RANK ? 1 : 0);
  static_assert(ROWS == 64 || ROWS == 128, "tensor-core M");
  static_assert(RED_OFF % 1024 == 0, "reduction slots start on a stage boundary");
  static_assert(STAGES >= 2, "pipeline needs two stages");
  static_assert(2 * STAGES + 3 <= static_cast<int>(BAR_BYTES / 8), "barrier area");
};

struct QArgs {
  const float *inv_lambda;
  uint8_t *xq;
  uint8_t *xs;
  uint16_t *lora_act;
  int M, K;
  float s_x, d_x, inv_d, inv_alpha;
  int chunks_per_split;
  uint32_t *err;
};

// Settles the undecided elements of one group (the non-zero nibbles of d0 / d1, where the two
// bracket ends gave different codes) with the correctly rounded quotient X_hat / eff, recomputed
// from the stage buffers (x0, x1: the group's two 16-byte pieces of X; il: its 16 inv_lambda
// values). Out of line so that the compiler keeps this rare path off the common one.
__device__ __noinline__ uint2 group_codes_settle(uint32_t x0, uint32_t x1, uint32_t il, float eff, uint32_t w0,
                                                 uint32_t w1, uint32_t d0, uint32_t d1) {
  uint32_t w[2] = {w0, w1};
  const uint32_t dd[2] = {d0, d1};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t m = dd[j];
    while (m) {
      const int nib = (__ffs(m) - 1) >> 2;
      const float x = __uint_as_float(ld_shared_u16((j ? x1 : x0) + 2 * nib) << 16);
      const float l = __uint_as_float(ld_shared_u32(il + 4 * (8 * j + nib)));
      const uint32_t c = e2m1_code1(__fdiv_rn(__fmul_rn(x, l), eff));
      w[j] = (w[j] & ~(0xFu << (4 * nib))) | (c << (4 * nib));
      m &= ~(0xFu << (4 * nib));
    }
  }
  return make_uint2(w[0], w[1]);
}

template <int RANK, bool QUANT>
__global__ void __launch_bounds__(QCfg<RANK, QUANT>::THREADS, 1)
    k1_quant_act_lora_down(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1,
                           QArgs a) {
  using C = QCfg<RANK, QUANT>;
  constexpr int ST = C::STAGES;
  constexpr int SUB = C::SUB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::DATA_BYTES);
  // bars: full[ST] | empty[ST] | accfull | recv | tmem holder
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_empty = bar_full + 8 * ST;
  const uint32_t bar_acc = bar_empty + 8 * ST;
  const uint32_t bar_recv = bar_acc + 8;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 2 * ST + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int nsplit = gridDim.x;
  const int m0 = blockIdx.y * C::ROWS;
  const int nch = a.K / 64;
  const int c_begin = split * a.chunks_per_split;
  int n_local = nch - c_begin;
  if (n_local > a.chunks_per_split) n_local = a.chunks_per_split;
  if (n_local < 0) n_local = 0;
  const int n_stages = (n_local + SUB - 1) / SUB;
  // split-K reduction: CTA j of the cluster owns rows [j rows_per, min(ROWS, (j + 1) rows_per))
  const int rows_per = (C::ROWS + nsplit - 1) / nsplit;
  const int own_r0 = min(C::ROWS, split * rows_per);
  const int own_r1 = min(C::ROWS, own_r0 + rows_per);
  auto x_tile = [&](int s, int u) { return smem + s * C::STAGE_BYTES + u * C::X_BYTES; };
  auto l1_tile = [&](int s, int u) { return smem + s * C::STAGE_BYTES + SUB * C::X_BYTES + u * C::L1_BYTES; };
  auto il_tile = [&](int s, int u) {
    return smem + s * C::STAGE_BYTES + SUB * (C::X_BYTES + C::L1_BYTES) + u * C::IL_BYTES;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, C::EMPTY_COUNT);
    }
    mbar_init(bar_acc, 1);
    mbar_init(bar_recv, 1);
    fence_mbar_init();
    // the other CTAs of the cluster each send RANK fp32 per owned row
    if (RANK) mbar_arrive_expect_tx(bar_recv, static_cast<uint32_t>((nsplit - 1) * (own_r1 - own_r0) * RANK * 4));
  }
  if (RANK && warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = RANK ? *tmem_holder : 0u;
  // With separate reduction slots every thread arrives on the cluster barrier now: a CTA's slots
  // and recv barrier (initialised and published with fence.mbarrier_init above) are ready for
  // the other CTAs' partials from the start.
  if constexpr (C::RED_SEPARATE) cluster_arrive_relaxed();
  // The prologue above overlaps the previous kernel of the stream; global memory only after it.
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      if (RANK) tma_prefetch_desc(&tm_l1);
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % ST;
        if (i >= ST && !mbar_wait_parked(bar_empty + 8 * s, ((i / ST) - 1) & 1, a.err, KID_QUANT, 1)) break;
        // chunks of this stage that lie inside the CTA's range (the last stage may hold one)
        const int nu = min(SUB, n_local - i * SUB);
        const uint32_t fb = bar_full + 8 * s;
        mbar_arrive_expect_tx(fb, nu * (C::X_BYTES + C::L1_BYTES + C::IL_BYTES));
        for (int u = 0; u < nu; ++u) {
          const int kx = (c_begin + i * SUB + u) * 64;
          tma_load_2d(smem_u32(x_tile(s, u)), &tm_x, kx, m0, fb);
          if (RANK) tma_load_2d(smem_u32(l1_tile(s, u)), &tm_l1, kx, 0, fb);
          if (QUANT) bulk_load(smem_u32(il_tile(s, u)), a.inv_lambda + kx, C::IL_BYTES, fb);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); one elected lane issues.
    if (RANK) {
      // kind::f16: D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9, 10-12 = 1), K-major,
      // N = RANK (bits 17-22 = N >> 3), M = ROWS (bits 24-28 = M >> 4).
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t(RANK) >> 3) << 17) |
                             ((uint32_t(C::ROWS) >> 4) << 24);
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % ST;
        if (!__all_sync(0xffffffffu, mbar_wait_parked(bar_full + 8 * s, (i / ST) & 1, a.err, KID_QUANT, 2))) break;
        tc_fence_after();
        const int nu = min(SUB, n_local - i * SUB);
        const uint64_t ad0 = umma_desc(smem_u32(x_tile(s, 0)), 16, 1024, 2);
        const uint64_t bd0 = umma_desc(smem_u32(l1_tile(s, 0)), 16, 1024, 2);
        if (elect_one()) {
          for (int u = 0; u < nu; ++u) {
            // chunk u's tiles sit u * X_BYTES and u * L1_BYTES further (descriptor units of 16 bytes)
            const uint64_t ad = ad0 + static_cast<uint64_t>(u * (C::X_BYTES >> 4));
            const uint64_t bd = bd0 + static_cast<uint64_t>(u * (C::L1_BYTES >> 4));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16(tbase, ad + 2u * k, bd + 2u * k, idesc, (i | u | k) != 0 ? 1u : 0u);
          }
          tc_commit(bar_empty + 8 * s);
        }
        __syncwarp();
      }
      if (elect_one()) tc_commit(bar_acc);
      __syncwarp();
    }
  } else if (QUANT && warp < C::RED_WARP0) {
    // ------------------------------------------------------------ quantizers
    const int qw = warp - 2;
    const int u = qw / C::WARPS_PER_CHUNK;  // chunk of the stage
    const int g = lane >> 3;                // 16-column group of the chunk
    const int rl = lane & 7;
    const int row = 16 * (qw % C::WARPS_PER_CHUNK) + rl;  // and row + 8 (same swizzle phase: row & 7 == rl)
    const int m = m0 + row;
    const uint32_t xoff0 = row * 128 + ((((2 * g) ^ rl)) << 4);
    const uint32_t xoff1 = row * 128 + ((((2 * g + 1) ^ rl)) << 4);
    const size_t row_bytes = static_cast<size_t>(a.K) / 2;
    // per stage the codes advance by SUB chunks of 32 bytes and the scales by SUB 512-byte blocks;
    // row + 8 sits 8 code rows further and 8 x 16 bytes further in the same scale block (the
    // tile starts at a multiple of 64 rows, so rows row and row + 8 share one 32-row group)
    uint8_t *xq_p = a.xq + static_cast<size_t>(m) * row_bytes + (c_begin + u) * 32 + 8 * g;
    uint8_t *xs_p = a.xs + scale_offset(m, (c_begin + u) * 4 + g, a.K / 16);
    const bool ok0 = m < a.M, ok1 = m + 8 < a.M;
    const float s_x = a.s_x, d_x = a.d_x, inv_d = a.inv_d;
    for (int i = 0; i < n_stages; ++i, xq_p += 32 * SUB, xs_p += 512 * SUB) {
      const int s = i % ST;
      if (!mbar_wait_parked(bar_full + 8 * s, (i / ST) & 1, a.err, KID_QUANT, 4)) break;
      if (i * SUB + u < n_local) {
        const uint32_t il4 = smem_u32(il_tile(s, u)) + g * 64;
        const uint4 l0 = ld_shared_u32x4(il4), l1 = ld_shared_u32x4(il4 + 16), l2 = ld_shared_u32x4(il4 + 32),
                    l3 = ld_shared_u32x4(il4 + 48);
        const f2 il[8] = {mk2(__uint_as_float(l0.x), __uint_as_float(l0.y)), mk2(__uint_as_float(l0.z), __uint_as_float(l0.w)),
                          mk2(__uint_as_float(l1.x), __uint_as_float(l1.y)), mk2(__uint_as_float(l1.z), __uint_as_float(l1.w)),
                          mk2(__uint_as_float(l2.x), __uint_as_float(l2.y)), mk2(__uint_as_float(l2.z), __uint_as_float(l2.w)),
                          mk2(__uint_as_float(l3.x), __uint_as_float(l3.y)), mk2(__uint_as_float(l3.z), __uint_as_float(l3.w))};
        const uint32_t xt = smem_u32(x_tile(s, u));
        // both rows' groups are independent and computed without branches, so they interleave
        float xh[2][16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 raw0 = ld_shared_u32x4(xt + h * 1024 + xoff0);
          const uint4 raw1 = ld_shared_u32x4(xt + h * 1024 + xoff1);
          const uint32_t w[8] = {raw0.x, raw0.y, raw0.z, raw0.w, raw1.x, raw1.y, raw1.z, raw1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) un2(mul2(mk2(bf16_lo(w[e]), bf16_hi(w[e])), il[e]), xh[h][2 * e], xh[h][2 * e + 1]);
        }
        Group16 q[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) q[h] = nvfp4_group16_fast(xh[h], s_x, d_x, inv_d);
        if (q[0].exact | q[1].exact) {  // rare: one branch for both groups
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (q[h].exact) {
              const uint2 c = group_codes_settle(xt + h * 1024 + xoff0, xt + h * 1024 + xoff1, il4, q[h].eff,
                                                 q[h].w0, q[h].w1, q[h].d0, q[h].d1);
              q[h].w0 = c.x;
              q[h].w1 = c.y;
            }
        }
        if (ok0) *reinterpret_cast<uint2 *>(xq_p) = make_uint2(q[0].w0, q[0].w1);
        if (ok1) *reinterpret_cast<uint2 *>(xq_p + 8 * row_bytes) = make_uint2(q[1].w0, q[1].w1);
        xs_p[0] = static_cast<uint8_t>(q[0].sc);
        xs_p[128] = static_cast<uint8_t>(q[1].sc);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    }
  }

  if constexpr (RANK > 0) {
    // ------------------------------------------------------------ split-K reduction
    // Each CTA keeps, in its stage memory, one slot per cluster rank for the rows it owns:
    // slot[src][row - own_r0] = partial of CTA src (RS fp32 per row). Partials of rows owned by
    // another CTA go there with st.async, counted on that CTA's recv barrier; the owner sums
    // the slots in rank order (deterministic) once its own writes and the remote bytes are in.
    // The stage memory of every CTA must be idle first: a split cluster barrier, arrived at as
    // soon as this CTA's quantizer warps and MMAs are done with it.
    // Failure path: if the wait for the peers' bytes (bar_recv) gives up after its time limit (a
    // peer CTA stalled), the owner records the error and exits without a final cluster barrier
    // (a barrier.cluster wait cannot be bounded); a peer that resumes later could then still store
    // into the exited CTA's shared memory. The recorded error marks every output of the launch as
    // invalid (svdq_last_device_error); on the normal path every byte has landed before the owner
    // reads the slots, so no store is in flight when a CTA exits.
    constexpr uint32_t RS = C::RED_STRIDE;
    const uint32_t slot_bytes = static_cast<uint32_t>(rows_per) * RS * 4u;
    uint8_t *red = smem + C::RED_OFF;
    const uint32_t red_base = smem_u32(red);
    // rows own_r0 .. own_r1 - 1: sum the slots in rank order, four columns per thread, and store
    // lora_act (threads t0, t0 + nthr, ...)
    auto sum_store = [&](int t0, int nthr) {
      constexpr int QUADS = RANK / 4;
      for (int idx = t0; idx < (own_r1 - own_r0) * QUADS; idx += nthr) {
        const int lr = idx / QUADS;
        const int c = 4 * (idx % QUADS);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < nsplit; ++src) {
          const float4 v =
              *reinterpret_cast<const float4 *>(red + src * slot_bytes + static_cast<uint32_t>(lr * RS + c) * 4u);
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        const int m = m0 + own_r0 + lr;
        if (m < a.M) {
          // lora_act row = [hi(0..RANK-1) | lo(0..RANK-1)], v ~ hi + lo with hi = bf16(v),
          // lo = bf16(v - hi): the pair carries ~16 significant bits of the fp32 value.
          const float v0 = __fmul_rn(acc.x, a.inv_alpha), v1 = __fmul_rn(acc.y, a.inv_alpha);
          const float v2 = __fmul_rn(acc.z, a.inv_alpha), v3 = __fmul_rn(acc.w, a.inv_alpha);
          const uint32_t h01 = pack_bf16x2(v0, v1), h23 = pack_bf16x2(v2, v3);
          const uint32_t l01 = pack_bf16x2(__fsub_rn(v0, bf16_lo(h01)), __fsub_rn(v1, bf16_hi(h01)));
          const uint32_t l23 = pack_bf16x2(__fsub_rn(v2, bf16_lo(h23)), __fsub_rn(v3, bf16_hi(h23)));
          uint16_t *out = a.lora_act + static_cast<size_t>(m) * (2 * RANK) + c;
          *reinterpret_cast<uint2 *>(out) = make_uint2(h01, h23);
          *reinterpret_cast<uint2 *>(out + RANK) = make_uint2(l01, l23);
        }
      }
    };
    // this CTA's partial of accumulator row `row` (vals: RANK fp32) into the owner's slot
    auto send_row = [&](int row, const uint32_t *vals, int c0, int nc, bool ok) {
      const int owner = row / rows_per;
      const uint32_t off =
          static_cast<uint32_t>(split) * slot_bytes + static_cast<uint32_t>((row - owner * rows_per) * RS + c0) * 4u;
      if (owner == split) {
        for (int j = 0; j < nc; j += 4)
          *reinterpret_cast<float4 *>(red + off + 4 * j) =
              ok ? make_float4(__uint_as_float(vals[j]), __uint_as_float(vals[j + 1]), __uint_as_float(vals[j + 2]),
                               __uint_as_float(vals[j + 3]))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const uint32_t dst = map_shared_rank(red_base + off, owner);
        const uint32_t rbar = map_shared_rank(bar_recv, owner);
        for (int j = 0; j < nc; j += 4)
          st_async_f32x4(dst + 4 * j,
                         ok ? make_float4(__uint_as_float(vals[j]), __uint_as_float(vals[j + 1]),
                                          __uint_as_float(vals[j + 2]), __uint_as_float(vals[j + 3]))
                            : make_float4(0.f, 0.f, 0.f, 0.f),
                         rbar);
      }
    };
    if constexpr (C::RED_SEPARATE) {
      if (warp >= C::RED_WARP0) {
        // Warp w reads the accumulator rows of tensor-memory quadrant w % 4, all RANK columns.
        const int quad = warp & 3;
        const bool row_ok = C::ROWS == 128 || lane < 16;
        const int row = C::ROWS == 128 ? quad * 32 + lane : quad * 16 + (lane & 15);
        const bool ok = mbar_wait_parked(bar_acc, 0, a.err, KID_QUANT, 5) && n_local > 0;
        tc_fence_after();
        const uint32_t taddr = tbase + (static_cast<uint32_t>(quad * 32) << 16);
        uint32_t r[RANK];
        if constexpr (RANK == 16) {
          tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
        } else {
#pragma unroll
          for (int c = 0; c < RANK / 32; ++c) tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
        }
        tmem_wait_ld();
        tc_fence_before();
        cluster_wait();  // every CTA of the cluster has initialised its recv barrier
        if (row_ok) send_row(row, r, 0, RANK, ok);
        named_bar_sync(2, 32 * C::RED_WARPS);
        mbar_wait_parked(bar_recv, 0, a.err, KID_QUANT, 6);
        sum_store(static_cast<int>(threadIdx.x) - 32 * C::RED_WARP0, 32 * C::RED_WARPS);
      } else {
        cluster_wait();
      }
    } else if (warp >= 2) {
      // A warp reads the 32 tensor-memory lanes of its quadrant (warp % 4). Accumulator row r
      // sits in lane r for M = 128 and in lane 32 (r / 16) + r % 16 for M = 64 (the upper 16
      // lanes of each quadrant then hold nothing).
      const int quad = warp & 3;
      const bool row_ok = C::ROWS == 128 || lane < 16;
      const int row = C::ROWS == 128 ? quad * 32 + lane : quad * 16 + (lane & 15);
      const int grp = (warp - 2) >> 2;  // 0..3: column group
      const bool ok = mbar_wait_parked(bar_acc, 0, a.err, KID_QUANT, 5) && n_local > 0;
      // every quantizer warp must be done reading the stage buffers (the MMA commit above covers
      // only the tensor-core reads)
      if (QUANT) named_bar_sync(1, 32 * C::QWARPS);
      cluster_arrive();
      tc_fence_after();
      const uint32_t taddr = tbase + (static_cast<uint32_t>(quad * 32) << 16);
      constexpr int CPG = RANK == 16 ? 16 : RANK / 4;  // columns per warp: rank 16 uses one group
      const int cb = grp * CPG;
      uint32_t r[CPG];
      if (RANK != 16 || grp == 0) {
        if constexpr (CPG == 8) tmem_ld8(taddr + cb, r);
        else if constexpr (CPG == 16) tmem_ld16(taddr + cb, r);
        else tmem_ld32(taddr + cb, r);
        tmem_wait_ld();
      }
      tc_fence_before();
      cluster_wait();
      if (row_ok && (RANK != 16 || grp == 0)) send_row(row, r, cb, CPG, ok);
      named_bar_sync(1, 32 * C::QWARPS);
      mbar_wait_parked(bar_recv, 0, a.err, KID_QUANT, 6);
      sum_store(static_cast<int>(threadIdx.x) - 64, 32 * C::QWARPS);
    } else {
      cluster_arrive();
      cluster_wait();
    }
  }

  __syncthreads();
  if (RANK && warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// Row tiles of K1: enough to cover the activation scale buffer's rows (M padded to 128).
int quant_tiles(int M) { return (M + 127) / 128 * (128 / kQuantRows); }

template <int RANK, bool QUANT>
cudaError_t set_attrs() {
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k1_quant_act_lora_down<RANK, QUANT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, QCfg<RANK, QUANT>::SMEM);
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  return cudaSuccess;
}

// Clusters of `splits` CTAs that can be resident at once (one query per device and size).
template <int RANK, bool QUANT>
int max_active_clusters(int splits) {
  static int cache[64][9] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || splits < 1 || splits > 8) return 0;
  if (cache[dev][splits]) return cache[dev][splits];
  if (set_attrs<RANK, QUANT>() != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(splits, 1, 1);
  cfg.blockDim = dim3(QCfg<RANK, QUANT>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = QCfg<RANK, QUANT>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k1_quant_act_lora_down<RANK, QUANT>, &cfg) != cudaSuccess) n = 0;
  cache[dev][splits] = n > 0 ? n : -1;
  return n;
}

// Cluster size along K: minimises (waves) x (chunks per CTA + 2), the 2 standing for the
// per-CTA fixed cost (pipeline fill, reduction); every CTA gets at least one chunk.
template <int RANK, bool QUANT>
int pick_splits_t(int M, int K) {
  const int tiles = quant_tiles(M);
  const int nch = K / 64;
  int best = 1;
  long best_cost = -1;
  for (int sp = 1; sp <= 8; ++sp) {
    const int cps = (nch + sp - 1) / sp;
    if ((sp - 1) * cps >= nch) continue;
    const int act = RANK ? max_active_clusters<RANK, QUANT>(sp) : 0;
    long waves = 1;
    if (act > 0) waves = (tiles + act - 1) / act;
    const long cost = waves * (cps + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = sp;
    }
  }
  return best;
}

template <int RANK, bool QUANT>
cudaError_t launch_t(const QuantLaunch &q) {
  using C = QCfg<RANK, QUANT>;
  auto kern = k1_quant_act_lora_down<RANK, QUANT>;
  cudaError_t e0 = set_attrs<RANK, QUANT>();
  if (e0 != cudaSuccess) return e0;
  QArgs a{q.inv_lambda, q.xq, q.xs, q.lora_act, q.M, q.K, q.s_x, q.d_x, 1.0f / q.d_x, q.inv_alpha, q.chunks_per_split, q.err};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(q.splits, quant_tiles(q.M), 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = q.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = q.splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = RANK ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, q.tm_x, q.tm_l1, a);
}

}  // namespace

int quant_act_splits(int M, int K, int rank, bool quantize, bool lora, int num_sms) {
  const int r = lora ? rank : 0;
  if (r == 0) {
    // no cross-CTA reduction: as many CTAs along K as fit one wave, none of them empty
    const int tiles = quant_tiles(M), nch = K / 64;
    int sp = num_sms / tiles;
    if (sp > nch) sp = nch;
    if (sp > 16) sp = 16;
    if (sp < 1) sp = 1;
    while (sp > 1 && (sp - 1) * ((nch + sp - 1) / sp) >= nch) --sp;
    return sp;
  }
  if (quantize) {
    switch (r) {
      case 16: return pick_splits_t<16, true>(M, K);
      case 32: return pick_splits_t<32, true>(M, K);
      case 64: return pick_splits_t<64, true>(M, K);
      case 128: return pick_splits_t<128, true>(M, K);
    }
  } else {
    switch (r) {
      case 16: return pick_splits_t<16, false>(M, K);
      case 32: return pick_splits_t<32, false>(M, K);
      case 64: return pick_splits_t<64, false>(M, K);
      case 128: return pick_splits_t<128, false>(M, K);
    }
  }
  return 1;
}

cudaError_t launch_quant_act(const QuantLaunch &q) {
  const int r = q.lora ? q.rank : 0;
  if (q.quantize) {
    switch (r) {
      case 0: return launch_t<0, true>(q);
      case 16: return launch_t<16, true>(q);
      case 32: return launch_t<32, true>(q);
      case 64: return launch_t<64, true>(q);
      case 128: return launch_t<128, true>(q);
    }
  } else {
    switch (r) {
      case 16: return launch_t<16, false>(q);
      case 32: return launch_t<32, false>(q);
      case 64: return launch_t<64, false>(q);
      case 128: return launch_t<128, false>(q);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace svdq
