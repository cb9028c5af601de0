// K2: block-scaled NVFP4 tensor-core GEMM whose output stage adds the low-rank up-projection
// and the bias and writes bf16 once.
//
// "Svdq Int4 Flux.1 Canny Dev" model card, "Nunchaku 引擎設計" (a)/(b): the up-projection and
// the 4-bit GEMM produce the same output, so one kernel serves both and the 16-bit output is
// written once.
//
// Persistent kernel of CTA pairs (clusters of two CTAs on two SMs). A pair owns an output tile
// of 256 x 256 (rows of X x rows of W) and computes it with cta_group::2 tensor-core MMAs of
// M = 256, N = 256: each CTA stages its own 128 rows of the activation tile and its own 128
// rows of the weight tile, the even CTA of the pair issues the MMAs for both, and each CTA's
// tensor memory holds the accumulator of its 128 rows (all 256 columns). Per SM and per 4-bit
// step this stages 32 KiB of operands for 512 tensor-core cycles; a one-CTA tile of 128 x 256
// needs 48 KiB.
//
// Per tile the k-loop is a sequence of pipeline steps through a 5-stage shared-memory ring
// (38 KiB per stage: operands and scale blocks):
//   - rank / kc low-rank steps, kc = min(rank, 32): per CTA the hi and lo planes of lora_act
//     (128 x kc bf16 each) and half of an L2t tile (128 x kc bf16); bf16 MMAs (K = 16 each),
//     hi and lo against the same L2t tile;
//   - K / 256 4-bit steps: per CTA 128 rows of xq and 128 rows of wq (128 bytes each, 128B
//     swizzle); four kind::mxf4nvf4 MMAs (K = 64 each).
// All steps accumulate into one fp32 accumulator. lora_act arrives pre-divided by
// alpha = s_x s_w, so the output stage computes Y = bf16(alpha * acc + bias) for every element.
//
// Scale factors reach tensor memory from shared memory. With each 4-bit step the producer
// bulk-copies three 2 KiB scale blocks into the stage (the CTA's activation block and the tile's
// two weight blocks, four k-blocks each), signalled on a per-stage sffull barrier. The MMA
// issuer copies the activation blocks with tcgen05.cp (one 32x128b.warpx4 copy per k-block, in
// both CTAs, in order with and overlapping the MMAs: four per step keep the copy unit, ~90
// cycles a block, inside the step's 512 MMA cycles). The eight weight blocks of a step would
// overrun the copy unit, so eight warps per CTA in two groups of four (one warp per 32-lane
// sub-partition, the groups taking alternate steps) read their lines and write them with
// tcgen05.st. Both paths produce the replicated layout the block-scaled MMA reads (lane i of
// every sub-partition holds rows i, i+32, i+64, i+96 of a block, one 32-bit column each).
// Staging the blocks with the stage gives them the ring's whole latency tolerance (loaded from
// L2 by the writers themselves, two steps ahead, they set the kernel's pace). A CTA holds the
// activation scales of its own 128 rows and the weight scales of all 256 rows of the tile, since
// its half of the MMA multiplies its rows by the whole of B (writing only the half of the weight
// scales that matches the CTA's B rows, or writing them in the even CTA only, fails the
// bit-exact layout tests).
//
// Warp roles (640 threads per CTA): warp 0 TMA producer; warp 1 tensor-memory owner and, in the
// even CTA, MMA issuer; warps 2..5 (even steps) and 6, 7, 16, 17 (odd steps) scale-factor
// writers; warps 8..15 output stage (warp w reaches lanes 32 (w % 4).. and drains columns
// 128 ((w - 8) / 4)..), which take 168 registers a thread from the other warpgroups
// (setmaxnreg); warps 18, 19 idle. The output stage drains the accumulator into a swizzled bf16 box in
// shared memory (one box of 64 columns per half, filled twice per tile), releases the
// accumulator once all its chunks are in registers, and writes the boxes with TMA stores (which
// clip the M / N edges).
//
// Synchronisation across the pair. Every barrier the MMA issuer waits on lives in the even CTA,
// and it waits on one per step and one per tile: each barrier result the issuing thread consumes
// costs the tensor pipe a bubble of about 200 cycles, because the MMA queue is short. The full
// barrier of a stage counts the even CTA producer's arrival (which expects the bytes of both
// CTAs' loads; the odd CTA's loads signal it across the pair) and one arrival per scale-writer
// warp of either CTA; accempty counts one arrival per output warp of either CTA. The MMA
// issuer's commits arrive on the empty and accfull barriers of both CTAs. Every wait is bounded:
// a thread whose wait gives up records the error and either leaves its loop or, where it shares
// named barriers, keeps stepping through them without touching tensor memory.
#include "common.cuh"
#include "internal.h"
#include "nvfp4.cuh"

namespace svdq {
namespace {

// Two fp32 values in one 64-bit register, for the packed f32x2 arithmetic of the fused QKV
// output stage (each lane of a packed op rounds like its scalar counterpart).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2_rn(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2_rn(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcp_approx_f(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU in its tanh form, 0.5 v (1 + tanh(u)) with u = sqrt(2 / pi) (v + 0.044715 v^3), through
// the identity 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2 u)):  v / (1 + 2^(v (c1 + c2 v^2))) with
// c1 = -2 sqrt(2 / pi) log2(e) and c2 = 0.044715 c1. One hardware base-2 exponential (relative
// error about 2^-22) and one reciprocal; no cancellation for negative v (the result goes smoothly
// to -0 as the exponential overflows to infinity).
__device__ __forceinline__ float gelu_tanh(float v) {
  constexpr float c1 = -2.3022082f;
  constexpr float c2 = -0.10294324f;
  const float t = __fmul_rn(v, v);
  const float e = ex2_approx(__fmul_rn(v, __fmaf_rn(c2, t, c1)));
  return __fmul_rn(v, rcp_approx_f(__fadd_rn(1.0f, e)));
}

// Sixteen fp32 values passed by value to the out-of-line exact path.
struct Vals16 {
  float v[16];
};
// x_hat = fp32(h inv_lambda) for a pair of values, recomputed where needed instead of kept live
// (volatile: the compiler must not merge the recomputation with the first one).
__device__ __forceinline__ void xhat2(float h0, float h1, float l0, float l1, float &x0, float &x1) {
  uint64_t r;
  asm volatile("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk2(h0, h1)), "l"(pk2(l0, l1)));
  upk2(r, x0, x1);
}

// The group quantizer of the activation kernel (same scale code, same reciprocal bracket: codes of
// x_hat (1 -/+ 2^-20) / eff through the reciprocal of eff) for x_hat = fp32(h inv_lambda), with the
// products formed from h and inv_lambda each time they are needed and the codes eight at a time, so
// that few values stay live in a thread that also holds a 128-column accumulator slice. h: the
// group's 16 values (fp32 bit patterns), il: its 16 inverse smoothing factors in shared memory.
// Returns true when an element is undecided: the caller then takes the codes from correctly
// rounded quotients.
__device__ __forceinline__ bool quant16_lean(const uint32_t *h, const float *il, float s, float d, float inv_d,
                                             uint32_t &w0, uint32_t &w1, uint32_t &sc, float &eff) {
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float4 l = *reinterpret_cast<const float4 *>(il + 4 * e);
    float x0, x1, x2, x3;
    xhat2(__uint_as_float(h[4 * e]), __uint_as_float(h[4 * e + 1]), l.x, l.y, x0, x1);
    xhat2(__uint_as_float(h[4 * e + 2]), __uint_as_float(h[4 * e + 3]), l.z, l.w, x2, x3);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3))));
  }
  sc = scale_code(amax, d, inv_d);
  const float sg = e4m3_value(sc);
  eff = __fmul_rn(sg, s);
  const float r = rcp_approx(eff);  // +inf when sg == 0; the codes are then forced to zero
  const f2 rl2 = mk2(__fmul_rn(r, kBracketLo), __fmul_rn(r, kBracketLo));
  const f2 rh2 = mk2(__fmul_rn(r, kBracketHi), __fmul_rn(r, kBracketHi));
  const bool zero = sg == 0.0f;
  uint32_t w[2], dd = 0;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float lo[8], hi[8];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float4 l = *reinterpret_cast<const float4 *>(il + 8 * hf + 4 * e);
      float x0, x1, x2, x3;
      xhat2(__uint_as_float(h[8 * hf + 4 * e]), __uint_as_float(h[8 * hf + 4 * e + 1]), l.x, l.y, x0, x1);
      xhat2(__uint_as_float(h[8 * hf + 4 * e + 2]), __uint_as_float(h[8 * hf + 4 * e + 3]), l.z, l.w, x2, x3);
      un2(mul2(mk2(x0, x1), rl2), lo[4 * e], lo[4 * e + 1]);
      un2(mul2(mk2(x2, x3), rl2), lo[4 * e + 2], lo[4 * e + 3]);
      un2(mul2(mk2(x0, x1), rh2), hi[4 * e], hi[4 * e + 1]);
      un2(mul2(mk2(x2, x3), rh2), hi[4 * e + 2], hi[4 * e + 3]);
    }
    const uint32_t l = e2m1x8_raw(lo), hc = e2m1x8_raw(hi);
    w[hf] = zero ? 0u : e2m1_clear_neg_zero(l);
    dd |= l ^ hc;
  }
  w0 = w[0];
  w1 = w[1];
  return !zero && dd != 0u;
}

// The codes of a group from correctly rounded quotients x_hat / eff (x_hat = fp32(h inv_lambda)).
__device__ __noinline__ uint2 group_codes_exact_h(Vals16 hv, const float *il, float eff) {
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(__fmul_rn(hv.v[i], il[i]), eff);
  return make_uint2(e2m1x8(q), e2m1x8(q + 8));
}

constexpr int BM = 128;      // rows of X per CTA
constexpr int BMP = 2 * BM;  // rows of X per pair tile
constexpr int BN = 256;      // rows of W per pair tile
constexpr int BNH = BN / 2;  // rows of W staged per CTA
constexpr int STAGES = 5;
constexpr uint32_t A_BYTES = BM * 128u;
constexpr uint32_t B_BYTES = BNH * 128u;
constexpr uint32_t SF_BLOCK = 512;  // scale bytes of 128 rows x 64 elements of K
// per 4-bit step: the CTA's activation scale block and the tile's two weight scale blocks
// (rows 0-127, 128-255), four k-blocks each, bulk-copied with the stage
constexpr uint32_t SF_OFF = A_BYTES + B_BYTES;
constexpr uint32_t SF_STAGE_BYTES = 3 * 4 * SF_BLOCK;                 // 6 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SF_STAGE_BYTES;  // 38 KiB
constexpr uint32_t DATA_BYTES = STAGES * STAGE_BYTES;
constexpr uint32_t YST_BYTES = BM * 64 * 2 * 2;  // bf16 output staging: one box of 128 rows x 64 columns per half
constexpr uint32_t BIAS_BYTES = BN * 4;
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM = DATA_BYTES + YST_BYTES + BIAS_BYTES + BAR_BYTES + 1024;
// Fused QKV output stage (QKNR): four ring stages instead of five make room for the rotary
// table rows of the tile (128 rows x 32 column pairs x (cos, sin) fp32, 32 KiB, one half of the
// head's pairs at a time) and the two normalization weight vectors.
constexpr int STAGES_QKNR = 4;
constexpr uint32_t ROPE_BYTES = 128 * 32 * 2 * 4;
constexpr uint32_t NORMW_BYTES = 2 * 2 * 128 * 4;
constexpr uint32_t SMEM_QKNR =
    STAGES_QKNR * STAGE_BYTES + ROPE_BYTES + YST_BYTES + BIAS_BYTES + NORMW_BYTES + BAR_BYTES + 1024;
// MLP pair (MLP): the up-projection's output stage quantizes GELU(alpha acc + b) for the down
// layer and feeds a bf16 hi / lo copy of it, 32 columns at a time, to a pair MMA against the down
// layer's L1s (four ring stages as for QKNR). Per CTA: the hi and lo planes of both halves' current
// 32 columns (128 rows x 64 bytes each, 64B swizzle), the tile's 256 columns of L1s (eight boxes of
// 32 columns x rank_d / 2 rows, rank_d <= 64) and the down layer's inverse smoothing factors.
constexpr int STAGES_MLP = 4;
constexpr uint32_t HBOX_BYTES = BM * 64u;            // one plane of one half: 128 rows x 32 bf16
constexpr uint32_t HBOXES_BYTES = 4 * HBOX_BYTES;   // [half][hi, lo]
constexpr uint32_t L1D_BOX_MAX = 32 * 64u;          // 32 rows (rank_d / 2 <= 32) x 32 bf16
constexpr uint32_t L1D_BYTES = 8 * L1D_BOX_MAX;
constexpr uint32_t ILD_BYTES = BN * 4;
constexpr uint32_t SMEM_MLP =
    STAGES_MLP * STAGE_BYTES + HBOXES_BYTES + L1D_BYTES + BIAS_BYTES + ILD_BYTES + BAR_BYTES + 1024;
constexpr uint32_t LA_COL0 = 448;  // down-projection partial accumulator (rank_d <= 64 columns)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 256;  // one scale slot per stage follows the accumulator
constexpr uint32_t SF_COLS = 48;   // per slot: 4 k-blocks x (4 SFA + 8 SFB) columns
// 20 warps = 5 warpgroups (registers are reallocated per warpgroup): warp 0 producer, warp 1
// MMA issuer, warps 2..7 and 16..17 scale writers (two per tensor-memory sub-partition), warps
// 8..15 output stage (warpgroups 2 and 3), warps 18..19 idle.
constexpr int EPI_WARP0 = 8;
constexpr int THREADS = 640;
// Registers per thread after reallocation: the output warpgroups hold a row's whole 128-column
// accumulator slice (4 x 32 fp32) before releasing it; the others need few.
constexpr uint32_t EPI_REGS = 168;
constexpr uint32_t OTHER_REGS = 48;
template <int OUT>
constexpr uint32_t epi_regs() { return EPI_REGS; }
template <int OUT>
constexpr uint32_t other_regs() { return OTHER_REGS; }
template <int OUT>
constexpr uint32_t reg_pool_needed() { return 32u * (8u * epi_regs<OUT>() + 12u * other_regs<OUT>()); }  // per CTA
static_assert(reg_pool_needed<0>() <= 96u * 640u, "register split");
// Arrivals the MMA issuer waits for, besides the producer's: per step one per writer warp of the
// step's group (four per CTA), per tile one per output warp, from both CTAs of the pair.
constexpr uint32_t SF_GROUP_WARPS = 4;
constexpr uint32_t EPI_WARPS = 8;
constexpr uint32_t FULL_COUNT = 1 + 2 * SF_GROUP_WARPS;
constexpr uint32_t ACCEMPTY_COUNT = 2 * EPI_WARPS;
constexpr int N_BARS = 4 * STAGES + 2 + 4;  // + rope_full, rope_empty (QKNR) or hfull, hempty, l1dfull, l1dfree (MLP)
static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1 KiB alignment of 128B-swizzled tiles");
static_assert(SF_COL0 + STAGES * SF_COLS <= TMEM_COLS, "scale slots exceed the tensor memory");
static_assert(SMEM_QKNR <= 232448, "shared memory per CTA");
static_assert(SMEM_MLP <= 232448, "shared memory per CTA");
static_assert(SF_COL0 + STAGES_MLP * SF_COLS <= LA_COL0 && LA_COL0 + 64 <= TMEM_COLS, "MLP tensor memory");
static_assert((STAGES_MLP * STAGE_BYTES) % 1024 == 0 && HBOXES_BYTES % 1024 == 0, "swizzled boxes stay aligned");
static_assert(N_BARS * 8 + 4 <= BAR_BYTES, "barrier area");

// Output stage of K2.
enum OutMode : int {
  OUT_PLAIN = 0,  // Y = bf16(alpha acc + b)
  OUT_ADDY = 1,   // Y = bf16(Y + alpha acc) (unfused up-projection)
  OUT_QKNR = 2,   // fused QKV: per-head Q/K RMS normalization and rotary embedding, then bf16
  OUT_GELU = 3,   // H = bf16(GELU(alpha acc + b)) (first layer of an unfused MLP pair)
  OUT_MLP = 4     // fused MLP pair: GELU, then the down layer's NVFP4 quantization and down-projection partials
};

struct GArgs {
  const uint8_t *xs;
  const uint8_t *ws;
  const float *bias;
  uint16_t *Y;
  int M, N, K;
  int Mt, Nt;  // pair tiles along M (256 rows) and N (256 rows of W)
  float alpha;
  uint32_t *err;
  // fused QKV output stage (QKNR): Y = [Q | K | V], qk_width = heads x 128 columns per section
  const float *norm_q;  // [128]
  const float *norm_k;  // [128]
  int qk_width;
  float eps;
  // fused MLP pair (MLP): the down layer's inverse smoothing factors (N of them), tensor scale
  // s_x (d = 6 s_x and its reciprocal), rank, outputs (codes M x N/2, block-layout scales with
  // mp_scales rows, fp32 partial down-projections [Nt][M][rank_d])
  const float *il_d;
  float sx_d, dx_d, inv_dx_d;
  int rank_d, mp_scales;
  uint8_t *xq_d;
  uint8_t *xs_d;
  float *part;
};

template <int RANK, bool FP4, int OUT>
__global__ void __launch_bounds__(THREADS, 1)
    k2_gemm_w4a4_lora_up(const __grid_constant__ CUtensorMap tm_xq, const __grid_constant__ CUtensorMap tm_wq,
                         const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_l2,
                         const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_rope,
                         GArgs a) {
  constexpr bool ADD_Y = OUT == OUT_ADDY;
  constexpr bool QKNR = OUT == OUT_QKNR;
  constexpr bool GELU = OUT == OUT_GELU;
  constexpr bool MLP = OUT == OUT_MLP;
  // tm_rope: the rotary table (QKNR) or the down layer's L1s, rank_d x N bf16 (MLP)
  const CUtensorMap &tm_aux = tm_rope;
  // Low-rank steps: kc columns of lora_act (hi and lo planes) and of L2t per step.
  constexpr int KC = RANK == 0 ? 32 : (RANK < 32 ? RANK : 32);
  constexpr int N_LORA = RANK == 0 ? 0 : RANK / KC;
  constexpr uint32_t LORA_ROW = KC * 2;  // bytes per row of a low-rank tile
  constexpr uint32_t LORA_SWZ = LORA_ROW == 64 ? 4u : 6u;
  constexpr uint32_t LORA_A_BYTES = BM * LORA_ROW;
  constexpr uint32_t LORA_B_BYTES = BNH * LORA_ROW;
  constexpr uint32_t LORA_LO_OFF = 8192u;  // lo plane inside the A slot
  static_assert(LORA_A_BYTES <= LORA_LO_OFF && LORA_LO_OFF + LORA_A_BYTES <= A_BYTES, "low-rank A slot");
  static_assert(LORA_B_BYTES <= B_BYTES, "low-rank B slot");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  static_assert(!(QKNR && ADD_Y), "the normalized output stage writes Y once");
  // Ring stages; a writer group meets the same (stage, step parity) pair again after
  // SF_PERIOD steps (2 ST for an odd stage count, ST for an even one).
  constexpr int ST = QKNR ? STAGES_QKNR : (MLP ? STAGES_MLP : STAGES);
  constexpr int SF_PERIOD = (ST % 2) ? 2 * ST : ST;
  static_assert(ST <= STAGES, "barrier area is sized for STAGES");
  // QKNR: the rotary rows of the tile (two 16 KiB boxes of 128 rows x 32 floats, 128B swizzle),
  // filled twice per tile (column pairs 0-31, then 32-63)
  uint8_t *rope_s = smem + ST * STAGE_BYTES;
  // MLP: the hi / lo boxes of both halves ([half][plane], 64B swizzle) and the tile's L1s boxes
  uint8_t *hbox = smem + ST * STAGE_BYTES;
  uint8_t *l1d = hbox + HBOXES_BYTES;
  uint8_t *ystage = rope_s + (QKNR ? ROPE_BYTES : 0u);
  float *bias_s = reinterpret_cast<float *>(MLP ? l1d + L1D_BYTES : ystage + YST_BYTES);
  // QKNR: each output group's copy of the Q and K normalization weights, [half][section][128]
  float *normw_s = bias_s + BN;
  // MLP: the down layer's inverse smoothing factors for the tile's 256 columns
  float *ild_s = bias_s + BN;
  uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(bias_s) + BIAS_BYTES +
                                                (QKNR ? NORMW_BYTES : (MLP ? ILD_BYTES : 0u)));
  // full[s] (used in the even CTA): stage s is loaded in both CTAs and both CTAs' scales for it
  // are in tensor memory; empty[s]: the MMAs reading stage s are done (both CTAs); accfull: the
  // accumulator is complete (both CTAs); accempty (used in the even CTA): both CTAs' output
  // stages have read it.
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_accfull = bar_empty + 8 * STAGES;
  const uint32_t bar_accempty = bar_accfull + 8;
  // sffull[s][p] (p = parity of the step): the stage's scale blocks have landed in this CTA (and,
  // by the producer's order, the MMAs that last read slot s are done). Even and odd steps have
  // barriers of their own, so each writer group waits on phases ten steps apart.
  const uint32_t bar_sf = bar_accempty + 8;
  // QKNR: rope_full (the pass's rotary rows have landed), rope_empty (the eight output warps of
  // this CTA are done reading them)
  const uint32_t bar_rope_full = bar_sf + 8 * 2 * STAGES;
  const uint32_t bar_rope_empty = bar_rope_full + 8;
  // MLP: hfull (even CTA: both CTAs' eight output warps wrote the pass's hi / lo rows), hempty (the
  // pass's down-projection MMAs are done; both CTAs), l1dfull (even CTA: the tile's L1s boxes landed
  // in both CTAs)
  // l1dfree (both CTAs: the MMAs that read the tile's L1s boxes are done; one phase per tile, so
  // the odd CTA's loader, which runs ahead of the passes, never waits on a phase two behind)
  const uint32_t bar_hfull = bar_sf + 8 * 2 * STAGES;
  const uint32_t bar_hempty = bar_hfull + 8;
  const uint32_t bar_l1dfull = bar_hempty + 8;
  const uint32_t bar_l1dfree = bar_l1dfull + 8;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + N_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();  // 0: issues the pair's MMAs; 1: its peer
  const int pid = blockIdx.x >> 1;           // pair (cluster) index
  const int npairs = gridDim.x >> 1;
  const int kblocks = a.K / 64;
  const int n_kt = FP4 ? (kblocks + 3) / 4 : 0;
  const int total = N_LORA + n_kt;  // steps per tile
  const int tiles = a.Mt * a.Nt;

  auto a_tile = [&](int s) { return smem + s * STAGE_BYTES; };
  auto b_tile = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, FULL_COUNT);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_accfull, 1);
    mbar_init(bar_accempty, ACCEMPTY_COUNT);
    for (int s = 0; s < 2 * STAGES; ++s) mbar_init(bar_sf + 8 * s, 1);
    if (QKNR) {
      mbar_init(bar_rope_full, 1);
      mbar_init(bar_rope_empty, EPI_WARPS);
    }
    if (MLP) {
      mbar_init(bar_hfull, 2 * EPI_WARPS);
      mbar_init(bar_hempty, 1);
      mbar_init(bar_l1dfull, 1);
      mbar_init(bar_l1dfree, 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and the pair's tensor memory allocated
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  // The prologue above overlaps the previous kernel of the stream; global memory only after it.
  grid_dep_wait();
  grid_dep_launch();

  if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 8) {
    setmaxnreg_inc<epi_regs<OUT>()>();
    // ------------------------------------------------------------ output stage
    // Two groups of four warps (named barriers 1 and 2), one per 128-column half of the tile;
    // the warps of a group cover the four 32-lane sub-partitions. Thread (row, half) loads
    // columns 128 half .. 128 half + 127 of its row (four 32-column chunks) into registers,
    // releases the accumulator to the next tile's MMAs, then converts and stores them.
    const int half = (warp - EPI_WARP0) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int et = (static_cast<int>(threadIdx.x) - EPI_WARP0 * 32) & 127;  // thread index in the group
    const uint32_t taddr = tbase + (static_cast<uint32_t>(quad * 32) << 16) + half * 128;
    const uint32_t accempty_lead = map_shared_rank(bar_accempty, 0);
    bool ok = true;
    uint32_t tcount = 0;
    for (int t = pid; t < tiles; t += npairs, ++tcount) {
      const int mt = t % a.Mt;
      const int nt = t / a.Mt;
      const int n0 = nt * BN;
      const int row0 = mt * BMP + static_cast<int>(crank) * BM;
      const int m = row0 + row;
      if constexpr (MLP) {
        // Fused MLP pair. h = GELU(alpha acc + b) (fp32, never rounded to 16 bits) becomes
        //  (1) the down layer's activation codes and scales: x_hat = fp32(h inv_lambda_d) quantized
        //      with s_x_d by the same group quantizer as the activation kernel (16 columns per group,
        //      the group lies in this thread's row);
        //  (2) the A operand, as the pair hi = bf16(h), lo = bf16(h - hi), of the pair MMAs that
        //      sum this tile's part of the down-projection h L1s_d in tensor memory (warp 18 of the
        //      even CTA issues them), 32 columns of the half per pass, four passes per tile.
        // After the fourth pass each thread stores its row's share of the tile's partial sums
        // (rank_d fp32 per row; half 0 the first rank_d / 2 columns) into slot nt of the partial
        // buffer, which a separate step adds in slot order.
        const int cbase = n0 + half * 128;  // first column of the half = first input channel of the down layer
        const bool lora_d = a.rank_d > 0;
        {
          const int e = half * 128 + et;
          bias_s[e] = (a.bias && n0 + e < a.N) ? __ldg(a.bias + n0 + e) : 0.0f;
          ild_s[e] = (n0 + e < a.N) ? __ldg(a.il_d + n0 + e) : 0.0f;
        }
        named_bar_sync(1 + half, 128);
        if (ok) ok = mbar_wait_parked(bar_accfull, tcount & 1, a.err, KID_GEMM, 4);
        ok = __all_sync(0xffffffffu, ok);
        uint32_t rr[4][32];
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, rr[c]);
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_wait_ld_dep(rr[c]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(accempty_lead);
        }
        const bool row_ok = m < a.M;
        const bool srow_ok = m < a.mp_scales;
        const size_t kd2 = static_cast<size_t>(a.N) / 2;  // bytes per row of the down layer's codes
        const uint32_t hfull_lead = map_shared_rank(bar_hfull, 0);
        uint8_t *hi_row = hbox + (half * 2 + 0) * HBOX_BYTES + row * 64;
        uint8_t *lo_row = hbox + (half * 2 + 1) * HBOX_BYTES + row * 64;
        const uint64_t al2 = pk2(a.alpha, a.alpha);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const int c0 = 32 * p;  // column of the half
          // h = GELU(alpha acc + b), in place of the accumulator values
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 b = *reinterpret_cast<const float2 *>(bias_s + half * 128 + c0 + 2 * e);
            const uint64_t v = fma2_rn(al2, pk2(__uint_as_float(rr[p][2 * e]), __uint_as_float(rr[p][2 * e + 1])),
                                       pk2(b.x, b.y));
            float v0, v1;
            upk2(v, v0, v1);
            rr[p][2 * e] = __float_as_uint(gelu_tanh(v0));
            rr[p][2 * e + 1] = __float_as_uint(gelu_tanh(v1));
          }
          if (lora_d) {
            // the hi / lo boxes are free once the MMAs of the previous pass are done
            const uint32_t pc = 4 * tcount + p;
            if (pc > 0 && ok)
              ok = __all_sync(0xffffffffu, mbar_wait_parked(bar_hempty, (pc - 1) & 1, a.err, KID_GEMM, 12));
            if (ok) {
#pragma unroll
              for (int c = 0; c < 4; ++c) {  // 16-byte chunk c: columns 8c .. 8c + 7, at c ^ ((row / 2) % 4)
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float x0 = __uint_as_float(rr[p][8 * c + 2 * i]), x1 = __uint_as_float(rr[p][8 * c + 2 * i + 1]);
                  hw[i] = pack_bf16x2(x0, x1);
                  lw[i] = pack_bf16x2(__fsub_rn(x0, bf16_lo(hw[i])), __fsub_rn(x1, bf16_hi(hw[i])));
                }
                const uint32_t off = static_cast<uint32_t>((c ^ ((row >> 1) & 3)) << 4);
                *reinterpret_cast<uint4 *>(hi_row + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(lo_row + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive_remote(hfull_lead);
            }
          }
          // the down layer's codes and scales of the pass's two groups
          const bool col_ok = cbase + c0 < a.N;  // N % 64 == 0: a pass lies wholly inside or outside
          uint32_t cw[4];
          uint32_t sc2 = 0;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float *ilq = ild_s + half * 128 + c0 + 16 * q;
            uint32_t w0, w1, sc;
            float eff;
            if (quant16_lean(&rr[p][16 * q], ilq, a.sx_d, a.dx_d, a.inv_dx_d, w0, w1, sc, eff)) {
              Vals16 hv;
#pragma unroll
              for (int i = 0; i < 16; ++i) hv.v[i] = __uint_as_float(rr[p][16 * q + i]);
              const uint2 c = group_codes_exact_h(hv, ilq, eff);
              w0 = c.x;
              w1 = c.y;
            }
            cw[2 * q] = w0;
            cw[2 * q + 1] = w1;
            sc2 |= sc << (8 * q);
          }
          if (ok && col_ok) {
            if (row_ok)
              *reinterpret_cast<uint4 *>(a.xq_d + static_cast<size_t>(m) * kd2 + (cbase + c0) / 2) =
                  make_uint4(cw[0], cw[1], cw[2], cw[3]);
            // padding rows of the scale buffer get zero scales, as the activation kernel writes them
            if (srow_ok)
              *reinterpret_cast<uint16_t *>(a.xs_d + scale_offset(m, (cbase + c0) / 16, a.N / 16)) =
                  static_cast<uint16_t>(row_ok ? sc2 : 0u);
          }
        }
        if (lora_d) {
          // the tile's partial down-projection: this warp's 32 rows, half `half` of the columns
          const uint32_t pc3 = 4 * tcount + 3;
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait_parked(bar_hempty, pc3 & 1, a.err, KID_GEMM, 13));
          if (ok) {
            tc_fence_after();
            const int hc = a.rank_d / 2;
            float *dst = a.part + (static_cast<size_t>(nt) * a.M + m) * a.rank_d + half * hc;
            for (int c8 = 0; c8 < hc; c8 += 8) {
              uint32_t v8[8];
              tmem_ld8(tbase + (static_cast<uint32_t>(quad * 32) << 16) + LA_COL0 + half * hc + c8, v8);
              tmem_wait_ld();
              if (row_ok) {
                *reinterpret_cast<float4 *>(dst + c8) = make_float4(__uint_as_float(v8[0]), __uint_as_float(v8[1]),
                                                                   __uint_as_float(v8[2]), __uint_as_float(v8[3]));
                *reinterpret_cast<float4 *>(dst + c8 + 4) = make_float4(
                    __uint_as_float(v8[4]), __uint_as_float(v8[5]), __uint_as_float(v8[6]), __uint_as_float(v8[7]));
              }
            }
            // the next tile's first down-projection MMA overwrites the partial: these reads come
            // before this warp's next arrival on hfull
            tc_fence_before();
          }
        }
        named_bar_sync(1 + half, 128);  // the group is done with this tile's bias_s / ild_s
      } else if constexpr (!ADD_Y) {
        // The group owns one staging box (128 rows x 64 columns, 16-byte chunk k of row r at
        // k ^ (r % 8)) and fills it twice per tile: columns 0-63 of its half, then 64-127.
        // The accumulator is released as soon as all four 32-column chunks are in registers.
        uint8_t *rowp = ystage + half * (BM * 128) + row * 128;
        auto convert_store = [&](const uint32_t(&v32)[32], int colh) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ch = ((colh & 63) >> 3) + q;
            const float4 b0 = *reinterpret_cast<const float4 *>(bias_s + half * 128 + colh + 8 * q);
            const float4 b1 = *reinterpret_cast<const float4 *>(bias_s + half * 128 + colh + 8 * q + 4);
            float v[8];
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              v[e] = fmaf(a.alpha, __uint_as_float(v32[8 * q + e]), bb[e]);
              if constexpr (GELU) v[e] = gelu_tanh(v[e]);
            }
            const uint32_t p0 = pack_bf16x2(v[0], v[1]);
            const uint32_t p1 = pack_bf16x2(v[2], v[3]);
            const uint32_t p2 = pack_bf16x2(v[4], v[5]);
            const uint32_t p3 = pack_bf16x2(v[6], v[7]);
            *reinterpret_cast<uint4 *>(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(p0, p1, p2, p3);
          }
        };
        // Fused QKV output stage: the half's 128 columns are one head. For a Q or K head,
        // u = v w / sqrt(mean(v^2) + eps) with v = alpha acc + bias (fp32, before any 16-bit
        // rounding), then each column pair (2i, 2i + 1) turns by the token's angle for pair i.
        auto bias_sumsq = [&](uint32_t(&v32)[32], int colh) {
          const uint64_t al2 = pk2(a.alpha, a.alpha);
          uint64_t sq0 = 0, sq1 = 0;  // packed (+0, +0)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 b = *reinterpret_cast<const float2 *>(bias_s + half * 128 + colh + 2 * e);
            const uint64_t v = fma2_rn(al2, pk2(__uint_as_float(v32[2 * e]), __uint_as_float(v32[2 * e + 1])),
                                       pk2(b.x, b.y));
            float lo, hi;
            upk2(v, lo, hi);
            v32[2 * e] = __float_as_uint(lo);
            v32[2 * e + 1] = __float_as_uint(hi);
            if (e & 1) sq1 = fma2_rn(v, v, sq1);
            else sq0 = fma2_rn(v, v, sq0);
          }
          float a0, a1, b0, b1;
          upk2(sq0, a0, a1);
          upk2(sq1, b0, b1);
          return (a0 + a1) + (b0 + b1);
        };
        // The pair's (cos, sin) of the token come from the staged rotary rows: box (colh & 63) / 32
        // of the current pass holds pairs 16 ((colh & 63) / 32) .. + 15 of each row, 16-byte
        // chunk k of row r at k ^ (r % 8).
        const uint32_t rope_row = smem_u32(rope_s) + row * 128;
        auto qk_store = [&](const uint32_t(&v32)[32], int colh, int sec, float inv) {
          const float *w = normw_s + (half * 2 + sec) * 128 + colh;
          const uint32_t rb = rope_row + ((colh & 63) >> 5) * (ROPE_BYTES / 2);
          const uint64_t inv2 = pk2(inv, inv);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ch = ((colh & 63) >> 3) + q;
            const uint4 c0 = ld_shared_u32x4(rb + (((2 * q) ^ (row & 7)) << 4));
            const uint4 c1 = ld_shared_u32x4(rb + (((2 * q + 1) ^ (row & 7)) << 4));
            const float4 w0 = *reinterpret_cast<const float4 *>(w + 8 * q);
            const float4 w1 = *reinterpret_cast<const float4 *>(w + 8 * q + 4);
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            const uint32_t cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t p[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              // (u0, u1) = (v0, v1) inv w;  z = (u0 c - u1 s, u1 c + u0 s)
              const uint64_t u = mul2_rn(mul2_rn(pk2(__uint_as_float(v32[8 * q + 2 * i]),
                                                     __uint_as_float(v32[8 * q + 2 * i + 1])), inv2),
                                         pk2(wv[2 * i], wv[2 * i + 1]));
              const float c = __uint_as_float(cs[2 * i]), sn = __uint_as_float(cs[2 * i + 1]);
              float u0, u1;
              upk2(u, u0, u1);
              const uint64_t z = fma2_rn(pk2(u1, u0), pk2(-sn, sn), mul2_rn(u, pk2(c, c)));
              float z0, z1;
              upk2(z, z0, z1);
              p[i] = pack_bf16x2(z0, z1);
            }
            *reinterpret_cast<uint4 *>(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(p[0], p[1], p[2], p[3]);
          }
        };
        // A pass of rotary rows: every output warp waits for it (so that no early arrival on
        // rope_empty can let the filler start the next pass over rows still being read) and
        // reports once it is done with it. Pass A (pairs 0-31) has phase parity 0, pass B 1.
        // Tiles whose two heads both lie in V get no rotary passes (the filler skips them too).
        const bool rope_tile = QKNR && n0 < 2 * a.qk_width;
        auto rope_wait = [&](uint32_t parity) {
          if (rope_tile && ok) ok = __all_sync(0xffffffffu, mbar_wait_parked(bar_rope_full, parity, a.err, KID_GEMM, 10));
        };
        auto rope_done = [&]() {
          if (rope_tile && ok) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_rope_empty);
          }
        };
        auto store_box = [&](int colh) {
          fence_proxy_async_smem();
          named_bar_sync(1 + half, 128);
          if (et == 0) {
            if (row0 < a.M && n0 + half * 128 + colh < a.N)
              tma_store_2d(&tm_y, smem_u32(ystage + half * (BM * 128)), n0 + half * 128 + colh, row0);
            bulk_commit();
          }
        };
        // the group's previous TMA store has finished reading the box, and its threads are done
        // with the previous bias values
        if (et == 0) bulk_wait_read0();
        {
          const int e = half * 128 + et;
          bias_s[e] = (a.bias && n0 + e < a.N) ? __ldg(a.bias + n0 + e) : 0.0f;
          if (QKNR && tcount == 0) {
            normw_s[(half * 2 + 0) * 128 + et] = __ldg(a.norm_q + et);
            normw_s[(half * 2 + 1) * 128 + et] = __ldg(a.norm_k + et);
          }
        }
        named_bar_sync(1 + half, 128);
        // section of this half's head: 0 Q, 1 K (normalized and rotated), 2 V
        const int sec = QKNR ? (n0 + half * 128) / a.qk_width : 2;
        float inv = 0.0f;
        // pass A of the tile's rotary rows is loaded while the tile's MMAs run: wait for it
        // before the accumulator's 128 columns take up the registers
        rope_wait(0);
        if (ok) ok = mbar_wait_parked(bar_accfull, tcount & 1, a.err, KID_GEMM, 4);
        ok = __all_sync(0xffffffffu, ok);
        uint32_t r0[32], r1[32], r2[32], r3[32];
        if (ok) {
          tc_fence_after();
          tmem_ld32(taddr, r0);
          tmem_ld32(taddr + 32, r1);
          tmem_ld32(taddr + 64, r2);
          tmem_ld32(taddr + 96, r3);
          tmem_wait_ld_dep(r0);
          tmem_wait_ld_dep(r1);
          tmem_wait_ld_dep(r2);
          tmem_wait_ld_dep(r3);
          // every column of this warp's rows is in registers: release the accumulator
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(accempty_lead);
          if (QKNR && sec < 2) {
            const float ss = (bias_sumsq(r0, 0) + bias_sumsq(r1, 32)) + (bias_sumsq(r2, 64) + bias_sumsq(r3, 96));
            inv = __frsqrt_rn(__fadd_rn(__fmul_rn(ss, 1.0f / 128.0f), a.eps));
            qk_store(r0, 0, sec, inv);
            qk_store(r1, 32, sec, inv);
          } else {
            convert_store(r0, 0);
            convert_store(r1, 32);
          }
          rope_done();
        }
        store_box(0);
        // the first store has finished reading the box
        if (et == 0) bulk_wait_read0();
        named_bar_sync(1 + half, 128);
        if (ok) {
          rope_wait(1);
          if (QKNR && sec < 2) {
            if (ok) {
              qk_store(r2, 64, sec, inv);
              qk_store(r3, 96, sec, inv);
            }
          } else {
            convert_store(r2, 64);
            convert_store(r3, 96);
          }
          rope_done();
        }
        store_box(64);
      } else {
        // Unfused up-projection: Y = bf16(Y + alpha * acc), one 32-column chunk at a time.
        if (ok) ok = mbar_wait_parked(bar_accfull, tcount & 1, a.err, KID_GEMM, 4);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_wait_ld_dep(r);
          if (c == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(accempty_lead);
          }
          const int n = n0 + half * 128 + c * 32;
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
    if (!ADD_Y && !MLP && et == 0) bulk_wait0();  // stores complete before the CTA exits
  } else {
    setmaxnreg_dec<other_regs<OUT>()>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
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
        for (int t = pid; t < tiles && ok; t += npairs) {
          const int mt = t % a.Mt;
          const int nt = t / a.Mt;
          const int row0 = mt * BMP + static_cast<int>(crank) * BM;  // this CTA's rows of X
          const int wrow0 = nt * BN + static_cast<int>(crank) * BNH;  // this CTA's rows of W
          for (int j = 0; j < total; ++j, ++it) {
            const int s = it % ST;
            // parked rather than spinning: the spinning loop's instructions cost the MMA warp
            // issue slots and the SM power, and under the power cap the step ran faster parked
            if (it >= ST && !mbar_wait_parked(bar_empty + 8 * s, ((it / ST) - 1) & 1, a.err, KID_GEMM, 1)) {
              ok = false;
              break;
            }
            const uint32_t fb = bar_full + 8 * s;
            const uint32_t fb_lead = map_shared_rank(fb, 0);
            const uint32_t at = smem_u32(a_tile(s));
            const uint32_t bt = smem_u32(b_tile(s));
            if (j < N_LORA) {
              mbar_arrive(bar_sf + 8 * (2 * s + (it & 1)));  // no scales for a low-rank step; the phase still advances
              if (crank == 0) mbar_arrive_expect_tx(fb, 2 * (2 * LORA_A_BYTES + LORA_B_BYTES));
              tma_load_2d_pair(at, &tm_la, j * KC, row0, fb_lead);
              tma_load_2d_pair(at + LORA_LO_OFF, &tm_la, RANK + j * KC, row0, fb_lead);
              tma_load_2d_pair(bt, &tm_l2, j * KC, wrow0, fb_lead);
            } else {
              const int kt = j - N_LORA;
              const int kbv = min(4, kblocks - 4 * kt);
              const int mb = 2 * mt + static_cast<int>(crank);  // this CTA's 128-row block of X
              const bool rows_ok = mb * BM < a.M;               // activation scales cover ceil(M / 128) blocks
              const uint32_t sfb = bar_sf + 8 * (2 * s + (it & 1));
              const uint32_t blk = static_cast<uint32_t>(kbv) * SF_BLOCK;
              mbar_arrive_expect_tx(sfb, (rows_ok ? 3u : 2u) * blk);
              if (rows_ok)
                bulk_load(at + SF_OFF, a.xs + (static_cast<size_t>(mb) * kblocks + 4 * kt) * SF_BLOCK, blk, sfb);
              bulk_load(at + SF_OFF + 4 * SF_BLOCK, a.ws + (static_cast<size_t>(2 * nt) * kblocks + 4 * kt) * SF_BLOCK,
                        blk, sfb);
              bulk_load(at + SF_OFF + 8 * SF_BLOCK,
                        a.ws + (static_cast<size_t>(2 * nt + 1) * kblocks + 4 * kt) * SF_BLOCK, blk, sfb);
              if (crank == 0) mbar_arrive_expect_tx(fb, 2 * (A_BYTES + B_BYTES));
              tma_load_2d_pair(at, &tm_xq, kt * 128, row0, fb_lead);
              tma_load_2d_pair(bt, &tm_wq, kt * 128, wrow0, fb_lead);
            }
          }
        }
        // The MMA issuer's last commits to this CTA's empty barriers have landed before it exits.
        for (uint32_t i = it > ST ? it - ST : 0; ok && i < it; ++i)
          ok = mbar_wait(bar_empty + 8 * (i % ST), (i / ST) & 1, a.err, KID_GEMM, 7);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer (even CTA)
      // The whole warp runs the loops, so the descriptor arithmetic stays warp-uniform (no
      // per-instruction register moves); one elected lane issues the MMAs and their commits.
      if (crank == 0) {
        // kind::mxf4nvf4: A, B e2m1 (bits 7-9, 10-12 = 1), K-major, N = 256 (bits 17-22),
        // scale type ue4m3 (bit 23 = 0), M = 256 across the pair (bits 24-28), scale ids 0, K = 64.
        const uint32_t idesc_fp4 = (1u << 7) | (1u << 10) | ((uint32_t(BN) >> 3) << 17) | ((uint32_t(BMP) >> 4) << 24);
        // kind::f16: D fp32, A, B bf16, N = 256, M = 256 across the pair.
        const uint32_t idesc_bf16 =
            (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t(BN) >> 3) << 17) | ((uint32_t(BMP) >> 4) << 24);
        uint32_t it = 0;
        uint32_t tcount = 0;
        bool ok = true;
        for (int t = pid; t < tiles && ok; t += npairs, ++tcount) {
          if (tcount > 0 && !__all_sync(0xffffffffu, mbar_wait(bar_accempty, (tcount - 1) & 1, a.err, KID_GEMM, 2))) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int j = 0; j < total; ++j, ++it) {
            const int s = it % ST;
            const uint32_t par = (it / ST) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, par, a.err, KID_GEMM, 3))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(a_tile(s));
            if (j < N_LORA) {
              const uint64_t ad = umma_desc(st, 16, 8 * LORA_ROW, LORA_SWZ);
              const uint64_t ald = umma_desc(st + LORA_LO_OFF, 16, 8 * LORA_ROW, LORA_SWZ);
              const uint64_t bd = umma_desc(st + A_BYTES, 16, 8 * LORA_ROW, LORA_SWZ);
              if (elect_one()) {
  #pragma unroll
                for (int k = 0; k < KC / 16; ++k) {
                  mma_bf16_pair(tbase, ad + 2u * k, bd + 2u * k, idesc_bf16, (j | k) != 0 ? 1u : 0u);
                  mma_bf16_pair(tbase, ald + 2u * k, bd + 2u * k, idesc_bf16, 1u);
                }
                tc_commit_pair_mc(bar_empty + 8 * s, 0x3);
              }
            } else {
              const int kt = j - N_LORA;
              const int kbv = min(4, kblocks - 4 * kt);
              const uint32_t tsf = tbase + SF_COL0 + SF_COLS * s;
              const uint64_t ad = umma_desc(st, 16, 1024, 2);
              const uint64_t bd = umma_desc(st + A_BYTES, 16, 1024, 2);
              if (elect_one()) {
                // activation scales: the copy unit replicates each CTA's 512-byte block into its
                // four sub-partitions, in order with (and overlapping) the MMAs
                for (int kb = 0; kb < kbv; ++kb) {
                  tmem_cp_32x128b_x4_pair(tsf + 4 * kb, umma_desc(st + SF_OFF + SF_BLOCK * kb, 0, 128, 0));
                  mma_nvfp4_pair(tbase, ad + 2u * kb, bd + 2u * kb, idesc_fp4, tsf + 4 * kb, tsf + 16 + 8 * kb,
                                 (j | kb) != 0 ? 1u : 0u);
                }
                tc_commit_pair_mc(bar_empty + 8 * s, 0x3);
              }
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) tc_commit_pair_mc(bar_accfull, 0x3);
          __syncwarp();
        }
        // both CTAs' output stages have released the last accumulator
        if (ok && tcount > 0) mbar_wait(bar_accempty, (tcount - 1) & 1, a.err, KID_GEMM, 8);
      }
    } else if (QKNR && warp == 18) {
      // ------------------------------------------------------------ rotary-row filler (QKNR)
      // Per tile two passes over this CTA's 128 rows of the (cos, sin) table: pairs 0-31 for
      // the output stage's first box of columns, then pairs 32-63. A pass reuses the buffer once
      // the eight output warps have read the previous one; the first pass of a tile is loaded
      // while the tile's MMAs run. Rows beyond M are filled with zeros by the copy (never stored).
      if (lane == 0) {
        tma_prefetch_desc(&tm_rope);
        const uint32_t rs = smem_u32(rope_s);
        uint32_t pass = 0;
        bool ok = true;
        for (int t = pid; t < tiles && ok; t += npairs) {
          const int row0 = (t % a.Mt) * BMP + static_cast<int>(crank) * BM;
          if ((t / a.Mt) * BN >= 2 * a.qk_width) continue;  // both heads in V: no rotation
          for (int ph = 0; ph < 2; ++ph, ++pass) {
            if (pass > 0 && !mbar_wait(bar_rope_empty, (pass - 1) & 1, a.err, KID_GEMM, 9)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar_rope_full, ROPE_BYTES);
            tma_load_2d(rs, &tm_rope, 64 * ph, row0, bar_rope_full);
            tma_load_2d(rs + ROPE_BYTES / 2, &tm_rope, 64 * ph + 32, row0, bar_rope_full);
          }
        }
        // the last pass has landed before the CTA can exit
        if (pass > 0) mbar_wait(bar_rope_full, (pass - 1) & 1, a.err, KID_GEMM, 11);
      }
    } else if (MLP && warp == 18) {
      // ------------------------------------------------------------ down-projection (MLP)
      // Per tile: both CTAs load their half of the down layer's L1s for the tile's 256 columns
      // (eight boxes of 32 columns x rank_d / 2 rows, 64B swizzle; counted on the even CTA's
      // l1dfull), once the MMAs that read the previous tile's boxes are done (l1dfree, committed
      // after each tile's fourth pass; a wait on hempty, four phases a tile, could return early in
      // the odd CTA, whose loader runs ahead: tests/test_mlp_down_protocol.py models both). In the even CTA the
      // warp then issues, per pass of 32 columns, the pair MMAs  D += hi L1s + lo L1s  (M = 256 across
      // the pair, N = rank_d, K = 16 each; both halves' boxes) and commits them to hempty in both
      // CTAs. D sits in columns LA_COL0.. of tensor memory; the first MMA of a tile starts it afresh.
      if (a.rank_d > 0) {
        const uint32_t hcr = static_cast<uint32_t>(a.rank_d) / 2;  // rows of L1s per CTA
        const uint32_t box = hcr * 64u;
        const uint32_t l1d_lead = map_shared_rank(bar_l1dfull, 0);
        // kind::f16: D fp32, A and B bf16, K-major, N = rank_d, M = 256 across the pair
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(a.rank_d) >> 3) << 17) |
                               ((uint32_t(BMP) >> 4) << 24);
        if (elect_one()) tma_prefetch_desc(&tm_aux);
        __syncwarp();
        uint32_t tcount = 0;
        bool ok = true;
        for (int t = pid; t < tiles && ok; t += npairs, ++tcount) {
          const int nt = t / a.Mt;
          if (tcount > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_l1dfree, (tcount - 1) & 1, a.err, KID_GEMM, 14));
            if (!ok) break;
          }
          if (elect_one()) {
            if (crank == 0) mbar_arrive_expect_tx(bar_l1dfull, 2u * 8u * box);
            for (int j = 0; j < 8; ++j)
              tma_load_2d_pair(smem_u32(l1d) + j * box, &tm_aux, nt * BN + 32 * j, static_cast<int>(crank * hcr),
                               l1d_lead);
          }
          __syncwarp();
          if (crank != 0) continue;
          ok = __all_sync(0xffffffffu, mbar_wait(bar_l1dfull, tcount & 1, a.err, KID_GEMM, 15));
          if (!ok) break;
          for (int p = 0; p < 4 && ok; ++p) {
            const uint32_t pc = 4 * tcount + p;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_hfull, pc & 1, a.err, KID_GEMM, 16));
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const uint64_t ahi = umma_desc(smem_u32(hbox) + (2 * hh) * HBOX_BYTES, 16, 512, 4);
                const uint64_t alo = umma_desc(smem_u32(hbox) + (2 * hh + 1) * HBOX_BYTES, 16, 512, 4);
                const uint64_t bd = umma_desc(smem_u32(l1d) + (4 * hh + p) * box, 16, 512, 4);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                  mma_bf16_pair(tbase + LA_COL0, ahi + 2u * k, bd + 2u * k, idesc, (p | hh | k) != 0 ? 1u : 0u);
                  mma_bf16_pair(tbase + LA_COL0, alo + 2u * k, bd + 2u * k, idesc, 1u);
                }
              }
              tc_commit_pair_mc(bar_hempty, 0x3);
              if (p == 3) tc_commit_pair_mc(bar_l1dfree, 0x3);
            }
            __syncwarp();
          }
        }
        // the last commit has arrived (in this CTA) before the CTA can exit
        if (ok && tcount > 0) mbar_wait(bar_l1dfree, (tcount - 1) & 1, a.err, KID_GEMM, 17);
      }
    } else if ((warp >= 2 && warp < EPI_WARP0) || warp == 16 || warp == 17) {
      // ------------------------------------------------------------ scale-factor writers
      // Warp (q, h) writes tensor-memory lanes 32 q .. 32 q + 31 for the steps of parity h (two
      // groups, so each warp's shared-memory reads, which queue behind the MMA operand reads and
      // the TMA fills, have two steps of time): lane i moves the 16-byte line i of the tile's two
      // weight blocks (8 columns) of each k-block from the stage's scale region into the step's
      // slot. Every step (low-rank ones too) is announced on the even CTA's full barrier by the
      // four warps of its group.
      const int h = (warp >= 2 && warp < 6) ? 0 : 1;  // warps 2..5 take the even steps, 6, 7, 16, 17 the odd ones
      const uint32_t full_lead = map_shared_rank(bar_full, 0);
      const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const int my_tiles = tiles > pid ? (tiles - 1 - pid) / npairs + 1 : 0;
      const int nsteps = my_tiles * total;
      for (int step = h; step < nsteps; step += 2) {
        const int s = step % ST;
        const int j = step % total;
        // sffull of this step: its scale blocks are in shared memory and slot s is free (parked,
        // as the producer's wait)
        if (!__all_sync(0xffffffffu, mbar_wait_parked(bar_sf + 8 * (2 * s + h), (step / SF_PERIOD) & 1, a.err, KID_GEMM, 6)))
          break;
        if (FP4 && j >= N_LORA) {
          const int kt = j - N_LORA;
          const int kbv = min(4, kblocks - 4 * kt);
          const uint32_t sft = smem_u32(a_tile(s)) + SF_OFF + lane * 16;
          const uint32_t tsf = tbase + lane_base + SF_COL0 + SF_COLS * s;
  #pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t sb[16];
  #pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int kb = 2 * hh + e;
              uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
              if (kb < kbv) {
                v0 = ld_shared_u32x4(sft + (4 + kb) * SF_BLOCK);
                v1 = ld_shared_u32x4(sft + (8 + kb) * SF_BLOCK);
              }
              sb[8 * e + 0] = v0.x; sb[8 * e + 1] = v0.y; sb[8 * e + 2] = v0.z; sb[8 * e + 3] = v0.w;
              sb[8 * e + 4] = v1.x; sb[8 * e + 5] = v1.y; sb[8 * e + 6] = v1.z; sb[8 * e + 7] = v1.w;
            }
            // slot columns: SFB k-block kb at 16 + 8 kb (rows 0-127, then 128-255); the SFA
            // columns (4 kb) are filled by the MMA issuer's copies
            tmem_st16(tsf + 16 + 16 * hh, sb);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(full_lead + 8 * s);
      }
    }
  }

  __syncthreads();
  tc_fence_before();
  cluster_sync_all();  // neither CTA frees the pair's tensor memory while the other still uses it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, TMEM_COLS);
  }
}

// Pairs that can be resident at once (clusters of two, one CTA per SM), per device.
template <int OUT>
constexpr uint32_t smem_bytes() {
  return OUT == OUT_QKNR ? SMEM_QKNR : (OUT == OUT_MLP ? SMEM_MLP : SMEM);
}

template <int RANK, bool FP4, int OUT>
int pair_slots(cudaError_t *err) {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return 0;
  }
  if (cache[dev] > 0) return cache[dev];
  auto kern = k2_gemm_w4a4_lora_up<RANK, FP4, OUT>;
  constexpr uint32_t smem = smem_bytes<OUT>();
  // setmaxnreg.inc would wait forever for registers the block was not launched with: the split
  // must fit the pool of the compiled kernel (registers per thread x threads).
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
      static_cast<uint32_t>(fa.numRegs) * THREADS < reg_pool_needed<OUT>() ||
      static_cast<uint32_t>(fa.numRegs) > epi_regs<OUT>() || static_cast<uint32_t>(fa.numRegs) < other_regs<OUT>()) {
    *err = cudaErrorLaunchOutOfResources;
    return 0;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) {
    *err = e;
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
  if (e != cudaSuccess || n <= 0) {
    *err = e != cudaSuccess ? e : cudaErrorLaunchOutOfResources;
    return 0;
  }
  cache[dev] = n;
  return n;
}

template <int RANK, bool FP4, int OUT>
cudaError_t launch_t(const GemmLaunch &g) {
  cudaError_t e = cudaSuccess;
  const int slots = pair_slots<RANK, FP4, OUT>(&e);
  if (slots <= 0) return e;
  GArgs a{};
  a.xs = g.xs;
  a.ws = g.ws;
  a.bias = g.bias;
  a.Y = g.Y;
  a.M = g.M;
  a.N = g.N;
  a.K = g.K;
  a.Mt = (g.M + BMP - 1) / BMP;
  a.Nt = (g.N + BN - 1) / BN;
  a.alpha = g.alpha;
  a.err = g.err;
  a.norm_q = g.norm_q;
  a.norm_k = g.norm_k;
  a.qk_width = g.qk_width;
  a.eps = g.eps;
  a.il_d = g.il_d;
  a.sx_d = g.sx_d;
  a.dx_d = 6.0f * g.sx_d;
  a.inv_dx_d = 1.0f / a.dx_d;
  a.rank_d = g.rank_d;
  a.mp_scales = g.mp_scales;
  a.xq_d = g.xq_d;
  a.xs_d = g.xs_d;
  a.part = g.part;
  const int tiles = a.Mt * a.Nt;
  const int pairs = tiles < slots ? tiles : slots;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<OUT>();
  cfg.stream = g.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const CUtensorMap &aux = OUT == OUT_QKNR ? g.tm_rope : (OUT == OUT_MLP ? g.tm_l1d : g.tm_y);
  return cudaLaunchKernelEx(&cfg, k2_gemm_w4a4_lora_up<RANK, FP4, OUT>, g.tm_xq, g.tm_wq, g.tm_la, g.tm_l2, g.tm_y,
                            aux, a);
}

template <bool FP4, int OUT>
cudaError_t launch_rank(const GemmLaunch &g) {
  switch (g.rank) {
    case 0:
      if constexpr (FP4) return launch_t<0, FP4, OUT>(g);
      return cudaErrorInvalidValue;
    case 16: return launch_t<16, FP4, OUT>(g);
    case 32: return launch_t<32, FP4, OUT>(g);
    case 64: return launch_t<64, FP4, OUT>(g);
    case 128: return launch_t<128, FP4, OUT>(g);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch &g) {
  if (!g.fp4) return g.add_y ? launch_rank<false, OUT_ADDY>(g) : cudaErrorInvalidValue;
  if (g.add_y) return cudaErrorInvalidValue;
  if (g.mlp) return launch_rank<true, OUT_MLP>(g);
  if (g.qk_norm_rope) return launch_rank<true, OUT_QKNR>(g);
  if (g.gelu) return launch_rank<true, OUT_GELU>(g);
  return launch_rank<true, OUT_PLAIN>(g);
}

// Down layer's low-rank branch from the fused MLP pair's partial sums: lora_act[m] = [hi | lo] of
// v = fp32(sum over slots s = 0 .. n_slots - 1, in that order, of part[s][m][:]) * inv_alpha.
__global__ void k_lora_reduce(const float *part, int n_slots, int M, int rank, float inv_alpha, uint16_t *lora_act) {
  const int quads = rank / 4;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= M * quads) return;
  const int m = idx / quads;
  const int c = 4 * (idx % quads);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const size_t stride = static_cast<size_t>(M) * rank;
  const float *p = part + static_cast<size_t>(m) * rank + c;
  for (int s = 0; s < n_slots; ++s, p += stride) {
    const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  const float v0 = __fmul_rn(acc.x, inv_alpha), v1 = __fmul_rn(acc.y, inv_alpha);
  const float v2 = __fmul_rn(acc.z, inv_alpha), v3 = __fmul_rn(acc.w, inv_alpha);
  const uint32_t h01 = pack_bf16x2(v0, v1), h23 = pack_bf16x2(v2, v3);
  const uint32_t l01 = pack_bf16x2(__fsub_rn(v0, bf16_lo(h01)), __fsub_rn(v1, bf16_hi(h01)));
  const uint32_t l23 = pack_bf16x2(__fsub_rn(v2, bf16_lo(h23)), __fsub_rn(v3, bf16_hi(h23)));
  uint16_t *out = lora_act + static_cast<size_t>(m) * (2 * rank) + c;
  *reinterpret_cast<uint2 *>(out) = make_uint2(h01, h23);
  *reinterpret_cast<uint2 *>(out + rank) = make_uint2(l01, l23);
}

cudaError_t launch_lora_reduce(const float *part, int n_slots, int M, int rank, float inv_alpha, uint16_t *lora_act,
                               cudaStream_t st) {
  const int n = M * (rank / 4);
  k_lora_reduce<<<(n + 255) / 256, 256, 0, st>>>(part, n_slots, M, rank, inv_alpha, lora_act);
  return cudaGetLastError();
}

int gemm_n_tiles(int N) { return (N + BN - 1) / BN; }

}  // namespace svdq
