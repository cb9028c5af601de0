// Internal launch interfaces between the C ABI layer (api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace svdq {

// K1 (and the unfused down-projection / quantize baselines).
// Rows per K1 tile: the TMA box height of X and the M of its tensor-core down-projection.
constexpr int kQuantRows = 64;
struct QuantLaunch {
  CUtensorMap tm_x;   // X, bf16 [M, K], box 64 x kQuantRows, 128B swizzle
  CUtensorMap tm_l1;  // L1t, bf16 [rank, K], box 64 x rank, 128B swizzle (unused at rank 0)
  const float *inv_lambda;
  uint8_t *xq;
  uint8_t *xs;
  uint16_t *lora_act;
  int M, K, rank;
  float s_x, d_x, inv_alpha;
  int splits;            // CTAs along K per 128-row tile (cluster size)
  int chunks_per_split;  // 64-column chunks per CTA
  bool quantize;         // write xq / xs
  bool lora;             // compute the down-projection
  uint32_t *err;
  cudaStream_t stream;
};
cudaError_t launch_quant_act(const QuantLaunch &q);
// Cluster size (CTAs along K per row tile) for K1 on the current device.
int quant_act_splits(int M, int K, int rank, bool quantize, bool lora, int num_sms);

// K2 (and the unfused 4-bit GEMM / up-projection baselines).
struct GemmLaunch {
  CUtensorMap tm_xq;  // xq, u8 [M, K/2], box 128 x 128, 128B swizzle
  CUtensorMap tm_wq;  // wq, u8 [N, K/2], box 128 x 128 (half a pair tile), 128B swizzle
  CUtensorMap tm_la;  // lora_act, bf16 [M, 2 rank] (hi | lo planes), box kc x 128
  CUtensorMap tm_l2;  // L2t, bf16 [N, rank], box kc x 128 (half a pair tile)
  CUtensorMap tm_y;   // Y, bf16 [M, N], box 64 x 128, 128B swizzle (output stores)
  CUtensorMap tm_rope;  // rotary table, fp32 [M, 128], box 32 x 128, 128B swizzle (QKNR only)
  const uint8_t *xs;  // activation scales (block layout, ceil(M / 128) row blocks)
  const uint8_t *ws;  // weight scales (block layout, rows padded to 256)
  const float *bias;
  uint16_t *Y;
  int M, N, K, rank;
  float alpha;
  bool fp4;    // run the block-scaled 4-bit product
  bool add_y;  // Y = bf16(Y + alpha * acc) instead of bf16(alpha * acc + bias)
  // Fused QKV output stage: per-head RMS normalization and rotary embedding of the Q and K
  // sections of Y = [Q | K | V] (head_dim 128, qk_width = heads x 128 columns per section).
  bool qk_norm_rope;
  const float *norm_q, *norm_k;  // [128] each
  int qk_width;
  float eps;
  bool gelu;  // H = bf16(GELU(alpha acc + bias)) instead of Y (first layer of an unfused MLP pair)
  // Fused MLP pair: GELU(alpha acc + bias) quantized for the down layer (codes, block scales with
  // mp_scales rows) plus fp32 partial down-projections [ceil(N / 256)][M][rank_d] against L1t_d.
  bool mlp;
  CUtensorMap tm_l1d;  // L1t_d, bf16 [rank_d, N], box 32 x rank_d / 2, 64B swizzle
  const float *il_d;
  float sx_d;
  int rank_d, mp_scales;
  uint8_t *xq_d, *xs_d;
  float *part;
  int num_sms;
  uint32_t *err;
  cudaStream_t stream;
};
cudaError_t launch_gemm(const GemmLaunch &g);
// Column tiles of K2 (256 rows of W each): the number of partial-sum slots of the fused MLP pair.
int gemm_n_tiles(int N);
// lora_act = [hi | lo] of (sum over n_slots slots of part[slot][m][:], in slot order) * inv_alpha.
cudaError_t launch_lora_reduce(const float *part, int n_slots, int M, int rank, float inv_alpha, uint16_t *lora_act,
                               cudaStream_t st);

// Unfused per-head Q/K normalization and rotary embedding of a bf16 Y = [Q | K | V], in place.
cudaError_t launch_qk_norm_rope(uint16_t *Y, int M, int heads, const float *norm_q, const float *norm_k,
                                const float *rope, float eps, cudaStream_t st);

// awq_w4a16 (awq.cu): int4 weights in groups of 64 with fp16 scales and zero points.
int awq_max_tokens();
size_t awq_smem_bytes(int M, int K);
size_t awq_packed_weight_bytes(int N, int K);
size_t awq_packed_sz_bytes(int N, int K);
cudaError_t launch_awq_quantize(const float *W, int N, int K, uint8_t *wq, uint16_t *scales, uint8_t *zeros,
                                cudaStream_t st);
cudaError_t launch_awq_pack(const uint8_t *wq, const uint16_t *scales, const uint8_t *zeros, int N, int K, uint8_t *wt,
                            uint8_t *szt, cudaStream_t st);
cudaError_t launch_awq_gemv(const uint16_t *X, int M, const uint8_t *wt, const uint8_t *szt, const float *bias, int N,
                            int K, uint16_t *Y, uint32_t *err, cudaStream_t st);

// Failure-path self-test (selftest.cu): bounded waits on an mbarrier nobody signals.
cudaError_t launch_selftest_wait(uint32_t *err, uint64_t limit_ns, cudaStream_t st);

// Offline preparation pieces (prepare.cu).
cudaError_t launch_col_absmax_f32(const float *A, int rows, int cols, float *out, cudaStream_t st);
cudaError_t launch_col_absmax_bf16(const uint16_t *A, int rows, int cols, float *out, cudaStream_t st);
cudaError_t launch_quantize_rows(const float *A, int rows, int K, float s, uint8_t *codes, uint8_t *scales,
                                 cudaStream_t st);

}  // namespace svdq

namespace svdq {

enum PrepStatus { PREP_OK = 0, PREP_CUDA, PREP_NO_SOLVER, PREP_SOLVER_FAILED, PREP_INTERNAL };

struct PrepPlan {
  int n_g = 0, side = 0, lwork = 0;
  size_t off_G = 0, off_evals = 0, off_V = 0, off_P = 0, off_Q = 0, off_sig = 0, off_R = 0, off_aw = 0, off_lam = 0,
         off_scal = 0, off_info = 0, off_work = 0, bytes = 0;
};

struct PrepArgs {
  const float *W;
  const float *act_absmax;
  int N, K, rank;
  PrepPlan plan;
  void *workspace;
  float *lambda_out;  // may be null
  float *inv_lambda;
  uint16_t *L1t, *L2t;
  uint8_t *wq, *wscales;
  size_t wscale_bytes;
  float *s_w, *s_x;  // host outputs
  float *R_out_host = nullptr;  // host, N x K: the fp32 residual the weight quantizer read (may be null)
  cudaStream_t stream;
};

PrepStatus prepare_plan(int N, int K, int rank, PrepPlan *plan);

// Smoothing stage with its scratch in a static device array (no allocation); K <= noalloc_max_k().
int noalloc_max_k();
cudaError_t smoothing_noalloc(const float *W, const float *act_absmax, int N, int K, float *lambda,
                              float *inv_lambda, float *x_tensor_scale, cudaStream_t st);
PrepStatus prepare_run(const PrepArgs &p);

}  // namespace svdq
