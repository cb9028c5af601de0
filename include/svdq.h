/*
 * libsvdq — SVDQuant NVFP4 W4A4 + low-rank linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer computes   Y = Q(X_hat) Q(R)^T + (X_hat L1) L2 + b
 * where X_hat = X diag(lambda)^-1 is the smoothed activation, W_hat = W diag(lambda) the
 * smoothed weight, W_hat^T ~ L1 L2 its rank-r SVD branch (bf16) and R = W_hat - (L1 L2)^T
 * the residual; Q() is NVFP4 quantization (e2m1 codes, one e4m3 scale per 16 elements
 * along K, one fp32 tensor scale).
 *   - outlier migration and low-rank split: "Svdq Int4 Flux.1 Canny Dev" model card,
 *     section "SVDQuant 概述", stages 1-3;
 *   - fusion of the down-projection with the activation quantizer and of the up-projection
 *     with the 4-bit GEMM: same card, section "Nunchaku 引擎設計", (a) and (b);
 *   - NVFP4, group size 16, rank 32: "Nunchaku Lite in Diffusers" (blog post), section
 *     on the quantization_config block ("التحميل الأصلي في الناشرون");
 *   - refusing unsupported GPUs with a clear error: same post, "دعم الأجهزة".
 *
 * Conventions for every entry point:
 *   - Shapes follow nn.Linear: X is M x K (tokens x in-features), W is N x K, Y is M x N.
 *     All matrices are row-major and contiguous.
 *   - "device" pointers are CUDA device (or managed) memory; "host" pointers are host memory.
 *     All buffers are owned by the caller; the library never allocates or frees them.
 *   - bf16 values are passed as uint16_t bit patterns.
 *   - stream is a cudaStream_t passed as void* (NULL = the legacy default stream). Unless a
 *     function says otherwise it only enqueues work and returns; results are ready when the
 *     stream reaches that point.
 *   - Device pointers must be 16-byte aligned.
 *   - Tensor scales (s_w, s_x, the s of svdq_quantize_rows) lie in [2^-116, 2^116]: there every
 *     non-zero group scale times s is a normal fp32 number, which the quantizers' exact
 *     division relies on. Others return SVDQ_ERR_INVALID_ARG.
 *   - Shape limits: M >= 1; K % 64 == 0; N % 16 == 0; rank in {0, 16, 32, 64, 128}.
 *     Other values return SVDQ_ERR_INVALID_ARG; misaligned pointers SVDQ_ERR_MISALIGNED.
 *     Arguments are checked before the device is queried, so these errors are reported the
 *     same way on any machine.
 *   - The first call on a device checks for compute capability 10.0 and returns
 *     SVDQ_ERR_UNSUPPORTED_ARCH on any other GPU. There is no fallback path.
 *   - Device-side waits are bounded; a kernel that gives up records a code that
 *     svdq_last_device_error() returns (and the kernel's outputs are then undefined).
 *
 * Storage formats:
 *   - NVFP4 codes: K-major, two e2m1 codes per byte, element 2i in the low nibble;
 *     a matrix with `rows` rows takes rows * K / 2 bytes.
 *   - Group scales (e4m3 codes): block layout consumed by the tensor-core GEMM. The scales
 *     of rows [128 b, 128 b + 128) and groups [4 c, 4 c + 4) (64 elements of K) fill one
 *     512-byte block at ((b * (K / 64)) + c) * 512; inside it, (row m, group g) sits at
 *     (m % 32) * 16 + ((m % 128) / 32) * 4 + g % 4. Rows are padded (with zero scales):
 *     activations to a multiple of 128, weights to a multiple of 256.
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,      /* a shape, rank or null pointer outside the contract */
  SVDQ_ERR_UNSUPPORTED_ARCH = 2, /* not a compute capability 10.0 GPU */
  SVDQ_ERR_MISALIGNED = 3,       /* a device pointer is not 16-byte aligned */
  SVDQ_ERR_CUDA = 4,             /* a CUDA runtime call or a kernel launch failed */
  SVDQ_ERR_TIMEOUT = 5,          /* a kernel gave up on a bounded wait */
  SVDQ_ERR_INTERNAL = 6,         /* an internal consistency check failed */
  SVDQ_ERR_UNAVAILABLE = 7       /* a runtime dependency (the eigen-solver library) is missing */
} svdq_status;

/* One prepared layer. Every pointer is a caller-allocated device buffer of the stated size;
 * svdq_prepare_weights fills them and the two scalar tensor scales. */
typedef struct svdq_layer {
  int32_t N, K, rank;
  int32_t group;            /* always 16 */
  float w_tensor_scale;     /* s_w = fp32(max|R| / 2688) (1 when R == 0) */
  float x_tensor_scale;     /* s_x = fp32(max_j fp32(a_x[j] inv_lambda[j]) / 2688), calibrated */
  uint8_t *wq;              /* N * K / 2 bytes: NVFP4 codes of R (fp32-rounded residual) */
  uint8_t *ws;              /* svdq_weight_scale_bytes(N, K) bytes: e4m3 group scales of R */
  float *inv_lambda;        /* K floats: fp32(1 / lambda_j) */
  float *lambda;            /* K floats: lambda_j (optional; written by prepare when not NULL) */
  uint16_t *L1t;            /* rank * K bf16: L1s = diag(lambda)^-1 L1 transposed (row j = column j
                               of L1s; the smoothing folded into the first factor); NULL if rank 0 */
  uint16_t *L2t;            /* N * rank bf16: L2 transposed (row n = column n of L2); NULL if rank 0 */
  float *bias;              /* N floats, or NULL for no bias */
} svdq_layer;

/* Human-readable name of a status code (static string). */
SVDQ_API const char *svdq_status_string(svdq_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
SVDQ_API int svdq_version(void);

/* Bytes of the weight group-scale buffer (rows padded to a multiple of 256). */
SVDQ_API size_t svdq_weight_scale_bytes(int N, int K);

/* Bytes of the activation group-scale buffer (rows padded to a multiple of 128). */
SVDQ_API size_t svdq_act_scale_bytes(int M, int K);

/* Calibration maxima a_x[j] = max_m |X[m, j]| over the rows of X (the activation side of
 * the smoothing factor; "SVDQuant 概述" stage 2).
 *   X       device, M x K bf16.
 *   absmax  device, K floats (overwritten).
 * Asynchronous on stream. */
SVDQ_API svdq_status svdq_act_absmax(const uint16_t *X, int M, int K, float *absmax, void *stream);

/* Workspace (device bytes) that svdq_prepare_weights needs for an N x K weight at this rank.
 * Loads the eigen-solver library on first use (SVDQ_ERR_UNAVAILABLE if it cannot). Returns 0
 * and sets *status on error when status is not NULL. */
SVDQ_API size_t svdq_prepare_workspace_bytes(int N, int K, int rank, svdq_status *status);

/* Offline step, once per layer ("SVDQuant 概述" stages 2 and 3; packing for the kernels):
 *   a_w[j] = max_n |W[n, j]|; lambda_j = fp32(fp32(sqrt a_x[j]) / fp32(sqrt a_w[j])), 1 when
 *   either is 0; inv_lambda_j = fp32(1 / lambda_j); W_hat = W diag(lambda) (fp64);
 *   truncated SVD W_hat^T = P S Q^T (fp64, from the eigen-decomposition of the smaller Gram
 *   matrix), sign fixed so that the largest-magnitude entry of each column of P is positive;
 *   L1s = bf16(diag(lambda)^-1 P_r S_r^1/2) (the smoothing folded into the first factor, so
 *   that the down-projection reads X itself: X_hat L1 = X diag(lambda)^-1 L1, "Nunchaku 引擎設計"
 *   (b)), L2 = bf16(S_r^1/2 Q_r^T); R = fp32(W_hat - (diag(lambda) L1s L2)^T) (fp64 before the
 *   final rounding); s_w, s_x as in svdq_layer; R quantized to NVFP4 with s_w.
 *   W           device, N x K fp32.
 *   bias        device, N fp32, or NULL. Copied into layer->bias when both are non-NULL.
 *   act_absmax  device, K fp32: calibration maxima a_x (e.g. from svdq_act_absmax).
 *   layer       in: N, K, rank and the device buffers; out: buffers filled, group = 16,
 *               w_tensor_scale and x_tensor_scale set.
 *   workspace   device, at least svdq_prepare_workspace_bytes(N, K, rank) bytes.
 * Synchronous: returns after the work on stream has finished. */
SVDQ_API svdq_status svdq_prepare_weights(const float *W, const float *bias, const float *act_absmax,
                                 int N, int K, int rank, svdq_layer *layer,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* svdq_prepare_weights from host memory, for offline preparation and for checking the weight
 * quantizer at full size: the same steps and outputs, plus the residual the quantizer read.
 *   W_host           host, N x K fp32.
 *   bias_host        host, N fp32, or NULL. Copied into layer->bias when both are non-NULL.
 *   act_absmax_host  host, K fp32 calibration maxima a_x.
 *   layer            as for svdq_prepare_weights (device buffers preallocated by the caller).
 *   R_out_host       host, N x K fp32, or NULL: receives R = fp32(W_hat - (diag(lambda) L1s L2)^T),
 *                    the matrix whose NVFP4 codes and scales land in layer->wq / layer->ws (two
 *                    fp64 routes to the SVD can differ in the last bits of R, so a test of the
 *                    weight quantizer takes R from here).
 * This offline entry point allocates and frees its own device memory (a copy of W, the maxima and
 * the workspace: N K 4 bytes plus svdq_prepare_workspace_bytes) with cudaMalloc / cudaFree.
 * Synchronous: returns after the work on stream has finished. */
SVDQ_API svdq_status svdq_prepare_weights_host(const float *W_host, const float *bias_host,
                                               const float *act_absmax_host, int N, int K, int rank,
                                               svdq_layer *layer, float *R_out_host, void *stream);

/* NVFP4 quantization of the rows of a fp32 matrix A (rows x K) with tensor scale s
 * ("التحميل الأصلي في الناشرون": nvfp4, group 16). Per 16-element group along K:
 *   amax = max|a|; scale = e4m3_rn_satfinite(fp32(amax / fp32(6 s)));
 *   code_i = 0 if scale == 0, else e2m1_rn_satfinite(fp32(a_i / fp32(scale * s)));
 *   a value that rounds to zero encodes as +0.
 *   A      device, rows x K fp32.
 *   codes  device, rows * K / 2 bytes (packed as described above).
 *   scales device, block layout with rows padded to a multiple of row_pad (128 or 256);
 *          the padding rows are written as zero scales.
 * Asynchronous on stream. */
SVDQ_API svdq_status svdq_quantize_rows(const float *A, int rows, int K, float s, int row_pad,
                               uint8_t *codes, uint8_t *scales, void *stream);

/* K1 — one pass over X ("Nunchaku 引擎設計" (b): the down-projection and the quantizer read
 * the same input, so they run as one kernel):
 *   X_hat[m, k] = fp32(X[m, k] * inv_lambda[k]);
 *   xq, xs   = NVFP4(X_hat) with tensor scale s_x (same rule as svdq_quantize_rows);
 *   v[m, :]  = fp32( (sum_k X[m, k] L1s[k, :]) / alpha ),  alpha = fp32(s_x * s_w), with L1s
 *              the smoothing-folded factor (so the sum equals X_hat L1), accumulated in fp32 on
 *              the tensor cores straight from the bf16 input. The 1/alpha pre-scaling lets K2
 *              add the branch to the same fp32 accumulator as the 4-bit product.
 *   lora_act row m = [hi | lo] (2 * rank bf16): hi = bf16(v), lo = bf16(v - hi), so hi + lo
 *              carries v with ~16 significant bits (no 16-bit rounding of the branch's
 *              intermediate before the up-projection).
 *   X         device, M x K bf16.
 *   xq        device, M * K / 2 bytes.
 *   xs        device, svdq_act_scale_bytes(M, K) bytes (padding rows written as zero).
 *   lora_act  device, M x (2 * rank) bf16 (unused and may be NULL when rank == 0).
 * Asynchronous on stream. */
SVDQ_API svdq_status svdq_quant_act_lora_down(const uint16_t *X, int M, const svdq_layer *layer,
                                     uint8_t *xq, uint8_t *xs, uint16_t *lora_act, void *stream);

/* K2 — block-scaled FP4 tensor-core GEMM with the up-projection in its output stage
 * ("Nunchaku 引擎設計" (b): the up-projection and the 4-bit GEMM share one output):
 *   acc[m, n] = sum_g xs[m,g] ws[n,g] sum_{k in g} e2m1(xq[m,k]) e2m1(wq[n,k])
 *               + sum_j (hi[m, j] + lo[m, j]) L2[j, n]                 (fp32, tensor memory)
 *   Y[m, n]   = bf16(alpha * acc[m, n] + bias[n]),  alpha = fp32(s_x * s_w).
 *   xq, xs, lora_act  as written by svdq_quant_act_lora_down.
 *   Y         device, M x N bf16 (written once).
 * Asynchronous on stream. */
SVDQ_API svdq_status svdq_gemm_w4a4_lora_up(const uint8_t *xq, const uint8_t *xs, const uint16_t *lora_act,
                                   int M, const svdq_layer *layer, uint16_t *Y, void *stream);

/* K2 with the output stage of the fused QKV projection ("Nunchaku Lite in Diffusers", section on
 * quantized models with structural rewrites: the engine's operator takes the concatenated
 * to_qkv projection together with the Q/K normalizations norm_q, norm_k and the rotary
 * embedding, which the default path runs as separate steps):
 *   Y = [Q | K | V] along N, each section heads x head_dim columns (head_dim must be 128, so
 *   layer->N == 3 * heads * 128); v = alpha * acc + bias as in svdq_gemm_w4a4_lora_up (fp32);
 *   for every head of Q and K:  u = v * w / sqrt(mean(v^2) + eps)  (w = norm_q_weight for Q,
 *   norm_k_weight for K), then each column pair (2i, 2i + 1) of the head turns by token m's
 *   angle for pair i:  (u0, u1) -> (u0 cos - u1 sin, u1 cos + u0 sin);  V: bf16(v) unchanged.
 *   The normalization reads the fp32 values before any 16-bit rounding; Y is written once.
 *   norm_q_weight, norm_k_weight  device, 128 fp32 each.
 *   rope                          device, M x 64 x 2 fp32: (cos, sin) per token and pair.
 *   eps                           > 0 or 0 (added to the mean square).
 * Errors: SVDQ_ERR_INVALID_ARG for head_dim != 128 or N != 3 * heads * 128; otherwise as
 * svdq_gemm_w4a4_lora_up. Asynchronous on stream. */
SVDQ_API svdq_status svdq_gemm_w4a4_lora_up_qk_norm_rope(const uint8_t *xq, const uint8_t *xs,
                                                         const uint16_t *lora_act, int M,
                                                         const svdq_layer *layer, int heads, int head_dim,
                                                         const float *norm_q_weight, const float *norm_k_weight,
                                                         const float *rope, float eps, uint16_t *Y,
                                                         void *stream);

/* Unfused baseline of the step above: the per-head normalization and rotary embedding of the
 * Q and K sections of a bf16 Y = [Q | K | V] that a plain projection has already written
 * (M x 3 * heads * 128, modified in place; it reads the 16-bit values back and rewrites them).
 * Same weights, table and eps as svdq_gemm_w4a4_lora_up_qk_norm_rope. Asynchronous on stream. */
SVDQ_API svdq_status svdq_qk_norm_rope(uint16_t *Y, int M, int heads, int head_dim, const float *norm_q_weight,
                                       const float *norm_k_weight, const float *rope, float eps, void *stream);

/* The FLUX feed-forward pair, Linear -> GELU (tanh form) -> Linear, with both linears SVDQuant
 * layers ("Nunchaku Lite in Diffusers", introduction of Nunchaku Lite: the engine's fused GELU / MLP
 * kernels). GELU(v) = 0.5 v (1 + tanh(sqrt(2 / pi) (v + 0.044715 v^3))).
 *
 * svdq_gemm_w4a4_lora_up_gelu_quant — the fused pair's middle: K2 of the up layer whose output
 * stage, instead of writing Y, computes h = GELU(alpha acc + bias) in fp32 and produces the down
 * layer's activations exactly as svdq_quant_act_lora_down would from an unrounded input h:
 *   xq_down, xs_down  NVFP4 codes / block scales of x_hat = fp32(h inv_lambda_down) with the down
 *                     layer's s_x (same quantizer, same formats; padding scale rows zero);
 *   lora_act_down     [hi | lo] of fp32(sum_k h[m, k] L1s_down[k, :]) / alpha_down, the sum formed
 *                     on the tensor cores from the bf16 pair hi = bf16(h), lo = bf16(h - hi) per
 *                     256 columns, and the per-tile partials added in tile order (deterministic).
 * The M x N_up intermediate never reaches memory in 16 bits. Requirements: down->K == up->N,
 * down->rank in {0, 16, 32, 64}.
 *   workspace  device, at least svdq_mlp_workspace_bytes(M, up->N, down->rank) bytes (the fp32
 *              partials; may be NULL at down rank 0). Owned by the caller, contents not kept.
 * Asynchronous on stream.
 *
 * svdq_gemm_w4a4_lora_up_gelu — the unfused pair's first layer: Y = bf16(GELU(alpha acc + bias)),
 * the bf16 intermediate that svdq_quant_act_lora_down of the down layer then reads back.
 *
 * svdq_mlp_forward — the fused pair: svdq_quant_act_lora_down (up), then the fused middle, then
 * svdq_gemm_w4a4_lora_up (down) writing Z (M x down->N bf16). Buffers as above. Asynchronous. */
SVDQ_API size_t svdq_mlp_workspace_bytes(int M, int N_up, int rank_down);
SVDQ_API svdq_status svdq_gemm_w4a4_lora_up_gelu_quant(const uint8_t *xq, const uint8_t *xs,
                                                       const uint16_t *lora_act, int M, const svdq_layer *up,
                                                       const svdq_layer *down, uint8_t *xq_down, uint8_t *xs_down,
                                                       uint16_t *lora_act_down, void *workspace,
                                                       size_t workspace_bytes, void *stream);
SVDQ_API svdq_status svdq_gemm_w4a4_lora_up_gelu(const uint8_t *xq, const uint8_t *xs, const uint16_t *lora_act,
                                                 int M, const svdq_layer *layer, uint16_t *H, void *stream);
SVDQ_API svdq_status svdq_mlp_forward(const uint16_t *X, int M, const svdq_layer *up, const svdq_layer *down,
                                      uint8_t *xq, uint8_t *xs, uint16_t *lora_act, uint8_t *xq_down,
                                      uint8_t *xs_down, uint16_t *lora_act_down, void *workspace,
                                      size_t workspace_bytes, uint16_t *Z, void *stream);

/* awq_w4a16 — the second kernel family ("Nunchaku Lite in Diffusers": 4-bit weights with 16-bit
 * activations for the adaptive-normalization / modulation projections, memory-bound and
 * precision-sensitive; quantization_config: int4, group_size 64).
 * Storage: wq N x K/2 bytes (element 2i of a row in the low nibble of byte i), scales N x K/64
 * fp16, zeros N x K/64 bytes; W_hat[n, k] = (q[n, k] - z[n, k/64]) * s[n, k/64]. K % 64 == 0.
 *
 * svdq_awq_quantize_weights: round-to-nearest per group of 64, decided in fp32:
 *   range = max - min (at least 1e-5), s = fp16(range / 15), z = clamp(rint(-min / s), 0, 15),
 *   q = clamp(rint(w / s) + z, 0, 15)  (rint: ties to even; divisions correctly rounded).
 *   W device N x K fp32 (16-byte aligned), |W| below ~4.9e5 (fp16 scale range).
 *   wq, scales, zeros device outputs (wq 16-byte aligned). Asynchronous on stream.
 *
 * svdq_awq_pack_weights: rearranges wq, scales and zeros (as above) into the layout the GEMV
 *   streams: per 16 rows x 64 columns a 512-byte tile of codes in tensor-core operand order and
 *   64 bytes of scales and zero points (fp16 s and fp16 128 + z per row; rows padded to a multiple
 *   of 16 with zeros).
 *   wq_packed  device, svdq_awq_packed_weight_bytes(N, K) bytes, 16-byte aligned.
 *   sz_packed  device, svdq_awq_packed_sz_bytes(N, K) bytes, 16-byte aligned.
 *   Done once per layer. Asynchronous on stream.
 *
 * svdq_awq_gemv_w4a16: Y[m, n] = bf16(sum_k X[m, k] W_hat[n, k] + bias[n]) for 1 <= M <= 8 tokens;
 *   the tensor cores sum exact products (128 + q) x in fp32 per group of 64, and the scale and
 *   zero point are applied per group in fp32: s (D - (128 + z) sum x). X device M x K bf16 (16-byte aligned); wq_packed, sz_packed from
 *   svdq_awq_pack_weights; bias device N fp32 or NULL; Y device M x N bf16. K <= 12288 (the
 *   staged activations take K/64 KiB of shared memory beside the warps' rings of weight tiles in
 *   flight) and ceil(N/16) * K/64 < 2^26 tiles; otherwise SVDQ_ERR_INVALID_ARG.
 *   Asynchronous on stream, launched as a programmatic dependent launch: it may start under the
 *   tail of the previous kernel of the stream and read wq_packed / sz_packed before waiting for
 *   that kernel (X, bias and Y only after the wait), so the packed weights must be complete before
 *   the kernel launched just before this call on the stream begins: pack them at load time, or
 *   put an event or a synchronization between svdq_awq_pack_weights and the first GEMV. A lost
 *   wait inside the kernel (about two seconds) sets the library's device error word. */
SVDQ_API svdq_status svdq_awq_quantize_weights(const float *W, int N, int K, uint8_t *wq, uint16_t *scales,
                                               uint8_t *zeros, void *stream);
SVDQ_API size_t svdq_awq_packed_weight_bytes(int N, int K);
SVDQ_API size_t svdq_awq_packed_sz_bytes(int N, int K);
SVDQ_API svdq_status svdq_awq_pack_weights(const uint8_t *wq, const uint16_t *scales, const uint8_t *zeros, int N,
                                           int K, uint8_t *wq_packed, uint8_t *sz_packed, void *stream);
SVDQ_API svdq_status svdq_awq_gemv_w4a16(const uint16_t *X, int M, const uint8_t *wq_packed, const uint8_t *sz_packed,
                                         const float *bias, int N, int K, uint16_t *Y, void *stream);

/* K1 then K2 on the same stream (the layer's forward pass). Buffers as above. */
SVDQ_API svdq_status svdq_linear_forward(const uint16_t *X, int M, const svdq_layer *layer,
                                uint8_t *xq, uint8_t *xs, uint16_t *lora_act,
                                uint16_t *Y, void *stream);

/* The forward pass from and to host memory: copies X_host (M x K bf16) to X_dev, runs
 * svdq_linear_forward, copies Y_dev (M x N bf16) back to Y_host. For M > 256 it runs in row
 * chunks of a multiple of 256 rows (up to 8): the kernels of a chunk run on stream while the next
 * chunk is copied in and the previous one copied out on two streams of the library's own (one per
 * copy direction, created on first use and ordered after the work already on stream), so the
 * copies of both directions overlap each other and the kernels; the result is the whole-M call's,
 * bit for bit. Pinned host buffers make the copies asynchronous (pageable ones work, without the
 * overlap). Synchronous: returns after the last copy out; concurrent calls on one device take
 * turns. */
SVDQ_API svdq_status svdq_linear_forward_host(const uint16_t *X_host, int M, const svdq_layer *layer,
                                     uint16_t *X_dev, uint8_t *xq, uint8_t *xs,
                                     uint16_t *lora_act, uint16_t *Y_dev, uint16_t *Y_host,
                                     void *stream);

/* Unfused baseline: the low-rank branch as separate kernels around the 4-bit GEMM
 * ("Nunchaku 引擎設計" (a): the branch run naively re-reads the 16-bit input in the
 * down-projection and re-writes the 16-bit output in the up-projection).
 *   svdq_baseline_lora_down: lora_act = hi/lo pair of sum_k X L1s / alpha (reads X).
 *   svdq_baseline_quantize:  xq, xs = NVFP4(X_hat) (reads X again).
 *   svdq_baseline_gemm_w4a4: Y = bf16(alpha * 4-bit product + bias) (no branch).
 *   svdq_baseline_lora_up:   Y = bf16(Y + alpha * lora_act L2) (reads and rewrites Y).
 * Same buffers and formats as the fused calls. Asynchronous on stream. */
SVDQ_API svdq_status svdq_baseline_lora_down(const uint16_t *X, int M, const svdq_layer *layer,
                                    uint16_t *lora_act, void *stream);
SVDQ_API svdq_status svdq_baseline_quantize(const uint16_t *X, int M, const svdq_layer *layer,
                                   uint8_t *xq, uint8_t *xs, void *stream);
SVDQ_API svdq_status svdq_baseline_gemm_w4a4(const uint8_t *xq, const uint8_t *xs, int M,
                                    const svdq_layer *layer, uint16_t *Y, void *stream);
SVDQ_API svdq_status svdq_baseline_lora_up(const uint16_t *lora_act, int M, const svdq_layer *layer,
                                  uint16_t *Y, void *stream);

/* Allocation-free variant of the smoothing stage of svdq_prepare_weights (this entry point has
 * no counterpart on the method's pages; it exists for callers that cannot allocate device memory
 * when they need it, e.g. code running under a fixed, pre-reserved memory budget or inside a
 * framework that forbids allocations after start-up, and so cannot pass a workspace):
 *   a_w[j] = max_n |W[n, j]|; lambda_j, inv_lambda_j and s_x exactly as svdq_prepare_weights
 *   computes them (s_x = fp32(max_j fp32(a_x[j] inv_lambda_j) / 2688), 1 when that maximum is 0).
 *   W                device, N x K fp32.
 *   act_absmax       device, K fp32 calibration maxima a_x.
 *   lambda           device, K fp32 (out).
 *   inv_lambda       device, K fp32 (out).
 *   x_tensor_scale   device, 1 fp32 (out).
 * Its scratch (K column maxima and one running maximum) is a static device array inside the
 * library sized for K <= 65536 (256 KiB, held on every GPU that loads the library until the
 * process exits); larger K, K % 64 != 0, N <= 0 or a NULL pointer return SVDQ_ERR_INVALID_ARG.
 * It calls no allocating routine. The first call on a device looks up the array's device address
 * (once per device), so make that first call before any stream capture; if that lookup fails,
 * every later call on that device returns SVDQ_ERR_CUDA for the rest of the process. All calls share the array and the call clears what must
 * start at zero; calls that overlap on the GPU (other streams, other threads) race on it.
 * Asynchronous on stream. */
SVDQ_API svdq_status svdq_smoothing_factors_noalloc(const float *W, const float *act_absmax, int N, int K,
                                                    float *lambda, float *inv_lambda, float *x_tensor_scale,
                                                    void *stream);

/* Group scales from the block layout (as svdq_quant_act_lora_down, svdq_quantize_rows and
 * svdq_prepare_weights write them) to row-major order: rowmajor[m * (K / 16) + g] = the e4m3
 * code of row m, group g, for m < rows. Pure host code, no device needed.
 *   blocked   host, at least ceil(rows / 128) * 128 * K / 16 bytes (the stored layout; padding
 *             rows are not read).
 *   rowmajor  host, rows * K / 16 bytes (out).
 * Errors: SVDQ_ERR_INVALID_ARG for NULL pointers, rows <= 0, K <= 0 or K % 64 != 0. */
SVDQ_API svdq_status svdq_unswizzle_scales(const uint8_t *blocked, int rows, int K, uint8_t *rowmajor);

/* Test hook for the architecture check. After svdq_test_override_capability(major, minor) every
 * entry point that would use the GPU acts as if the device reported compute capability
 * major.minor: anything other than 10.0 returns SVDQ_ERR_UNSUPPORTED_ARCH before any CUDA call,
 * so the refusal path can be exercised on any machine; 10.0 falls through to the real check (the
 * hook can make a B200 look unsupported, never the reverse). major < 0 removes the override.
 * Argument checks still come first. Returns SVDQ_ERR_INVALID_ARG for major > 99 or minor
 * outside 0..9. Process-wide; not meant for production use. */
SVDQ_API svdq_status svdq_test_override_capability(int major, int minor);

/* Failure-path self-test. Launches one CTA whose bounded waits (the same code every kernel of
 * the library uses) wait on an mbarrier that nothing signals; each gives up after limit_us
 * microseconds (1 .. 1000000) and records the timeout as a stalled kernel would, and the kernel
 * then returns normally: no trap, no fault, the context stays usable. A following
 * svdq_last_device_error returns SVDQ_ERR_TIMEOUT with *code = (5 << 16) | (1 << 8) | 1.
 * Asynchronous on stream. */
SVDQ_API svdq_status svdq_selftest_wait_timeout(uint32_t limit_us, void *stream);

/* Reads and clears the device-side error word after synchronizing stream. *code is 0 when
 * no kernel gave up on a wait; otherwise (kernel id << 16) | (site << 8) | 1.
 * Returns SVDQ_ERR_TIMEOUT when *code != 0. */
SVDQ_API svdq_status svdq_last_device_error(void *stream, uint32_t *code);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
