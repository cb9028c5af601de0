// C ABI of libsvdq: argument checks, architecture check, TMA tensor-map encoding and kernel
// launches. Every entry point is declared and documented in include/svdq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "svdq.h"

namespace svdq {

__device__ uint32_t g_error_word;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::once_flag once;
  svdq_status arch = SVDQ_OK;
  int num_sms = 0;
  uint32_t *err = nullptr;
};
DeviceState g_dev[kMaxDevices];

// Compute capability that svdq_test_override_capability asks device_check to assume
// (major * 10 + minor), or -1. It can only make a supported GPU look unsupported.
std::atomic<int> g_cap_override{-1};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

void init_encode() {
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}

// Checks the current device once: compute capability 10.0 ("دعم الأجهزة": unsupported GPUs
// get a clear error instead of wrong output) and records the SM count and the error word.
// Copy streams and events of svdq_linear_forward_host's pipelined path, per device, created on
// first use (a mutex serialises the calls that share them).
constexpr int kHostChunks = 8;
struct HostPipe {
  std::once_flag once;
  bool ok = false;
  std::mutex mu;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t in_done[kHostChunks] = {}, fwd_done[kHostChunks] = {};
};
HostPipe g_pipe[kMaxDevices];

svdq_status device_check(DeviceState **out) {
  const int ov = g_cap_override.load(std::memory_order_relaxed);
  if (ov >= 0 && ov != 100) return SVDQ_ERR_UNSUPPORTED_ARCH;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_INTERNAL;
  DeviceState &d = g_dev[dev];
  std::call_once(d.once, [&]() {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      d.arch = SVDQ_ERR_CUDA;
      return;
    }
    if (major != 10 || minor != 0) {
      d.arch = SVDQ_ERR_UNSUPPORTED_ARCH;
      return;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) {
      d.arch = SVDQ_ERR_CUDA;
      return;
    }
    d.err = static_cast<uint32_t *>(p);
  });
  if (d.arch != SVDQ_OK) return d.arch;
  *out = &d;
  return SVDQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

bool rank_ok(int r) { return r == 0 || r == 16 || r == 32 || r == 64 || r == 128; }

// Tensor scales the quantizers handle exactly: with s in [2^-116, 2^116] every non-zero group
// scale times s (at least 2^-9 s) is a normal fp32 number whose reciprocal is finite, and 6 s,
// 448 s and 1 / (6 s) are finite.
bool scale_ok(float s) { return s >= 0x1p-116f && s <= 0x1p116f; }

svdq_status check_layer(const svdq_layer *L) {
  if (!L) return SVDQ_ERR_INVALID_ARG;
  if (L->N <= 0 || L->K <= 0 || (L->K % 64) != 0 || (L->N % 16) != 0 || !rank_ok(L->rank))
    return SVDQ_ERR_INVALID_ARG;
  if (!L->wq || !L->ws || !L->inv_lambda) return SVDQ_ERR_INVALID_ARG;
  if (L->rank > 0 && (!L->L1t || !L->L2t)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(L->wq) || !aligned16(L->ws) || !aligned16(L->inv_lambda) || !aligned16(L->bias) ||
      !aligned16(L->L1t) || !aligned16(L->L2t))
    return SVDQ_ERR_MISALIGNED;
  if (!scale_ok(L->x_tensor_scale) || !scale_ok(L->w_tensor_scale)) return SVDQ_ERR_INVALID_ARG;
  return SVDQ_OK;
}

bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  std::call_once(g_encode_once, init_encode);
  if (!g_encode) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for_row_bytes(uint32_t b) {
  return b >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : (b == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

float alpha_of(const svdq_layer *L) { return L->x_tensor_scale * L->w_tensor_scale; }

HostPipe *host_pipe(DeviceState *d) {
  HostPipe &p = g_pipe[d - g_dev];
  std::call_once(p.once, [&]() {
    bool ok = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&p.end, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kHostChunks; ++i)
      ok = cudaEventCreateWithFlags(&p.in_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&p.fwd_done[i], cudaEventDisableTiming) == cudaSuccess;
    p.ok = ok;
  });
  return p.ok ? &p : nullptr;
}

svdq_status run_quant(const uint16_t *X, int M, const svdq_layer *L, uint8_t *xq, uint8_t *xs, uint16_t *la,
                      bool quantize, bool lora, void *stream) {
  // argument checks first: they need no device, so a bad call is reported the same way on any
  // machine
  svdq_status st = check_layer(L);
  if (st != SVDQ_OK) return st;
  if (!X || M <= 0) return SVDQ_ERR_INVALID_ARG;
  if (quantize && (!xq || !xs)) return SVDQ_ERR_INVALID_ARG;
  if (lora && L->rank > 0 && !la) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(xq) || !aligned16(xs) || !aligned16(la)) return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  st = device_check(&d);
  if (st != SVDQ_OK) return st;
  if (!quantize && (!lora || L->rank == 0)) return SVDQ_OK;
  QuantLaunch q;
  memset(&q, 0, sizeof(q));
  const int K = L->K, r = lora ? L->rank : 0;
  if (!make_map(&q.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, static_cast<uint64_t>(K) * 2, 64, kQuantRows,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_map(&q.tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L->L1t, K, r, static_cast<uint64_t>(K) * 2, 64, r,
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    q.tm_l1 = q.tm_x;
  }
  q.inv_lambda = L->inv_lambda;
  q.xq = xq;
  q.xs = xs;
  q.lora_act = la;
  q.M = M;
  q.K = K;
  q.rank = L->rank;
  q.s_x = L->x_tensor_scale;
  q.d_x = 6.0f * L->x_tensor_scale;
  q.inv_alpha = 1.0f / alpha_of(L);
  q.splits = quant_act_splits(M, K, L->rank, quantize, lora, d->num_sms);
  q.chunks_per_split = (K / 64 + q.splits - 1) / q.splits;
  q.quantize = quantize;
  q.lora = lora;
  q.err = d->err;
  q.stream = static_cast<cudaStream_t>(stream);
  return launch_quant_act(q) == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

struct QkNormRope {
  int heads;
  const float *norm_q, *norm_k, *rope;
  float eps;
};

// Output of the fused MLP pair's first GEMM: the down layer's activations.
struct MlpOut {
  const svdq_layer *down;
  uint8_t *xq, *xs;
  uint16_t *la;  // M x 2 rank_down bf16 ([hi | lo])
  float *part;   // [ceil(N_up / 256)][M][rank_down] fp32
};

svdq_status run_gemm(const uint8_t *xq, const uint8_t *xs, const uint16_t *la, int M, const svdq_layer *L,
                     uint16_t *Y, bool fp4, bool add_y, bool lora, void *stream, const QkNormRope *qk = nullptr,
                     bool gelu = false, const MlpOut *mlp = nullptr) {
  svdq_status st = check_layer(L);
  if (st != SVDQ_OK) return st;
  if (M <= 0 || (!Y && !mlp)) return SVDQ_ERR_INVALID_ARG;
  if (fp4 && (!xq || !xs)) return SVDQ_ERR_INVALID_ARG;
  const int r = lora ? L->rank : 0;
  if (r > 0 && !la) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(xs) || !aligned16(la) || !aligned16(Y)) return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  st = device_check(&d);
  if (st != SVDQ_OK) return st;
  if (!fp4 && r == 0) return SVDQ_OK;
  GemmLaunch g;
  memset(&g, 0, sizeof(g));
  const int K = L->K, N = L->N;
  if (fp4) {
    if (!make_map(&g.tm_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, K / 2, M, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&g.tm_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, L->wq, K / 2, N, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  }
  if (r > 0) {
    const uint32_t kc = r < 32 ? r : 32;
    const CUtensorMapSwizzle sw = swizzle_for_row_bytes(kc * 2);
    if (!make_map(&g.tm_la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, la, 2 * r, M, static_cast<uint64_t>(r) * 4, kc, 128, sw) ||
        !make_map(&g.tm_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L->L2t, r, N, static_cast<uint64_t>(r) * 2, kc, 128, sw))
      return SVDQ_ERR_CUDA;
  }
  if (Y && !make_map(&g.tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, N, M, static_cast<uint64_t>(N) * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  if (!Y) g.tm_y = g.tm_xq;  // the fused MLP pair writes no Y
  if (!fp4) {
    g.tm_xq = g.tm_la;
    g.tm_wq = g.tm_l2;
  }
  if (r == 0) {
    g.tm_la = g.tm_xq;
    g.tm_l2 = g.tm_wq;
  }
  g.xs = xs;
  g.ws = L->ws;
  g.bias = L->bias;
  g.Y = Y;
  g.M = M;
  g.N = N;
  g.K = K;
  g.rank = r;
  g.alpha = alpha_of(L);
  g.fp4 = fp4;
  g.add_y = add_y;
  if (qk) {
    g.qk_norm_rope = true;
    g.norm_q = qk->norm_q;
    g.norm_k = qk->norm_k;
    g.qk_width = qk->heads * 128;
    g.eps = qk->eps;
    // rotary table [M][64 pairs][cos, sin] as M rows of 128 fp32, staged 32 floats x 128 rows per box
    if (!make_map(&g.tm_rope, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, qk->rope, 128, M, 512, 32, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  }
  g.gelu = gelu;
  if (mlp) {
    const svdq_layer *D = mlp->down;
    g.mlp = true;
    g.il_d = D->inv_lambda;
    g.sx_d = D->x_tensor_scale;
    g.rank_d = D->rank;
    g.mp_scales = static_cast<int>(round_up(static_cast<size_t>(M), 128));
    g.xq_d = mlp->xq;
    g.xs_d = mlp->xs;
    g.part = mlp->part;
    if (D->rank > 0) {
      // L1t of the down layer: rank_d rows of N (= its K) bf16; boxes of 32 columns x rank_d / 2 rows
      if (!make_map(&g.tm_l1d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D->L1t, N, D->rank, static_cast<uint64_t>(N) * 2, 32,
                    D->rank / 2, CU_TENSOR_MAP_SWIZZLE_64B))
        return SVDQ_ERR_CUDA;
    } else {
      g.tm_l1d = g.tm_xq;
    }
  }
  g.num_sms = d->num_sms;
  g.err = d->err;
  g.stream = static_cast<cudaStream_t>(stream);
  if (launch_gemm(g) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (mlp && mlp->down->rank > 0) {
    const svdq_layer *D = mlp->down;
    const float inv_alpha_d = 1.0f / alpha_of(D);
    if (launch_lora_reduce(mlp->part, gemm_n_tiles(N), M, D->rank, inv_alpha_d, mlp->la,
                           g.stream) != cudaSuccess)
      return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" {

const char *svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED_ARCH: return "unsupported GPU: libsvdq needs compute capability 10.0 (B200, sm_100a)";
    case SVDQ_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case SVDQ_ERR_INTERNAL: return "internal error";
    case SVDQ_ERR_UNAVAILABLE: return "eigen-solver library (libcusolver.so.11) not found";
  }
  return "unknown status";
}

int svdq_version(void) { return 100; }

size_t svdq_weight_scale_bytes(int N, int K) {
  if (N <= 0 || K <= 0) return 0;
  return round_up(static_cast<size_t>(N), 256) * static_cast<size_t>(K / 16);
}

size_t svdq_act_scale_bytes(int M, int K) {
  if (M <= 0 || K <= 0) return 0;
  return round_up(static_cast<size_t>(M), 128) * static_cast<size_t>(K / 16);
}

svdq_status svdq_act_absmax(const uint16_t *X, int M, int K, float *absmax, void *stream) {
  if (!X || !absmax || M <= 0 || K <= 0) return SVDQ_ERR_INVALID_ARG;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  return launch_col_absmax_bf16(X, M, K, absmax, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SVDQ_OK
                                                                                                   : SVDQ_ERR_CUDA;
}

size_t svdq_prepare_workspace_bytes(int N, int K, int rank, svdq_status *status) {
  PrepPlan plan;
  svdq_status st = SVDQ_OK;
  if (N <= 0 || K <= 0 || K % 64 || N % 16 || !rank_ok(rank)) st = SVDQ_ERR_INVALID_ARG;
  if (st == SVDQ_OK) {
    const PrepStatus ps = prepare_plan(N, K, rank, &plan);
    if (ps == PREP_NO_SOLVER) st = SVDQ_ERR_UNAVAILABLE;
    else if (ps != PREP_OK) st = SVDQ_ERR_CUDA;
  }
  if (status) *status = st;
  return st == SVDQ_OK ? plan.bytes : 0;
}

svdq_status svdq_prepare_weights(const float *W, const float *bias, const float *act_absmax, int N, int K, int rank,
                                 svdq_layer *layer, void *workspace, size_t workspace_bytes, void *stream) {
  if (!W || !act_absmax || !layer || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || K % 64 || N % 16 || !rank_ok(rank)) return SVDQ_ERR_INVALID_ARG;
  if (layer->N != N || layer->K != K || layer->rank != rank) return SVDQ_ERR_INVALID_ARG;
  if (!layer->wq || !layer->ws || !layer->inv_lambda || (rank > 0 && (!layer->L1t || !layer->L2t)))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(act_absmax) || !aligned16(workspace) || !aligned16(layer->wq) ||
      !aligned16(layer->ws) || !aligned16(layer->inv_lambda) || !aligned16(layer->lambda) ||
      !aligned16(layer->L1t) || !aligned16(layer->L2t) || !aligned16(layer->bias) || !aligned16(bias))
    return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  PrepArgs p;
  const PrepStatus ps = prepare_plan(N, K, rank, &p.plan);
  if (ps == PREP_NO_SOLVER) return SVDQ_ERR_UNAVAILABLE;
  if (ps != PREP_OK) return SVDQ_ERR_CUDA;
  if (workspace_bytes < p.plan.bytes) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  p.W = W;
  p.act_absmax = act_absmax;
  p.N = N;
  p.K = K;
  p.rank = rank;
  p.workspace = workspace;
  p.lambda_out = layer->lambda;
  p.inv_lambda = layer->inv_lambda;
  p.L1t = layer->L1t;
  p.L2t = layer->L2t;
  p.wq = layer->wq;
  p.wscales = layer->ws;
  p.wscale_bytes = svdq_weight_scale_bytes(N, K);
  float s_w = 0.0f, s_x = 0.0f;
  p.s_w = &s_w;
  p.s_x = &s_x;
  p.stream = s;
  const PrepStatus rs = prepare_run(p);
  if (rs == PREP_SOLVER_FAILED) return SVDQ_ERR_INTERNAL;
  if (rs != PREP_OK) return SVDQ_ERR_CUDA;
  if (bias && layer->bias && bias != layer->bias) {
    if (cudaMemcpyAsync(layer->bias, bias, sizeof(float) * N, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return SVDQ_ERR_CUDA;
  }
  layer->group = 16;
  layer->w_tensor_scale = s_w;
  layer->x_tensor_scale = s_x;
  return SVDQ_OK;
}

svdq_status svdq_prepare_weights_host(const float *W_host, const float *bias_host, const float *act_absmax_host, int N,
                                      int K, int rank, svdq_layer *layer, float *R_out_host, void *stream) {
  if (!W_host || !act_absmax_host || !layer) return SVDQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || K % 64 || N % 16 || !rank_ok(rank)) return SVDQ_ERR_INVALID_ARG;
  if (layer->N != N || layer->K != K || layer->rank != rank) return SVDQ_ERR_INVALID_ARG;
  if (!layer->wq || !layer->ws || !layer->inv_lambda || (rank > 0 && (!layer->L1t || !layer->L2t)))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(layer->wq) || !aligned16(layer->ws) || !aligned16(layer->inv_lambda) || !aligned16(layer->lambda) ||
      !aligned16(layer->L1t) || !aligned16(layer->L2t) || !aligned16(layer->bias))
    return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  svdq_status ws_st = SVDQ_OK;
  const size_t ws_bytes = svdq_prepare_workspace_bytes(N, K, rank, &ws_st);
  if (ws_st != SVDQ_OK) return ws_st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t wbytes = static_cast<size_t>(N) * K * sizeof(float);
  // one offline allocation: W, the calibration maxima and the workspace, 256-byte aligned pieces
  const size_t off_ax = (wbytes + 255) & ~size_t(255);
  const size_t off_ws = off_ax + ((static_cast<size_t>(K) * sizeof(float) + 255) & ~size_t(255));
  void *buf = nullptr;
  if (cudaMalloc(&buf, off_ws + ws_bytes) != cudaSuccess) return SVDQ_ERR_CUDA;
  uint8_t *base = static_cast<uint8_t *>(buf);
  st = SVDQ_OK;
  if (cudaMemcpyAsync(base, W_host, wbytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(base + off_ax, act_absmax_host, sizeof(float) * K, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      (bias_host && layer->bias &&
       cudaMemcpyAsync(layer->bias, bias_host, sizeof(float) * N, cudaMemcpyHostToDevice, s) != cudaSuccess))
    st = SVDQ_ERR_CUDA;
  if (st == SVDQ_OK) {
    PrepArgs p;
    const PrepStatus ps = prepare_plan(N, K, rank, &p.plan);
    if (ps != PREP_OK) st = ps == PREP_NO_SOLVER ? SVDQ_ERR_UNAVAILABLE : SVDQ_ERR_CUDA;
    if (st == SVDQ_OK) {
      float s_w = 0.0f, s_x = 0.0f;
      p.W = reinterpret_cast<const float *>(base);
      p.act_absmax = reinterpret_cast<const float *>(base + off_ax);
      p.N = N;
      p.K = K;
      p.rank = rank;
      p.workspace = base + off_ws;
      p.lambda_out = layer->lambda;
      p.inv_lambda = layer->inv_lambda;
      p.L1t = layer->L1t;
      p.L2t = layer->L2t;
      p.wq = layer->wq;
      p.wscales = layer->ws;
      p.wscale_bytes = svdq_weight_scale_bytes(N, K);
      p.s_w = &s_w;
      p.s_x = &s_x;
      p.R_out_host = R_out_host;
      p.stream = s;
      const PrepStatus rs = prepare_run(p);
      if (rs == PREP_SOLVER_FAILED) st = SVDQ_ERR_INTERNAL;
      else if (rs != PREP_OK) st = SVDQ_ERR_CUDA;
      if (st == SVDQ_OK) {
        layer->group = 16;
        layer->w_tensor_scale = s_w;
        layer->x_tensor_scale = s_x;
      }
    }
  }
  if (cudaStreamSynchronize(s) != cudaSuccess) st = SVDQ_ERR_CUDA;
  if (cudaFree(buf) != cudaSuccess && st == SVDQ_OK) st = SVDQ_ERR_CUDA;
  return st;
}

svdq_status svdq_smoothing_factors_noalloc(const float *W, const float *act_absmax, int N, int K, float *lambda,
                                           float *inv_lambda, float *x_tensor_scale, void *stream) {
  if (!W || !act_absmax || !lambda || !inv_lambda || !x_tensor_scale || N <= 0 || K <= 0 || K % 64 != 0 ||
      K > noalloc_max_k())
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(act_absmax) || !aligned16(lambda) || !aligned16(inv_lambda))
    return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  return smoothing_noalloc(W, act_absmax, N, K, lambda, inv_lambda, x_tensor_scale,
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVDQ_OK
             : SVDQ_ERR_CUDA;
}

svdq_status svdq_quantize_rows(const float *A, int rows, int K, float s, int row_pad, uint8_t *codes, uint8_t *scales,
                               void *stream) {
  if (!A || !codes || !scales || rows <= 0 || K <= 0 || K % 64 || !scale_ok(s) || (row_pad != 128 && row_pad != 256))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(codes) || !aligned16(scales)) return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const size_t sbytes = round_up(static_cast<size_t>(rows), row_pad) * (K / 16);
  if (cudaMemsetAsync(scales, 0, sbytes, cs) != cudaSuccess) return SVDQ_ERR_CUDA;
  return launch_quantize_rows(A, rows, K, s, codes, scales, cs) == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

svdq_status svdq_quant_act_lora_down(const uint16_t *X, int M, const svdq_layer *layer, uint8_t *xq, uint8_t *xs,
                                     uint16_t *lora_act, void *stream) {
  return run_quant(X, M, layer, xq, xs, lora_act, true, true, stream);
}

svdq_status svdq_gemm_w4a4_lora_up(const uint8_t *xq, const uint8_t *xs, const uint16_t *lora_act, int M,
                                   const svdq_layer *layer, uint16_t *Y, void *stream) {
  return run_gemm(xq, xs, lora_act, M, layer, Y, true, false, true, stream);
}

size_t svdq_mlp_workspace_bytes(int M, int N_up, int rank_down) {
  if (M <= 0 || N_up <= 0 || N_up % 64 || !(rank_down == 0 || rank_down == 16 || rank_down == 32 || rank_down == 64))
    return 0;
  return static_cast<size_t>(gemm_n_tiles(N_up)) * static_cast<size_t>(M) * static_cast<size_t>(rank_down) * 4u;
}

svdq_status svdq_gemm_w4a4_lora_up_gelu(const uint8_t *xq, const uint8_t *xs, const uint16_t *lora_act, int M,
                                        const svdq_layer *layer, uint16_t *H, void *stream) {
  return run_gemm(xq, xs, lora_act, M, layer, H, true, false, true, stream, nullptr, true);
}

svdq_status svdq_gemm_w4a4_lora_up_gelu_quant(const uint8_t *xq, const uint8_t *xs, const uint16_t *lora_act, int M,
                                              const svdq_layer *up, const svdq_layer *down, uint8_t *xq_down,
                                              uint8_t *xs_down, uint16_t *lora_act_down, void *workspace,
                                              size_t workspace_bytes, void *stream) {
  if (!up || !down) return SVDQ_ERR_INVALID_ARG;
  svdq_status st = check_layer(down);
  if (st != SVDQ_OK) return st;
  if (down->K != up->N || down->rank > 64 || M <= 0) return SVDQ_ERR_INVALID_ARG;
  if (!xq_down || !xs_down) return SVDQ_ERR_INVALID_ARG;
  if (down->rank > 0 && (!lora_act_down || !workspace || workspace_bytes < svdq_mlp_workspace_bytes(M, up->N, down->rank)))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(xq_down) || !aligned16(xs_down) || !aligned16(lora_act_down) || !aligned16(workspace))
    return SVDQ_ERR_MISALIGNED;
  const MlpOut mo{down, xq_down, xs_down, lora_act_down, static_cast<float *>(workspace)};
  return run_gemm(xq, xs, lora_act, M, up, nullptr, true, false, true, stream, nullptr, false, &mo);
}

svdq_status svdq_mlp_forward(const uint16_t *X, int M, const svdq_layer *up, const svdq_layer *down, uint8_t *xq,
                             uint8_t *xs, uint16_t *lora_act, uint8_t *xq_down, uint8_t *xs_down,
                             uint16_t *lora_act_down, void *workspace, size_t workspace_bytes, uint16_t *Z,
                             void *stream) {
  svdq_status st = svdq_quant_act_lora_down(X, M, up, xq, xs, lora_act, stream);
  if (st != SVDQ_OK) return st;
  st = svdq_gemm_w4a4_lora_up_gelu_quant(xq, xs, lora_act, M, up, down, xq_down, xs_down, lora_act_down, workspace,
                                         workspace_bytes, stream);
  if (st != SVDQ_OK) return st;
  return svdq_gemm_w4a4_lora_up(xq_down, xs_down, lora_act_down, M, down, Z, stream);
}

namespace {
svdq_status check_qk_args(int N, int heads, int head_dim, const float *wq, const float *wk, const float *rope,
                          float eps) {
  if (heads <= 0 || head_dim != 128 || N != 3 * heads * 128 || !wq || !wk || !rope || !(eps >= 0.0f))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(wq) || !aligned16(wk) || !aligned16(rope)) return SVDQ_ERR_MISALIGNED;
  return SVDQ_OK;
}
}  // namespace

svdq_status svdq_gemm_w4a4_lora_up_qk_norm_rope(const uint8_t *xq, const uint8_t *xs, const uint16_t *lora_act,
                                                int M, const svdq_layer *layer, int heads, int head_dim,
                                                const float *norm_q_weight, const float *norm_k_weight,
                                                const float *rope, float eps, uint16_t *Y, void *stream) {
  if (!layer) return SVDQ_ERR_INVALID_ARG;
  svdq_status st = check_qk_args(layer->N, heads, head_dim, norm_q_weight, norm_k_weight, rope, eps);
  if (st != SVDQ_OK) return st;
  const QkNormRope qk{heads, norm_q_weight, norm_k_weight, rope, eps};
  return run_gemm(xq, xs, lora_act, M, layer, Y, true, false, true, stream, &qk);
}

svdq_status svdq_qk_norm_rope(uint16_t *Y, int M, int heads, int head_dim, const float *norm_q_weight,
                              const float *norm_k_weight, const float *rope, float eps, void *stream) {
  if (!Y || M <= 0 || heads <= 0) return SVDQ_ERR_INVALID_ARG;
  svdq_status st = check_qk_args(3 * heads * head_dim, heads, head_dim, norm_q_weight, norm_k_weight, rope, eps);
  if (st != SVDQ_OK) return st;
  if (!aligned16(Y)) return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  st = device_check(&d);
  if (st != SVDQ_OK) return st;
  return launch_qk_norm_rope(Y, M, heads, norm_q_weight, norm_k_weight, rope, eps, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? SVDQ_OK
             : SVDQ_ERR_CUDA;
}

svdq_status svdq_awq_quantize_weights(const float *W, int N, int K, uint8_t *wq, uint16_t *scales, uint8_t *zeros,
                                      void *stream) {
  if (!W || !wq || !scales || !zeros || N <= 0 || K <= 0 || K % 64) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(wq)) return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  return launch_awq_quantize(W, N, K, wq, scales, zeros, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVDQ_OK
             : SVDQ_ERR_CUDA;
}

size_t svdq_awq_packed_weight_bytes(int N, int K) {
  return (N > 0 && K > 0 && K % 64 == 0) ? awq_packed_weight_bytes(N, K) : 0;
}

size_t svdq_awq_packed_sz_bytes(int N, int K) { return (N > 0 && K > 0 && K % 64 == 0) ? awq_packed_sz_bytes(N, K) : 0; }

svdq_status svdq_awq_pack_weights(const uint8_t *wq, const uint16_t *scales, const uint8_t *zeros, int N, int K,
                                  uint8_t *wq_packed, uint8_t *sz_packed, void *stream) {
  if (!wq || !scales || !zeros || !wq_packed || !sz_packed || N <= 0 || K <= 0 || K % 64) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(wq_packed) || !aligned16(sz_packed)) return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  return launch_awq_pack(wq, scales, zeros, N, K, wq_packed, sz_packed, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? SVDQ_OK
             : SVDQ_ERR_CUDA;
}

svdq_status svdq_awq_gemv_w4a16(const uint16_t *X, int M, const uint8_t *wq_packed, const uint8_t *sz_packed,
                                const float *bias, int N, int K, uint16_t *Y, void *stream) {
  if (!X || !wq_packed || !sz_packed || !Y || N <= 0 || K <= 0 || K % 64 || M <= 0 || M > awq_max_tokens() ||
      awq_smem_bytes(M, K) > 227u * 1024u)
    return SVDQ_ERR_INVALID_ARG;
  // the documented tile limit (the pack kernel runs 32 threads per tile, a grid of < 2^31 threads)
  if (static_cast<uint64_t>((N + 15) / 16) * static_cast<uint64_t>(K / 64) >= (1ull << 26)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(wq_packed) || !aligned16(sz_packed)) return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  return launch_awq_gemv(X, M, wq_packed, sz_packed, bias, N, K, Y, d->err, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? SVDQ_OK
             : SVDQ_ERR_CUDA;
}

svdq_status svdq_linear_forward(const uint16_t *X, int M, const svdq_layer *layer, uint8_t *xq, uint8_t *xs,
                                uint16_t *lora_act, uint16_t *Y, void *stream) {
  svdq_status st = svdq_quant_act_lora_down(X, M, layer, xq, xs, lora_act, stream);
  if (st != SVDQ_OK) return st;
  return svdq_gemm_w4a4_lora_up(xq, xs, lora_act, M, layer, Y, stream);
}

svdq_status svdq_linear_forward_host(const uint16_t *X_host, int M, const svdq_layer *layer, uint16_t *X_dev,
                                     uint8_t *xq, uint8_t *xs, uint16_t *lora_act, uint16_t *Y_dev, uint16_t *Y_host,
                                     void *stream) {
  if (!X_host || !Y_host || !X_dev || !Y_dev || !layer || M <= 0) return SVDQ_ERR_INVALID_ARG;
  svdq_status st = check_layer(layer);
  if (st != SVDQ_OK) return st;
  if (!xq || !xs || (layer->rank > 0 && !lora_act)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X_dev) || !aligned16(Y_dev) || !aligned16(xq) || !aligned16(xs) || !aligned16(lora_act))
    return SVDQ_ERR_MISALIGNED;
  DeviceState *d = nullptr;
  st = device_check(&d);
  if (st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int K = layer->K, N = layer->N, r = layer->rank;
  // Row chunks (multiples of 256 rows: whole K2 tiles and whole 128-row scale blocks, so each
  // chunk's kernels write exactly the bytes the whole-M call would): the copy in of chunk i + 1
  // and the copy out of chunk i - 1 run on their own streams while chunk i's kernels run on
  // `stream`; the two copy directions use separate copy engines of the full-duplex link.
  const int chunk = static_cast<int>(round_up(static_cast<size_t>((M + kHostChunks - 1) / kHostChunks), 256));
  const int n_chunks = (M + chunk - 1) / chunk;
  HostPipe *hp = n_chunks > 1 ? host_pipe(d) : nullptr;
  if (!hp) {
    const size_t xb = static_cast<size_t>(M) * K * 2, yb = static_cast<size_t>(M) * N * 2;
    if (cudaMemcpyAsync(X_dev, X_host, xb, cudaMemcpyHostToDevice, s) != cudaSuccess) return SVDQ_ERR_CUDA;
    st = svdq_linear_forward(X_dev, M, layer, xq, xs, lora_act, Y_dev, stream);
    if (st != SVDQ_OK) return st;
    if (cudaMemcpyAsync(Y_host, Y_dev, yb, cudaMemcpyDeviceToHost, s) != cudaSuccess) return SVDQ_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(hp->mu);
  auto fail = [&]() {
    cudaStreamSynchronize(hp->in);
    cudaStreamSynchronize(hp->out);
    cudaStreamSynchronize(s);
    return SVDQ_ERR_CUDA;
  };
  // the copies wait for the work already enqueued on `stream` (which may still use the buffers)
  if (cudaEventRecord(hp->start, s) != cudaSuccess || cudaStreamWaitEvent(hp->in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->start, 0) != cudaSuccess)
    return fail();
  for (int i = 0; i < n_chunks; ++i) {
    const int r0 = i * chunk, mc = M - r0 < chunk ? M - r0 : chunk;
    const size_t x0 = static_cast<size_t>(r0) * K, y0 = static_cast<size_t>(r0) * N;
    if (cudaMemcpyAsync(X_dev + x0, X_host + x0, static_cast<size_t>(mc) * K * 2, cudaMemcpyHostToDevice, hp->in) !=
            cudaSuccess ||
        cudaEventRecord(hp->in_done[i], hp->in) != cudaSuccess || cudaStreamWaitEvent(s, hp->in_done[i], 0) != cudaSuccess)
      return fail();
    st = svdq_linear_forward(X_dev + x0, mc, layer, xq + x0 / 2, xs + static_cast<size_t>(r0) * (K / 16),
                             r > 0 ? lora_act + static_cast<size_t>(r0) * 2 * r : lora_act, Y_dev + y0, stream);
    if (st != SVDQ_OK) {
      fail();
      return st;
    }
    if (cudaEventRecord(hp->fwd_done[i], s) != cudaSuccess || cudaStreamWaitEvent(hp->out, hp->fwd_done[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(Y_host + y0, Y_dev + y0, static_cast<size_t>(mc) * N * 2, cudaMemcpyDeviceToHost, hp->out) !=
            cudaSuccess)
      return fail();
  }
  // `stream` is ordered after the last copy out
  if (cudaEventRecord(hp->end, hp->out) != cudaSuccess || cudaStreamWaitEvent(s, hp->end, 0) != cudaSuccess)
    return fail();
  return cudaStreamSynchronize(s) == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

svdq_status svdq_baseline_lora_down(const uint16_t *X, int M, const svdq_layer *layer, uint16_t *lora_act,
                                    void *stream) {
  return run_quant(X, M, layer, nullptr, nullptr, lora_act, false, true, stream);
}

svdq_status svdq_baseline_quantize(const uint16_t *X, int M, const svdq_layer *layer, uint8_t *xq, uint8_t *xs,
                                   void *stream) {
  return run_quant(X, M, layer, xq, xs, nullptr, true, false, stream);
}

svdq_status svdq_baseline_gemm_w4a4(const uint8_t *xq, const uint8_t *xs, int M, const svdq_layer *layer, uint16_t *Y,
                                    void *stream) {
  return run_gemm(xq, xs, nullptr, M, layer, Y, true, false, false, stream);
}

svdq_status svdq_baseline_lora_up(const uint16_t *lora_act, int M, const svdq_layer *layer, uint16_t *Y,
                                  void *stream) {
  if (layer && layer->rank == 0) return SVDQ_OK;
  return run_gemm(nullptr, nullptr, lora_act, M, layer, Y, false, true, true, stream);
}

svdq_status svdq_selftest_wait_timeout(uint32_t limit_us, void *stream) {
  if (limit_us < 1 || limit_us > 1000000) return SVDQ_ERR_INVALID_ARG;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  return launch_selftest_wait(d->err, static_cast<uint64_t>(limit_us) * 1000ull, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? SVDQ_OK
             : SVDQ_ERR_CUDA;
}

svdq_status svdq_unswizzle_scales(const uint8_t *blocked, int rows, int K, uint8_t *rowmajor) {
  if (!blocked || !rowmajor || rows <= 0 || K <= 0 || K % 64) return SVDQ_ERR_INVALID_ARG;
  const uint32_t ng = static_cast<uint32_t>(K / 16);
  for (uint32_t m = 0; m < static_cast<uint32_t>(rows); ++m)
    for (uint32_t g = 0; g < ng; ++g) rowmajor[static_cast<size_t>(m) * ng + g] = blocked[scale_offset(m, g, ng)];
  return SVDQ_OK;
}

svdq_status svdq_test_override_capability(int major, int minor) {
  if (major < 0) {
    g_cap_override.store(-1, std::memory_order_relaxed);
    return SVDQ_OK;
  }
  if (major > 99 || minor < 0 || minor > 9) return SVDQ_ERR_INVALID_ARG;
  g_cap_override.store(major * 10 + minor, std::memory_order_relaxed);
  return SVDQ_OK;
}

svdq_status svdq_last_device_error(void *stream, uint32_t *code) {
  if (!code) return SVDQ_ERR_INVALID_ARG;
  DeviceState *d = nullptr;
  svdq_status st = device_check(&d);
  if (st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SVDQ_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, d->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (v && cudaMemset(d->err, 0, sizeof(v)) != cudaSuccess) return SVDQ_ERR_CUDA;
  *code = v;
  return v ? SVDQ_ERR_TIMEOUT : SVDQ_OK;
}

}  // extern "C"
