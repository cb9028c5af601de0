// Offline preparation of one layer on the GPU: smoothing factors, the rank-r SVD split of the
// smoothed weight, the fp32 residual and its NVFP4 packing.
//
// "Svdq Int4 Flux.1 Canny Dev" model card, "SVDQuant 概述":
//   stage 2 — outliers move from activations to weights with a per-input-channel factor
//             lambda_j = sqrt(max|X_j|) / sqrt(max|W_j|);
//   stage 3 — the SVD splits the smoothed weight into a 16-bit low-rank branch and a residual.
//
// The truncated SVD of W_hat^T (K x N) comes from the fp64 eigen-decomposition of the smaller
// Gram matrix (W_hat^T W_hat when K <= N, else W_hat W_hat^T), computed by cuSOLVER's
// dsyevd, which is loaded at run time. The other factor is recovered by one fp64 projection
// (Q_r = W_hat P_r S_r^-1, or P_r = W_hat^T Q_r S_r^-1).
#include <dlfcn.h>
#include <stdlib.h>

#include <cusolverDn.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "nvfp4.cuh"

namespace svdq {

// ------------------------------------------------------------------ column maxima
// out must be zero on entry; non-negative floats order like their bit patterns.
__global__ void k_col_absmax_f32(const float *A, int rows, int cols, float *out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int r0 = blockIdx.y * 256;
  const int r1 = min(rows, r0 + 256);
  float mx = 0.0f;
  for (int r = r0; r < r1; ++r) mx = fmaxf(mx, fabsf(A[static_cast<size_t>(r) * cols + c]));
  atomicMax(reinterpret_cast<unsigned int *>(out) + c, __float_as_uint(mx));
}

__global__ void k_col_absmax_bf16(const uint16_t *A, int rows, int cols, float *out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int r0 = blockIdx.y * 256;
  const int r1 = min(rows, r0 + 256);
  float mx = 0.0f;
  for (int r = r0; r < r1; ++r)
    mx = fmaxf(mx, fabsf(__uint_as_float(static_cast<uint32_t>(A[static_cast<size_t>(r) * cols + c]) << 16)));
  atomicMax(reinterpret_cast<unsigned int *>(out) + c, __float_as_uint(mx));
}

template <typename T>
static cudaError_t col_absmax(const T *A, int rows, int cols, float *out, cudaStream_t st,
                              void (*kern)(const T *, int, int, float *)) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * cols, st);
  if (e != cudaSuccess) return e;
  dim3 grid((cols + 255) / 256, (rows + 255) / 256);
  kern<<<grid, 256, 0, st>>>(A, rows, cols, out);
  return cudaGetLastError();
}

cudaError_t launch_col_absmax_f32(const float *A, int rows, int cols, float *out, cudaStream_t st) {
  return col_absmax<float>(A, rows, cols, out, st, k_col_absmax_f32);
}
cudaError_t launch_col_absmax_bf16(const uint16_t *A, int rows, int cols, float *out, cudaStream_t st) {
  return col_absmax<uint16_t>(A, rows, cols, out, st, k_col_absmax_bf16);
}

// ------------------------------------------------------------------ smoothing
// lambda_j = fp32(fp32(sqrt a_x) / fp32(sqrt a_w)) (1 when either maximum is 0),
// inv_lambda_j = fp32(1 / lambda_j); axh_max collects max_j fp32(a_x inv_lambda_j) (zeroed first).
__global__ void k_smoothing(const float *a_x, const float *a_w, int K, float *lam, float *inv_lam,
                            float *axh_max) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const float ax = a_x[j], aw = a_w[j];
  float l = 1.0f;
  if (ax > 0.0f && aw > 0.0f) l = __fdiv_rn(__fsqrt_rn(ax), __fsqrt_rn(aw));
  const float il = __fdiv_rn(1.0f, l);
  if (lam) lam[j] = l;
  inv_lam[j] = il;
  atomicMax(reinterpret_cast<unsigned int *>(axh_max), __float_as_uint(__fmul_rn(ax, il)));
}

// ------------------------------------------------------------------ Gram matrix (fp64)
// side 0: G[i][j] = sum_n What[n][i] What[n][j]  (K x K)
// side 1: G[i][j] = sum_k What[i][k] What[j][k]  (N x N)
// with What[n][k] = W[n][k] * lambda[k] in fp64. 64 x 64 tiles, 16-deep slabs, 4 x 4 per thread.
__global__ void __launch_bounds__(256) k_gram(const float *W, const float *lam, int N, int K, int side, double *G) {
  __shared__ double As[16][65];
  __shared__ double Bs[16][65];
  const int n_out = side == 0 ? K : N;
  const int depth = side == 0 ? N : K;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[4][4] = {};
  for (int t0 = 0; t0 < depth; t0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      int tt, ii;
      if (side == 0) {
        tt = e / 64;
        ii = e % 64;
      } else {
        ii = e / 16;
        tt = e % 16;
      }
      const int t = t0 + tt;
      double va = 0.0, vb = 0.0;
      if (t < depth) {
        if (side == 0) {
          if (i0 + ii < n_out) va = static_cast<double>(W[static_cast<size_t>(t) * K + i0 + ii]) * lam[i0 + ii];
          if (j0 + ii < n_out) vb = static_cast<double>(W[static_cast<size_t>(t) * K + j0 + ii]) * lam[j0 + ii];
        } else {
          if (i0 + ii < n_out) va = static_cast<double>(W[static_cast<size_t>(i0 + ii) * K + t]) * lam[t];
          if (j0 + ii < n_out) vb = static_cast<double>(W[static_cast<size_t>(j0 + ii) * K + t]) * lam[t];
        }
      }
      As[tt][ii] = va;
      Bs[tt][ii] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
      double av[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        av[u] = As[tt][ty + 16 * u];
        bv[u] = Bs[tt][tx + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(av[u], bv[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int i = i0 + ty + 16 * u, j = j0 + tx + 16 * v;
      if (i < n_out && j < n_out) G[static_cast<size_t>(i) * n_out + j] = acc[u][v];
    }
}

// ------------------------------------------------------------------ top-r factors
// E: eigenvectors (column c of the column-major n x n matrix in E[c * n ..]), eigenvalues
// ascending. V[i][j] = eigenvector of the (j+1)-th largest eigenvalue; sig[j] = its sqrt.
__global__ void k_extract(const double *E, const double *evals, int n, int r, double *V, double *sig) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < r) sig[idx] = sqrt(fmax(evals[n - 1 - idx], 0.0));
  if (idx >= n * r) return;
  const int i = idx / r, j = idx % r;
  V[idx] = E[static_cast<size_t>(n - 1 - j) * n + i];
}

// side 0 (V = P, K x r): Out = Q (N x r), Q[n][j] = sum_k What[n][k] P[k][j] / sig[j]
// side 1 (V = Q, N x r): Out = P (K x r), P[k][j] = sum_n What[n][k] Q[n][j] / sig[j]
__global__ void k_project(const float *W, const float *lam, int N, int K, int r, int side, const double *V,
                          const double *sig, double *Out) {
  const int rows = side == 0 ? N : K;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * r) return;
  const int o = idx / r, j = idx % r;
  double acc = 0.0;
  if (side == 0) {
    for (int k = 0; k < K; ++k) acc = fma(static_cast<double>(W[static_cast<size_t>(o) * K + k]) * lam[k], V[k * r + j], acc);
  } else {
    for (int n = 0; n < N; ++n)
      acc = fma(static_cast<double>(W[static_cast<size_t>(n) * K + o]) * lam[o], V[static_cast<size_t>(n) * r + j], acc);
  }
  Out[idx] = sig[j] > 0.0 ? acc / sig[j] : 0.0;
}

// Sign convention: the largest-magnitude entry of column j of P (first on ties) is positive;
// Q's column follows. One block per column.
__global__ void k_fix_sign(double *P, int K, double *Q, int N, int r) {
  const int j = blockIdx.x;
  __shared__ double best_v[256];
  __shared__ int best_i[256];
  double bv = -1.0;
  int bi = 0x7FFFFFFF;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double v = fabs(P[static_cast<size_t>(k) * r + j]);
    if (v > bv || (v == bv && k < bi)) {
      bv = v;
      bi = k;
    }
  }
  best_v[threadIdx.x] = bv;
  best_i[threadIdx.x] = bi;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      const double v2 = best_v[threadIdx.x + w];
      const int i2 = best_i[threadIdx.x + w];
      if (v2 > best_v[threadIdx.x] || (v2 == best_v[threadIdx.x] && i2 < best_i[threadIdx.x])) {
        best_v[threadIdx.x] = v2;
        best_i[threadIdx.x] = i2;
      }
    }
    __syncthreads();
  }
  const bool flip = P[static_cast<size_t>(best_i[0]) * r + j] < 0.0;
  __syncthreads();
  if (!flip) return;
  for (int k = threadIdx.x; k < K; k += blockDim.x) P[static_cast<size_t>(k) * r + j] = -P[static_cast<size_t>(k) * r + j];
  for (int n = threadIdx.x; n < N; n += blockDim.x) Q[static_cast<size_t>(n) * r + j] = -Q[static_cast<size_t>(n) * r + j];
}

// fp64 -> bf16, round to nearest even, written from the IEEE definitions: the significand is
// rounded at the bit that bf16 keeps (7 fraction bits in the normal range; a fixed quantum of
// 2^-133 below 2^-126), then the exactly representable result is re-encoded.
__device__ uint16_t f64_to_bf16_rne(double x) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  const uint16_t sign = static_cast<uint16_t>((u >> 48) & 0x8000u);
  const uint64_t a = u & 0x7FFFFFFFFFFFFFFFull;
  if (a == 0) return sign;
  const int e = static_cast<int>(a >> 52) - 1023;  // inputs here are normal doubles
  const int drop = 45 + (e < -126 ? (-126 - e) : 0);
  if (drop > 53) return sign;
  const uint64_t sig = (a & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  uint64_t q = sig >> drop;
  const uint64_t rem = sig & ((1ull << drop) - 1);
  const uint64_t half = 1ull << (drop - 1);
  if (rem > half || (rem == half && (q & 1))) ++q;
  const double v = static_cast<double>(q) * ldexp(1.0, e - 52 + drop);  // exact
  const float f = static_cast<float>(v);                                 // exact
  return static_cast<uint16_t>(sign | (__float_as_uint(f) >> 16));
}

__device__ __forceinline__ double bf16_to_f64(uint16_t b) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}

// L1t[j][k] = bf16(P[k][j] sqrt(sig_j) / lambda_k) (the smoothing folded into the first factor,
// so that the down-projection reads X itself), L2t[n][j] = bf16(sqrt(sig_j) Q[n][j]).
__global__ void k_make_branch(const double *P, const double *Q, const double *sig, const float *lam, int K, int N,
                              int r, uint16_t *L1t, uint16_t *L2t) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < K * r) {
    const int k = idx / r, j = idx % r;
    L1t[static_cast<size_t>(j) * K + k] = f64_to_bf16_rne(P[idx] * sqrt(sig[j]) / static_cast<double>(lam[k]));
  }
  if (idx < N * r) {
    const int j = idx % r;
    L2t[idx] = f64_to_bf16_rne(sqrt(sig[j]) * Q[idx]);
  }
}

// R[n][k] = fp32(W[n][k] lambda[k] - sum_j lambda[k] L1s[k][j] L2[j][n]) in fp64 (each product
// exact); rmax collects max|R|.
__global__ void k_residual(const float *W, const float *lam, const uint16_t *L1t, const uint16_t *L2t, int N, int K,
                           int r, float *R, float *rmax) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  float mx = 0.0f;
  if (idx < static_cast<size_t>(N) * K) {
    const int n = static_cast<int>(idx / K), k = static_cast<int>(idx % K);
    const double lk = static_cast<double>(lam[k]);
    double lr = 0.0;
    for (int j = 0; j < r; ++j)
      lr += (lk * bf16_to_f64(L1t[static_cast<size_t>(j) * K + k])) * bf16_to_f64(L2t[static_cast<size_t>(n) * r + j]);
    const double what = static_cast<double>(W[idx]) * lk;
    const float v = __double2float_rn(what - lr);
    R[idx] = v;
    mx = fabsf(v);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned int *>(rmax), __float_as_uint(mx));
}

// ------------------------------------------------------------------ NVFP4 rows
// One thread per 16-element group; scales of padding rows are zeroed by the caller.
__global__ void k_quantize_rows(const float *A, int rows, int K, float s, float d, float inv_d, uint8_t *codes,
                                uint8_t *scales) {
  const int ng = K / 16;
  const size_t gi = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gi >= static_cast<size_t>(rows) * ng) return;
  const int row = static_cast<int>(gi / ng), g = static_cast<int>(gi % ng);
  const float4 *src = reinterpret_cast<const float4 *>(A + static_cast<size_t>(row) * K + 16 * g);
  float v[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 t = src[q];
    v[4 * q] = t.x;
    v[4 * q + 1] = t.y;
    v[4 * q + 2] = t.z;
    v[4 * q + 3] = t.w;
  }
  uint2 w;
  const uint32_t sc = nvfp4_group16(v, s, d, inv_d, w.x, w.y);
  *reinterpret_cast<uint2 *>(codes + static_cast<size_t>(row) * (K / 2) + 8 * g) = w;
  scales[scale_offset(row, g, ng)] = static_cast<uint8_t>(sc);
}

cudaError_t launch_quantize_rows(const float *A, int rows, int K, float s, uint8_t *codes, uint8_t *scales,
                                 cudaStream_t st) {
  const float d = 6.0f * s;  // fp32 multiply, round to nearest
  const size_t groups = static_cast<size_t>(rows) * (K / 16);
  const unsigned blocks = static_cast<unsigned>((groups + 255) / 256);
  k_quantize_rows<<<blocks, 256, 0, st>>>(A, rows, K, s, d, 1.0f / d, codes, scales);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ allocation-free smoothing
// Some callers cannot allocate device memory at the point where they need a layer's smoothing
// factors (for example code that runs with a fixed, pre-reserved memory budget, or inside a
// framework that forbids allocation after start-up). This variant of the smoothing stage keeps
// its scratch (the K column maxima of W and the running maximum behind s_x) in a file-scope
// device array instead of the caller's workspace. Every GPU that loads the library holds the
// array until the process exits; all calls share it, so calls that overlap on the GPU race.
constexpr int kNoAllocMaxK = 65536;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxK + 64];

// s = fp32(amax / 2688) (6 x 448), 1 when amax is zero.
__global__ void k_tensor_scale_from_max(const float *amax, float *s_out) {
  const float m = *amax;
  *s_out = m > 0.0f ? __fdiv_rn(m, 2688.0f) : 1.0f;
}

namespace {
struct NoAllocSlot {
  std::once_flag once;
  float *ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
NoAllocSlot g_noalloc_slot[64];
}  // namespace

int noalloc_max_k() { return kNoAllocMaxK; }

cudaError_t smoothing_noalloc(const float *W, const float *act_absmax, int N, int K, float *lambda,
                              float *inv_lambda, float *x_tensor_scale, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || K > kNoAllocMaxK) return cudaErrorInvalidValue;
  NoAllocSlot &slot = g_noalloc_slot[dev];
  // Once per device, with that device current: the device address of the array (host code
  // only sees a host-side stand-in for the symbol).
  std::call_once(slot.once, [&]() {
    void *p = nullptr;
    slot.err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    slot.ptr = static_cast<float *>(p);
  });
  if (slot.err != cudaSuccess) return slot.err;
  float *a_w = slot.ptr;                 // K floats (zeroed by launch_col_absmax_f32)
  float *axh_max = slot.ptr + kNoAllocMaxK;  // one float, zeroed here
  e = cudaMemsetAsync(axh_max, 0, sizeof(float), st);
  if (e != cudaSuccess) return e;
  e = launch_col_absmax_f32(W, N, K, a_w, st);
  if (e != cudaSuccess) return e;
  k_smoothing<<<(K + 255) / 256, 256, 0, st>>>(act_absmax, a_w, K, lambda, inv_lambda, axh_max);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_tensor_scale_from_max<<<1, 1, 0, st>>>(axh_max, x_tensor_scale);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ eigen-solver (dlopen)
namespace {
using fn_create = cusolverStatus_t (*)(cusolverDnHandle_t *);
using fn_destroy = cusolverStatus_t (*)(cusolverDnHandle_t);
using fn_set_stream = cusolverStatus_t (*)(cusolverDnHandle_t, cudaStream_t);
using fn_syevd_bs = cusolverStatus_t (*)(cusolverDnHandle_t, cusolverEigMode_t, cublasFillMode_t, int, const double *,
                                         int, const double *, int *);
using fn_syevd = cusolverStatus_t (*)(cusolverDnHandle_t, cusolverEigMode_t, cublasFillMode_t, int, double *, int,
                                      double *, double *, int, int *);
struct Solver {
  bool loaded = false;
  fn_create create = nullptr;
  fn_destroy destroy = nullptr;
  fn_set_stream set_stream = nullptr;
  fn_syevd_bs syevd_bs = nullptr;
  fn_syevd syevd = nullptr;
};
Solver g_solver;
std::once_flag g_solver_once;

void load_solver() {
  const char *names[3] = {getenv("SVDQ_CUSOLVER_PATH"), "libcusolver.so.11",
#ifdef SVDQ_CUSOLVER_HINT
                          SVDQ_CUSOLVER_HINT
#else
                          nullptr
#endif
  };
  void *h = nullptr;
  for (const char *n : names) {
    if (!n || !*n) continue;
    h = dlopen(n, RTLD_NOW | RTLD_GLOBAL);
    if (h) break;
  }
  if (!h) return;
  g_solver.create = reinterpret_cast<fn_create>(dlsym(h, "cusolverDnCreate"));
  g_solver.destroy = reinterpret_cast<fn_destroy>(dlsym(h, "cusolverDnDestroy"));
  g_solver.set_stream = reinterpret_cast<fn_set_stream>(dlsym(h, "cusolverDnSetStream"));
  g_solver.syevd_bs = reinterpret_cast<fn_syevd_bs>(dlsym(h, "cusolverDnDsyevd_bufferSize"));
  g_solver.syevd = reinterpret_cast<fn_syevd>(dlsym(h, "cusolverDnDsyevd"));
  g_solver.loaded = g_solver.create && g_solver.destroy && g_solver.set_stream && g_solver.syevd_bs && g_solver.syevd;
}

bool solver_ready() {
  std::call_once(g_solver_once, load_solver);
  return g_solver.loaded;
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }
}  // namespace

// Workspace carve-up (each piece 256-byte aligned):
//   G n_g^2 f64 | evals n_g f64 | V n_g*r f64 | P K*r f64 | Q N*r f64 | sig r f64 |
//   R N*K f32 | a_w K f32 | lambda K f32 | scalars 4 f32 | info int | syevd work lwork f64
PrepStatus prepare_plan(int N, int K, int rank, PrepPlan *plan) {
  plan->n_g = K <= N ? K : N;
  plan->side = K <= N ? 0 : 1;
  plan->lwork = 0;
  if (rank > 0) {
    if (!solver_ready()) return PREP_NO_SOLVER;
    cusolverDnHandle_t h;
    if (g_solver.create(&h) != CUSOLVER_STATUS_SUCCESS) return PREP_SOLVER_FAILED;
    int lwork = 0;
    const cusolverStatus_t s = g_solver.syevd_bs(h, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, plan->n_g,
                                                 nullptr, plan->n_g, nullptr, &lwork);
    g_solver.destroy(h);
    if (s != CUSOLVER_STATUS_SUCCESS) return PREP_SOLVER_FAILED;
    plan->lwork = lwork;
  }
  const size_t ng = plan->n_g, r = rank;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  plan->off_G = take(rank ? ng * ng * 8 : 0);
  plan->off_evals = take(rank ? ng * 8 : 0);
  plan->off_V = take(ng * r * 8);
  plan->off_P = take(static_cast<size_t>(K) * r * 8);
  plan->off_Q = take(static_cast<size_t>(N) * r * 8);
  plan->off_sig = take(r * 8);
  plan->off_R = take(static_cast<size_t>(N) * K * 4);
  plan->off_aw = take(static_cast<size_t>(K) * 4);
  plan->off_lam = take(static_cast<size_t>(K) * 4);
  plan->off_scal = take(16);
  plan->off_info = take(16);
  plan->off_work = take(static_cast<size_t>(plan->lwork) * 8);
  plan->bytes = off;
  return PREP_OK;
}

PrepStatus prepare_run(const PrepArgs &p) {
  const PrepPlan &plan = p.plan;
  uint8_t *base = static_cast<uint8_t *>(p.workspace);
  double *G = reinterpret_cast<double *>(base + plan.off_G);
  double *evals = reinterpret_cast<double *>(base + plan.off_evals);
  double *V = reinterpret_cast<double *>(base + plan.off_V);
  double *P = reinterpret_cast<double *>(base + plan.off_P);
  double *Q = reinterpret_cast<double *>(base + plan.off_Q);
  double *sig = reinterpret_cast<double *>(base + plan.off_sig);
  float *R = reinterpret_cast<float *>(base + plan.off_R);
  float *a_w = reinterpret_cast<float *>(base + plan.off_aw);
  float *lam = reinterpret_cast<float *>(base + plan.off_lam);
  float *scal = reinterpret_cast<float *>(base + plan.off_scal);  // [0] max|R|, [1] max a_x inv_lambda
  int *info = reinterpret_cast<int *>(base + plan.off_info);
  double *work = reinterpret_cast<double *>(base + plan.off_work);
  const int N = p.N, K = p.K, r = p.rank;
  cudaStream_t st = p.stream;

#define PCHK(x)                               \
  do {                                        \
    if ((x) != cudaSuccess) return PREP_CUDA; \
  } while (0)

  PCHK(launch_col_absmax_f32(p.W, N, K, a_w, st));
  PCHK(cudaMemsetAsync(scal, 0, 16, st));
  k_smoothing<<<(K + 255) / 256, 256, 0, st>>>(p.act_absmax, a_w, K, lam, p.inv_lambda, scal + 1);
  PCHK(cudaGetLastError());
  if (p.lambda_out) PCHK(cudaMemcpyAsync(p.lambda_out, lam, sizeof(float) * K, cudaMemcpyDeviceToDevice, st));

  if (r > 0) {
    const int ng = plan.n_g;
    dim3 gg((ng + 63) / 64, (ng + 63) / 64);
    k_gram<<<gg, 256, 0, st>>>(p.W, lam, N, K, plan.side, G);
    PCHK(cudaGetLastError());
    cusolverDnHandle_t h;
    if (g_solver.create(&h) != CUSOLVER_STATUS_SUCCESS) return PREP_SOLVER_FAILED;
    cusolverStatus_t cs = g_solver.set_stream(h, st);
    if (cs == CUSOLVER_STATUS_SUCCESS)
      cs = g_solver.syevd(h, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, ng, G, ng, evals, work, plan.lwork,
                          info);
    if (cs != CUSOLVER_STATUS_SUCCESS) {
      g_solver.destroy(h);
      return PREP_SOLVER_FAILED;
    }
    int hinfo = 0;
    PCHK(cudaMemcpyAsync(&hinfo, info, sizeof(int), cudaMemcpyDeviceToHost, st));
    PCHK(cudaStreamSynchronize(st));
    g_solver.destroy(h);
    if (hinfo != 0) return PREP_SOLVER_FAILED;

    const int nr = ng * r;
    k_extract<<<(nr + 255) / 256, 256, 0, st>>>(G, evals, ng, r, V, sig);
    PCHK(cudaGetLastError());
    double *Pdst = plan.side == 0 ? P : Q;  // the factor that came from the eigenvectors
    PCHK(cudaMemcpyAsync(Pdst, V, sizeof(double) * nr, cudaMemcpyDeviceToDevice, st));
    const int prow = plan.side == 0 ? N : K;
    k_project<<<(prow * r + 255) / 256, 256, 0, st>>>(p.W, lam, N, K, r, plan.side, V, sig,
                                                      plan.side == 0 ? Q : P);
    PCHK(cudaGetLastError());
    k_fix_sign<<<r, 256, 0, st>>>(P, K, Q, N, r);
    PCHK(cudaGetLastError());
    const int nb = (K > N ? K : N) * r;
    k_make_branch<<<(nb + 255) / 256, 256, 0, st>>>(P, Q, sig, lam, K, N, r, p.L1t, p.L2t);
    PCHK(cudaGetLastError());
  }
  const size_t nk = static_cast<size_t>(N) * K;
  k_residual<<<static_cast<unsigned>((nk + 255) / 256), 256, 0, st>>>(p.W, lam, p.L1t, p.L2t, N, K, r, R, scal);
  PCHK(cudaGetLastError());
  float hs[2];
  PCHK(cudaMemcpyAsync(hs, scal, sizeof(hs), cudaMemcpyDeviceToHost, st));
  PCHK(cudaStreamSynchronize(st));
  // s = fp32(amax / 2688), 1 when amax is 0 (host fp32 division rounds to nearest).
  const float s_w = hs[0] > 0.0f ? hs[0] / 2688.0f : 1.0f;
  const float s_x = hs[1] > 0.0f ? hs[1] / 2688.0f : 1.0f;
  PCHK(cudaMemsetAsync(p.wscales, 0, p.wscale_bytes, st));
  PCHK(launch_quantize_rows(R, N, K, s_w, p.wq, p.wscales, st));
  if (p.R_out_host) PCHK(cudaMemcpyAsync(p.R_out_host, R, sizeof(float) * nk, cudaMemcpyDeviceToHost, st));
  PCHK(cudaStreamSynchronize(st));
  *p.s_w = s_w;
  *p.s_x = s_x;
  return PREP_OK;
#undef PCHK
}

}  // namespace svdq
