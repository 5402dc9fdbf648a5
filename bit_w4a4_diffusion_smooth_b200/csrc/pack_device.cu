// GPU-side calibration and offline pack of one SVDQuant layer.
//
// The offline workflow on the pages quantizes the weights to 4 bits and
// produces the low-rank branch from calibration data ("Diffusers × Nunchaku
// 4-bit", donmalab.com, section "自行量化模型的流程"; the calibration samples
// decide the scales and the low-rank correction: remio.ai, section
// "基准测试展示了性能提升，但并非普遍结论").  svdq_pack_weights does this on the host;
// this file does the same steps on the GPU, so a model's layers pack in
// milliseconds each instead of seconds:
//   calibration   act_absmax[k] = max over calibration rows of |X[m][k]|
//                 (svdq_calibrate_absmax, accumulating over batches);
//   smoothing     lambda_j = sqrt(absmaxX_j / absmaxW_j), inv_lambda = f32(1/lambda),
//                 W' = W / inv_lambda in float64;
//   top-r SVD     randomized subspace iteration in float64 (oversampling 48,
//                 10 power iterations, each basis re-orthonormalized by
//                 Cholesky QR twice, an eigen-decomposition of the Gram matrix
//                 when Cholesky meets a vanishing direction), then a
//                 Rayleigh-Ritz step: L1 = U_r Sigma_r, L2 = V_r^T, in bf16;
//   residual      R = W' - L1 L2 (float64, the bf16 factors), rounded to f32;
//   NVFP4         s_w = f32(max|R|) / 2688 and the blocks of 16 along K of
//                 every output column into the 256-row weight bundle, in the
//                 f32 steps of the host pack and the activation kernel;
//   s_a           max_j f32(absmaxX_j inv_lambda_j) / 2688.
// The float64 products run on cuBLAS (plain GEMMs); the p x p factorizations
// (p = rank + 48) run on the host between them, so the call synchronizes its
// stream.  Everything else is kernels of this file.
#include <cublas_v2.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <numeric>
#include <string>
#include <vector>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int kOversample = 48;
constexpr int kPowerIters = 10;

// ---------------------------------------------------------------- calibration
// Block (x: 256 groups of 8 columns, y: a range of rows); one 16-byte load of
// 8 bf16 per thread and row, then an atomic max per column on the float bits
// (non-negative floats order like their bit patterns).
__global__ void calib_absmax_kernel(const uint16_t *X, int M, int K, int ldx, int rows_per_block,
                                    unsigned int *amax_bits) {
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= K / 8) return;
  const int r0 = blockIdx.y * rows_per_block, r1 = min(M, r0 + rows_per_block);
  float mx[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int m = r0; m < r1; ++m) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<size_t>(m) * ldx) + g);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      mx[2 * j] = fmaxf(mx[2 * j], fabsf(__uint_as_float(w[j] << 16)));
      mx[2 * j + 1] = fmaxf(mx[2 * j + 1], fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
  }
  if (r0 < r1)
#pragma unroll
    for (int j = 0; j < 8; ++j) atomicMax(amax_bits + 8 * g + j, __float_as_uint(mx[j]));
}

// ---------------------------------------------------------------- pack kernels
// One block per input channel j: absmax of W's row j, the smoothing factor,
// and row j of W' = W / inv_lambda in float64.
__global__ void smooth_kernel(const uint16_t *W, int N, const float *act_absmax, float *inv_lambda, double *Wp) {
  __shared__ float red[32];
  const int j = blockIdx.x;
  const uint16_t *row = W + static_cast<size_t>(j) * N;
  float aw = 0.0f;
  for (int n = threadIdx.x; n < N; n += blockDim.x) aw = fmaxf(aw, fabsf(__uint_as_float(uint32_t(row[n]) << 16)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) aw = fmaxf(aw, __shfl_xor_sync(0xFFFFFFFFu, aw, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = aw;
  __syncthreads();
  if (threadIdx.x < 32) {
    aw = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) aw = fmaxf(aw, __shfl_xor_sync(0xFFFFFFFFu, aw, o));
    if (threadIdx.x == 0) {
      const double ax = static_cast<double>(act_absmax[j]), awd = static_cast<double>(aw);
      const double lam = (ax > 0.0 && awd > 0.0) ? sqrt(ax / awd) : 1.0;
      red[0] = __double2float_rn(1.0 / lam);
      inv_lambda[j] = red[0];
    }
  }
  __syncthreads();
  const double inv = static_cast<double>(red[0]);
  for (int n = threadIdx.x; n < N; n += blockDim.x)
    Wp[static_cast<size_t>(j) * N + n] = static_cast<double>(__uint_as_float(uint32_t(row[n]) << 16)) / inv;
}

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

// Standard normal draws for the random test matrix: element i takes two
// uniforms from splitmix64 (a counter-based generator) of (seed, 2i) and
// (seed, 2i + 1), through Box-Muller.
__global__ void gaussian_kernel(uint64_t seed, size_t n, double *out) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint64_t a = splitmix64(seed ^ (2 * i)), b = splitmix64(seed ^ (2 * i + 1) ^ 0x5851F42D4C957F2Dull);
  const double u1 = (static_cast<double>(a >> 11) + 1.0) * 0x1.0p-53;  // (0, 1]
  const double u2 = static_cast<double>(b >> 11) * 0x1.0p-53;          // [0, 1)
  out[i] = sqrt(-2.0 * log(u1)) * cospi(2.0 * u2);
}

// sigma_i = || column i of Gt [N][r] ||, one block per column.
__global__ void colnorm_kernel(const double *Gt, int N, int r, double *sigma) {
  __shared__ double red[32];
  const int i = blockIdx.x;
  double s = 0.0;
  for (int n = threadIdx.x; n < N; n += blockDim.x) s += Gt[static_cast<size_t>(n) * r + i] * Gt[static_cast<size_t>(n) * r + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x / 32); ++w) t += red[w];
    sigma[i] = sqrt(t);
  }
}

// bf16 bit pattern of the nearest bf16 to v (ties to even), in one rounding:
// the spacing of bf16 around |v| is 2^(e-7), floored at 2^-133.
__device__ __forceinline__ uint16_t bf16_bits_from_double(double v) {
  if (v == 0.0) return signbit(v) ? 0x8000 : 0;
  const double a = fabs(v);
  int e2;
  frexp(a, &e2);
  const int e = max(e2 - 1, -126);
  const double quantum = ldexp(1.0, e - 7);
  const double r = rint(a / quantum) * quantum;
  const float f = __double2float_rn(copysign(r, v));  // exact: at most 8 significant bits
  return static_cast<uint16_t>(__float_as_uint(f) >> 16);
}

// L1 = Ur . Sigma (bf16): l1t [r][K] bits and the rounded values L1r [K][r].
__global__ void l1_kernel(const double *Ur, const double *sigma, int K, int r, uint16_t *l1t, double *L1r) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= K * r) return;
  const int j = idx / r, i = idx % r;
  const uint16_t b = bf16_bits_from_double(Ur[idx] * sigma[i]);
  l1t[static_cast<size_t>(i) * K + j] = b;
  L1r[idx] = static_cast<double>(__uint_as_float(uint32_t(b) << 16));
}

// L2 = Sigma^-1 (Ur^T W') (bf16): the 256-row low-rank tiles of L2^T (columns
// >= r zero) and the rounded values L2r [r][N].
__global__ void l2_kernel(const double *Gt, const double *sigma, int N, int r, uint8_t *l2t, double *L2r) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * SVDQ_LR_STRIDE) return;
  const int n = idx / SVDQ_LR_STRIDE, i = idx % SVDQ_LR_STRIDE;
  uint16_t b = 0;
  if (i < r) {
    const double s = sigma[i];
    b = bf16_bits_from_double(s > 0.0 ? Gt[static_cast<size_t>(n) * r + i] / s : 0.0);
    L2r[static_cast<size_t>(i) * N + n] = static_cast<double>(__uint_as_float(uint32_t(b) << 16));
  }
  *reinterpret_cast<uint16_t *>(l2t + lowrank_offset(n, i, 256)) = b;
}

// f32(R), its absolute maximum (atomic on the float bits), and the optional
// float32 copy of R [K][N].
__global__ void residual_f32_kernel(const double *R, size_t n, float *residual, unsigned int *amax_bits) {
  float mx = 0.0f;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float f = __double2float_rn(R[i]);
    if (residual) residual[i] = f;
    mx = fmaxf(mx, fabsf(f));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(mx));
}

// The fp32 tensor scale of a non-negative maximum: f32(amax) / 2688, 1 when 0.
__device__ __forceinline__ float tensor_scale(float amax) { return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f); }

__global__ void s_w_kernel(const unsigned int *amax_bits, float *s_w) { *s_w = tensor_scale(__uint_as_float(*amax_bits)); }

// NVFP4 of R along K for every output column: thread per (column n, block of
// 16 rows of R), the same f32 steps as the activation kernel and the host
// pack; codes and the four replicas of the block scale into the bundle.
__global__ void quant_weight_kernel(const double *R, int K, int N, const float *s_w_ptr, uint8_t *bundle) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * (K / 16)) return;
  const int n = idx % N, kb = idx / N;          // consecutive threads: consecutive columns (coalesced)
  const float s_w = *s_w_ptr;
  const float d = __fmul_rn(6.0f, s_w);
  float x[16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    x[i] = __double2float_rn(R[static_cast<size_t>(16 * kb + i) * N + n]);
    amax = fmaxf(amax, fabsf(x[i]));
  }
  const uint32_t sb = dev::cvt_e4m3(__fdiv_rn(amax, d));
  const float scale = sb < 127u ? __fmul_rn(dev::e4m3_value(sb), s_w) : 0.0f;
  const float rinv = scale == 0.0f ? 0.0f : __frcp_rn(scale);
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float2 a = dev::mul2_rn(make_float2(x[8 * h], x[8 * h + 1]), make_float2(rinv, rinv));
    const float2 b = dev::mul2_rn(make_float2(x[8 * h + 2], x[8 * h + 3]), make_float2(rinv, rinv));
    const float2 c = dev::mul2_rn(make_float2(x[8 * h + 4], x[8 * h + 5]), make_float2(rinv, rinv));
    const float2 e = dev::mul2_rn(make_float2(x[8 * h + 6], x[8 * h + 7]), make_float2(rinv, rinv));
    w[h] = dev::cvt_e2m1x4(a.x, a.y, b.x, b.y) | (dev::cvt_e2m1x4(c.x, c.y, e.x, e.y) << 16);
  }
  *reinterpret_cast<uint2 *>(bundle + bundle_code_offset(n, 16 * kb, K, 256)) = make_uint2(w[0], w[1]);
#pragma unroll
  for (int rep = 0; rep < 4; ++rep) bundle[bundle_scale_offset(n, 16 * kb, K, 256, rep)] = static_cast<uint8_t>(sb);
}

// s_a = max_j f32(absmaxX_j * inv_lambda_j) / 2688 (one block).
__global__ void s_a_kernel(const float *act_absmax, const float *inv_lambda, int K, float *s_a) {
  __shared__ float red[32];
  float mx = 0.0f;
  for (int j = threadIdx.x; j < K; j += blockDim.x) mx = fmaxf(mx, __fmul_rn(act_absmax[j], inv_lambda[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x / 32); ++w) mx = fmaxf(mx, red[w]);
    mx = fmaxf(mx, red[0]);
    *s_a = tensor_scale(mx);
  }
}

// ---------------------------------------------------------------- host side
struct Workspace {
  double *Wp, *Om, *Y, *Y2, *Z, *G, *T, *Ur, *Gt, *L1r, *L2r, *sigma;
  unsigned int *amax;
};

size_t align_up(size_t v) { return (v + 255) / 256 * 256; }

// Byte offsets of the workspace parts (Wp first); returns the total.
size_t workspace_layout(int K, int N, int r, int p, Workspace *ws, char *base) {
  const size_t sizes[] = {
      sizeof(double) * K * N,  sizeof(double) * N * p, sizeof(double) * K * p, sizeof(double) * K * p,
      sizeof(double) * N * p,  sizeof(double) * p * p, sizeof(double) * p * p, sizeof(double) * K * std::max(r, 1),
      sizeof(double) * N * std::max(r, 1), sizeof(double) * K * std::max(r, 1), sizeof(double) * std::max(r, 1) * N,
      sizeof(double) * 64, 256};
  double **slots[] = {&ws->Wp, &ws->Om, &ws->Y, &ws->Y2, &ws->Z, &ws->G, &ws->T, &ws->Ur, &ws->Gt, &ws->L1r,
                      &ws->L2r, &ws->sigma};
  size_t off = 0;
  for (int i = 0; i < 12; ++i) {
    if (base) *slots[i] = reinterpret_cast<double *>(base + off);
    off += align_up(sizes[i]);
  }
  if (base) ws->amax = reinterpret_cast<unsigned int *>(base + off);
  off += align_up(sizes[12]);
  return off;
}

int oversampled(int K, int N, int r) { return std::min(std::min(K, N), r + kOversample); }

cublasHandle_t cublas_handle(int *rc) {
  static std::mutex mu;
  static cublasHandle_t handles[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    *rc = fail(SVDQ_ERR_CUDA, "svdq_pack_weights_device: no current device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && cublasCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) {
    handles[dev] = nullptr;
    *rc = fail(SVDQ_ERR_CUDA, "svdq_pack_weights_device: cublasCreate failed");
    return nullptr;
  }
  *rc = SVDQ_OK;
  return handles[dev];
}

// Row-major products through column-major cuBLAS: a row-major [a x b] matrix
// is the column-major [b x a] matrix with leading dimension b.
struct Gemm {
  cublasHandle_t h;
  bool ok = true;
  // C [m x n] = A [m x k] . B [k x n]          (all row-major)
  void ab(int m, int n, int k, const double *A, const double *B, double *C, double alpha = 1.0, double beta = 0.0) {
    ok = ok && cublasDgemm(h, CUBLAS_OP_N, CUBLAS_OP_N, n, m, k, &alpha, B, n, A, k, &beta, C, n) ==
                   CUBLAS_STATUS_SUCCESS;
  }
  // C [m x n] = A^T . B with A [k x m], B [k x n] (row-major)
  void atb(int m, int n, int k, const double *A, const double *B, double *C) {
    const double one = 1.0, zero = 0.0;
    ok = ok && cublasDgemm(h, CUBLAS_OP_N, CUBLAS_OP_T, n, m, k, &one, B, n, A, m, &zero, C, n) ==
                   CUBLAS_STATUS_SUCCESS;
  }
};

// Orthonormal basis of the columns of Y [rows][p] (row-major, device), into Y:
// Cholesky QR twice (G = Y^T Y = R^T R, Y <- Y R^-1); when a pivot vanishes
// (a rank-deficient Y) the pass uses the eigen-decomposition of G instead and
// drops the directions whose eigenvalue is below 1e-24 of the largest.
bool orthonormalize(Gemm &g, double *Y, double *Y2, int rows, int p, double *G, double *T, cudaStream_t s,
                    std::vector<double> &hg, std::vector<double> &hm) {
  for (int pass = 0; pass < 2; ++pass) {
    g.atb(p, p, rows, Y, Y, G);
    if (!g.ok || cudaMemcpyAsync(hg.data(), G, sizeof(double) * p * p, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return false;
    // Cholesky: G = L L^T (L lower); M = L^-T so that Y M has orthonormal columns
    std::vector<double> L(static_cast<size_t>(p) * p, 0.0);
    bool chol = true;
    double dmax = 0.0;
    for (int i = 0; i < p; ++i) dmax = std::max(dmax, hg[static_cast<size_t>(i) * p + i]);
    for (int j = 0; j < p && chol; ++j) {
      double d = hg[static_cast<size_t>(j) * p + j];
      for (int k = 0; k < j; ++k) d -= L[static_cast<size_t>(j) * p + k] * L[static_cast<size_t>(j) * p + k];
      if (!(d > 1e-20 * dmax)) {
        chol = false;
        break;
      }
      const double ljj = std::sqrt(d);
      L[static_cast<size_t>(j) * p + j] = ljj;
      for (int i = j + 1; i < p; ++i) {
        double v = hg[static_cast<size_t>(i) * p + j];
        for (int k = 0; k < j; ++k) v -= L[static_cast<size_t>(i) * p + k] * L[static_cast<size_t>(j) * p + k];
        L[static_cast<size_t>(i) * p + j] = v / ljj;
      }
    }
    std::fill(hm.begin(), hm.end(), 0.0);
    if (chol) {
      // Linv lower triangular (forward substitution), M = Linv^T (upper)
      std::vector<double> Li(static_cast<size_t>(p) * p, 0.0);
      for (int c = 0; c < p; ++c) {
        Li[static_cast<size_t>(c) * p + c] = 1.0 / L[static_cast<size_t>(c) * p + c];
        for (int i = c + 1; i < p; ++i) {
          double v = 0.0;
          for (int k = c; k < i; ++k) v -= L[static_cast<size_t>(i) * p + k] * Li[static_cast<size_t>(k) * p + c];
          Li[static_cast<size_t>(i) * p + c] = v / L[static_cast<size_t>(i) * p + i];
        }
      }
      for (int i = 0; i < p; ++i)
        for (int j = 0; j < p; ++j) hm[static_cast<size_t>(i) * p + j] = Li[static_cast<size_t>(j) * p + i];
    } else {
      std::vector<double> C(hg.begin(), hg.end()), V;
      jacobi_eigen(C, p, V);
      double lmax = 0.0;
      for (int i = 0; i < p; ++i) lmax = std::max(lmax, C[static_cast<size_t>(i) * p + i]);
      for (int c = 0; c < p; ++c) {
        const double lam = C[static_cast<size_t>(c) * p + c];
        const double f = lam > 1e-24 * lmax && lam > 0.0 ? 1.0 / std::sqrt(lam) : 0.0;
        for (int i = 0; i < p; ++i) hm[static_cast<size_t>(i) * p + c] = V[static_cast<size_t>(i) * p + c] * f;
      }
    }
    if (cudaMemcpyAsync(T, hm.data(), sizeof(double) * p * p, cudaMemcpyHostToDevice, s) != cudaSuccess) return false;
    g.ab(rows, p, p, Y, T, Y2);
    if (!g.ok || cudaMemcpyAsync(Y, Y2, sizeof(double) * rows * p, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return false;
  }
  return true;
}

int cuda_fail(const char *what, cudaError_t e) {
  return fail(SVDQ_ERR_CUDA, std::string("svdq_pack_weights_device: ") + what + ": " + cudaGetErrorString(e));
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_calibrate_absmax(const void *X, int M, int K, int ldx, float *act_absmax, svdq_stream_t stream) {
  if (!X || !act_absmax) return fail(SVDQ_ERR_INVALID_ARG, "svdq_calibrate_absmax: null pointer");
  if (M < 1 || K < 8 || K % 8 || ldx < K || ldx % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_calibrate_absmax: need M >= 1, K % 8 == 0, ldx >= K, ldx % 8 == 0");
  if (!aligned16(X) || !aligned16(act_absmax))
    return fail(SVDQ_ERR_ALIGNMENT, "svdq_calibrate_absmax: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  const int gx = (K / 8 + 255) / 256;
  const int want_y = std::max(1, (4 * st->sm_count) / gx);
  const int gy = std::min(want_y, M);
  const int rows_per_block = (M + gy - 1) / gy;
  DependentLaunch dl(dim3(gx, (M + rows_per_block - 1) / rows_per_block), dim3(256), 0,
                     reinterpret_cast<cudaStream_t>(stream));
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, calib_absmax_kernel, static_cast<const uint16_t *>(X), M, K, ldx,
                                     rows_per_block, reinterpret_cast<unsigned int *>(act_absmax));
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(SVDQ_ERR_CUDA, std::string("svdq_calibrate_absmax launch: ") + cudaGetErrorString(e));
  return ok();
}

extern "C" int svdq_pack_device_workspace_size(int K, int N, int rank, size_t *bytes) {
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARG, "svdq_pack_device_workspace_size: null pointer");
  if (K < 64 || K % 64 || N < 8 || N % 8 || rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16 || rank > std::min(K, N))
    return fail(SVDQ_ERR_SHAPE, "svdq_pack_device_workspace_size: need K % 64 == 0, N % 8 == 0, rank a multiple "
                                "of 16 in [0, min(64, K, N)]");
  Workspace ws{};
  *bytes = workspace_layout(K, N, rank, oversampled(K, N, rank), &ws, nullptr);
  return ok();
}

extern "C" int svdq_pack_weights_device(const void *W, int K, int N, const float *act_absmax, int rank, uint64_t seed,
                                        float *inv_lambda, void *l1t, uint8_t *l2t, uint8_t *w_bundle, float *s_w,
                                        float *s_a, float *residual, void *workspace, svdq_stream_t stream) {
  static const char *fn = "svdq_pack_weights_device";
  if (!W || !act_absmax || !inv_lambda || !l2t || !w_bundle || !s_w || !s_a || !workspace || (rank > 0 && !l1t))
    return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  size_t ws_bytes = 0;
  int rc = svdq_pack_device_workspace_size(K, N, rank, &ws_bytes);
  if (rc != SVDQ_OK) return rc;
  if (!aligned16(W) || !aligned16(act_absmax) || !aligned16(inv_lambda) || !aligned16(l2t) || !aligned16(w_bundle) ||
      !aligned16(workspace) || (l1t && !aligned16(l1t)) || (residual && !aligned16(residual)))
    return fail(SVDQ_ERR_ALIGNMENT, std::string(fn) + ": pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int p = oversampled(K, N, rank), r = rank;
  Workspace ws{};
  workspace_layout(K, N, r, p, &ws, static_cast<char *>(workspace));

  // 1. smoothing and W'
  smooth_kernel<<<K, 256, 0, s>>>(static_cast<const uint16_t *>(W), N, act_absmax, inv_lambda, ws.Wp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("smoothing", e);

  // 2. top-r basis of W' and the factors
  e = cudaMemsetAsync(l2t, 0, lowrank_bytes(N, 256), s);
  if (e != cudaSuccess) return cuda_fail("memset", e);
  if (r > 0) {
    cublasHandle_t h = cublas_handle(&rc);
    if (!h) return rc;
    if (cublasSetStream(h, s) != CUBLAS_STATUS_SUCCESS) return fail(SVDQ_ERR_CUDA, std::string(fn) + ": cublasSetStream");
    Gemm g{h};
    std::vector<double> hg(static_cast<size_t>(p) * p), hm(static_cast<size_t>(p) * p);
    const size_t n_om = static_cast<size_t>(N) * p;
    gaussian_kernel<<<static_cast<unsigned>((n_om + 255) / 256), 256, 0, s>>>(seed, n_om, ws.Om);
    g.ab(K, p, N, ws.Wp, ws.Om, ws.Y);                                  // Y = W' Omega
    bool okq = orthonormalize(g, ws.Y, ws.Y2, K, p, ws.G, ws.T, s, hg, hm);
    for (int it = 0; it < kPowerIters && okq; ++it) {
      g.atb(N, p, K, ws.Wp, ws.Y, ws.Z);                                 // Z = W'^T Q
      okq = orthonormalize(g, ws.Z, ws.Om, N, p, ws.G, ws.T, s, hg, hm);
      g.ab(K, p, N, ws.Wp, ws.Z, ws.Y);                                 // Y = W' Z
      okq = okq && orthonormalize(g, ws.Y, ws.Y2, K, p, ws.G, ws.T, s, hg, hm);
    }
    if (!okq || !g.ok) return fail(SVDQ_ERR_CUDA, std::string(fn) + ": subspace iteration failed");
    // Rayleigh-Ritz: B^T = W'^T Q [N][p], C = B B^T = Z^T Z [p][p]; top r eigenvectors
    g.atb(N, p, K, ws.Wp, ws.Y, ws.Z);
    g.atb(p, p, N, ws.Z, ws.Z, ws.G);
    e = cudaMemcpyAsync(hg.data(), ws.G, sizeof(double) * p * p, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess || !g.ok) return cuda_fail("Rayleigh-Ritz", e);
    std::vector<double> V;
    jacobi_eigen(hg, p, V);
    std::vector<int> order(p);
    std::iota(order.begin(), order.end(), 0);
    std::sort(order.begin(), order.end(), [&](int a, int b) {
      return hg[static_cast<size_t>(a) * p + a] > hg[static_cast<size_t>(b) * p + b];
    });
    std::vector<double> vsel(static_cast<size_t>(p) * r);
    for (int t = 0; t < p; ++t)
      for (int i = 0; i < r; ++i) vsel[static_cast<size_t>(t) * r + i] = V[static_cast<size_t>(t) * p + order[i]];
    e = cudaMemcpyAsync(ws.T, vsel.data(), sizeof(double) * p * r, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail("copy", e);
    g.ab(K, r, p, ws.Y, ws.T, ws.Ur);                                   // Ur = Q V_r
    g.atb(N, r, K, ws.Wp, ws.Ur, ws.Gt);                                // Gt = W'^T Ur = (Sigma_r V_r^T)^T
    colnorm_kernel<<<r, 256, 0, s>>>(ws.Gt, N, r, ws.sigma);
    l1_kernel<<<(K * r + 255) / 256, 256, 0, s>>>(ws.Ur, ws.sigma, K, r, static_cast<uint16_t *>(l1t), ws.L1r);
    l2_kernel<<<(N * SVDQ_LR_STRIDE + 255) / 256, 256, 0, s>>>(ws.Gt, ws.sigma, N, r, l2t, ws.L2r);
    g.ab(K, N, r, ws.L1r, ws.L2r, ws.Wp, -1.0, 1.0);                    // R = W' - L1 L2, in place
    if (!g.ok) return fail(SVDQ_ERR_CUDA, std::string(fn) + ": residual GEMM failed");
    // the call's work stays ordered on `s`; the caller may free the workspace once it is done
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail("factors", e);
  }

  // 3. f32 residual, s_w, the weight bundle, s_a
  e = cudaMemsetAsync(ws.amax, 0, 256, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(w_bundle, 0, bundle_bytes(N, K, 256), s);
  if (e != cudaSuccess) return cuda_fail("memset", e);
  const size_t kn = static_cast<size_t>(K) * N;
  residual_f32_kernel<<<4 * st->sm_count, 256, 0, s>>>(ws.Wp, kn, residual, ws.amax);
  s_w_kernel<<<1, 1, 0, s>>>(ws.amax, s_w);
  quant_weight_kernel<<<(N * (K / 16) + 255) / 256, 256, 0, s>>>(ws.Wp, K, N, s_w, w_bundle);
  s_a_kernel<<<1, 256, 0, s>>>(act_absmax, inv_lambda, K, s_a);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail("quantization", e);
  return ok();
}
