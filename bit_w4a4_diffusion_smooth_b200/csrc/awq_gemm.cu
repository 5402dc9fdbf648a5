// AWQ W4A16 for many rows: the GEMM path beside K3's GEMV.
//
// The pages give the modulation / adaptive-norm projections 4-bit weights and
// 16-bit activations (web page "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定
// 适用范围", remio.ai, section "Nunchaku Diffusers 支持改变了加载路径").  K3 reads
// the packed weights once per block of 16 rows, which is right for the few
// rows a modulation layer has and wasteful for hundreds.  With many rows the
// weights are worth expanding once:
//   1. awq_dequant_kernel: w = f32(inv_awq[k] * (q - z) * s), the layer's
//      weight with the AWQ input scale folded into its rows, split into two
//      K x N bf16 matrices W_hi = bf16(w) and W_lo = bf16(w - W_hi) in the
//      caller's workspace (together ~16 significant bits, as the GEMV's hi/lo
//      split of X^ keeps).  One CTA per (quad of 64 columns, group of 64
//      along K): it decodes the group's 2 KB of packed words (the fragment
//      order of svdq.h) into 64 x 64 tiles in shared memory and writes them
//      out as full 128-byte rows.
//   2. D = X . W_hi, then D += X . W_lo: two bf16 GEMMs with fp32 output
//      through cuBLASLt (plain library GEMMs) into the workspace;
//   3. awq_finalize_kernel: Y = bf16(D + bias), one rounding.
// The weight expansion costs one pass over 4*K*N bytes; the GEMMs then run at
// tensor-core rate instead of ceil(M/16) passes over the packed weights.
#include <cublasLt.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <string>

#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int DQ_THREADS = 128;   // 4 words per thread: one (quad, group) = 4 blocks x 128 words

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__global__ void __launch_bounds__(DQ_THREADS) awq_dequant_kernel(const uint32_t *qweight, const uint16_t *scales,
                                                                  const uint16_t *zeros, const float *inv_awq,
                                                                  int K, int N, uint16_t *w_hi, uint16_t *w_lo) {
  __shared__ __align__(16) uint16_t tile[2][64][64 + 8];   // hi / lo, [k in group][column in quad], padded rows
  const int quad = blockIdx.x, grp = blockIdx.y, G = K / 64;
  const size_t base = (static_cast<size_t>(quad) * G + grp) * 4 * 128;   // this (quad, group)'s 512 words
  const size_t sz = (static_cast<size_t>(quad) * G + grp) * 64;          // its 64 scales and zero points
  for (int w = threadIdx.x; w < 512; w += DQ_THREADS) {
    const int blk = w / 128, lane = (w % 128) / 4, j = w % 4;
    const int g = lane / 4, t = lane % 4;
    const uint32_t word = __ldg(qweight + base + w);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = g + ((i & 1) ? 8 : 0);
      const int kq = 2 * t + ((i & 2) ? 8 : 0) + ((i & 4) ? 1 : 0);
      const int k = 16 * j + kq, col = blk * 16 + c;
      const float q = static_cast<float>((word >> (4 * i)) & 0xFu);
      const float s = bf16_to_f32(__ldg(scales + sz + col)), z = bf16_to_f32(__ldg(zeros + sz + col));
      const float v = __fmul_rn(__fmul_rn(__ldg(inv_awq + grp * 64 + k), q - z), s);
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));   // v - hi is exact in f32
      tile[0][k][col] = *reinterpret_cast<const uint16_t *>(&h);
      tile[1][k][col] = *reinterpret_cast<const uint16_t *>(&l);
    }
  }
  __syncthreads();
  // 2 x 64 rows of 128 bytes: thread -> (matrix, row, 16-byte chunk)
  for (int e = threadIdx.x; e < 2 * 64 * 8; e += DQ_THREADS) {
    const int hl = e / 512, k = (e / 8) % 64, ch = e % 8;
    const uint4 v = *reinterpret_cast<const uint4 *>(&tile[hl][k][ch * 8]);
    *reinterpret_cast<uint4 *>((hl ? w_lo : w_hi) + static_cast<size_t>(grp * 64 + k) * N + quad * 64 + ch * 8) = v;
  }
}

// Y = bf16(D + bias): one thread per 4 consecutive outputs of a row.
__global__ void awq_finalize_kernel(const float *D, const uint16_t *bias, int M, int N, uint16_t *Y, int ldy) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int n4 = N / 4;
  if (idx >= static_cast<size_t>(M) * n4) return;
  const int m = static_cast<int>(idx / n4), n = static_cast<int>(idx % n4) * 4;
  const float4 d = *reinterpret_cast<const float4 *>(D + static_cast<size_t>(m) * N + n);
  float b[4] = {0.f, 0.f, 0.f, 0.f};
  if (bias) {
    const uint2 bb = *reinterpret_cast<const uint2 *>(bias + n);
    b[0] = __uint_as_float(bb.x << 16);
    b[1] = __uint_as_float(bb.x & 0xFFFF0000u);
    b[2] = __uint_as_float(bb.y << 16);
    b[3] = __uint_as_float(bb.y & 0xFFFF0000u);
  }
  const __nv_bfloat162 y0 = __floats2bfloat162_rn(__fadd_rn(d.x, b[0]), __fadd_rn(d.y, b[1]));
  const __nv_bfloat162 y1 = __floats2bfloat162_rn(__fadd_rn(d.z, b[2]), __fadd_rn(d.w, b[3]));
  uint2 o;
  o.x = *reinterpret_cast<const uint32_t *>(&y0);
  o.y = *reinterpret_cast<const uint32_t *>(&y1);
  *reinterpret_cast<uint2 *>(Y + static_cast<size_t>(m) * ldy + n) = o;
}

cublasLtHandle_t lt_handle(int *rc) {
  static std::mutex mu;
  static cublasLtHandle_t handles[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    *rc = fail(SVDQ_ERR_CUDA, "awq_linear_w4a16_gemm: no current device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && cublasLtCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) {
    handles[dev] = nullptr;
    *rc = fail(SVDQ_ERR_CUDA, "awq_linear_w4a16_gemm: cublasLtCreate failed");
    return nullptr;
  }
  *rc = SVDQ_OK;
  return handles[dev];
}

// D^T [N x M] (=|+=) W^T [N x K] . X^T [K x M], column-major views of the row-major buffers; D fp32, ld N.
int lt_gemm(cublasLtHandle_t h, const uint16_t *w, const void *X, float *D, float beta, int M, int N, int K, int ldx,
            cudaStream_t stream) {
  static const char *fn = "awq_linear_w4a16_gemm";
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  int rc = SVDQ_OK;
  bool ok = cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) == CUBLAS_STATUS_SUCCESS;
  const cublasOperation_t no = CUBLAS_OP_N;
  ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &no, sizeof(no)) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &no, sizeof(no)) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, N, K, N) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, K, M, ldx) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, N, M, N) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS;
  const size_t no_ws = 0;
  ok = ok && cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &no_ws,
                                                  sizeof(no_ws)) == CUBLAS_STATUS_SUCCESS;
  cublasLtMatmulHeuristicResult_t heur;
  std::memset(&heur, 0, sizeof(heur));
  int found = 0;
  ok = ok && cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &heur, &found) == CUBLAS_STATUS_SUCCESS &&
       found > 0;
  if (!ok) {
    rc = fail(SVDQ_ERR_CUDA, std::string(fn) + ": no cuBLASLt algorithm for the bf16 GEMM");
  } else {
    const float alpha = 1.0f;
    if (cublasLtMatmul(h, op, &alpha, w, la, X, lb, &beta, D, lc, D, lc, &heur.algo, nullptr, 0, stream) !=
        CUBLAS_STATUS_SUCCESS)
      rc = fail(SVDQ_ERR_CUDA, std::string(fn) + ": cublasLtMatmul failed");
  }
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return rc;
}

}  // namespace
}  // namespace svdq

using namespace svdq;

// Workspace: W_hi and W_lo (K x N bf16 each), then D (M x N fp32).
extern "C" int awq_gemm_workspace_size(int M, int K, int N, size_t *bytes) {
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARG, "awq_gemm_workspace_size: null pointer");
  if (M < 1 || K < 64 || K % 64 || N < 64 || N % 64)
    return fail(SVDQ_ERR_SHAPE, "awq_gemm_workspace_size: need M >= 1, K % 64 == 0 and N % 64 == 0");
  *bytes = static_cast<size_t>(K) * static_cast<size_t>(N) * 4 + static_cast<size_t>(M) * static_cast<size_t>(N) * 4;
  return ok();
}

namespace {
int check_expand(const char *fn, const float *inv_awq, const uint32_t *qweight, const void *scales, const void *zeros,
                 int K, int N, int group, const void *workspace) {
  if (!inv_awq || !qweight || !scales || !zeros || !workspace)
    return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (group != 64) return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": group must be 64");
  if (K < 64 || K % 64 || N < 64 || N % 64)
    return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": need K % 64 == 0 and N % 64 == 0");
  if (!aligned16(inv_awq) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(workspace))
    return fail(SVDQ_ERR_ALIGNMENT, std::string(fn) + ": pointers must be 16-byte aligned");
  return SVDQ_OK;
}
int check_gemm(const char *fn, const void *X, int M, int K, int ldx, const void *bias, int N, const void *Y, int ldy,
               const void *workspace) {
  if (!X || !Y || !workspace) return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (M < 1 || K < 64 || K % 64 || N < 64 || N % 64 || ldx < K || ldx % 8 || ldy < N || ldy % 8)
    return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": need M >= 1, K % 64 == 0, N % 64 == 0, ldx >= K, ldy >= N, "
                                                  "ldx/ldy % 8 == 0");
  if (!aligned16(X) || !aligned16(Y) || !aligned16(workspace) || (bias && !aligned16(bias)))
    return fail(SVDQ_ERR_ALIGNMENT, std::string(fn) + ": pointers must be 16-byte aligned");
  return SVDQ_OK;
}
int enqueue_expand(const char *fn, const float *inv_awq, const uint32_t *qweight, const void *scales,
                   const void *zeros, int K, int N, void *workspace, cudaStream_t s) {
  uint16_t *w_hi = static_cast<uint16_t *>(workspace);
  uint16_t *w_lo = w_hi + static_cast<size_t>(K) * N;
  awq_dequant_kernel<<<dim3(N / 64, K / 64), DQ_THREADS, 0, s>>>(
      qweight, static_cast<const uint16_t *>(scales), static_cast<const uint16_t *>(zeros), inv_awq, K, N, w_hi, w_lo);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + " launch: " + cudaGetErrorString(e));
  return SVDQ_OK;
}
int enqueue_gemm(const char *fn, const void *X, int M, int K, int ldx, const void *bias, int N, void *Y, int ldy,
                 void *workspace, cudaStream_t s) {
  int rc = SVDQ_OK;
  cublasLtHandle_t h = lt_handle(&rc);
  if (!h) return rc;
  const uint16_t *w_hi = static_cast<const uint16_t *>(workspace);
  const uint16_t *w_lo = w_hi + static_cast<size_t>(K) * N;
  float *D = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + static_cast<size_t>(K) * N * 4);
  rc = lt_gemm(h, w_hi, X, D, 0.0f, M, N, K, ldx, s);
  if (rc == SVDQ_OK) rc = lt_gemm(h, w_lo, X, D, 1.0f, M, N, K, ldx, s);
  if (rc != SVDQ_OK) return rc;
  const size_t total = static_cast<size_t>(M) * (N / 4);
  awq_finalize_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      D, static_cast<const uint16_t *>(bias), M, N, static_cast<uint16_t *>(Y), ldy);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + " launch: " + cudaGetErrorString(e));
  return SVDQ_OK;
}
}  // namespace

extern "C" int awq_expand_weights(const float *inv_awq, const uint32_t *qweight, const void *scales, const void *zeros,
                                  int K, int N, int group, void *workspace, svdq_stream_t stream) {
  static const char *fn = "awq_expand_weights";
  int rc = check_expand(fn, inv_awq, qweight, scales, zeros, K, N, group, workspace);
  if (rc != SVDQ_OK) return rc;
  if (!current_device_state()) return SVDQ_ERR_NOT_INITIALIZED;
  rc = enqueue_expand(fn, inv_awq, qweight, scales, zeros, K, N, workspace, reinterpret_cast<cudaStream_t>(stream));
  return rc == SVDQ_OK ? ok() : rc;
}

extern "C" int awq_linear_w4a16_expanded(const void *X, int M, int K, int ldx, const void *bias, int N, void *Y,
                                         int ldy, void *workspace, svdq_stream_t stream) {
  static const char *fn = "awq_linear_w4a16_expanded";
  int rc = check_gemm(fn, X, M, K, ldx, bias, N, Y, ldy, workspace);
  if (rc != SVDQ_OK) return rc;
  if (!current_device_state()) return SVDQ_ERR_NOT_INITIALIZED;
  rc = enqueue_gemm(fn, X, M, K, ldx, bias, N, Y, ldy, workspace, reinterpret_cast<cudaStream_t>(stream));
  return rc == SVDQ_OK ? ok() : rc;
}

extern "C" int awq_linear_w4a16_gemm(const void *X, int M, int K, int ldx, const float *inv_awq,
                                     const uint32_t *qweight, const void *scales, const void *zeros, int group,
                                     const void *bias, int N, void *Y, int ldy, void *workspace,
                                     svdq_stream_t stream) {
  static const char *fn = "awq_linear_w4a16_gemm";
  int rc = check_expand(fn, inv_awq, qweight, scales, zeros, K, N, group, workspace);
  if (rc == SVDQ_OK) rc = check_gemm(fn, X, M, K, ldx, bias, N, Y, ldy, workspace);
  if (rc != SVDQ_OK) return rc;
  if (!current_device_state()) return SVDQ_ERR_NOT_INITIALIZED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rc = enqueue_expand(fn, inv_awq, qweight, scales, zeros, K, N, workspace, s);
  if (rc == SVDQ_OK) rc = enqueue_gemm(fn, X, M, K, ldx, bias, N, Y, ldy, workspace, s);
  return rc == SVDQ_OK ? ok() : rc;
}
