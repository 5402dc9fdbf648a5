// K2, re-quantizing variant: the W4A4 GEMM of one SVDQ linear whose output is
// the input of the next SVDQ linear (MLP fc1 -> fc2).  The pages fuse the
// low-rank down-projection with the quantization of a layer's input (web page
// "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定适用范围", remio.ai, section
// "SVDQuant 将棘手数值移出 4 位路径"); here that fusion moves into the epilogue of
// the layer that produces the input, so the bf16 activation between the two
// layers never travels through memory and the next layer needs no pass of K1.
//
// One call = three stream operations:
//   1. the fp32 accumulator of the next layer's low-rank input is cleared;
//   2. the GEMM (gemm_w4a4_kernel<EPI, RQ>): per 128 x 256 output tile the
//      epilogue writes the next layer's codes and block scales (one tile of
//      its bundle) and adds bf16(x^) . L1_next over the tile's columns into
//      the accumulator;
//   3. finalize_lowrank_kernel: U_next = bf16(sum / (s_a_next s_w_next)) in
//      the 128-row low-rank tile layout, zero past the rank and past M.
#include "gemm_w4a4_kernel.cuh"

namespace svdq {
namespace w4a4 {
namespace {

// One thread per (row, column pair) of the 128-row padded U tiles.
__global__ void finalize_lowrank_kernel(const float *acc, int M, int rows_padded, int rq, const float *s_a,
                                        const float *s_w, uint8_t *U) {
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int row = idx / (SVDQ_LR_STRIDE / 2), cp = idx % (SVDQ_LR_STRIDE / 2);
  if (row >= rows_padded) return;
  uint32_t o = 0;
  if (row < M && 2 * cp < rq) {
    const float alpha = __fmul_rn(__ldg(s_a), __ldg(s_w));
    const float2 v = *reinterpret_cast<const float2 *>(acc + static_cast<size_t>(row) * rq + 2 * cp);
    __nv_bfloat162 h = __floats2bfloat162_rn(__fdiv_rn(v.x, alpha), __fdiv_rn(v.y, alpha));
    o = *reinterpret_cast<uint32_t *>(&h);
  }
  *reinterpret_cast<uint32_t *>(U + lowrank_offset(row, 2 * cp, 128)) = o;
}

}  // namespace
}  // namespace w4a4
}  // namespace svdq

using namespace svdq;
using namespace svdq::w4a4;

extern "C" int svdq_requant_workspace_size(int M, int next_rank, size_t *bytes) {
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARG, "svdq_requant_workspace_size: null pointer");
  if (M < 1 || next_rank < 0 || next_rank > SVDQ_LR_STRIDE || next_rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_requant_workspace_size: need M >= 1 and next_rank in {0, 16, 32, 48, 64}");
  *bytes = static_cast<size_t>(M) * static_cast<size_t>(next_rank) * sizeof(float);
  return ok();
}

extern "C" int svdq_linear_w4a4_requant(const uint8_t *a_bundle, const void *U, const float *s_a,
                                        const uint8_t *w_bundle, const void *l2t, const float *s_w,
                                        const void *bias, int M, int N, int K, int rank, int epilogue,
                                        int gelu_col_begin, void *Y, int ldy, const float *next_inv_lambda,
                                        const void *next_l1t, int next_rank, const float *next_s_a,
                                        const float *next_s_w, uint8_t *next_a_bundle, void *next_U,
                                        float *workspace, svdq_stream_t stream) {
  static const char *fn = "svdq_linear_w4a4_requant";
  if (!next_inv_lambda || !next_s_a || !next_s_w || !next_a_bundle ||
      (next_rank > 0 && (!next_l1t || !next_U || !workspace)))
    return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": null pointer (next layer)");
  if (N % 64) return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": N (the next layer's K) must be a multiple of 64");
  if (next_rank < 0 || next_rank > SVDQ_LR_STRIDE || next_rank % 16)
    return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": next_rank must be a multiple of 16 in [0, 64]");
  if (!aligned16(next_inv_lambda) || !aligned16(next_a_bundle) ||
      (next_rank > 0 && (!aligned16(next_l1t) || !aligned16(next_U) || !aligned16(workspace))))
    return fail(SVDQ_ERR_ALIGNMENT, std::string(fn) + ": pointers must be 16-byte aligned");
  Maps maps;
  Params p;
  DeviceState *st = nullptr;
  int rc = setup_gemm(fn, a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, epilogue, gelu_col_begin, Y,
                      ldy, true, &maps, &p, &st);
  if (rc != SVDQ_OK) return rc;
  p.nx_inv = next_inv_lambda;
  p.nx_l1t = static_cast<const uint16_t *>(next_l1t);
  p.nx_s_a = next_s_a;
  p.nx_s_w = next_s_w;
  p.nx_bundle = next_a_bundle;
  p.nx_acc = workspace;
  p.nx_ks = bundle_ks(N);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (next_rank > 0) {
    cudaError_t e = cudaMemsetAsync(workspace, 0, static_cast<size_t>(M) * next_rank * sizeof(float), s);
    if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + ": clearing the workspace: " +
                                                         cudaGetErrorString(e));
  }
  switch (next_rank) {
    case 0: rc = launch_gemm<0>(fn, maps, p, st->sm_count, s); break;
    case 16: rc = launch_gemm<16>(fn, maps, p, st->sm_count, s); break;
    case 32: rc = launch_gemm<32>(fn, maps, p, st->sm_count, s); break;
    case 48: rc = launch_gemm<48>(fn, maps, p, st->sm_count, s); break;
    default: rc = launch_gemm<64>(fn, maps, p, st->sm_count, s); break;
  }
  if (rc != SVDQ_OK || next_rank == 0) return rc == SVDQ_OK ? ok() : rc;
  const int rows_padded = (M + 127) / 128 * 128;
  const int threads = 256, total = rows_padded * (SVDQ_LR_STRIDE / 2);
  DependentLaunch dl(dim3((total + threads - 1) / threads), dim3(threads), 0, s);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, finalize_lowrank_kernel, static_cast<const float *>(workspace), M,
                                     rows_padded, next_rank, next_s_a, next_s_w, static_cast<uint8_t *>(next_U));
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + " launch: " + cudaGetErrorString(e));
  return ok();
}

// Allocation-free form of svdq_linear_w4a4_requant: the fp32 partial sums of
// the next layer's low-rank input live in a fixed array of this library's
// device image instead of a caller buffer.  It serves callers that can hand
// the library only the tensors of the layer and no scratch buffer: plugins of
// an inference engine whose interface passes inputs and outputs alone, or
// code that must not call cudaMalloc in the middle of a pipeline (it can
// synchronize the device) and keeps no memory pool of its own.
constexpr size_t kStaticScratchFloats = 262144;   // 1 MiB: M * next_rank <= 262144
static __device__ __align__(256) float g_requant_scratch[kStaticScratchFloats];

namespace {
// Device address of g_requant_scratch, looked up once per device (with that
// device current): in host code the array's name is only a host-side stand-in.
float *static_scratch_address(int *status_out) {
  static std::mutex mu;
  static float *addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    *status_out = fail(SVDQ_ERR_CUDA, "svdq_linear_w4a4_requant_noalloc: no current device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_requant_scratch);
    if (e != cudaSuccess) {
      *status_out = fail(SVDQ_ERR_CUDA, std::string("svdq_linear_w4a4_requant_noalloc: cudaGetSymbolAddress: ") +
                                            cudaGetErrorString(e));
      return nullptr;
    }
    addr[dev] = static_cast<float *>(p);
  }
  *status_out = SVDQ_OK;
  return addr[dev];
}
}  // namespace

extern "C" int svdq_linear_w4a4_requant_noalloc(const uint8_t *a_bundle, const void *U, const float *s_a,
                                                const uint8_t *w_bundle, const void *l2t, const float *s_w,
                                                const void *bias, int M, int N, int K, int rank, int epilogue,
                                                int gelu_col_begin, void *Y, int ldy, const float *next_inv_lambda,
                                                const void *next_l1t, int next_rank, const float *next_s_a,
                                                const float *next_s_w, uint8_t *next_a_bundle, void *next_U,
                                                svdq_stream_t stream) {
  if (M < 1 || next_rank < 0 || static_cast<size_t>(M) * static_cast<size_t>(next_rank > 0 ? next_rank : 0) >
                                    kStaticScratchFloats)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_w4a4_requant_noalloc: M * next_rank must be at most " +
                                    std::to_string(kStaticScratchFloats) + " (the fixed scratch array)");
  if (current_device_state() == nullptr) return SVDQ_ERR_NOT_INITIALIZED;
  int rc = SVDQ_OK;
  float *scratch = static_scratch_address(&rc);
  if (!scratch) return rc;
  return svdq_linear_w4a4_requant(a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, epilogue,
                                  gelu_col_begin, Y, ldy, next_inv_lambda, next_l1t, next_rank, next_s_a, next_s_w,
                                  next_a_bundle, next_U, scratch, stream);
}
