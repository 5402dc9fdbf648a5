// Dynamic activation scale: the optional pre-pass that takes the activation
// tensor scale from the tensor itself instead of from calibration.
//
// The pages say calibration decides the quantization scales (web page
// "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定适用范围", remio.ai, section
// "基准测试展示了性能提升，但并非普遍结论"); the static s_a of svdq_pack_weights is
// calibrated once, this pass recomputes it for every call:
//   s_a = f32(max_{m,k} |f32(x[m][k] * inv_lambda[k])|) / 2688   (1 when the max is 0)
// in the same f32 steps svdq_quantize_act takes, so that handing its result to
// svdq_quantize_act / svdq_linear_w4a4 is a dynamic-scale layer.
//
// One read of X (16-byte loads, grid sized to the SM count); per block a
// shuffle + shared-memory max; blocks combine through an atomic max on the
// float bits (non-negative floats order like their bit patterns) in a small
// workspace, and the last block to finish (ticket counter in the same
// workspace) writes s_a.  The entry point clears the workspace first.
#include <cuda_runtime.h>

#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int AMAX_THREADS = 512;

__global__ void __launch_bounds__(AMAX_THREADS)
    act_amax_kernel(const uint16_t *X, int M, int K, int ldx, const float *inv_lambda, unsigned int *ws,
                    float *s_a_out) {
  __shared__ float warp_max[AMAX_THREADS / 32];
  __shared__ bool last;
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();
  const int k8 = K / 8;                                   // 8 bf16 (16 bytes) per load
  const long long total = static_cast<long long>(M) * k8;
  float mx = 0.0f;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i / k8), k = static_cast<int>(i % k8) * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<size_t>(m) * ldx + k));
    const float4 i0 = __ldg(reinterpret_cast<const float4 *>(inv_lambda + k));
    const float4 i1 = __ldg(reinterpret_cast<const float4 *>(inv_lambda + k + 4));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const float iv[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      mx = fmaxf(mx, fabsf(__fmul_rn(__uint_as_float(w[j] << 16), iv[2 * j])));
      mx = fmaxf(mx, fabsf(__fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), iv[2 * j + 1])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    mx = threadIdx.x < AMAX_THREADS / 32 ? warp_max[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (threadIdx.x == 0) {
      atomicMax(&ws[0], __float_as_uint(mx));
      __threadfence();
      last = atomicAdd(&ws[1], 1u) == gridDim.x - 1;
    }
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    const float amax = __uint_as_float(atomicMax(&ws[0], 0u));   // every block's maximum is in
    *s_a_out = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
  }
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_act_amax(const void *X, int M, int K, int ldx, const float *inv_lambda, void *workspace,
                             float *s_a, svdq_stream_t stream) {
  if (!X || !inv_lambda || !workspace || !s_a) return fail(SVDQ_ERR_INVALID_ARG, "svdq_act_amax: null pointer");
  if (M < 1 || K < 64 || K % 64 || ldx < K || ldx % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_act_amax: need M >= 1, K % 64 == 0, ldx >= K, ldx % 8 == 0");
  if (!aligned16(X) || !aligned16(inv_lambda) || !aligned16(workspace) || !aligned16(s_a))
    return fail(SVDQ_ERR_ALIGNMENT, "svdq_act_amax: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, SVDQ_AMAX_WORKSPACE_BYTES, s);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_act_amax: memset: ") + cudaGetErrorString(e));
  const long long loads = static_cast<long long>(M) * (K / 8);
  const long long want = (loads + AMAX_THREADS - 1) / AMAX_THREADS;
  const int grid = static_cast<int>(want < 4LL * st->sm_count ? want : 4LL * st->sm_count);
  DependentLaunch dl(dim3(grid), dim3(AMAX_THREADS), 0, s);
  e = cudaLaunchKernelEx(&dl.cfg, act_amax_kernel, static_cast<const uint16_t *>(X), M, K, ldx, inv_lambda,
                         static_cast<unsigned int *>(workspace), s_a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_act_amax launch: ") + cudaGetErrorString(e));
  return ok();
}
