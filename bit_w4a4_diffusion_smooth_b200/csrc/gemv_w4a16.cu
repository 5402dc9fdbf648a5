// K3: AWQ W4A16 projection for small row counts (modulation / adaLN layers).
//
// The pages give these precision-sensitive, low-compute projections 4-bit
// weights and 16-bit activations (web page "Nunchaku Diffusers 支持降低显存占用，
// 但硬件仍决定适用范围", remio.ai, section "Nunchaku Diffusers 支持改变了加载路径").
// With M <= 16 rows the layer is a pass over the weights: the kernel streams
// every weight byte once, in 16-byte coalesced loads, and keeps the
// arithmetic below the memory time:
//   * dequantization in registers: two nibbles at a time become a bf16 pair
//     (128 + q) by one mask-and-or, one bf16x2 subtraction of (128 + z)
//     gives (q - z) exactly;
//   * the products run on the tensor cores as Y^T = W_deq^T . X^T
//     (mma.sync m16n8k16: 16 output columns x 16 k per instruction, the rows
//     of X in the 8-wide N slot); X^ = f32(x * inv_awq) is split into
//     bf16 hi + lo parts so the result keeps ~fp32 accuracy;
//   * per group of 64 k the fp32 partial is scaled by s[n][g] in registers;
//   * a CTA owns NBC blocks of 16 columns, its 16 warps split K by groups,
//     partials are added through shared memory.
// The weight layout (qweight) is the MMA fragment order; see svdq.h.
#include <cuda_runtime.h>

#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int THREADS = 512;
constexpr int WARPS = THREADS / 32;

struct Params {
  int M, K, N, ldx, ldy, G;
  const uint16_t *X;
  const float *inv;
  const uint4 *qw;
  const uint16_t *scales, *zeros, *bias;
  uint16_t *Y;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
// (q - z) for the two nibbles at bits [s, s+4) and [s+16, s+20) of w, as bf16x2.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t w, int s, uint32_t z128) {
  uint32_t t = ((w >> s) & 0x000F000Fu) | 0x43004300u;  // bf16 (128 + q) in each half
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&t);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&z128);
  __nv_bfloat162 d = __hsub2(a, b);
  return *reinterpret_cast<uint32_t *>(&d);
}

// B fragments (hi and lo bf16 parts of X^) of one k16 step for rows nt*8+g.
template <int NT>
__device__ __forceinline__ void load_x_frag(const Params &p, int k, int g8, uint32_t (&bh)[NT][2],
                                            uint32_t (&bl)[NT][2]) {
  const float2 i0 = p.inv ? __ldg(reinterpret_cast<const float2 *>(p.inv + k)) : make_float2(1.f, 1.f);
  const float2 i1 = p.inv ? __ldg(reinterpret_cast<const float2 *>(p.inv + k + 8)) : make_float2(1.f, 1.f);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int m = nt * 8 + g8;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (m < p.M) {
      const uint32_t w0 = __ldg(reinterpret_cast<const uint32_t *>(p.X + static_cast<size_t>(m) * p.ldx + k));
      const uint32_t w1 = __ldg(reinterpret_cast<const uint32_t *>(p.X + static_cast<size_t>(m) * p.ldx + k + 8));
      x[0] = __fmul_rn(__uint_as_float(w0 << 16), i0.x);
      x[1] = __fmul_rn(__uint_as_float(w0 & 0xFFFF0000u), i0.y);
      x[2] = __fmul_rn(__uint_as_float(w1 << 16), i1.x);
      x[3] = __fmul_rn(__uint_as_float(w1 & 0xFFFF0000u), i1.y);
    }
    float h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
      l[i] = x[i] - h[i];  // exact
    }
    bh[nt][0] = pack_bf16x2(h[0], h[1]);
    bh[nt][1] = pack_bf16x2(h[2], h[3]);
    bl[nt][0] = pack_bf16x2(l[0], l[1]);
    bl[nt][1] = pack_bf16x2(l[2], l[3]);
  }
}

template <int NT, int NBC>
__global__ void __launch_bounds__(THREADS, 1) awq_gemv_kernel(Params p) {
  extern __shared__ float red[];  // [WARPS][NBC][NT][32][4]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t = lane & 3;
  const int cb0 = blockIdx.x * NBC;

  float tot[NBC][NT][4];
#pragma unroll
  for (int a = 0; a < NBC; ++a)
#pragma unroll
    for (int b = 0; b < NT; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) tot[a][b][e] = 0.0f;

#pragma unroll 1
  for (int grp = warp; grp < p.G; grp += WARPS) {
    // weights, scales and zero points of this group for the CTA's column blocks
    uint4 wq[NBC];
    float s_lo[NBC], s_hi[NBC];
    uint32_t z_lo[NBC], z_hi[NBC];
#pragma unroll
    for (int cb = 0; cb < NBC; ++cb) {
      wq[cb] = __ldg(p.qw + (static_cast<size_t>(cb0 + cb) * p.G + grp) * 32 + lane);
      const int n = (cb0 + cb) * 16 + g8;
      s_lo[cb] = bf16_bits_to_float(__ldg(p.scales + static_cast<size_t>(n) * p.G + grp));
      s_hi[cb] = bf16_bits_to_float(__ldg(p.scales + static_cast<size_t>(n + 8) * p.G + grp));
      const float zl = bf16_bits_to_float(__ldg(p.zeros + static_cast<size_t>(n) * p.G + grp));
      const float zh = bf16_bits_to_float(__ldg(p.zeros + static_cast<size_t>(n + 8) * p.G + grp));
      z_lo[cb] = pack_bf16x2(128.0f + zl, 128.0f + zl);
      z_hi[cb] = pack_bf16x2(128.0f + zh, 128.0f + zh);
    }
    float c[NBC][NT][4];
#pragma unroll
    for (int a = 0; a < NBC; ++a)
#pragma unroll
      for (int b = 0; b < NT; ++b)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[a][b][e] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t bh[NT][2], bl[NT][2];
      load_x_frag<NT>(p, grp * 64 + 16 * j + 2 * t, g8, bh, bl);
#pragma unroll
      for (int cb = 0; cb < NBC; ++cb) {
        const uint32_t w = j == 0 ? wq[cb].x : j == 1 ? wq[cb].y : j == 2 ? wq[cb].z : wq[cb].w;
        uint32_t a[4];
        a[0] = dequant_pair(w, 0, z_lo[cb]);   // column g,   k 2t, 2t+1
        a[1] = dequant_pair(w, 4, z_hi[cb]);   // column g+8, k 2t, 2t+1
        a[2] = dequant_pair(w, 8, z_lo[cb]);   // column g,   k 2t+8, 2t+9
        a[3] = dequant_pair(w, 12, z_hi[cb]);  // column g+8, k 2t+8, 2t+9
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          dev::mma_bf16_16816(c[cb][nt], a, bh[nt][0], bh[nt][1]);
          dev::mma_bf16_16816(c[cb][nt], a, bl[nt][0], bl[nt][1]);
        }
      }
    }
#pragma unroll
    for (int cb = 0; cb < NBC; ++cb)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        tot[cb][nt][0] = __fmaf_rn(s_lo[cb], c[cb][nt][0], tot[cb][nt][0]);
        tot[cb][nt][1] = __fmaf_rn(s_lo[cb], c[cb][nt][1], tot[cb][nt][1]);
        tot[cb][nt][2] = __fmaf_rn(s_hi[cb], c[cb][nt][2], tot[cb][nt][2]);
        tot[cb][nt][3] = __fmaf_rn(s_hi[cb], c[cb][nt][3], tot[cb][nt][3]);
      }
  }

#pragma unroll
  for (int cb = 0; cb < NBC; ++cb)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[(((warp * NBC + cb) * NT + nt) * 32 + lane) * 4 + e] = tot[cb][nt][e];
  __syncthreads();

  constexpr int SLOTS = NBC * NT * 32 * 4;
  for (int slot = threadIdx.x; slot < SLOTS; slot += THREADS) {
    float v = 0.0f;
#pragma unroll 4
    for (int w = 0; w < WARPS; ++w) v += red[w * SLOTS + slot];
    const int e = slot & 3, ln = (slot >> 2) & 31, nt = (slot >> 7) % NT, cb = (slot >> 7) / NT;
    const int n = (cb0 + cb) * 16 + (ln >> 2) + (e >= 2 ? 8 : 0);
    const int m = nt * 8 + 2 * (ln & 3) + (e & 1);
    if (m < p.M && n < p.N) {
      if (p.bias) v += bf16_bits_to_float(p.bias[n]);
      __nv_bfloat16 h = __float2bfloat16_rn(v);
      p.Y[static_cast<size_t>(m) * p.ldy + n] = *reinterpret_cast<uint16_t *>(&h);
    }
  }
}

template <int NT, int NBC>
int launch(const Params &p, cudaStream_t stream) {
  const int smem = WARPS * NBC * NT * 32 * 4 * static_cast<int>(sizeof(float));
  cudaError_t e = cudaFuncSetAttribute(awq_gemv_kernel<NT, NBC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("awq_linear_w4a16: ") + cudaGetErrorString(e));
  const int grid = p.N / (16 * NBC);
  awq_gemv_kernel<NT, NBC><<<grid, THREADS, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("awq_linear_w4a16 launch: ") + cudaGetErrorString(e));
  return ok();
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int awq_linear_w4a16(const void *X, int M, int K, int ldx, const float *inv_awq, const uint32_t *qweight,
                                const void *scales, const void *zeros, int group, const void *bias, int N, void *Y,
                                int ldy, svdq_stream_t stream) {
  if (!X || !qweight || !scales || !zeros || !Y) return fail(SVDQ_ERR_INVALID_ARG, "awq_linear_w4a16: null pointer");
  if (group != 64) return fail(SVDQ_ERR_SHAPE, "awq_linear_w4a16: group must be 64");
  if (M < 1 || M > 16 || K < 64 || K % 64 || N < 16 || N % 16 || ldx < K || ldx % 8 || ldy < N || ldy % 8)
    return fail(SVDQ_ERR_SHAPE,
                "awq_linear_w4a16: need 1 <= M <= 16, K % 64 == 0, N % 16 == 0, ldx >= K, ldy >= N, ldx/ldy % 8 == 0");
  if (!aligned16(X) || !aligned16(qweight) || (inv_awq && !aligned16(inv_awq)) || !aligned16(Y))
    return fail(SVDQ_ERR_ALIGNMENT, "awq_linear_w4a16: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  Params p;
  p.M = M;
  p.K = K;
  p.N = N;
  p.ldx = ldx;
  p.ldy = ldy;
  p.G = K / 64;
  p.X = static_cast<const uint16_t *>(X);
  p.inv = inv_awq;
  p.qw = reinterpret_cast<const uint4 *>(qweight);
  p.scales = static_cast<const uint16_t *>(scales);
  p.zeros = static_cast<const uint16_t *>(zeros);
  p.bias = static_cast<const uint16_t *>(bias);
  p.Y = static_cast<uint16_t *>(Y);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int blocks16 = N / 16;
  if (M <= 8) {
    if (blocks16 % 4 == 0) return launch<1, 4>(p, s);
    if (blocks16 % 2 == 0) return launch<1, 2>(p, s);
    return launch<1, 1>(p, s);
  }
  if (blocks16 % 2 == 0) return launch<2, 2>(p, s);
  return launch<2, 1>(p, s);
}
