// K3: AWQ W4A16 projection for small row counts (modulation / adaLN layers).
//
// The pages give these precision-sensitive, low-compute projections 4-bit
// weights and 16-bit activations (web page "Nunchaku Diffusers 支持降低显存占用，
// 但硬件仍决定适用范围", remio.ai, section "Nunchaku Diffusers 支持改变了加载路径").
// With up to 16 rows the layer is one pass over the weights and the kernel
// is bound by how many weight bytes are in flight:
//   * one CTA per quad of 64 output columns, its 16 warps split K by groups
//     of 64; before any arithmetic each warp requests all of its groups'
//     weights (4 x 16 bytes per lane and group: the four 16-column blocks),
//     scales and zero points, so a CTA has 48 KB in flight (K = 3072);
//   * the products run on the tensor cores as Y^T = W^T . X^T (mma.sync
//     m16n8k16: 16 output columns x 16 k per instruction, the rows of X in
//     the 8-wide slot); X^ = f32(x * inv_awq) is split into bf16 hi + lo
//     parts (hi + lo carries ~16 significant bits), one MMA each;
//   * dequantization in registers: two nibbles at a time become a bf16 pair
//     (128 + q) by one mask-and-or, one bf16x2 subtraction of (128 + z)
//     gives (q - z) exactly;
//   * per group the fp32 partial is scaled by s in registers; the warps'
//     partials are added through shared memory.
// More than 16 rows (a batch of modulation vectors) run as blocks of 16 rows
// on the grid's second dimension; each block is one more pass over the
// weights, mostly from L2.
// The weight layout (qweight) is the MMA fragment order; see svdq.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }
// bf16 (128 + q) for the two nibbles at bits [0, 4) and [16, 20) of w.
__device__ __forceinline__ uint32_t nib_pair(uint32_t w) { return (w & 0x000F000Fu) | 0x43004300u; }

// The 4 A fragments (16 columns x 16 k) of k16-step word w: (128 + q) as bf16.
__device__ __forceinline__ void a_frags(uint32_t w, uint32_t (&a)[4]) {
  a[0] = nib_pair(w);         // column g,   k 2t, 2t+1
  a[1] = nib_pair(w >> 4);    // column g+8, k 2t, 2t+1
  a[2] = nib_pair(w >> 8);    // column g,   k 2t+8, 2t+9
  a[3] = nib_pair(w >> 12);   // column g+8, k 2t+8, 2t+9
}

// ===========================================================================
// Direct kernel: one CTA per quad and block of 8 NT rows, 16 warps split K by groups.
constexpr int D_THREADS = 512;
constexpr int D_WARPS = D_THREADS / 32;

struct Params {
  int M, K, N, ldx, ldy, G;
  const uint16_t *X;
  const float *inv;
  const uint4 *qw;
  const uint16_t *scales, *zeros, *bias;
  uint16_t *Y;
};

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

// (q - z) for the two nibbles at bits [s, s+4) and [s+16, s+20) of w, as bf16x2.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t w, int s, uint32_t z128) {
  uint32_t t = nib_pair(w >> s);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&t);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&z128);
  __nv_bfloat162 d = __hsub2(a, b);
  return *reinterpret_cast<uint32_t *>(&d);
}

template <int NT, int GPW>
__global__ void __launch_bounds__(D_THREADS, 1) awq_gemv_kernel(Params p) {
  extern __shared__ float red[];  // [WARPS][4][NT][32][4]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t = lane & 3;
  const int quad = blockIdx.x;
  {  // this CTA's block of 8 NT rows
    const int r0 = static_cast<int>(blockIdx.y) * 8 * NT;
    p.X += static_cast<size_t>(r0) * p.ldx;
    p.Y += static_cast<size_t>(r0) * p.ldy;
    p.M = min(8 * NT, p.M - r0);
  }
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();

  float tot[4][NT][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < NT; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) tot[a][b][e] = 0.0f;

#pragma unroll 1
  for (int base = 0; base < p.G; base += D_WARPS * GPW) {
  // every weight, scale and zero point of this slice, requested before any arithmetic:
  // groups base + warp, base + warp + 16, ... of the quad, 4 column blocks each
  uint4 wq[GPW][4];
  uint32_t sp[GPW][4], zp[GPW][4];  // bf16 of columns g (low half) and g + 8 (high half)
#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int grp = base + warp + D_WARPS * i;
    const size_t blk = static_cast<size_t>(quad) * p.G + (grp < p.G ? grp : 0);
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
      if (grp < p.G) {
        wq[i][cb] = __ldg(p.qw + (blk * 4 + cb) * 32 + lane);
        const size_t gb = blk * 64 + cb * 16 + g8;
        sp[i][cb] = static_cast<uint32_t>(__ldg(p.scales + gb)) | (static_cast<uint32_t>(__ldg(p.scales + gb + 8)) << 16);
        zp[i][cb] = static_cast<uint32_t>(__ldg(p.zeros + gb)) | (static_cast<uint32_t>(__ldg(p.zeros + gb + 8)) << 16);
      } else {
        wq[i][cb] = make_uint4(0, 0, 0, 0);
        sp[i][cb] = zp[i][cb] = 0;
      }
    }
  }

#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int grp = base + warp + D_WARPS * i;
    if (grp >= p.G) break;
    uint32_t z_lo[4], z_hi[4];
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
      const float zl = bf16_bits_to_float(zp[i][cb] & 0xFFFFu), zh = bf16_bits_to_float(zp[i][cb] >> 16);
      z_lo[cb] = pack_bf16x2(128.0f + zl, 128.0f + zl);
      z_hi[cb] = pack_bf16x2(128.0f + zh, 128.0f + zh);
    }
    float c[4][NT][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < NT; ++b)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[a][b][e] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t bh[NT][2], bl[NT][2];
      load_x_frag<NT>(p, grp * 64 + 16 * j + 2 * t, g8, bh, bl);
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        const uint4 &w4 = wq[i][cb];
        const uint32_t w = j == 0 ? w4.x : j == 1 ? w4.y : j == 2 ? w4.z : w4.w;
        uint32_t a[4];
        a[0] = dequant_pair(w, 0, z_lo[cb]);
        a[1] = dequant_pair(w, 4, z_hi[cb]);
        a[2] = dequant_pair(w, 8, z_lo[cb]);
        a[3] = dequant_pair(w, 12, z_hi[cb]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          dev::mma_bf16_16816(c[cb][nt], a, bh[nt][0], bh[nt][1]);
          dev::mma_bf16_16816(c[cb][nt], a, bl[nt][0], bl[nt][1]);
        }
      }
    }
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
      const float s_lo = bf16_bits_to_float(sp[i][cb] & 0xFFFFu), s_hi = bf16_bits_to_float(sp[i][cb] >> 16);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        tot[cb][nt][0] = __fmaf_rn(s_lo, c[cb][nt][0], tot[cb][nt][0]);
        tot[cb][nt][1] = __fmaf_rn(s_lo, c[cb][nt][1], tot[cb][nt][1]);
        tot[cb][nt][2] = __fmaf_rn(s_hi, c[cb][nt][2], tot[cb][nt][2]);
        tot[cb][nt][3] = __fmaf_rn(s_hi, c[cb][nt][3], tot[cb][nt][3]);
      }
    }
  }
  }

#pragma unroll
  for (int cb = 0; cb < 4; ++cb)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[(((warp * 4 + cb) * NT + nt) * 32 + lane) * 4 + e] = tot[cb][nt][e];
  __syncthreads();

  constexpr int SLOTS = 4 * NT * 32 * 4;
  for (int slot = threadIdx.x; slot < SLOTS; slot += D_THREADS) {
    float v = 0.0f;
#pragma unroll 4
    for (int w = 0; w < D_WARPS; ++w) v += red[w * SLOTS + slot];
    const int e = slot & 3, ln = (slot >> 2) & 31, nt = (slot >> 7) % NT, cb = (slot >> 7) / NT;
    const int n = quad * 64 + cb * 16 + (ln >> 2) + (e >= 2 ? 8 : 0);
    const int m = nt * 8 + 2 * (ln & 3) + (e & 1);
    if (m < p.M) {
      if (p.bias) v += bf16_bits_to_float(p.bias[n]);
      __nv_bfloat16 h = __float2bfloat16_rn(v);
      p.Y[static_cast<size_t>(m) * p.ldy + n] = *reinterpret_cast<uint16_t *>(&h);
    }
  }
}

template <int NT, int GPW>
int launch_direct(const Params &p, cudaStream_t stream) {
  const int smem = D_WARPS * 4 * NT * 32 * 4 * static_cast<int>(sizeof(float));
  cudaError_t e =
      cudaFuncSetAttribute(awq_gemv_kernel<NT, GPW>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("awq_linear_w4a16: ") + cudaGetErrorString(e));
  DependentLaunch dl(dim3(p.N / 64, (p.M + 8 * NT - 1) / (8 * NT)), dim3(D_THREADS), smem, stream);
  e = cudaLaunchKernelEx(&dl.cfg, awq_gemv_kernel<NT, GPW>, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("awq_linear_w4a16 launch: ") + cudaGetErrorString(e));
  return ok();
}

// Groups per warp (G / 16 rounded up, at most 3 for one row block of X and 1
// for two, which keeps every operand in registers) picks the instantiation;
// a longer K is walked in slices.
int launch_direct_g(const Params &p, cudaStream_t stream) {
  if (p.M > 8) return launch_direct<2, 1>(p, stream);
  const int gpw = (p.G + D_WARPS - 1) / D_WARPS;
  if (gpw <= 1) return launch_direct<1, 1>(p, stream);
  if (gpw == 2) return launch_direct<1, 2>(p, stream);
  return launch_direct<1, 3>(p, stream);
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int awq_linear_w4a16(const void *X, int M, int K, int ldx, const float *inv_awq, const uint32_t *qweight,
                                const void *scales, const void *zeros, int group, const void *bias, int N, void *Y,
                                int ldy, svdq_stream_t stream) {
  if (!X || !qweight || !scales || !zeros || !Y) return fail(SVDQ_ERR_INVALID_ARG, "awq_linear_w4a16: null pointer");
  if (group != 64) return fail(SVDQ_ERR_SHAPE, "awq_linear_w4a16: group must be 64");
  if (M < 1 || M > 65535 * 16 || K < 64 || K % 64 || N < 64 || N % 64 || ldx < K || ldx % 8 || ldy < N ||
      ldy % 8)
    return fail(SVDQ_ERR_SHAPE, "awq_linear_w4a16: need 1 <= M <= 1048560, K % 64 == 0, N % 64 == 0, ldx >= K, "
                                "ldy >= N, ldx/ldy % 8 == 0");
  if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
      (inv_awq && !aligned16(inv_awq)) || !aligned16(Y))
    return fail(SVDQ_ERR_ALIGNMENT, "awq_linear_w4a16: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int G = K / 64;

  Params p;
  p.M = M;
  p.K = K;
  p.N = N;
  p.ldx = ldx;
  p.ldy = ldy;
  p.G = G;
  p.X = static_cast<const uint16_t *>(X);
  p.inv = inv_awq;
  p.qw = reinterpret_cast<const uint4 *>(qweight);
  p.scales = static_cast<const uint16_t *>(scales);
  p.zeros = static_cast<const uint16_t *>(zeros);
  p.bias = static_cast<const uint16_t *>(bias);
  p.Y = static_cast<uint16_t *>(Y);
  return launch_direct_g(p, s);
}
