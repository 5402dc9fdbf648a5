// INT4 W4A4 GEMM with the low-rank up-projection, bias and GELU fused in:
// the entry point, and the kernel for widths that are not whole 256-column
// tiles (the others run on the tensor cores, int4_gemm_tc.cu).
//
// The pages ship an INT4 W4A4 variant beside NVFP4 for GPUs without NVFP4
// tensor cores (web page "Diffusers × Nunchaku 4-bit", donmalab.com, section
// "實務上的影響與硬體要求"); its 4-bit branch is, in this library's reading,
// symmetric INT4 in groups of 64 along K with one bf16 scale per row or output
// column and group:
//   Y = epilogue( sum_g (s_a[m,g] s_w[n,g]) sum_{k in g} q_a[m,k] q_w[n,k]
//                 + U . L2 + bias )
// B200's tensor cores have no 4-bit integer MMA (the warp-level s4 MMA
// measured 40 times slower than the 8-bit one: it is emulated), so:
//   * one CTA per 128 x 128 output tile, 8 warps of 64 x 32; the K loop walks
//     the groups of 64 through a ring of 4 stages filled by 16-byte async
//     copies (codes of 128 rows and 128 columns, 4 KB each, and their 128 + 128
//     bf16 scales);
//   * each group's codes are unpacked once per CTA into 8-bit two's-complement
//     tiles in shared memory (16-byte chunks xor-swizzled by row pairs, so the
//     ldmatrix reads are conflict-free) and multiplied with the 8-bit warp MMA
//     (mma.sync m16n8k32 s8, int32 accumulation: exact, |partial| <= 4096);
//   * the group's first MMA starts from the integer bits of the float
//     1.5 * 2^23 instead of zero, so the int32 result is the bit pattern of
//     1.5 * 2^23 + partial (exact, |partial| < 2^22): one subtraction gives
//     the partial as a float, added into fp32 accumulators with the two
//     scales: acc += s_a * (s_w * partial);
//   * after the last group, U . L2 (bf16 warp MMAs from the 128-row tiles of
//     U and the 256-row tiles of L2T, into the same accumulators), bias,
//     GELU and bf16 stores.
#include <cuda_runtime.h>

#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 128, THREADS = 256, STAGES = 4;
constexpr int A4_OFF = 0, B4_OFF = 4096, SA_OFF = 8192, SB_OFF = 8448, STAGE_BYTES = 8704;
constexpr int A8_OFF = STAGES * STAGE_BYTES, B8_OFF = A8_OFF + 8192;
constexpr int SMEM_BYTES = B8_OFF + 8192;                  // 51,200
constexpr int LR_TILE = 128 * 128;                         // U or L2T rows of this tile: 16 KB each
static_assert(2 * LR_TILE <= STAGES * STAGE_BYTES, "the low-rank tiles fit the drained ring");

struct Params {
  const uint8_t *a_codes, *w_codes;
  const uint16_t *a_scales, *w_scales, *bias;
  const uint8_t *U, *l2t;
  uint16_t *Y;
  int M, N, K, ldy, ld_sa, rank, gelu_col_begin;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dev::smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// Eight 4-bit two's-complement values (element i at bits 4i) -> eight int8 in two words.
__device__ __forceinline__ uint2 unpack8(uint32_t w) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;   // elements 0,2,4,6 / 1,3,5,7
  uint32_t a = prmt(lo, hi, 0x5140u), b = prmt(lo, hi, 0x7362u);     // elements 0..3 / 4..7, one per byte
  a |= (a & 0x08080808u) * 0x1Eu;                                     // sign bit 3 -> bits 4..7 of its byte
  b |= (b & 0x08080808u) * 0x1Eu;
  return make_uint2(a, b);
}
// Byte offset of 16-byte chunk ch (0..3) of row r in a [rows][64 B] int8 tile.
__device__ __forceinline__ uint32_t i8_off(int r, int ch) { return static_cast<uint32_t>(r * 64 + ((ch ^ (r >> 1)) & 3) * 16); }
// Byte offset of 16-byte chunk ch (0..7) of row r in a 128-byte-swizzled low-rank tile.
__device__ __forceinline__ uint32_t lr_off(int r, int ch) { return static_cast<uint32_t>(r * 128 + ((ch ^ r) & 7) * 16); }
__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// The first k32 step of a group: D = A . B + C with C = the bits of 1.5 * 2^23 in every element, so
// that after the group D holds the bits of the float 1.5 * 2^23 + partial (exact for |partial| < 2^22).
__device__ __forceinline__ void mma_s8_biased(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%10,%10,%10,%10};"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0x4B400000));
}
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1) int4_gemm_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int g8 = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int wm = (warp & 1) * 64, wn = (warp >> 1) * 32;    // the warp's 64 x 32 sub-tile
  const int G = p.K / 64;
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();

  auto load_group = [&](int g) {   // group g into ring slot g % STAGES (an empty commit past the end)
    if (g < G) {
      uint8_t *st = smem + (g % STAGES) * STAGE_BYTES;
      const int r = tid >> 1, h = tid & 1;
      cp_async16(st + A4_OFF + tid * 16, p.a_codes + static_cast<size_t>(m0 + r) * (p.K / 2) + g * 32 + h * 16);
      cp_async16(st + B4_OFF + tid * 16, p.w_codes + static_cast<size_t>(n0 + r) * (p.K / 2) + g * 32 + h * 16);
      if (tid < 16) cp_async16(st + SA_OFF + tid * 16, p.a_scales + static_cast<size_t>(g) * p.ld_sa + m0 + tid * 8);
      else if (tid < 32)
        cp_async16(st + SB_OFF + (tid - 16) * 16, p.w_scales + static_cast<size_t>(g) * p.N + n0 + (tid - 16) * 8);
    }
    cp_async_commit();
  };

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;

#pragma unroll
  for (int g = 0; g < STAGES - 1; ++g) load_group(g);

  const uint32_t a8 = dev::smem_u32(smem + A8_OFF), b8 = dev::smem_u32(smem + B8_OFF);
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();                      // group g has landed; every warp is done with the int8 tiles
    load_group(g + STAGES - 1);           // into the slot read by the unpack of group g - 1
    const uint8_t *st = smem + (g % STAGES) * STAGE_BYTES;
    {  // unpack: thread tid takes 32 codes of row tid >> 1 of A and of B
      const int r = tid >> 1, h = tid & 1;
      const uint4 qa = *reinterpret_cast<const uint4 *>(st + A4_OFF + tid * 16);
      const uint4 qb = *reinterpret_cast<const uint4 *>(st + B4_OFF + tid * 16);
      const uint2 a0 = unpack8(qa.x), a1 = unpack8(qa.y), a2 = unpack8(qa.z), a3 = unpack8(qa.w);
      const uint2 b0 = unpack8(qb.x), b1 = unpack8(qb.y), b2 = unpack8(qb.z), b3 = unpack8(qb.w);
      *reinterpret_cast<uint4 *>(smem + A8_OFF + i8_off(r, 2 * h)) = make_uint4(a0.x, a0.y, a1.x, a1.y);
      *reinterpret_cast<uint4 *>(smem + A8_OFF + i8_off(r, 2 * h + 1)) = make_uint4(a2.x, a2.y, a3.x, a3.y);
      *reinterpret_cast<uint4 *>(smem + B8_OFF + i8_off(r, 2 * h)) = make_uint4(b0.x, b0.y, b1.x, b1.y);
      *reinterpret_cast<uint4 *>(smem + B8_OFF + i8_off(r, 2 * h + 1)) = make_uint4(b2.x, b2.y, b3.x, b3.y);
    }
    __syncthreads();                      // the int8 tiles of group g are complete
    // B fragments of the warp's 4 column tiles x 2 k32 steps; column scales
    uint32_t bf[4][2][2];
#pragma unroll
    for (int np = 0; np < 2; ++np)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t q[4];
        const int row = wn + np * 16 + (lane >> 4) * 8 + (lane & 7);
        ldmatrix_x4(b8 + i8_off(row, 2 * kk + ((lane >> 3) & 1)), q);
        bf[2 * np][kk][0] = q[0];
        bf[2 * np][kk][1] = q[1];
        bf[2 * np + 1][kk][0] = q[2];
        bf[2 * np + 1][kk][1] = q[3];
      }
    const uint16_t *sa = reinterpret_cast<const uint16_t *>(st + SA_OFF);
    const uint16_t *sb = reinterpret_cast<const uint16_t *>(st + SB_OFF);
    float swc[4][2];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const uint32_t pair = *reinterpret_cast<const uint32_t *>(sb + wn + nt * 8 + 2 * t);
      swc[nt][0] = bf16f(pair & 0xFFFFu);
      swc[nt][1] = bf16f(pair >> 16);
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      int part[4][4];   // bits of the float 1.5 * 2^23 + the group's int32 partial
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t af[4];
        ldmatrix_x4(a8 + i8_off(wm + mt * 16 + (lane & 15), 2 * kk + (lane >> 4)), af);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          if (kk == 0)
            mma_s8_biased(part[nt], af, bf[nt][kk][0], bf[nt][kk][1]);
          else
            mma_s8(part[nt], af, bf[nt][kk][0], bf[nt][kk][1]);
        }
      }
      const float sa0 = bf16f(sa[wm + mt * 16 + g8]), sa1 = bf16f(sa[wm + mt * 16 + g8 + 8]);
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float f = __int_as_float(part[nt][e]) - 12582912.0f;   // the partial, exactly
          acc[mt][nt][e] = __fmaf_rn(e < 2 ? sa0 : sa1, __fmul_rn(swc[nt][e & 1], f), acc[mt][nt][e]);
        }
    }
  }
  cp_async_wait<0>();
  __syncthreads();                        // the ring is free for the low-rank tiles
  if (p.rank > 0) {
    // U rows m0..m0+127 (one 128-row tile) and L2T rows n0..n0+127 (half of a 256-row tile), copied
    // as they are: the 128-byte swizzle depends on the row modulo 8 only
    const uint8_t *ug = p.U + static_cast<size_t>(m0) * 128;
    const uint8_t *lg = p.l2t + static_cast<size_t>(n0 / 256) * 256 * 128 + static_cast<size_t>(n0 % 256) * 128;
    for (int i = tid; i < LR_TILE / 16; i += THREADS) {
      cp_async16(smem + i * 16, ug + i * 16);
      cp_async16(smem + LR_TILE + i * 16, lg + i * 16);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    const uint32_t us = dev::smem_u32(smem), ls = dev::smem_u32(smem + LR_TILE);
#pragma unroll 1
    for (int kk = 0; kk < p.rank / 16; ++kk) {
      uint32_t lb[4][2];
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t q[4];
        ldmatrix_x4(ls + lr_off(wn + np * 16 + (lane >> 4) * 8 + (lane & 7), 2 * kk + ((lane >> 3) & 1)), q);
        lb[2 * np][0] = q[0];
        lb[2 * np][1] = q[1];
        lb[2 * np + 1][0] = q[2];
        lb[2 * np + 1][1] = q[3];
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t af[4];
        ldmatrix_x4(us + lr_off(wm + mt * 16 + (lane & 15), 2 * kk + (lane >> 4)), af);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) dev::mma_bf16_16816(acc[mt][nt], af, lb[nt][0], lb[nt][1]);
      }
    }
  }

  // epilogue: + bias, GELU on columns >= gelu_col_begin, bf16 out (rows past M are not written)
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const int c = n0 + wn + nt * 8 + 2 * t;
    float b0 = 0.0f, b1 = 0.0f;
    if (p.bias) {
      const uint32_t bb = __ldg(reinterpret_cast<const uint32_t *>(p.bias + c));
      b0 = bf16f(bb & 0xFFFFu);
      b1 = bf16f(bb >> 16);
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = m0 + wm + mt * 16 + g8 + 8 * h;
        float2 y = make_float2(acc[mt][nt][2 * h] + b0, acc[mt][nt][2 * h + 1] + b1);
        if constexpr (EPI == SVDQ_EPILOGUE_GELU_ERF) {
          const float2 gy = dev::gelu_erf2(y);
          y = make_float2(c >= p.gelu_col_begin ? gy.x : y.x, c + 1 >= p.gelu_col_begin ? gy.y : y.y);
        } else if constexpr (EPI == SVDQ_EPILOGUE_GELU_TANH) {
          y = make_float2(c >= p.gelu_col_begin ? dev::gelu_tanh(y.x) : y.x,
                          c + 1 >= p.gelu_col_begin ? dev::gelu_tanh(y.y) : y.y);
        }
        if (r < p.M) {
          __nv_bfloat162 o = __floats2bfloat162_rn(y.x, y.y);
          *reinterpret_cast<__nv_bfloat162 *>(p.Y + static_cast<size_t>(r) * p.ldy + c) = o;
        }
      }
  }
}

template <int EPI>
int launch(const Params &p, cudaStream_t stream) {
  const int rc = smem_optin_once<int4_gemm_kernel<EPI>>(SMEM_BYTES, "svdq_linear_int4");
  if (rc != SVDQ_OK) return rc;
  DependentLaunch dl(dim3(p.N / BN, (p.M + BM - 1) / BM), dim3(THREADS), SMEM_BYTES, stream);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, int4_gemm_kernel<EPI>, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_int4 launch: ") + cudaGetErrorString(e));
  return ok();
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_linear_int4(const uint8_t *a_codes, const void *a_scales, const void *U, const uint8_t *w_codes,
                                const void *w_scales, const void *l2t, const void *bias, int M, int N, int K, int rank,
                                int epilogue, int gelu_col_begin, void *Y, int ldy, svdq_stream_t stream) {
  if (!a_codes || !a_scales || !w_codes || !w_scales || !Y || (rank > 0 && (!U || !l2t)))
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_int4: null pointer");
  if (epilogue < SVDQ_EPILOGUE_NONE || epilogue > SVDQ_EPILOGUE_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_int4: unknown epilogue");
  if (M < 1 || K < 64 || K % 64 || N < 128 || N % 128 || ldy < N || ldy % 8 || gelu_col_begin < 0 ||
      gelu_col_begin > N)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_int4: need M >= 1, K % 64 == 0, N % 128 == 0, ldy >= N, ldy % 8 == 0, "
                                "0 <= gelu_col_begin <= N");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_int4: rank must be a multiple of 16 in [0, 64]");
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (rank > 0 && (!aligned16(U) || !aligned16(l2t))))
    return fail(SVDQ_ERR_ALIGNMENT, "svdq_linear_int4: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // widths in whole 256-column tiles: the tcgen05 kernel (fp16 operands from the codes, no per-group
  // rescale); otherwise the 8-bit warp-MMA kernel below
  if (N % 256 == 0)
    return launch_int4_tc(a_codes, a_scales, U, w_codes, w_scales, l2t, bias, M, N, K, rank, epilogue, gelu_col_begin,
                          Y, ldy, st->status_word, s);
  Params p;
  p.a_codes = a_codes;
  p.w_codes = w_codes;
  p.a_scales = static_cast<const uint16_t *>(a_scales);
  p.w_scales = static_cast<const uint16_t *>(w_scales);
  p.bias = static_cast<const uint16_t *>(bias);
  p.U = static_cast<const uint8_t *>(U);
  p.l2t = static_cast<const uint8_t *>(l2t);
  p.Y = static_cast<uint16_t *>(Y);
  p.M = M;
  p.N = N;
  p.K = K;
  p.ldy = ldy;
  p.ld_sa = (M + 127) / 128 * 128;
  p.rank = rank;
  p.gelu_col_begin = gelu_col_begin;
  switch (epilogue) {
    case SVDQ_EPILOGUE_GELU_ERF: return launch<SVDQ_EPILOGUE_GELU_ERF>(p, s);
    case SVDQ_EPILOGUE_GELU_TANH: return launch<SVDQ_EPILOGUE_GELU_TANH>(p, s);
    default: return launch<SVDQ_EPILOGUE_NONE>(p, s);
  }
}
