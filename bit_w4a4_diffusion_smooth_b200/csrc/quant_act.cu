// K1: activation quantization fused with the low-rank down-projection.
//
// The pages fuse the input quantization of the 4-bit GEMM with the low-rank
// down-projection so that the 16-bit branch costs no extra pass over X (web
// page "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定适用范围", remio.ai,
// section "SVDQuant 将棘手数值移出 4 位路径").  One read of X produces:
//   * the NVFP4 codes and ue4m3 block scales of X^ = X . diag(inv_lambda),
//     written straight into the 128-row operand bundle the GEMM streams;
//   * U = (bf16(X^) . L1) / (s_a s_w), the low-rank activations the GEMM adds,
//     written as 128-row swizzled tiles.
//
// Design (X is read once, ~0.3 B written per byte read):
//   * one CTA per 32 rows, 16 compute warps + 1 TMA warp; a 4-stage ring of
//     [32 rows x 256 cols] bf16 tiles of X, [rank x 256] tiles of L1^T and
//     256-float slices of inv_lambda, loaded by TMA / bulk copies; X and L1^T
//     land with the 128-byte swizzle (conflict-free for the row-wise pass and
//     for ldmatrix);
//   * quantize pass: each lane owns one 16-element block of one row: two
//     16-byte loads, the block maximum in registers, one f32 division for the
//     block scale, and 1/scale from a per-CTA table of all 128 scale codes
//     (the tensor scale is fixed per call, so f32(1 / f32(e4m3 * s_a)) has
//     only 128 possible values); the block's 8 code bytes go out as one
//     8-byte store, four lanes' scale bytes as one 32-bit store, and X^ is
//     written back in place as bf16;
//   * down-projection pass: each warp owns one 16 x 8 tile of U and a share
//     of the stage's 16 k16-slices (mma.sync, bf16 in, fp32 accumulate); at
//     most 4 partial sums per output are added at the end;
//   * the compute warps meet at named barriers; every mbarrier wait is
//     bounded (try_wait + %globaltimer) and decided warp-uniformly - a warp
//     whose wait runs out records SVDQ_ERR_TIMEOUT, skips its work and keeps
//     meeting the others at the barriers, so the block always finishes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 32;             // rows per CTA
constexpr int KC = kStageK;        // columns per stage (one bundle k-stage)
constexpr int STAGES = 4;
constexpr int CWARPS = 16;         // compute warps
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int X_BOX = BM * 128;    // one [32 x 64] bf16 box, 128-byte rows
constexpr int X_STAGE = 4 * X_BOX;
constexpr int INV_BYTES = KC * 4;

struct Params {
  int M, K, KS;
  const float *inv_lambda;
  const float *s_a, *s_w;
  uint8_t *bundle;
  uint8_t *U;
  unsigned int *status;
  unsigned long long limit_ns;
};

template <int RANK>
__host__ __device__ constexpr int stage_bytes() {
  return X_STAGE + 4 * RANK * 128 + INV_BYTES;
}
template <int RANK>
__host__ __device__ constexpr int smem_bytes() {
  return 1024 + STAGES * stage_bytes<RANK>() + 128 * 4 + 256;
}

// Byte offset of the 16-byte chunk holding column c (0..63, multiple of 8) of
// row r inside a 128-byte-swizzled box of 128-byte rows.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ r) & 7) << 4));
}

// x^ = f32(x * inv) for the 8 bf16 of `w`, into out[0..7].
__device__ __forceinline__ void smooth8(const uint4 &w, const float4 &i0, const float4 &i1, float (&out)[8]) {
  out[0] = __fmul_rn(__uint_as_float(w.x << 16), i0.x);
  out[1] = __fmul_rn(__uint_as_float(w.x & 0xFFFF0000u), i0.y);
  out[2] = __fmul_rn(__uint_as_float(w.y << 16), i0.z);
  out[3] = __fmul_rn(__uint_as_float(w.y & 0xFFFF0000u), i0.w);
  out[4] = __fmul_rn(__uint_as_float(w.z << 16), i1.x);
  out[5] = __fmul_rn(__uint_as_float(w.z & 0xFFFF0000u), i1.y);
  out[6] = __fmul_rn(__uint_as_float(w.w << 16), i1.z);
  out[7] = __fmul_rn(__uint_as_float(w.w & 0xFFFF0000u), i1.w);
}
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Warps of the down-projection: (16-row half mt, 8-column tile nt) pairs, the
// k16-slices of a stage split KSPLIT ways between warps with the same pair.
template <int RANK>
struct LrSplit {
  static constexpr int NT8 = RANK > 0 ? RANK / 8 : 1;
  static constexpr int P = 2 * NT8;
  static constexpr int PP = P <= 4 ? 4 : P <= 8 ? 8 : 16;   // pairs rounded up to a power of 2
  static constexpr int KSPLIT = CWARPS / PP;                 // 4, 2 or 1
  static constexpr int SLICES = 16 / KSPLIT;                 // k16-slices per warp and stage
};

template <int RANK>
__global__ void __launch_bounds__(THREADS, 1)
    quant_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1, Params p) {
  using LS = LrSplit<RANK>;
  constexpr int L1_BOX = RANK * 128;
  constexpr int STAGE = stage_bytes<RANK>();
  constexpr int INV_OFF = X_STAGE + 4 * L1_BOX;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *rinv_tab = reinterpret_cast<float *>(smem + STAGES * STAGE);   // [128]
  uint64_t *full = reinterpret_cast<uint64_t *>(rinv_tab + 128);
  uint64_t *empty = full + STAGES;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], CWARPS);
    }
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();
  const float s_a = __ldg(p.s_a);
  if (threadIdx.x < 128) {
    // 1 / (scale of code c): the same two f32 roundings as the quantizer
    // definition, f32(e4m3(c) * s_a) then f32(1 / that)
    const uint32_t c = threadIdx.x;
    const float scale = c < 127u ? __fmul_rn(dev::e4m3_value(c), s_a) : 0.0f;
    rinv_tab[c] = scale == 0.0f ? 0.0f : __frcp_rn(scale);
  }
  __syncthreads();

  if (warp == CWARPS) {
    // ------------------------------------------------------------ TMA warp
    if (lane == 0) {
      dev::prefetch_tmap(&tm_x);
      if (RANK > 0) dev::prefetch_tmap(&tm_l1);
      int issued = 0;
      for (int c = 0; c < p.KS; ++c) {
        const int s = c % STAGES;
        if (!dev::mbar_wait(&empty[s], ((c / STAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
          *abort_flag = 1;
          dev::report(p.status, SVDQ_ERR_TIMEOUT);
          break;
        }
        const int nbox = min(4, (p.K - c * KC) / 64);
        dev::mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox * (X_BOX + L1_BOX + 256)));
        uint8_t *st = smem + s * STAGE;
        for (int b = 0; b < nbox; ++b) {
          dev::tma_load_2d(st + b * X_BOX, &tm_x, &full[s], c * KC + b * 64, m0);
          if (RANK > 0) dev::tma_load_2d(st + X_STAGE + b * L1_BOX, &tm_l1, &full[s], c * KC + b * 64, 0);
        }
        dev::bulk_load(st + INV_OFF, p.inv_lambda + c * KC, static_cast<uint32_t>(nbox * 256), &full[s]);
        ++issued;
      }
      // every issued copy lands before the block leaves
      for (int c = max(0, issued - STAGES); c < issued; ++c)
        dev::mbar_wait(&full[c % STAGES], (c / STAGES) & 1, p.limit_ns, nullptr);
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  // quantize pass: lane -> (row r, 16-block jb of box b)
  const int b = warp >> 2;                        // 64-column box of the stage
  const int r = (warp & 3) * 8 + (lane & 7);      // row within the CTA's 32
  const int jb = lane >> 3;                       // block within the box
  const int rt = m0 % 128 + r;                    // row inside the 128-row bundle tile
  const int m_blk = m0 / 128;
  const float d6 = __fmul_rn(6.0f, s_a);
  // down-projection pass: this warp's 16 x 8 tile of U and its k16-slices
  const int pi = warp % LS::PP, kq = warp / LS::PP;
  const int mt = pi & 1, nt = pi >> 1;
  const bool lr_active = RANK > 0 && nt < LS::NT8;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  bool failed = false;

  for (int c = 0; c < p.KS; ++c) {
    const int s = c % STAGES;
    const uint32_t ph = (c / STAGES) & 1;
    if (!failed && !dev::mbar_wait_warp(&full[s], ph, p.limit_ns, abort_flag)) {
      *abort_flag = 1;
      dev::report(p.status, SVDQ_ERR_TIMEOUT);
      failed = true;
    }
    const int nbox = min(4, (p.K - c * KC) / 64);
    uint8_t *st = smem + s * STAGE;
    if (!failed) {
      const bool col_ok = b < nbox;                 // columns past K quantize as zeros
      uint8_t *chunk0 = st + b * X_BOX + sw_off(r, 16 * jb);
      uint8_t *chunk1 = st + b * X_BOX + sw_off(r, 16 * jb + 8);
      float xh[16];
      if (col_ok) {
        const float4 *iv = reinterpret_cast<const float4 *>(st + INV_OFF + (b * 64 + 16 * jb) * 4);
        const uint4 w0 = *reinterpret_cast<const uint4 *>(chunk0);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(chunk1);
        float lo[8], hi[8];
        smooth8(w0, iv[0], iv[1], lo);
        smooth8(w1, iv[2], iv[3], hi);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          xh[i] = lo[i];
          xh[8 + i] = hi[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) xh[i] = 0.0f;
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(xh[i]));
      const uint32_t sb = dev::cvt_e4m3(__fdiv_rn(amax, d6));
      const float rinv = rinv_tab[sb];
      uint32_t q[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i)
        q[i >> 2] |= dev::cvt_e2m1x2(__fmul_rn(xh[2 * i], rinv), __fmul_rn(xh[2 * i + 1], rinv)) << (8 * (i & 3));
      // the block's 8 code bytes: byte 8 (4 b + jb) of the row, 128-byte swizzle
      uint8_t *tile = p.bundle + (static_cast<size_t>(m_blk) * p.KS + c) * bundle_tile_bytes(128);
      const int j = 4 * b + jb;
      *reinterpret_cast<uint2 *>(tile + rt * 128 + ((((j >> 1) ^ rt) & 7) << 4) + 8 * (j & 1)) = make_uint2(q[0], q[1]);
      // the 4 block scales of this row in box b -> one word of atom b
      const uint32_t word = __shfl_sync(0xFFFFFFFFu, sb, lane & 7) | (__shfl_sync(0xFFFFFFFFu, sb, (lane & 7) + 8) << 8) |
                            (__shfl_sync(0xFFFFFFFFu, sb, (lane & 7) + 16) << 16) |
                            (__shfl_sync(0xFFFFFFFFu, sb, (lane & 7) + 24) << 24);
      if (jb == 0)
        *reinterpret_cast<uint32_t *>(tile + 128 * 128 + b * 512 + (rt & 31) * 16 + ((rt >> 5) & 3) * 4) = word;
      if (RANK > 0 && col_ok) {
        *reinterpret_cast<uint4 *>(chunk0) =
            make_uint4(bf16x2(xh[0], xh[1]), bf16x2(xh[2], xh[3]), bf16x2(xh[4], xh[5]), bf16x2(xh[6], xh[7]));
        *reinterpret_cast<uint4 *>(chunk1) = make_uint4(bf16x2(xh[8], xh[9]), bf16x2(xh[10], xh[11]),
                                                       bf16x2(xh[12], xh[13]), bf16x2(xh[14], xh[15]));
      }
    }

    if (RANK > 0) {
      dev::named_barrier(1, CWARPS * 32);           // every warp's bf16(X^) is in place
      if (!failed && lr_active) {
#pragma unroll
        for (int i = 0; i < LS::SLICES; i += 2) {    // two k16-slices (of one box) per step
          const int slice = kq * LS::SLICES + i;
          const int sbx = slice >> 2;
          if (sbx < nbox) {
            const int kc = (slice & 3) * 16;
            const uint32_t xbase = dev::smem_u32(st + sbx * X_BOX);
            const uint32_t lbase = dev::smem_u32(st + X_STAGE + sbx * L1_BOX);
            uint32_t a0[4], a1[4], bq[4];
            const int ar = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            dev::ldmatrix_x4(xbase + sw_off(ar, kc + (lane >> 4) * 8), a0[0], a0[1], a0[2], a0[3]);
            dev::ldmatrix_x4(xbase + sw_off(ar, kc + 16 + (lane >> 4) * 8), a1[0], a1[1], a1[2], a1[3]);
            // B: rows 8 nt .. +7 of L1^T; lanes 0-15 slice i (k 0-7, 8-15), lanes 16-31 slice i + 1
            dev::ldmatrix_x4(lbase + sw_off(nt * 8 + (lane & 7), kc + ((lane >> 3) & 3) * 8), bq[0], bq[1], bq[2],
                             bq[3]);
            dev::mma_bf16_16816(acc, a0, bq[0], bq[1]);
            dev::mma_bf16_16816(acc, a1, bq[2], bq[3]);
          }
        }
      }
      // the next TMA load into this stage must come after our generic writes
      dev::fence_proxy_async();
    }
    __syncwarp();
    if (lane == 0 && !failed) dev::mbar_arrive(&empty[s]);
  }

  // ---- U = (sum of the warps' partial products) / (s_a s_w), bf16, 128-row tiles
  const int tid = threadIdx.x;  // 0..511
  if (RANK > 0) {
    dev::named_barrier(1, CWARPS * 32);            // the stage buffers are free: reuse for the partials
    float *red = reinterpret_cast<float *>(smem);  // [KSPLIT][BM][RANK]
    if (lr_active) {
      const int g = lane >> 2, t = lane & 3;
      float *base = red + kq * BM * RANK;
      const int row = mt * 16 + g, col = nt * 8 + 2 * t;
      base[row * RANK + col] = acc[0];
      base[row * RANK + col + 1] = acc[1];
      base[(row + 8) * RANK + col] = acc[2];
      base[(row + 8) * RANK + col + 1] = acc[3];
    }
    dev::named_barrier(1, CWARPS * 32);
  }
  const float alpha = __fmul_rn(s_a, __ldg(p.s_w));
  for (int idx = tid; idx < BM * (SVDQ_LR_STRIDE / 8); idx += CWARPS * 32) {
    const int rr = idx >> 3, cc = idx & 7;   // row, 8-column chunk
    const int m = m0 + rr;
    uint32_t o[4] = {0, 0, 0, 0};
    if (RANK > 0 && 8 * cc < RANK && !failed) {
      const float *red = reinterpret_cast<const float *>(smem);
      float v[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < LS::KSPLIT; ++w) sum += red[(w * BM + rr) * RANK + 8 * cc + jj];
        v[jj] = __fdiv_rn(sum, alpha);
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) o[jj] = bf16x2(v[2 * jj], v[2 * jj + 1]);
    }
    *reinterpret_cast<uint4 *>(p.U + lowrank_offset(m, 8 * cc, 128)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

template <int RANK>
int launch(const CUtensorMap &tx, const CUtensorMap &tl, const Params &p, int grid, cudaStream_t stream) {
  const int smem = smem_bytes<RANK>();
  cudaError_t e = cudaFuncSetAttribute(quant_act_kernel<RANK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_quantize_act: ") + cudaGetErrorString(e));
  DependentLaunch dl(dim3(grid), dim3(THREADS), smem, stream);
  e = cudaLaunchKernelEx(&dl.cfg, quant_act_kernel<RANK>, tx, tl, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_quantize_act launch: ") + cudaGetErrorString(e));
  return ok();
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_quantize_act(const void *X, int M, int K, int ldx, const float *inv_lambda, const void *l1t,
                                 int rank, const float *s_a, const float *s_w, uint8_t *a_bundle, void *U,
                                 svdq_stream_t stream) {
  if (!X || !inv_lambda || !s_a || !s_w || !a_bundle || !U || (rank > 0 && !l1t))
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_quantize_act: null pointer");
  if (M < 1 || K < 64 || K % 64 || ldx < K || ldx % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_quantize_act: need M >= 1, K % 64 == 0, ldx >= K, ldx % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_quantize_act: rank must be a multiple of 16 in [0, 64]");
  if (!aligned16(X) || !aligned16(inv_lambda) || !aligned16(a_bundle) || !aligned16(U) ||
      (rank > 0 && !aligned16(l1t)))
    return fail(SVDQ_ERR_ALIGNMENT, "svdq_quantize_act: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;

  Params p;
  p.M = M;
  p.K = K;
  p.KS = bundle_ks(K);
  p.inv_lambda = inv_lambda;
  p.s_a = s_a;
  p.s_w = s_w;
  p.bundle = a_bundle;
  p.U = static_cast<uint8_t *>(U);
  p.status = st->status_word;
  p.limit_ns = kWaitLimitNs;

  CUtensorMap tx, tl;
  int rc = encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                          static_cast<uint64_t>(ldx) * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != SVDQ_OK) return rc;
  if (rank > 0) {
    rc = encode_tmap_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, l1t, static_cast<uint64_t>(K),
                        static_cast<uint64_t>(rank), static_cast<uint64_t>(K) * 2, 64, static_cast<uint32_t>(rank),
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != SVDQ_OK) return rc;
  } else {
    tl = tx;
  }
  const int grid = (M + 127) / 128 * (128 / BM);   // every row of every 128-row tile
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (rank) {
    case 0: return launch<0>(tx, tl, p, grid, s);
    case 16: return launch<16>(tx, tl, p, grid, s);
    case 32: return launch<32>(tx, tl, p, grid, s);
    case 48: return launch<48>(tx, tl, p, grid, s);
    default: return launch<64>(tx, tl, p, grid, s);
  }
}
