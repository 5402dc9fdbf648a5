// K1: activation quantization fused with the low-rank down-projection.
//
// The pages fuse the input quantization of the 4-bit GEMM with the low-rank
// down-projection so that the 16-bit branch costs no extra pass over X (web
// page "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定适用范围", remio.ai,
// section "SVDQuant 将棘手数值移出 4 位路径").  One read of X produces:
//   * the NVFP4 codes and ue4m3 block scales of X^ = X . diag(inv_lambda),
//   * U = (bf16(X^) . L1) / (s_a s_w), the low-rank activations the GEMM adds.
//
// Design (memory bound: X is read once, ~0.3 B written per byte read):
//   * one CTA per 32 rows, 8 compute warps + 1 TMA warp; a 4-stage ring of
//     [32 rows x 256 cols] bf16 tiles of X and [rank x 256] tiles of L1^T,
//     loaded by TMA with the 128-byte swizzle (conflict-free for both the
//     row-wise quantize pass and ldmatrix);
//   * quantize pass: each warp owns 4 rows, each lane 8 consecutive
//     elements (two lanes per 16-block, one shuffle for the block max),
//     16-byte shared loads, 128-byte coalesced code stores; X^ is written
//     back in place as bf16;
//   * down-projection pass: warp w multiplies its 32-column slice of the
//     tile with mma.sync (bf16 in, fp32 accumulate), partial sums are added
//     across warps once at the end;
//   * every wait is bounded (mbarrier try_wait + %globaltimer); a wait that
//     runs out records SVDQ_ERR_TIMEOUT and the block leaves cleanly.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 32;             // rows per CTA
constexpr int KC = 256;            // columns per stage
constexpr int STAGES = 4;
constexpr int CWARPS = 8;          // compute warps
constexpr int THREADS = (CWARPS + 1) * 32;
constexpr int X_BOX = BM * 128;    // one [32 x 64] bf16 box, 128-byte rows
constexpr int X_STAGE = 4 * X_BOX;

struct Params {
  int M, K, m_pad;
  const float *inv_lambda;
  const float *s_a, *s_w;
  uint8_t *codes, *scales;
  uint16_t *U;
  unsigned int *status;
  unsigned long long limit_ns;
};

template <int RANK>
__host__ __device__ constexpr int stage_bytes() {
  return X_STAGE + 4 * RANK * 128;
}
template <int RANK>
__host__ __device__ constexpr int smem_bytes() {
  return 1024 + STAGES * stage_bytes<RANK>() + 256;
}

// Byte offset of the 16-byte chunk holding column c (0..63, multiple of 8) of
// row r inside a 128-byte-swizzled box of 128-byte rows.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ r) & 7) << 4));
}

template <int RANK>
__global__ void __launch_bounds__(THREADS, 1)
    quant_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1, Params p) {
  constexpr int NP = RANK / 16;           // pairs of 8-wide MMA column tiles
  constexpr int L1_BOX = RANK * 128;
  constexpr int STAGE = stage_bytes<RANK>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE);
  uint64_t *empty = full + STAGES;
  uint64_t *ready = empty + STAGES;       // X^ written back, per stage
  uint64_t *sync = ready + STAGES;        // two end-of-loop syncs
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sync + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;
  const int nchunks = (p.K + KC - 1) / KC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], CWARPS);
      dev::mbar_init(&ready[s], CWARPS);
    }
    dev::mbar_init(sync, CWARPS);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  __syncthreads();

  if (warp == CWARPS) {
    // ------------------------------------------------------------ TMA warp
    if (lane == 0) {
      dev::prefetch_tmap(&tm_x);
      if (RANK > 0) dev::prefetch_tmap(&tm_l1);
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int s = c % STAGES;
        const uint32_t ph = (c / STAGES) & 1;
        if (!dev::mbar_wait(&empty[s], ph ^ 1, p.limit_ns, abort_flag)) {
          *abort_flag = 1;
          dev::report(p.status, SVDQ_ERR_TIMEOUT);
          break;
        }
        const int nbox = min(4, (p.K - c * KC) / 64);
        dev::mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox * (X_BOX + L1_BOX)));
        uint8_t *st = smem + s * STAGE;
        for (int b = 0; b < nbox; ++b) {
          dev::tma_load_2d(st + b * X_BOX, &tm_x, &full[s], c * KC + b * 64, m0);
          if (RANK > 0) dev::tma_load_2d(st + X_STAGE + b * L1_BOX, &tm_l1, &full[s], c * KC + b * 64, 0);
        }
        ++issued;
      }
      if (*abort_flag) {
        // Let copies already in flight land before the block exits.
        for (int c = max(0, issued - STAGES); c < issued; ++c)
          dev::mbar_wait(&full[c % STAGES], (c / STAGES) & 1, p.limit_ns, nullptr);
      }
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  float acc[2][2 * NP + 1][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2 * NP + 1; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[a][b][e] = 0.0f;

  const float s_a = __ldg(p.s_a);
  const float d6 = __fmul_rn(6.0f, s_a);
  bool ok = true;

  for (int c = 0; c < nchunks && ok; ++c) {
    const int s = c % STAGES;
    const uint32_t ph = (c / STAGES) & 1;
    if (!dev::mbar_wait(&full[s], ph, p.limit_ns, abort_flag)) {
      ok = false;
      break;
    }
    const int nbox = min(4, (p.K - c * KC) / 64);
    uint8_t *st = smem + s * STAGE;
    const int col = c * KC + 8 * lane;        // first of this lane's 8 columns
    const int box = lane >> 3;
    const bool col_ok = box < nbox;

    float inv[8];
    if (col_ok) {
      const float4 i0 = __ldg(reinterpret_cast<const float4 *>(p.inv_lambda + col));
      const float4 i1 = __ldg(reinterpret_cast<const float4 *>(p.inv_lambda + col + 4));
      inv[0] = i0.x; inv[1] = i0.y; inv[2] = i0.z; inv[3] = i0.w;
      inv[4] = i1.x; inv[5] = i1.y; inv[6] = i1.z; inv[7] = i1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) inv[i] = 0.0f;
    }

    // ---- quantize pass: rows 4*warp .. 4*warp+3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = warp * 4 + i;
      const int m = m0 + r;
      uint8_t *chunk = st + box * X_BOX + sw_off(r, (8 * lane) & 63);
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (col_ok) raw = *reinterpret_cast<const uint4 *>(chunk);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      float xh[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        xh[2 * j] = __fmul_rn(__uint_as_float(w[j] << 16), inv[2 * j]);
        xh[2 * j + 1] = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), inv[2 * j + 1]);
      }
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(xh[j]));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      const uint32_t sb = dev::cvt_e4m3(__fdiv_rn(amax, d6));
      const float scale = __fmul_rn(dev::e4m3_value(sb), s_a);
      const float rinv = scale == 0.0f ? 0.0f : __frcp_rn(scale);
      uint32_t packed = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        packed |= dev::cvt_e2m1x2(__fmul_rn(xh[2 * j], rinv), __fmul_rn(xh[2 * j + 1], rinv)) << (8 * j);
      if (col_ok && m < p.M)
        *reinterpret_cast<uint32_t *>(p.codes + static_cast<size_t>(m) * (p.K / 2) + col / 2) = packed;
      // four consecutive block scales (lanes 8q, 8q+2, 8q+4, 8q+6) -> one word
      const int base = lane & ~7;
      const uint32_t word = __shfl_sync(0xFFFFFFFFu, sb, base) | (__shfl_sync(0xFFFFFFFFu, sb, base + 2) << 8) |
                            (__shfl_sync(0xFFFFFFFFu, sb, base + 4) << 16) |
                            (__shfl_sync(0xFFFFFFFFu, sb, base + 6) << 24);
      if ((lane & 7) == 0 && col_ok && m < p.m_pad)
        *reinterpret_cast<uint32_t *>(p.scales + sf_offset(m, col / 16, p.K)) = word;
      if (RANK > 0 && col_ok) {
        uint4 o;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(xh[0], xh[1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(xh[2], xh[3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(xh[4], xh[5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(xh[6], xh[7]);
        o.x = *reinterpret_cast<uint32_t *>(&h0);
        o.y = *reinterpret_cast<uint32_t *>(&h1);
        o.z = *reinterpret_cast<uint32_t *>(&h2);
        o.w = *reinterpret_cast<uint32_t *>(&h3);
        *reinterpret_cast<uint4 *>(chunk) = o;
      }
    }

    // ---- down-projection pass: warp w takes columns [32w, 32w+32) of the tile
    if (RANK > 0) {
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&ready[s]);
      if (!dev::mbar_wait(&ready[s], ph, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      const int kbox = warp >> 1;
      if (kbox < nbox) {
        const uint32_t xbase = dev::smem_u32(st + kbox * X_BOX);
        const uint32_t lbase = dev::smem_u32(st + X_STAGE + kbox * L1_BOX);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const int kc = (warp & 1) * 32 + ks * 16;
          uint32_t a[2][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int r = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            dev::ldmatrix_x4(xbase + sw_off(r, kc + (lane >> 4) * 8), a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
          }
#pragma unroll
          for (int np = 0; np < NP; ++np) {
            const int n = np * 16 + (lane & 7) + (lane >> 4) * 8;
            uint32_t b0, b1, b2, b3;
            dev::ldmatrix_x4(lbase + sw_off(n, kc + ((lane >> 3) & 1) * 8), b0, b1, b2, b3);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              dev::mma_bf16_16816(acc[mt][2 * np], a[mt], b0, b1);
              dev::mma_bf16_16816(acc[mt][2 * np + 1], a[mt], b2, b3);
            }
          }
        }
      }
    }
    // the next TMA load into this stage must come after our generic writes
    if (RANK > 0) dev::fence_proxy_async();
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[s]);
  }

  if (!ok) {
    *abort_flag = 1;
    dev::report(p.status, SVDQ_ERR_TIMEOUT);
    return;
  }

  // ---- U = (sum of the warps' partial products) / (s_a s_w), bf16, [M][64]
  const int tid = threadIdx.x;  // 0..255
  if (RANK > 0) {
    // every warp is done with the stage buffers -> reuse them for partials
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(sync);
    if (!dev::mbar_wait(sync, 0, p.limit_ns, abort_flag)) {
      *abort_flag = 1;
      dev::report(p.status, SVDQ_ERR_TIMEOUT);
      return;
    }
    float *red = reinterpret_cast<float *>(smem);  // [CWARPS][BM][RANK]
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2 * NP; ++nt) {
        const int r = mt * 16 + g, n = nt * 8 + 2 * t;
        float *base = red + (warp * BM) * RANK;
        base[r * RANK + n] = acc[mt][nt][0];
        base[r * RANK + n + 1] = acc[mt][nt][1];
        base[(r + 8) * RANK + n] = acc[mt][nt][2];
        base[(r + 8) * RANK + n + 1] = acc[mt][nt][3];
      }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(sync);
    if (!dev::mbar_wait(sync, 1, p.limit_ns, abort_flag)) {
      *abort_flag = 1;
      dev::report(p.status, SVDQ_ERR_TIMEOUT);
      return;
    }
    const float alpha = __fmul_rn(s_a, __ldg(p.s_w));
    for (int idx = tid; idx < BM * SVDQ_LR_STRIDE; idx += CWARPS * 32) {
      const int r = idx / SVDQ_LR_STRIDE, j = idx % SVDQ_LR_STRIDE;
      const int m = m0 + r;
      if (m >= p.M) continue;
      float v = 0.0f;
      if (j < RANK) {
#pragma unroll
        for (int w = 0; w < CWARPS; ++w) v += red[(w * BM + r) * RANK + j];
        v = __fdiv_rn(v, alpha);
      }
      __nv_bfloat16 h = __float2bfloat16_rn(v);
      p.U[static_cast<size_t>(m) * SVDQ_LR_STRIDE + j] = *reinterpret_cast<uint16_t *>(&h);
    }
  } else {
    for (int idx = tid; idx < BM * SVDQ_LR_STRIDE; idx += CWARPS * 32) {
      const int r = idx / SVDQ_LR_STRIDE, j = idx % SVDQ_LR_STRIDE;
      if (m0 + r < p.M) p.U[static_cast<size_t>(m0 + r) * SVDQ_LR_STRIDE + j] = 0;
    }
  }
}

template <int RANK>
int launch(const CUtensorMap &tx, const CUtensorMap &tl, const Params &p, int grid, cudaStream_t stream) {
  const int smem = smem_bytes<RANK>();
  cudaError_t e = cudaFuncSetAttribute(quant_act_kernel<RANK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_quantize_act: ") + cudaGetErrorString(e));
  quant_act_kernel<RANK><<<grid, THREADS, smem, stream>>>(tx, tl, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_quantize_act launch: ") + cudaGetErrorString(e));
  return ok();
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_quantize_act(const void *X, int M, int K, int ldx, const float *inv_lambda, const void *l1t,
                                 int rank, const float *s_a, const float *s_w, uint8_t *codes, uint8_t *scales,
                                 void *U, svdq_stream_t stream) {
  if (!X || !inv_lambda || !s_a || !s_w || !codes || !scales || !U || (rank > 0 && !l1t))
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_quantize_act: null pointer");
  if (M < 1 || K < 64 || K % 64 || ldx < K || ldx % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_quantize_act: need M >= 1, K % 64 == 0, ldx >= K, ldx % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_quantize_act: rank must be a multiple of 16 in [0, 64]");
  if (!aligned16(X) || !aligned16(inv_lambda) || !aligned16(codes) || !aligned16(scales) || !aligned16(U) ||
      (rank > 0 && !aligned16(l1t)))
    return fail(SVDQ_ERR_ALIGNMENT, "svdq_quantize_act: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;

  Params p;
  p.M = M;
  p.K = K;
  p.m_pad = (M + 127) / 128 * 128;
  p.inv_lambda = inv_lambda;
  p.s_a = s_a;
  p.s_w = s_w;
  p.codes = codes;
  p.scales = scales;
  p.U = static_cast<uint16_t *>(U);
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
  const int grid = p.m_pad / BM;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (rank) {
    case 0: return launch<0>(tx, tl, p, grid, s);
    case 16: return launch<16>(tx, tl, p, grid, s);
    case 32: return launch<32>(tx, tl, p, grid, s);
    case 48: return launch<48>(tx, tl, p, grid, s);
    default: return launch<64>(tx, tl, p, grid, s);
  }
}
