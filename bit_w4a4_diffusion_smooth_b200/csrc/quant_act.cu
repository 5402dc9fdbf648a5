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
// Design (memory bound: X is read once, ~0.3 B written per byte read):
//   * one CTA per 32 rows, 16 compute warps + 1 TMA warp; a 4-stage ring of
//     [32 rows x 256 cols] bf16 tiles of X, [rank x 256] tiles of L1^T and
//     256-float slices of inv_lambda, loaded by TMA / bulk copies; X and L1^T
//     land with the 128-byte swizzle (conflict-free for the row-wise pass and
//     for ldmatrix);
//   * quantize pass: each warp owns 2 rows, each lane 8 consecutive elements
//     (two lanes per 16-block, one shuffle for the block max); codes go out
//     as one 128-byte row segment per warp and row, four block scales per
//     32-bit store; X^ is written back in place as bf16;
//   * down-projection pass: warp w multiplies k16-slice w of the tile with
//     mma.sync (bf16 in, fp32 accumulate); partial sums are added across the
//     warps once at the end;
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
  return 1024 + STAGES * stage_bytes<RANK>() + 256;
}

// Byte offset of the 16-byte chunk holding column c (0..63, multiple of 8) of
// row r inside a 128-byte-swizzled box of 128-byte rows.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ r) & 7) << 4));
}

__device__ __forceinline__ void fail_wait(volatile int *abort_flag, unsigned int *status) {
  *abort_flag = 1;
  dev::report(status, SVDQ_ERR_TIMEOUT);
}

template <int RANK>
__global__ void __launch_bounds__(THREADS, 1)
    quant_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1, Params p) {
  constexpr int NP = RANK / 16;           // pairs of 8-wide MMA column tiles
  constexpr int L1_BOX = RANK * 128;
  constexpr int STAGE = stage_bytes<RANK>();
  constexpr int INV_OFF = X_STAGE + 4 * L1_BOX;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE);
  uint64_t *empty = full + STAGES;
  uint64_t *ready = empty + STAGES;       // X^ written back, per stage
  uint64_t *sync = ready + STAGES;        // two end-of-loop syncs
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sync + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;

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
      for (int c = 0; c < p.KS; ++c) {
        const int s = c % STAGES;
        if (!dev::mbar_wait(&empty[s], ((c / STAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
          fail_wait(abort_flag, p.status);
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
  const int m_blk = m0 / 128;
  const int r_base = m0 % 128;            // row of this CTA's first row inside its 128-row tile

  for (int c = 0; c < p.KS; ++c) {
    const int s = c % STAGES;
    const uint32_t ph = (c / STAGES) & 1;
    if (!dev::mbar_wait(&full[s], ph, p.limit_ns, abort_flag)) {
      fail_wait(abort_flag, p.status);
      return;
    }
    const int nbox = min(4, (p.K - c * KC) / 64);
    uint8_t *st = smem + s * STAGE;
    const int box = lane >> 3;
    const bool col_ok = box < nbox;       // columns past K quantize as zeros
    uint8_t *tile = p.bundle + (static_cast<size_t>(m_blk) * p.KS + c) * bundle_tile_bytes(128);

    float inv[8];
    if (col_ok) {
      const float4 i0 = *reinterpret_cast<const float4 *>(st + INV_OFF + 32 * lane);
      const float4 i1 = *reinterpret_cast<const float4 *>(st + INV_OFF + 32 * lane + 16);
      inv[0] = i0.x; inv[1] = i0.y; inv[2] = i0.z; inv[3] = i0.w;
      inv[4] = i1.x; inv[5] = i1.y; inv[6] = i1.z; inv[7] = i1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) inv[i] = 0.0f;
    }

    // ---- quantize pass: rows 2*warp, 2*warp+1
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = warp * 2 + i;
      const int rt = r_base + r;          // row inside the 128-row bundle tile
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
      // this lane's 4 code bytes: byte 4*lane of the row, 128-byte swizzle
      *reinterpret_cast<uint32_t *>(tile + rt * 128 + ((((lane >> 2) ^ rt) & 7) << 4) + (lane & 3) * 4) = packed;
      // four consecutive block scales (lanes 8q, 8q+2, 8q+4, 8q+6) -> one word of atom q
      const int base = lane & ~7;
      const uint32_t word = __shfl_sync(0xFFFFFFFFu, sb, base) | (__shfl_sync(0xFFFFFFFFu, sb, base + 2) << 8) |
                            (__shfl_sync(0xFFFFFFFFu, sb, base + 4) << 16) |
                            (__shfl_sync(0xFFFFFFFFu, sb, base + 6) << 24);
      if ((lane & 7) == 0)
        *reinterpret_cast<uint32_t *>(tile + 128 * 128 + box * 512 + (rt & 31) * 16 + ((rt >> 5) & 3) * 4) = word;
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

    // ---- down-projection pass: warp w takes columns [16w, 16w+16) of the tile
    if (RANK > 0) {
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&ready[s]);
      if (!dev::mbar_wait(&ready[s], ph, p.limit_ns, abort_flag)) {
        fail_wait(abort_flag, p.status);
        return;
      }
      const int kbox = warp >> 2;
      if (kbox < nbox) {
        const uint32_t xbase = dev::smem_u32(st + kbox * X_BOX);
        const uint32_t lbase = dev::smem_u32(st + X_STAGE + kbox * L1_BOX);
        const int kc = (warp & 3) * 16;
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
      // the next TMA load into this stage must come after our generic writes
      dev::fence_proxy_async();
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[s]);
  }

  // ---- U = (sum of the warps' partial products) / (s_a s_w), bf16, 128-row tiles
  const int tid = threadIdx.x;  // 0..511
  if (RANK > 0) {
    // every warp is done with the stage buffers -> reuse them for partials
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(sync);
    if (!dev::mbar_wait(sync, 0, p.limit_ns, abort_flag)) {
      fail_wait(abort_flag, p.status);
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
      fail_wait(abort_flag, p.status);
      return;
    }
  }
  const float alpha = __fmul_rn(s_a, __ldg(p.s_w));
  for (int idx = tid; idx < BM * (SVDQ_LR_STRIDE / 8); idx += CWARPS * 32) {
    const int r = idx >> 3, cc = idx & 7;   // row, 8-column chunk
    const int m = m0 + r;
    uint32_t o[4] = {0, 0, 0, 0};
    if (RANK > 0 && 8 * cc < RANK) {
      const float *red = reinterpret_cast<const float *>(smem);
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < CWARPS; ++w) sum += red[(w * BM + r) * RANK + 8 * cc + j];
        v[j] = __fdiv_rn(sum, alpha);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        o[j] = *reinterpret_cast<uint32_t *>(&h);
      }
    }
    *reinterpret_cast<uint4 *>(p.U + lowrank_offset(m, 8 * cc, 128)) = make_uint4(o[0], o[1], o[2], o[3]);
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
