// K2: W4A4 GEMM with the low-rank up-projection fused in.
//
// The pages fuse the 16-bit low-rank up-projection into the 4-bit GEMM so the
// correction branch does not eat the W4A4 gain (web page "Nunchaku Diffusers
// 支持降低显存占用，但硬件仍决定适用范围", remio.ai, section "SVDQuant 将棘手数值移出
// 4 位路径").  Per 128 x 256 output tile:
//   acc  = U_tile . L2T_tile^T                 tcgen05.mma kind::f16 (bf16)
//   acc += sum_k (qa sa)(qw sw)                tcgen05.mma kind::mxf4nvf4,
//                                               block16 ue4m3 scales in TMEM
//   Y    = bf16( epilogue( s_a s_w acc + bias ) )
// U arrives pre-divided by s_a s_w, so both branches share one fp32
// accumulator and one scale in the epilogue.
//
// Structure (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: A/B code tiles (128-byte swizzle), scale-factor
//               atoms (bulk copies), the U / L2T tiles of the low-rank stage
//   warp 1      owns TMEM (512 columns) and issues tcgen05.cp / tcgen05.mma
//               from one thread; commits release pipeline stages
//   warps 2..9  epilogue: drain the 128 x 256 fp32 accumulator from TMEM
//               (each warp: its 32-lane quarter, 128 columns), release it to
//               the MMA warp at once, then scale, add bias, GELU, store bf16
// Pipeline: 4 stages of {A 16 KB, B 32 KB, SFA 2 KB, SFB 4 KB}; one stage
// carries 256 K-elements (4 MMAs of K = 64).  A tile's first stage carries
// the low-rank operands (rank / 16 MMAs of K = 16).
// Every wait is bounded; a wait that runs out records SVDQ_ERR_TIMEOUT, the
// other roles see the abort flag, in-flight work is drained and TMEM freed.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 256;
constexpr int BK_BYTES = 128;                // 256 e2m1 elements per row per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;       // 16384
constexpr int B_BYTES = BN * BK_BYTES;       // 32768
constexpr int SFA_BYTES = 4 * 512;           // 4 atoms: 128 rows x 16 scales
constexpr int SFB_BYTES = 2 * 4 * 512;       // 2 row blocks of 128
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
constexpr int THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SFA_COL = 256, SFB_COL = 272;

// Instruction descriptors (tcgen05 instruction-descriptor bit fields):
// [4,6) accumulator format (1 = f32), [7,10) A format, [10,13) B format,
// [17,23) N >> 3, [24,29) M >> 4; block-scaled: [23] scale format
// (0 = ue4m3), [29,31) / [4,6) scale-factor ids (0), A/B K-major (bits 15/16 = 0).
constexpr uint32_t IDESC_BF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);

struct Params {
  int M, N, K, rank, epilogue, gelu_col_begin, ldy;
  int num_m_blk, num_tiles, k_stages, kb_total;
  const uint8_t *sfa, *sfb;
  const float *s_a, *s_w;
  const uint16_t *bias;
  uint16_t *Y;
  unsigned int *status;
  unsigned long long limit_ns;
};

__device__ __forceinline__ float gelu_erf(float y) { return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_tanh(float y) {
  return 0.5f * y * (1.0f + tanhf(0.79788456080286536f * (y + 0.044715f * y * y * y)));
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_l2, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tmem_full = empty + STAGES;
  uint64_t *tmem_empty = tmem_full + 1;
  uint64_t *drain = tmem_empty + 1;
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_lr = p.rank > 0;
  const int stages_per_tile = p.k_stages + (has_lr ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], 1);
    }
    dev::mbar_init(tmem_full, 1);
    dev::mbar_init(tmem_empty, EPI_WARPS);
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == 1) {
    dev::tmem_alloc(tmem_base_slot, TMEM_COLS);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      dev::prefetch_tmap(&tm_a);
      dev::prefetch_tmap(&tm_b);
      if (has_lr) {
        dev::prefetch_tmap(&tm_u);
        dev::prefetch_tmap(&tm_l2);
      }
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % p.num_m_blk, n_blk = tile / p.num_m_blk;
        for (int st = 0; st < stages_per_tile; ++st, ++it) {
          const int s = it % STAGES;
          if (!dev::mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *sa = smem + s * STAGE_BYTES;
          uint8_t *sb = sa + A_BYTES;
          uint8_t *ssfa = sb + B_BYTES;
          uint8_t *ssfb = ssfa + SFA_BYTES;
          if (has_lr && st == 0) {
            dev::mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
            dev::tma_load_2d(sa, &tm_u, &full[s], 0, m_blk * BM);
            dev::tma_load_2d(sb, &tm_l2, &full[s], 0, n_blk * BN);
          } else {
            const int ks = st - (has_lr ? 1 : 0);
            const int nkb = min(4, p.kb_total - ks * 4);
            const bool b1_ok = (n_blk * 2 + 1) * 128 < p.N;
            const uint32_t sf_bytes = static_cast<uint32_t>(nkb * 512);
            dev::mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES + sf_bytes * (b1_ok ? 3u : 2u));
            dev::tma_load_2d(sa, &tm_a, &full[s], ks * BK_BYTES, m_blk * BM);
            dev::tma_load_2d(sb, &tm_b, &full[s], ks * BK_BYTES, n_blk * BN);
            dev::bulk_load(ssfa, p.sfa + (static_cast<size_t>(m_blk) * p.kb_total + ks * 4) * 512, sf_bytes, &full[s]);
            dev::bulk_load(ssfb, p.sfb + (static_cast<size_t>(n_blk * 2) * p.kb_total + ks * 4) * 512, sf_bytes,
                           &full[s]);
            if (b1_ok)
              dev::bulk_load(ssfb + 2048, p.sfb + (static_cast<size_t>(n_blk * 2 + 1) * p.kb_total + ks * 4) * 512,
                             sf_bytes, &full[s]);
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        dev::report(p.status, SVDQ_ERR_TIMEOUT);
        for (int j = max(0, it - STAGES); j < it; ++j)  // let issued copies land
          dev::mbar_wait(&full[j % STAGES], (j / STAGES) & 1, p.limit_ns, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, tcount = 0;
      bool ok = true, issued_any = false;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
        const int n_blk = tile / p.num_m_blk;
        const bool b1_ok = (n_blk * 2 + 1) * 128 < p.N;
        if (!dev::mbar_wait(tmem_empty, (tcount & 1) ^ 1, p.limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        for (int st = 0; st < stages_per_tile; ++st, ++it) {
          const int s = it % STAGES;
          if (!dev::mbar_wait(&full[s], (it / STAGES) & 1, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t sa = dev::smem_u32(smem + s * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t ssfa = sb + B_BYTES;
          const uint32_t ssfb = ssfa + SFA_BYTES;
          if (has_lr && st == 0) {
            for (int j = 0; j < p.rank / 16; ++j) {  // K = 16 bf16 = 32 bytes per MMA
              dev::umma_bf16(tmem, dev::desc_sw128(sa + 32 * j), dev::desc_sw128(sb + 32 * j), IDESC_BF16,
                             accumulate);
              accumulate = 1;
            }
          } else {
            const int ks = st - (has_lr ? 1 : 0);
            const int nkb = min(4, p.kb_total - ks * 4);
            for (int kb = 0; kb < nkb; ++kb) {
              dev::tmem_cp_32x128b_x4(tmem + SFA_COL + 4 * kb, dev::desc_sf(ssfa + 512 * kb));
              dev::tmem_cp_32x128b_x4(tmem + SFB_COL + 8 * kb, dev::desc_sf(ssfb + 512 * kb));
              if (b1_ok) dev::tmem_cp_32x128b_x4(tmem + SFB_COL + 8 * kb + 4, dev::desc_sf(ssfb + 2048 + 512 * kb));
            }
            for (int kb = 0; kb < nkb; ++kb) {  // K = 64 e2m1 = 32 bytes per MMA
              dev::umma_nvfp4(tmem, dev::desc_sw128(sa + 32 * kb), dev::desc_sw128(sb + 32 * kb), IDESC_NVFP4,
                              tmem + SFA_COL + 4 * kb, tmem + SFB_COL + 8 * kb, accumulate);
              accumulate = 1;
            }
          }
          issued_any = true;
          dev::tc_commit(&empty[s]);  // stage s is free once these MMAs finish
        }
        if (!ok) break;
        dev::tc_commit(tmem_full);    // accumulator ready for the epilogue
      }
      if (!ok) {
        *abort_flag = 1;
        dev::report(p.status, SVDQ_ERR_TIMEOUT);
      }
      if (issued_any) {  // make sure the tensor core is idle before TMEM is freed
        dev::tc_commit(drain);
        dev::mbar_wait(drain, 0, p.limit_ns, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;       // which 128 of the 256 columns
    const float alpha = __fmul_rn(__ldg(p.s_a), __ldg(p.s_w));
    int tcount = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      const int m_blk = tile % p.num_m_blk, n_blk = tile / p.num_m_blk;
      if (!dev::mbar_wait(tmem_full, tcount & 1, p.limit_ns, abort_flag)) {
        *abort_flag = 1;
        dev::report(p.status, SVDQ_ERR_TIMEOUT);
        break;
      }
      dev::tc_fence_after();
      uint32_t v[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(half * 128);
#pragma unroll
      for (int c = 0; c < 4; ++c) dev::tmem_ld_32x32b_x32(taddr + 32 * c, v[c]);
      dev::tmem_wait_ld();
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(tmem_empty);  // the MMA warp may start the next tile

      const int row = m_blk * BM + 32 * q + lane;
      const int col0 = n_blk * BN + half * 128;
      if (row < p.M) {
        uint16_t *yrow = p.Y + static_cast<size_t>(row) * p.ldy;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int col = col0 + 32 * c + 8 * g;
            if (col >= p.N) continue;
            float b[8];
            if (p.bias) {
              const uint4 bb = __ldg(reinterpret_cast<const uint4 *>(p.bias + col));
              const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                b[2 * j] = __uint_as_float(bw[j] << 16);
                b[2 * j + 1] = __uint_as_float(bw[j] & 0xFFFF0000u);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) b[j] = 0.0f;
            }
            uint32_t out[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float y0 = __fmaf_rn(alpha, __uint_as_float(v[c][8 * g + 2 * j]), b[2 * j]);
              float y1 = __fmaf_rn(alpha, __uint_as_float(v[c][8 * g + 2 * j + 1]), b[2 * j + 1]);
              if (p.epilogue != SVDQ_EPILOGUE_NONE) {
                const bool act0 = col + 2 * j >= p.gelu_col_begin, act1 = col + 2 * j + 1 >= p.gelu_col_begin;
                if (p.epilogue == SVDQ_EPILOGUE_GELU_ERF) {
                  if (act0) y0 = gelu_erf(y0);
                  if (act1) y1 = gelu_erf(y1);
                } else {
                  if (act0) y0 = gelu_tanh(y0);
                  if (act1) y1 = gelu_tanh(y1);
                }
              }
              __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
              out[j] = *reinterpret_cast<uint32_t *>(&h);
            }
            *reinterpret_cast<uint4 *>(yrow + col) = make_uint4(out[0], out[1], out[2], out[3]);
          }
        }
      }
    }
  }

  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_linear_w4a4(const uint8_t *a_codes, const uint8_t *a_scales, const void *U, const float *s_a,
                                const uint8_t *w_codes, const uint8_t *w_scales, const void *l2t, const float *s_w,
                                const void *bias, int M, int N, int K, int rank, int epilogue, int gelu_col_begin,
                                void *Y, int ldy, svdq_stream_t stream) {
  if (!a_codes || !a_scales || !s_a || !w_codes || !w_scales || !s_w || !Y || (rank > 0 && (!U || !l2t)))
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_w4a4: null pointer");
  if (epilogue < SVDQ_EPILOGUE_NONE || epilogue > SVDQ_EPILOGUE_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_w4a4: unknown epilogue");
  if (M < 1 || K < 64 || K % 64 || N < 8 || N % 8 || ldy < N || ldy % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_w4a4: need M >= 1, K % 64 == 0, N % 8 == 0, ldy >= N, ldy % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_w4a4: rank must be a multiple of 16 in [0, 64]");
  if (gelu_col_begin < 0 || gelu_col_begin > N)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_w4a4: gelu_col_begin outside [0, N]");
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (rank > 0 && (!aligned16(U) || !aligned16(l2t))))
    return fail(SVDQ_ERR_ALIGNMENT, "svdq_linear_w4a4: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;

  Params p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.rank = rank;
  p.epilogue = epilogue;
  p.gelu_col_begin = gelu_col_begin;
  p.ldy = ldy;
  p.num_m_blk = (M + BM - 1) / BM;
  const int num_n_blk = (N + BN - 1) / BN;
  p.num_tiles = p.num_m_blk * num_n_blk;
  p.kb_total = K / 64;
  p.k_stages = (p.kb_total + 3) / 4;
  p.sfa = a_scales;
  p.sfb = w_scales;
  p.s_a = s_a;
  p.s_w = s_w;
  p.bias = static_cast<const uint16_t *>(bias);
  p.Y = static_cast<uint16_t *>(Y);
  p.status = st->status_word;
  p.limit_ns = kWaitLimitNs;

  CUtensorMap ta, tb, tu, tl;
  int rc = encode_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, static_cast<uint64_t>(K / 2),
                          static_cast<uint64_t>(M), static_cast<uint64_t>(K / 2), BK_BYTES, BM,
                          CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != SVDQ_OK) return rc;
  rc = encode_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, static_cast<uint64_t>(K / 2),
                      static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), BK_BYTES, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != SVDQ_OK) return rc;
  if (rank > 0) {
    rc = encode_tmap_2d(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, U, SVDQ_LR_STRIDE, static_cast<uint64_t>(M),
                        SVDQ_LR_STRIDE * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != SVDQ_OK) return rc;
    rc = encode_tmap_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, l2t, SVDQ_LR_STRIDE, static_cast<uint64_t>(N),
                        SVDQ_LR_STRIDE * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != SVDQ_OK) return rc;
  } else {
    tu = ta;
    tl = tb;
  }

  cudaError_t e = cudaFuncSetAttribute(gemm_w4a4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_w4a4: ") + cudaGetErrorString(e));
  const int grid = std::min(p.num_tiles, st->sm_count);
  gemm_w4a4_kernel<<<grid, THREADS, SMEM_BYTES, reinterpret_cast<cudaStream_t>(stream)>>>(ta, tb, tu, tl, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_w4a4 launch: ") + cudaGetErrorString(e));
  return ok();
}
