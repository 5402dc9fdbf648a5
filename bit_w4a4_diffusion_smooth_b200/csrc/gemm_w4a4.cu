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
// Structure (one CTA per SM, persistent over output tiles, 12 warps):
//   warps 0, 3  producers: one bulk copy per stage each - the activation
//               bundle tile (128 rows x 256 K: swizzled codes + block scales,
//               18 KB) and the weight bundle tile (256 rows, 36 KB); at the
//               start of a tile the U and L2T tiles of the low-rank branch
//   warp 1      owns TMEM (512 columns), issues tcgen05.mma from one thread
//   warp 2      moves each stage's block scales from shared memory into that
//               stage's own TMEM columns (tcgen05.cp 32x128b.warpx4); issued
//               from its own warp the copies overlap the MMAs, issued from
//               the MMA thread they would serialize with them
//   warps 4..11 epilogue: drain the 128 x 256 fp32 accumulator (each warp its
//               32-lane quarter, 128 columns), hand TMEM back at once, then
//               scale, add bias, GELU, round to bf16 into a 128-byte-swizzled
//               staging tile and write it with TMA stores
// Pipeline: 3 stages of 54 KB (the two bundle tiles, which are laid out in
// memory exactly as the MMA reads them from shared memory); TMEM holds the
// accumulator (256 columns) and 3 x 48 columns of block scales.
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
constexpr int STAGES = 3;
constexpr int A_TILE = BM * 144;              // activation bundle tile: codes 16 KB + scales 2 KB
constexpr int B_TILE = BN * 144;              // weight bundle tile: codes 32 KB + scales 4 KB
constexpr int SFA_OFF = BM * 128;
constexpr int B_OFF = A_TILE;                 // 18432, a multiple of 1024
constexpr int SFB_OFF = B_OFF + BN * 128;
constexpr int STAGE_BYTES = A_TILE + B_TILE;  // 55296
constexpr int U_TILE = BM * 128, L2_TILE = BN * 128;
constexpr int EPI_WARPS = 8;
constexpr int EPI_TILE_BYTES = 32 * 128;      // 32 rows x 64 bf16, 128-byte swizzle
constexpr int EPI_OFF = STAGES * STAGE_BYTES;
constexpr int BAR_OFF = EPI_OFF + EPI_WARPS * EPI_TILE_BYTES;
constexpr int SMEM_BYTES = 1024 + BAR_OFF + 256;
constexpr int THREADS = (4 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL = 256;              // stage s: SFA at +48s (+4 kb), SFB at +48s+16 (+8 kb, +4 per row block)

// Instruction descriptors (tcgen05 instruction-descriptor bit fields):
// [4,6) accumulator format (1 = f32), [7,10) A format, [10,13) B format,
// [17,23) N >> 3, [24,29) M >> 4; block-scaled: [23] scale format
// (0 = ue4m3), [29,31) / [4,6) scale-factor ids (0), A/B K-major (bits 15/16 = 0).
constexpr uint32_t IDESC_BF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);

__device__ __forceinline__ uint32_t sfa_col(int s, int kb) { return SF_COL + 48 * s + 4 * kb; }
__device__ __forceinline__ uint32_t sfb_col(int s, int kb) { return SF_COL + 48 * s + 16 + 8 * kb; }

struct Params {
  int M, N, K, rank, epilogue, gelu_col_begin;
  int num_m_blk, num_tiles, k_stages, lr_stages, kb_total;
  const uint8_t *a_bundle, *w_bundle, *u, *l2t;
  const float *s_a, *s_w;
  const uint16_t *bias;
  unsigned int *status;
  unsigned long long limit_ns;
};

__device__ __forceinline__ float gelu_erf(float y) { return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_tanh(float y) {
  return 0.5f * y * (1.0f + tanhf(0.79788456080286536f * (y + 0.044715f * y * y * y)));
}

__device__ __forceinline__ void abort_all(volatile int *abort_flag, unsigned int *status) {
  *abort_flag = 1;
  dev::report(status, SVDQ_ERR_TIMEOUT);
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap tm_y, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + BAR_OFF);
  uint64_t *sf_full = full + STAGES;
  uint64_t *empty = sf_full + STAGES;
  uint64_t *tmem_full = empty + STAGES;
  uint64_t *tmem_empty = tmem_full + 1;
  uint64_t *drain_mma = tmem_empty + 1;
  uint64_t *drain_cp = drain_mma + 1;
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(drain_cp + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stages_per_tile = p.lr_stages + p.k_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      dev::mbar_init(&full[s], 2);            // one arrival per producer warp
      dev::mbar_init(&sf_full[s], 1);
      dev::mbar_init(&empty[s], 1);
    }
    dev::mbar_init(tmem_full, 1);
    dev::mbar_init(tmem_empty, EPI_WARPS);
    dev::mbar_init(drain_mma, 1);
    dev::mbar_init(drain_cp, 1);
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

  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ producers (0: activations, 3: weights)
    if (lane == 0) {
      const bool act = warp == 0;
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
          uint8_t *dst = smem + s * STAGE_BYTES + (act ? 0 : B_OFF);
          const uint8_t *src;
          uint32_t bytes;
          if (st < p.lr_stages) {
            src = act ? p.u + static_cast<size_t>(m_blk) * U_TILE : p.l2t + static_cast<size_t>(n_blk) * L2_TILE;
            bytes = act ? U_TILE : L2_TILE;
          } else {
            const int ks = st - p.lr_stages;
            src = act ? p.a_bundle + (static_cast<size_t>(m_blk) * p.k_stages + ks) * A_TILE
                      : p.w_bundle + (static_cast<size_t>(n_blk) * p.k_stages + ks) * B_TILE;
            bytes = act ? A_TILE : B_TILE;
          }
          dev::mbar_arrive_expect_tx(&full[s], bytes);
          dev::bulk_load(dst, src, bytes, &full[s]);
        }
      }
      if (!ok) {
        abort_all(abort_flag, p.status);
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
        if (!dev::mbar_wait(tmem_empty, (tcount & 1) ^ 1, p.limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        for (int st = 0; st < stages_per_tile; ++st, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!dev::mbar_wait(&sf_full[s], ph, p.limit_ns, abort_flag) ||
              !dev::mbar_wait(&full[s], ph, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t sa = dev::smem_u32(smem + s * STAGE_BYTES);
          const uint32_t sb = sa + B_OFF;
          if (st < p.lr_stages) {
            for (int j = 0; j < p.rank / 16; ++j) {  // K = 16 bf16 = 32 bytes per MMA
              dev::umma_bf16(tmem, dev::desc_sw128(sa + 32 * j), dev::desc_sw128(sb + 32 * j), IDESC_BF16,
                             accumulate);
              accumulate = 1;
            }
          } else {
            const int nkb = min(4, p.kb_total - 4 * (st - p.lr_stages));
            for (int kb = 0; kb < nkb; ++kb) {  // K = 64 e2m1 = 32 bytes per MMA
              dev::umma_nvfp4(tmem, dev::desc_sw128(sa + 32 * kb), dev::desc_sw128(sb + 32 * kb), IDESC_NVFP4,
                              tmem + sfa_col(s, kb), tmem + sfb_col(s, kb), accumulate);
              accumulate = 1;
            }
          }
          issued_any = true;
          dev::tc_commit(&empty[s]);  // stage s (shared memory and TMEM scales) free once these MMAs finish
        }
        if (!ok) break;
        dev::tc_commit(tmem_full);    // accumulator ready for the epilogue
      }
      if (!ok) abort_all(abort_flag, p.status);
      if (issued_any) {  // the tensor core must be idle before TMEM is freed
        dev::tc_commit(drain_mma);
        dev::mbar_wait(drain_mma, 0, p.limit_ns, nullptr);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale-factor copies
    if (lane == 0) {
      int it = 0;
      bool ok = true, issued_any = false;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int n_blk = tile / p.num_m_blk;
        const bool b1_ok = (n_blk * 2 + 1) * 128 < p.N;
        for (int st = 0; st < stages_per_tile; ++st, ++it) {
          const int s = it % STAGES;
          if (!dev::mbar_wait(&full[s], (it / STAGES) & 1, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          if (st >= p.lr_stages) {
            const int nkb = min(4, p.kb_total - 4 * (st - p.lr_stages));
            const uint32_t ssfa = dev::smem_u32(smem + s * STAGE_BYTES + SFA_OFF);
            const uint32_t ssfb = dev::smem_u32(smem + s * STAGE_BYTES + SFB_OFF);
            for (int kb = 0; kb < nkb; ++kb) {
              dev::tmem_cp_32x128b_x4(tmem + sfa_col(s, kb), dev::desc_sf(ssfa + 512 * kb));
              dev::tmem_cp_32x128b_x4(tmem + sfb_col(s, kb), dev::desc_sf(ssfb + 512 * kb));
              if (b1_ok) dev::tmem_cp_32x128b_x4(tmem + sfb_col(s, kb) + 4, dev::desc_sf(ssfb + 2048 + 512 * kb));
            }
            issued_any = true;
          }
          dev::tc_commit(&sf_full[s]);  // arrives once this stage's copies have landed
        }
      }
      if (!ok) abort_all(abort_flag, p.status);
      if (issued_any) {
        dev::tc_commit(drain_cp);
        dev::mbar_wait(drain_cp, 0, p.limit_ns, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 4;
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int half = e >> 2;                // which 128 of the 256 columns
    uint8_t *stage_out = smem + EPI_OFF + e * EPI_TILE_BYTES;
    const float alpha = __fmul_rn(__ldg(p.s_a), __ldg(p.s_w));
    int tcount = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      const int m_blk = tile % p.num_m_blk, n_blk = tile / p.num_m_blk;
      if (!dev::mbar_wait(tmem_full, tcount & 1, p.limit_ns, abort_flag)) {
        abort_all(abort_flag, p.status);
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

      const int row0 = m_blk * BM + 32 * q;
      const int col0 = n_blk * BN + half * 128;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {        // two 64-column chunks
        if (lane == 0) dev::bulk_wait_group_read<0>();  // staging tile free again
        __syncwarp();
#pragma unroll
        for (int g = 0; g < 8; ++g) {         // 8 columns (16 bytes) at a time
          const int c = 2 * c2 + (g >> 2);
          const int col = col0 + 64 * c2 + 8 * g;
          float b[8];
          if (p.bias && col + 8 <= p.N) {
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
            float y0 = __fmaf_rn(alpha, __uint_as_float(v[c][8 * (g & 3) + 2 * j]), b[2 * j]);
            float y1 = __fmaf_rn(alpha, __uint_as_float(v[c][8 * (g & 3) + 2 * j + 1]), b[2 * j + 1]);
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
          // row `lane` of the 32 x 64 staging tile, 16-byte chunk g, 128-byte swizzle
          *reinterpret_cast<uint4 *>(stage_out + lane * 128 + ((g ^ (lane & 7)) << 4)) =
              make_uint4(out[0], out[1], out[2], out[3]);
        }
        dev::fence_proxy_async();  // make the generic writes visible to the TMA store
        __syncwarp();
        if (lane == 0 && row0 < p.M && col0 + 64 * c2 < p.N) {  // the TMA clips the ragged edges
          dev::tma_store_2d(&tm_y, stage_out, col0 + 64 * c2, row0);
          dev::bulk_commit_group();
        }
      }
    }
    if (lane == 0) dev::bulk_wait_group<0>();
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

extern "C" int svdq_linear_w4a4(const uint8_t *a_bundle, const void *U, const float *s_a, const uint8_t *w_bundle,
                                const void *l2t, const float *s_w, const void *bias, int M, int N, int K, int rank,
                                int epilogue, int gelu_col_begin, void *Y, int ldy, svdq_stream_t stream) {
  if (!a_bundle || !s_a || !w_bundle || !s_w || !Y || (rank > 0 && (!U || !l2t)))
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_w4a4: null pointer");
  if (epilogue < SVDQ_EPILOGUE_NONE || epilogue > SVDQ_EPILOGUE_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_w4a4: unknown epilogue");
  if (M < 1 || K < 64 || K % 64 || N < 8 || N % 8 || ldy < N || ldy % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_w4a4: need M >= 1, K % 64 == 0, N % 8 == 0, ldy >= N, ldy % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_w4a4: rank must be a multiple of 16 in [0, 64]");
  if (gelu_col_begin < 0 || gelu_col_begin > N)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_w4a4: gelu_col_begin outside [0, N]");
  if (!aligned16(a_bundle) || !aligned16(w_bundle) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (rank > 0 && (!aligned16(U) || !aligned16(l2t))))
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
  p.num_m_blk = (M + BM - 1) / BM;
  const int num_n_blk = (N + BN - 1) / BN;
  p.num_tiles = p.num_m_blk * num_n_blk;
  p.kb_total = K / 64;
  p.k_stages = bundle_ks(K);
  p.lr_stages = rank > 0 ? 1 : 0;
  p.a_bundle = a_bundle;
  p.w_bundle = w_bundle;
  p.u = static_cast<const uint8_t *>(U);
  p.l2t = static_cast<const uint8_t *>(l2t);
  p.s_a = s_a;
  p.s_w = s_w;
  p.bias = static_cast<const uint16_t *>(bias);
  p.status = st->status_word;
  p.limit_ns = kWaitLimitNs;

  CUtensorMap ty;
  int rc = encode_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                          static_cast<uint64_t>(ldy) * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != SVDQ_OK) return rc;
  cudaError_t e = cudaFuncSetAttribute(gemm_w4a4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_w4a4: ") + cudaGetErrorString(e));
  const int grid = std::min(p.num_tiles, st->sm_count);
  gemm_w4a4_kernel<<<grid, THREADS, SMEM_BYTES, reinterpret_cast<cudaStream_t>(stream)>>>(ty, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_w4a4 launch: ") + cudaGetErrorString(e));
  return ok();
}
