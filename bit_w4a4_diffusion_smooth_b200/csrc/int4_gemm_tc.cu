// INT4 W4A4 GEMM on the 5th-generation tensor cores (tcgen05), for N a
// multiple of 256.
//
// The layer is the INT4 variant of the pages' W4A4 layer (donmalab.com,
// "Diffusers × Nunchaku 4-bit", section "實務上的影響與硬體要求"; this library
// reads it as symmetric INT4 in groups of 64 along K with bf16 scales):
//   Y = epilogue( sum_g (s_a[m,g] s_w[n,g]) sum_{k in g} q_a q_w + U . L2 + bias )
// tcgen05 has no 4-bit integer kind, and an 8-bit integer MMA would leave a
// per-group rescale of every output to the CUDA cores.  Instead every code is
// turned, once per tile, into the exact half-precision value q * s (|q| <= 8
// takes 4 significant bits and the bf16 scale 8, so the product has at most 11
// and is exact in fp16 whenever it lies in fp16's normal range), and the
// tensor cores multiply those: the fp32 accumulation then sums exactly the
// products the layer defines, with no per-group work after the MMA.
//
// One CTA per 128 x 256 output tile, 16 warps:
//   warp 0       producer: per group of 64 along K, TMA copies of the 128 x 32
//                and 256 x 32 bytes of codes and bulk copies of their scales
//                into a ring of 4 load slots; first, once, the tile's U and L2T
//                rows (their low-rank tile layouts are the MMA operand image)
//   warp 1       owns TMEM (256 columns, the fp32 accumulator) and issues, from
//                one thread, the low-rank MMAs (kind::f16, bf16) and then 4
//                MMAs per group (kind::f16, fp16 operands, M 128, N 256, K 16)
//                from a ring of 2 converted slots, committing each slot back
//   warps 4..11  converters: half-precision q * s of the slot's 384 rows into
//                the 128-byte-swizzled K-major layout (16 KB of A, 32 KB of B)
//   warps 12..15 epilogue: TMEM -> registers (lane quarter = warp % 4), bias,
//                GELU, bf16 rows to global memory
// The pair form below (a cluster of 2 CTAs per 256 x 256 tile, cta_group::2
// MMAs) is the one launched: each SM converts a third less per group.
// Inside every 8-element chunk both operands hold k in the same permuted order
// (k, k+4 pairs, so one mask-and-or makes a pair), which leaves the products'
// sum unchanged.  Every wait is bounded: a wait that runs out records
// SVDQ_ERR_TIMEOUT, raises the CTA's abort flag and every role leaves for the
// final barrier, after which TMEM is freed once the tensor cores are idle.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 256, LSTAGES = 4, CSTAGES = 2;
constexpr int THREADS = 16 * 32;
constexpr int A4_BYTES = BM * 32, B4_BYTES = BN * 32, SA_BYTES = BM * 2, SB_BYTES = BN * 2;
constexpr int LSTAGE = 13312;                                   // 13,056 bytes used, 1 KB multiple
constexpr int A16_BYTES = BM * 128, B16_BYTES = BN * 128;       // 16 KB, 32 KB
constexpr int CSTAGE = A16_BYTES + B16_BYTES;
constexpr int CONV_OFF = 0;
constexpr int LR_OFF = CONV_OFF + CSTAGES * CSTAGE;             // U 16 KB + L2T 32 KB
constexpr int LOAD_OFF = LR_OFF + A16_BYTES + B16_BYTES;
constexpr int BAR_OFF = LOAD_OFF + LSTAGES * LSTAGE;
constexpr int SMEM_BYTES = 1024 + BAR_OFF + 256;
constexpr uint32_t TMEM_COLS = 256;
static_assert(A4_BYTES + B4_BYTES + SA_BYTES + SB_BYTES <= LSTAGE, "a load slot holds one group");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
// instruction descriptors: f32 accumulate (bit 4), A/B fp16 (0) or bf16 (1) at bits 7 and 10,
// N >> 3 at bit 17, M >> 4 at bit 24, both operands K-major
constexpr uint32_t IDESC_F16 = (1u << 4) | ((BN >> 3) << 17) | ((BM >> 4) << 24);
constexpr uint32_t IDESC_BF16 = IDESC_F16 | (1u << 7) | (1u << 10);

struct TcParams {
  const uint16_t *a_scales, *w_scales, *bias;
  const uint8_t *U, *l2t;
  uint16_t *Y;
  int M, N, K, ldy, ld_sa, rank, gelu_col_begin;
  unsigned int *status;
  unsigned long long limit_ns;
};
struct TcMaps {
  CUtensorMap a, b;
};

// Four fp16 pairs of one word of eight codes (element i at bits 4i), in the
// permuted k order (i, i + 4): pair i = (q_i s, q_{i+4} s), exact.
__device__ __forceinline__ uint4 dequant8(uint32_t x, __half2 s2) {
  const __half2 bias = __floats2half2_rn(1032.0f, 1032.0f);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // nibble -> fp16 1024 + (q + 8): the offset-binary code (q xor 8 on the low 4 bits) in the mantissa
    uint32_t t;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t) : "r"(x >> (4 * i)), "r"(0x000F000Fu), "r"(0x64086408u));
    const __half2 q = __hsub2(*reinterpret_cast<__half2 *>(&t), bias);       // q, exact
    const __half2 v = __hmul2(q, s2);                                         // q s, exact
    o[i] = *reinterpret_cast<const uint32_t *>(&v);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1) int4_gemm_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *load_full = reinterpret_cast<uint64_t *>(smem + BAR_OFF);
  uint64_t *load_empty = load_full + LSTAGES;
  uint64_t *conv_full = load_empty + LSTAGES;
  uint64_t *conv_empty = conv_full + CSTAGES;
  uint64_t *lr_full = conv_empty + CSTAGES;
  uint64_t *tmem_full = lr_full + 1;
  uint64_t *drain = tmem_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int G = p.K / 64;
  if (threadIdx.x == 0) {
    for (int s = 0; s < LSTAGES; ++s) {
      dev::mbar_init(&load_full[s], 1);
      dev::mbar_init(&load_empty[s], 8);
    }
    for (int c = 0; c < CSTAGES; ++c) {
      dev::mbar_init(&conv_full[c], 8);
      dev::mbar_init(&conv_empty[c], 1);
    }
    dev::mbar_init(lr_full, 1);
    dev::mbar_init(tmem_full, 1);
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == 1) {
    dev::tmem_alloc(tmem_slot, TMEM_COLS);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();

  auto fail_wait = [&]() {
    *abort_flag = 1;
    dev::report(p.status, SVDQ_ERR_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      dev::prefetch_tmap(&maps.a);
      dev::prefetch_tmap(&maps.b);
      if (p.rank > 0) {
        dev::mbar_arrive_expect_tx(lr_full, A16_BYTES + B16_BYTES);
        dev::bulk_load(smem + LR_OFF, p.U + static_cast<size_t>(m0) * 128, A16_BYTES, lr_full);
        dev::bulk_load(smem + LR_OFF + A16_BYTES, p.l2t + static_cast<size_t>(n0) * 128, B16_BYTES, lr_full);
      }
      int issued = 0;
      for (int g = 0; g < G; ++g) {
        const int s = g % LSTAGES;
        if (!dev::mbar_wait(&load_empty[s], ((g / LSTAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
          fail_wait();
          break;
        }
        uint8_t *st = smem + LOAD_OFF + s * LSTAGE;
        dev::mbar_arrive_expect_tx(&load_full[s], A4_BYTES + B4_BYTES + SA_BYTES + SB_BYTES);
        dev::tma_load_2d(st, &maps.a, &load_full[s], g * 32, m0);
        dev::tma_load_2d(st + A4_BYTES, &maps.b, &load_full[s], g * 32, n0);
        dev::bulk_load(st + A4_BYTES + B4_BYTES, p.a_scales + static_cast<size_t>(g) * p.ld_sa + m0, SA_BYTES,
                       &load_full[s]);
        dev::bulk_load(st + A4_BYTES + B4_BYTES + SA_BYTES, p.w_scales + static_cast<size_t>(g) * p.N + n0, SB_BYTES,
                       &load_full[s]);
        ++issued;
      }
      // every copy issued lands before the block leaves
      if (p.rank > 0) dev::mbar_wait(lr_full, 0, p.limit_ns, nullptr);
      for (int g = max(0, issued - LSTAGES); g < issued; ++g)
        dev::mbar_wait(&load_full[g % LSTAGES], (g / LSTAGES) & 1, p.limit_ns, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true, issued_any = false;
      uint32_t accumulate = 0;
      if (p.rank > 0) {
        if (!dev::mbar_wait(lr_full, 0, p.limit_ns, abort_flag)) {
          fail_wait();
          ok = false;
        } else {
          dev::tc_fence_after();
          const uint32_t ua = dev::smem_u32(smem + LR_OFF), lb = ua + A16_BYTES;
          for (int j = 0; j < p.rank / 16; ++j) {   // K = 16 bf16 = 32 bytes per MMA
            dev::umma_bf16(tmem, dev::desc_sw128(ua + 32 * j), dev::desc_sw128(lb + 32 * j), IDESC_BF16, accumulate);
            accumulate = 1;
          }
          issued_any = true;
        }
      }
      for (int g = 0; g < G && ok; ++g) {
        const int c = g % CSTAGES;
        if (!dev::mbar_wait(&conv_full[c], (g / CSTAGES) & 1, p.limit_ns, abort_flag)) {
          fail_wait();
          ok = false;
          break;
        }
        dev::tc_fence_after();
        const uint32_t sa = dev::smem_u32(smem + CONV_OFF + c * CSTAGE), sb = sa + A16_BYTES;
        for (int j = 0; j < 4; ++j) {                 // K = 16 fp16 = 32 bytes per MMA
          dev::umma_bf16(tmem, dev::desc_sw128(sa + 32 * j), dev::desc_sw128(sb + 32 * j), IDESC_F16, accumulate);
          accumulate = 1;
        }
        issued_any = true;
        dev::tc_commit(&conv_empty[c]);               // the slot is free once these MMAs have read it
      }
      if (ok) dev::tc_commit(tmem_full);
      if (issued_any) {                               // the tensor cores are idle before TMEM is freed
        dev::tc_commit(drain);
        dev::mbar_wait(drain, 0, p.limit_ns, nullptr);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ converters
    const int ct = (warp - 4) * 32 + lane;           // 0..255
    for (int g = 0; g < G; ++g) {
      const int s = g % LSTAGES, c = g % CSTAGES;
      if (!dev::mbar_wait_warp(&load_full[s], (g / LSTAGES) & 1, p.limit_ns, abort_flag) ||
          !dev::mbar_wait_warp(&conv_empty[c], ((g / CSTAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
        fail_wait();
        break;
      }
      const uint8_t *st = smem + LOAD_OFF + s * LSTAGE;
      const uint16_t *sc = reinterpret_cast<const uint16_t *>(st + A4_BYTES + B4_BYTES);   // A then B scales
      uint8_t *cv = smem + CONV_OFF + c * CSTAGE;
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        // half-row hr of the 384 rows (A 0..127, B 128..383): 32 codes, k 32 h .. 32 h + 31
        const int hr = ct + 256 * j, row = hr >> 1, h = hr & 1;
        const uint4 q = *reinterpret_cast<const uint4 *>(st + row * 32 + h * 16);   // A rows then B rows
        const __half s16 = __float2half_rn(__uint_as_float(static_cast<uint32_t>(sc[row]) << 16));
        const __half2 s2 = __halves2half2(s16, s16);
        const int r = row < BM ? row : row - BM;
        uint8_t *tile = cv + (row < BM ? 0 : A16_BYTES) + r * 128;
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int chunk = 4 * h + w;                 // 16-byte chunk of the row's 128 bytes
          *reinterpret_cast<uint4 *>(tile + (((chunk ^ r) & 7) << 4)) = dequant8(words[w], s2);
        }
      }
      dev::fence_proxy_async();                      // the tensor cores read what the threads wrote
      __syncwarp();
      if (lane == 0) {
        dev::mbar_arrive(&load_empty[s]);
        dev::mbar_arrive(&conv_full[c]);
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    if (dev::mbar_wait_warp(tmem_full, 0, p.limit_ns, abort_flag)) {
      dev::tc_fence_after();
      const int row = 32 * q + lane, grow = m0 + row;
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        dev::tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * cb, v);
        dev::tmem_wait_ld();
        const int c0 = n0 + 32 * cb;
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = c0 + 2 * i;
          float2 y = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          if (p.bias) {
            const uint32_t bb = __ldg(reinterpret_cast<const uint32_t *>(p.bias + c));
            y.x += __uint_as_float(bb << 16);
            y.y += __uint_as_float(bb & 0xFFFF0000u);
          }
          if constexpr (EPI == SVDQ_EPILOGUE_GELU_ERF) {
            const float2 gy = dev::gelu_erf2(y);
            y = make_float2(c >= p.gelu_col_begin ? gy.x : y.x, c + 1 >= p.gelu_col_begin ? gy.y : y.y);
          } else if constexpr (EPI == SVDQ_EPILOGUE_GELU_TANH) {
            y = make_float2(c >= p.gelu_col_begin ? dev::gelu_tanh(y.x) : y.x,
                            c + 1 >= p.gelu_col_begin ? dev::gelu_tanh(y.y) : y.y);
          }
          __nv_bfloat162 h2 = __floats2bfloat162_rn(y.x, y.y);
          packed[i] = *reinterpret_cast<uint32_t *>(&h2);
        }
        if (grow < p.M) {
          uint4 *dst = reinterpret_cast<uint4 *>(p.Y + static_cast<size_t>(grow) * p.ldy + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
    } else {
      fail_wait();
    }
  }
  // warps 2 and 3 have no role; every warp meets here once
  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Pair form: a cluster of 2 CTAs per 256 x 256 tile (cta_group::2 MMAs, M 256).
// CTA h holds rows 128 h .. of the tile's A and output columns 128 h .. of its
// B, converts only those (128 + 128 rows per group instead of 128 + 256) and
// serves only its half of B to the tensor cores: a third less shared-memory
// traffic per group than the single-CTA form.  The even CTA's thread issues
// the MMAs once both CTAs' converters have arrived on its barrier; commits
// multicast to both CTAs; each CTA drains its own 128 accumulator rows.
constexpr int P_LSTAGES = 4, P_CSTAGES = 3;
constexpr int P_A4 = 128 * 32, P_B4 = 128 * 32, P_SA = 256, P_SB = 256;
constexpr int P_LSTAGE = 9216;                                   // 8,704 bytes used
constexpr int P_HALF16 = 128 * 128;                              // 16 KB: 128 rows of 64 fp16
constexpr int P_CSTAGE = 2 * P_HALF16;
constexpr int P_CONV_OFF = 0;
constexpr int P_LR_OFF = P_CONV_OFF + P_CSTAGES * P_CSTAGE;      // U rows + L2T half, 16 KB each
constexpr int P_LOAD_OFF = P_LR_OFF + 2 * P_HALF16;
constexpr int P_BAR_OFF = P_LOAD_OFF + P_LSTAGES * P_LSTAGE;
constexpr int P_SMEM_BYTES = 1024 + P_BAR_OFF + 256;
static_assert(P_A4 + P_B4 + P_SA + P_SB <= P_LSTAGE, "a pair load slot holds one group");
static_assert(P_SMEM_BYTES <= 227 * 1024, "shared memory");
constexpr bool kPair = true;   // the pair form runs the tcgen05 INT4 GEMM
constexpr uint32_t IDESC_F16_PAIR = (1u << 4) | ((256 >> 3) << 17) | ((256 >> 4) << 24);
constexpr uint32_t IDESC_BF16_PAIR = IDESC_F16_PAIR | (1u << 7) | (1u << 10);

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    int4_gemm_pair_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *load_full = reinterpret_cast<uint64_t *>(smem + P_BAR_OFF);   // local
  uint64_t *load_empty = load_full + P_LSTAGES;                          // local
  uint64_t *conv_full = load_empty + P_LSTAGES;                          // even CTA: both CTAs' converters
  uint64_t *conv_empty = conv_full + P_CSTAGES;                          // both: the multicast commit
  uint64_t *lr_local = conv_empty + P_CSTAGES;                           // local low-rank bytes
  uint64_t *lr_pair = lr_local + 1;                                      // even CTA: both CTAs' low-rank rows
  uint64_t *tmem_full = lr_pair + 1;                                     // both
  uint64_t *drain = tmem_full + 1;                                       // even CTA
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t h = dev::cluster_ctarank();
  const int n0 = blockIdx.y * BN, m0 = static_cast<int>(blockIdx.x) * BM;    // blockIdx.x = 2 * pair + h
  const int nb0 = n0 + 128 * static_cast<int>(h);                            // this CTA's B rows
  const bool a_live = m0 < p.ld_sa;          // the odd CTA of a last, half pair has no rows
  const int G = p.K / 64;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P_LSTAGES; ++s) {
      dev::mbar_init(&load_full[s], 1);
      dev::mbar_init(&load_empty[s], 8);
    }
    for (int c = 0; c < P_CSTAGES; ++c) {
      dev::mbar_init(&conv_full[c], 16);
      dev::mbar_init(&conv_empty[c], 1);
    }
    dev::mbar_init(lr_local, 1);
    dev::mbar_init(lr_pair, 2);
    dev::mbar_init(tmem_full, 1);
    dev::mbar_init(drain, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == 1) {
    dev::tmem_alloc_pair(tmem_slot, TMEM_COLS);
    dev::tmem_relinquish_pair();
  }
  dev::tc_fence_before();
  __syncwarp();
  dev::cluster_sync();                       // both CTAs' barriers exist before anyone arrives remotely
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();
  const uint32_t peer_abort = dev::mapa(dev::smem_u32(const_cast<int *>(abort_flag)), h ^ 1u);
  auto fail_wait = [&]() {
    *abort_flag = 1;
    dev::st_cluster_u32(peer_abort, 1u);
    dev::report(p.status, SVDQ_ERR_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      dev::prefetch_tmap(&maps.a);
      dev::prefetch_tmap(&maps.b);
      if (p.rank > 0) {
        dev::mbar_arrive_expect_tx(lr_local, (a_live ? P_HALF16 : 0) + P_HALF16);
        if (a_live) dev::bulk_load(smem + P_LR_OFF, p.U + static_cast<size_t>(m0) * 128, P_HALF16, lr_local);
        dev::bulk_load(smem + P_LR_OFF + P_HALF16, p.l2t + static_cast<size_t>(nb0) * 128, P_HALF16, lr_local);
      }
      int issued = 0;
      bool lr_sent = p.rank == 0;
      for (int g = 0; g < G; ++g) {
        const int s = g % P_LSTAGES;
        if (!lr_sent && g == P_LSTAGES) {
          // the first ring of loads is in flight: once this CTA's low-rank rows have landed, tell the
          // even CTA, whose MMA thread starts with them (it must not wait for the whole loop, which
          // itself waits on slots that only those MMAs free)
          if (!dev::mbar_wait(lr_local, 0, p.limit_ns, abort_flag)) {
            fail_wait();
            break;
          }
          dev::mbar_arrive_cluster(dev::mapa(dev::smem_u32(lr_pair), 0));
          lr_sent = true;
        }
        if (!dev::mbar_wait(&load_empty[s], ((g / P_LSTAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
          fail_wait();
          break;
        }
        uint8_t *st = smem + P_LOAD_OFF + s * P_LSTAGE;
        // a CTA without rows loads no A codes or scales: its converters use scale 0, so its codes never count
        dev::mbar_arrive_expect_tx(&load_full[s], (a_live ? P_A4 + P_SA : 0) + P_B4 + P_SB);
        if (a_live) dev::tma_load_2d(st, &maps.a, &load_full[s], g * 32, m0);
        dev::tma_load_2d(st + P_A4, &maps.b, &load_full[s], g * 32, nb0);
        if (a_live)
          dev::bulk_load(st + P_A4 + P_B4, p.a_scales + static_cast<size_t>(g) * p.ld_sa + m0, P_SA, &load_full[s]);
        dev::bulk_load(st + P_A4 + P_B4 + P_SA, p.w_scales + static_cast<size_t>(g) * p.N + nb0, P_SB, &load_full[s]);
        ++issued;
      }
      if (!lr_sent && issued == G) {   // G <= P_LSTAGES: the loop never reached the hand-off
        if (dev::mbar_wait(lr_local, 0, p.limit_ns, abort_flag))
          dev::mbar_arrive_cluster(dev::mapa(dev::smem_u32(lr_pair), 0));
        else
          fail_wait();
      }
      for (int g = max(0, issued - P_LSTAGES); g < issued; ++g)
        dev::mbar_wait(&load_full[g % P_LSTAGES], (g / P_LSTAGES) & 1, p.limit_ns, nullptr);
      if (p.rank > 0) dev::mbar_wait(lr_local, 0, p.limit_ns, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (h == 0 && lane == 0) {
      bool ok = true, issued_any = false;
      uint32_t accumulate = 0;
      if (p.rank > 0) {
        if (!dev::mbar_wait_cluster(lr_pair, 0, p.limit_ns, abort_flag)) {
          fail_wait();
          ok = false;
        } else {
          dev::tc_fence_after();
          const uint32_t ua = dev::smem_u32(smem + P_LR_OFF), lb = ua + P_HALF16;
          for (int j = 0; j < p.rank / 16; ++j) {
            dev::umma_bf16_pair(tmem, dev::desc_sw128(ua + 32 * j), dev::desc_sw128(lb + 32 * j), IDESC_BF16_PAIR,
                                accumulate);
            accumulate = 1;
          }
          issued_any = true;
        }
      }
      for (int g = 0; g < G && ok; ++g) {
        const int c = g % P_CSTAGES;
        if (!dev::mbar_wait(&conv_full[c], (g / P_CSTAGES) & 1, p.limit_ns, abort_flag)) {
          fail_wait();
          ok = false;
          break;
        }
        dev::tc_fence_after();
        const uint32_t sa = dev::smem_u32(smem + P_CONV_OFF + c * P_CSTAGE), sb = sa + P_HALF16;
        for (int j = 0; j < 4; ++j) {
          dev::umma_bf16_pair(tmem, dev::desc_sw128(sa + 32 * j), dev::desc_sw128(sb + 32 * j), IDESC_F16_PAIR,
                              accumulate);
          accumulate = 1;
        }
        issued_any = true;
        dev::tc_commit_pair_mc(&conv_empty[c], 0x3);   // both CTAs' slot c is free once these MMAs have read it
      }
      if (ok) dev::tc_commit_pair_mc(tmem_full, 0x3);
      if (issued_any) {
        dev::tc_commit_pair(drain);
        dev::mbar_wait(drain, 0, p.limit_ns, nullptr);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ converters (both CTAs)
    const int ct = (warp - 4) * 32 + lane;           // 0..255
    for (int g = 0; g < G; ++g) {
      const int s = g % P_LSTAGES, c = g % P_CSTAGES;
      if (!dev::mbar_wait_warp(&load_full[s], (g / P_LSTAGES) & 1, p.limit_ns, abort_flag) ||
          !dev::mbar_wait_warp(&conv_empty[c], ((g / P_CSTAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
        fail_wait();
        break;
      }
      const uint8_t *st = smem + P_LOAD_OFF + s * P_LSTAGE;
      const uint16_t *sc = reinterpret_cast<const uint16_t *>(st + P_A4 + P_B4);   // A then B scales
      uint8_t *cv = smem + P_CONV_OFF + c * P_CSTAGE;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        // half-row hr of the 256 rows (A 0..127, B 128..255): 32 codes, k 32 h .. 32 h + 31
        const int hr = ct + 256 * j, row = hr >> 1, hh = hr & 1;
        const uint4 q = *reinterpret_cast<const uint4 *>(st + row * 32 + hh * 16);
        const uint16_t sbits = (row < 128 && !a_live) ? 0 : sc[row];
        const __half s16 = __float2half_rn(__uint_as_float(static_cast<uint32_t>(sbits) << 16));
        const __half2 s2 = __halves2half2(s16, s16);
        const int r = row & 127;
        uint8_t *tile = cv + (row < 128 ? 0 : P_HALF16) + r * 128;
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int chunk = 4 * hh + w;
          *reinterpret_cast<uint4 *>(tile + (((chunk ^ r) & 7) << 4)) = dequant8(words[w], s2);
        }
      }
      dev::fence_proxy_async();                      // the tensor cores read what the threads wrote
      __syncwarp();
      if (lane == 0) {
        dev::mbar_arrive(&load_empty[s]);
        dev::mbar_arrive_remote(dev::mapa(dev::smem_u32(&conv_full[c]), 0));
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    if (dev::mbar_wait_warp(tmem_full, 0, p.limit_ns, abort_flag)) {
      dev::tc_fence_after();
      const int row = 32 * q + lane, grow = m0 + row;
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        dev::tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * cb, v);
        dev::tmem_wait_ld();
        const int c0 = n0 + 32 * cb;
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = c0 + 2 * i;
          float2 y = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          if (p.bias) {
            const uint32_t bb = __ldg(reinterpret_cast<const uint32_t *>(p.bias + c));
            y.x += __uint_as_float(bb << 16);
            y.y += __uint_as_float(bb & 0xFFFF0000u);
          }
          if constexpr (EPI == SVDQ_EPILOGUE_GELU_ERF) {
            const float2 gy = dev::gelu_erf2(y);
            y = make_float2(c >= p.gelu_col_begin ? gy.x : y.x, c + 1 >= p.gelu_col_begin ? gy.y : y.y);
          } else if constexpr (EPI == SVDQ_EPILOGUE_GELU_TANH) {
            y = make_float2(c >= p.gelu_col_begin ? dev::gelu_tanh(y.x) : y.x,
                            c + 1 >= p.gelu_col_begin ? dev::gelu_tanh(y.y) : y.y);
          }
          __nv_bfloat162 h2 = __floats2bfloat162_rn(y.x, y.y);
          packed[i] = *reinterpret_cast<uint32_t *>(&h2);
        }
        if (grow < p.M) {
          uint4 *dst = reinterpret_cast<uint4 *>(p.Y + static_cast<size_t>(grow) * p.ldy + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
    } else {
      fail_wait();
    }
  }
  dev::tc_fence_before();
  __syncwarp();
  dev::cluster_sync();                       // no MMA of the pair still reads either CTA's shared memory
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

template <int EPI>
int launch_pair(const TcMaps &maps, const TcParams &p, cudaStream_t stream) {
  const int rc = smem_optin_once<int4_gemm_pair_kernel<EPI>>(P_SMEM_BYTES, "svdq_linear_int4");
  if (rc != SVDQ_OK) return rc;
  DependentLaunch dl(dim3(2 * ((p.ld_sa + 255) / 256), p.N / BN), dim3(THREADS), P_SMEM_BYTES, stream);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, int4_gemm_pair_kernel<EPI>, maps, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_int4 launch: ") + cudaGetErrorString(e));
  return ok();
}

template <int EPI>
int launch(const TcMaps &maps, const TcParams &p, cudaStream_t stream) {
  const int rc = smem_optin_once<int4_gemm_tc_kernel<EPI>>(SMEM_BYTES, "svdq_linear_int4");
  if (rc != SVDQ_OK) return rc;
  DependentLaunch dl(dim3(p.N / BN, (p.M + BM - 1) / BM), dim3(THREADS), SMEM_BYTES, stream);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, int4_gemm_tc_kernel<EPI>, maps, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_int4 launch: ") + cudaGetErrorString(e));
  return ok();
}

}  // namespace

// The tcgen05 INT4 GEMM (N % 256 == 0); arguments already checked by svdq_linear_int4.
int launch_int4_tc(const uint8_t *a_codes, const void *a_scales, const void *U, const uint8_t *w_codes,
                   const void *w_scales, const void *l2t, const void *bias, int M, int N, int K, int rank, int epilogue,
                   int gelu_col_begin, void *Y, int ldy, unsigned int *status, cudaStream_t stream) {
  TcMaps maps;
  const int mp = (M + BM - 1) / BM * BM;
  int rc = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, static_cast<uint64_t>(K / 2),
                          static_cast<uint64_t>(mp), static_cast<uint64_t>(K / 2), 32, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc != SVDQ_OK) return rc;
  rc = encode_tmap_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, static_cast<uint64_t>(K / 2),
                      static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), 32, kPair ? 128 : BN,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc != SVDQ_OK) return rc;
  TcParams p;
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
  p.ld_sa = mp;
  p.rank = rank;
  p.gelu_col_begin = gelu_col_begin;
  p.status = status;
  p.limit_ns = kWaitLimitNs;
  if (kPair) {
    switch (epilogue) {
      case SVDQ_EPILOGUE_GELU_ERF: return launch_pair<SVDQ_EPILOGUE_GELU_ERF>(maps, p, stream);
      case SVDQ_EPILOGUE_GELU_TANH: return launch_pair<SVDQ_EPILOGUE_GELU_TANH>(maps, p, stream);
      default: return launch_pair<SVDQ_EPILOGUE_NONE>(maps, p, stream);
    }
  }
  switch (epilogue) {
    case SVDQ_EPILOGUE_GELU_ERF: return launch<SVDQ_EPILOGUE_GELU_ERF>(maps, p, stream);
    case SVDQ_EPILOGUE_GELU_TANH: return launch<SVDQ_EPILOGUE_GELU_TANH>(maps, p, stream);
    default: return launch<SVDQ_EPILOGUE_NONE>(maps, p, stream);
  }
}

}  // namespace svdq
