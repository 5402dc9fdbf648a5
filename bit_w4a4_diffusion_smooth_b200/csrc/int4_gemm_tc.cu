// INT4 W4A4 GEMM on the 5th-generation tensor cores (tcgen05), for N a
// multiple of 128 (256-column tiles; a last tile of 128 columns when N % 256
// is 128).
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
// SM pairs, persistent.  A cluster of 2 CTAs (one per SM) computes 256 x 256
// output tiles with cta_group::2 MMAs (M 256, N 256, K 16): CTA h holds rows
// 128h.. of the tile's activations and weight rows (output columns) 128h.. of
// its weights, converts only those (128 + 128 rows per group of 64) and
// serves its half of the weight tile to both SMs' tensor cores.  Each pair
// walks a contiguous run of tiles, m fastest.  TMEM holds two 256-column fp32
// accumulators, so the epilogue of one tile runs while the MMAs of the next
// fill the other.  Roles, 24 warps per CTA:
//   warp 0       producer: per group of 64 along K, TMA copies of the CTA's
//                128 x 32 bytes of activation codes and 128 x 32 bytes of
//                weight codes and bulk copies of their scales, into a ring of
//                4 load slots
//   warp 1       owns TMEM (pair allocation); in the even CTA one thread
//                issues per tile the low-rank MMAs (kind::f16, bf16, straight
//                from the U and L2T tiles, whose layout is the operand image)
//                and then 4 MMAs per group (kind::f16, fp16 operands) from a
//                ring of 4 converted slots, committing each slot back to both
//                CTAs (multicast commit)
//   warp 2       low-rank loader: per tile the CTA's U rows and L2T rows, then
//                tells the even CTA they have landed
//   warps 4..19  converters, 4 teams of 4 warps; team j takes the groups
//                g = j mod 4, so four groups are converted at once: half-
//                precision q * s of the group's 256 rows into the
//                128-byte-swizzled K-major layout (4 half rows of 32 codes per
//                thread), then a CTA-scope arrive on the even CTA's barrier
//                (the hand-off CUTLASS's SM100 mixed-input pipeline makes: no
//                cluster-scope fence per group).  With all 16 warps on one
//                group at a time the conversion was a latency chain per group
//   warps 20..23 epilogue: TMEM -> registers (lane quarter = warp % 4), bias,
//                GELU, bf16 rows to global memory, then the accumulator is
//                handed back to the even CTA
// Inside every 8-element chunk both operands hold k in the same permuted order
// (k, k+4 pairs, so one mask-and-or makes a pair), which leaves the products'
// sum unchanged.  Every wait is bounded: a wait that runs out records
// SVDQ_ERR_TIMEOUT, raises both CTAs' abort flags and every role leaves for
// the final cluster barrier, after which TMEM is freed once the tensor cores
// are idle.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int BN = 256;                                          // output columns per pair tile
constexpr int LSTAGES = 4, CSTAGES = 4;
constexpr int NCONV = 16;                                        // converter warps per CTA
constexpr int TEAMS = 4;                                         // teams of converters take groups in turn
constexpr int TEAM_WARPS = NCONV / TEAMS;
constexpr int CONV_WARP0 = 4, EPI_WARP0 = CONV_WARP0 + NCONV;
constexpr int THREADS = (EPI_WARP0 + 4) * 32;
constexpr int HALF_ROWS = 512;                                   // 256 rows x 2 halves of 32 codes per group
constexpr int HR_PER_THREAD = HALF_ROWS / (TEAM_WARPS * 32);
constexpr int A4 = 128 * 32, B4 = 128 * 32, SA = 256, SB = 256;  // one group: codes and scales of 128 + 128 rows
constexpr int LSTAGE = 9216;                                     // 8,704 bytes used
constexpr int HALF16 = 128 * 128;                                // 16 KB: 128 rows of 64 fp16 (or bf16)
constexpr int CSTAGE = 2 * HALF16;                               // A rows, then B rows
constexpr int CONV_OFF = 0;
constexpr int LR_OFF = CONV_OFF + CSTAGES * CSTAGE;              // U rows, then L2T rows
constexpr int LOAD_OFF = LR_OFF + 2 * HALF16;
constexpr int BAR_OFF = LOAD_OFF + LSTAGES * LSTAGE;
constexpr int SMEM_BYTES = 1024 + BAR_OFF + 256;
constexpr uint32_t TMEM_COLS = 512;                              // two 256-column accumulators
static_assert(A4 + B4 + SA + SB <= LSTAGE, "a load slot holds one group");
static_assert(HALF_ROWS % (TEAM_WARPS * 32) == 0 && NCONV % TEAMS == 0, "a team splits the half rows evenly");
static_assert(LSTAGES % TEAMS == 0, "a load slot always serves the same team");
// A team that reaches group g finished g - TEAMS, which needs only the MMAs up to
// g - TEAMS - CSTAGES; the slot of g must then be at most one phase behind the
// one the team waits for (an mbarrier parity wait cannot tell phases two apart).
static_assert(TEAMS <= CSTAGES, "no converter team runs two phases ahead of a slot");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
// instruction descriptors: f32 accumulate (bit 4), A/B fp16 (0) or bf16 (1) at bits 7 and 10,
// N >> 3 at bit 17, M >> 4 at bit 24 (M 256: the pair), both operands K-major
constexpr uint32_t IDESC_F16 = (1u << 4) | ((256 >> 3) << 17) | ((256 >> 4) << 24);
constexpr uint32_t IDESC_BF16 = IDESC_F16 | (1u << 7) | (1u << 10);
// a last tile of 128 columns (N % 256 == 128): N 128, each CTA serving 64 weight rows
constexpr uint32_t IDESC_F16_HALF = (1u << 4) | ((128 >> 3) << 17) | ((256 >> 4) << 24);
constexpr uint32_t IDESC_BF16_HALF = IDESC_F16_HALF | (1u << 7) | (1u << 10);

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
// permuted k order (i, i + 4): pair i = (q_i s, q_{i+4} s), exact.  One
// mask-and-xor per pair puts the offset-binary code u = q + 8 (the nibble with
// its top bit flipped) into an fp16 mantissa: at bits 0..3 under the exponent
// of 1024 (value 1024 + u), at bits 4..7 under the exponent of 64 (whose
// mantissa bit 4 weighs 1: value 64 + u), so one shift by 8 serves the four
// pairs; subtracting 1032 or 72 gives q exactly, and the multiply q s.
__device__ __forceinline__ uint4 dequant8(uint32_t x, __half2 s2) {
  const __half2 b1024 = __floats2half2_rn(1032.0f, 1032.0f), b64 = __floats2half2_rn(72.0f, 72.0f);
  const uint32_t y = x >> 8;
  uint32_t t[4];
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[0]) : "r"(x), "r"(0x000F000Fu), "r"(0x64086408u));
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[1]) : "r"(x), "r"(0x00F000F0u), "r"(0x54805480u));
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[2]) : "r"(y), "r"(0x000F000Fu), "r"(0x64086408u));
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t[3]) : "r"(y), "r"(0x00F000F0u), "r"(0x54805480u));
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 q = __hsub2(*reinterpret_cast<__half2 *>(&t[i]), (i & 1) ? b64 : b1024);   // q, exact
    const __half2 v = __hmul2(q, s2);                                                       // q s, exact
    o[i] = *reinterpret_cast<const uint32_t *>(&v);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Pair tile t: its 256-row block of activations (m fastest) and 256-column block of weights; a
// last block of 128 columns (N % 256 == 128) is a half tile, whose CTAs serve 64 weight rows each.
struct PairTile {
  int m2, nt;
  bool half;
};
__device__ __forceinline__ PairTile pair_tile(int t, int tiles_m, int N) {
  const int nt = t / tiles_m;
  return PairTile{t % tiles_m, nt, (nt + 1) * BN > N};
}
// this CTA's first weight row of the tile
__device__ __forceinline__ int weight_row0(const PairTile &pt, uint32_t h) {
  return pt.nt * BN + (pt.half ? 64 : 128) * static_cast<int>(h);
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    int4_gemm_tc_kernel(const __grid_constant__ TcMaps maps, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *load_full = reinterpret_cast<uint64_t *>(smem + BAR_OFF);   // local: producer -> converters
  uint64_t *load_empty = load_full + LSTAGES;                          // local: converters -> producer
  uint64_t *conv_full = load_empty + LSTAGES;                          // even CTA: both CTAs' converters
  uint64_t *conv_empty = conv_full + CSTAGES;                          // both: the multicast commit
  uint64_t *lr_local = conv_empty + CSTAGES;                           // local low-rank bytes
  uint64_t *lr_pair = lr_local + 1;                                    // even CTA: both CTAs' low-rank rows
  uint64_t *lr_empty = lr_pair + 1;                                    // both: the low-rank MMAs are done
  uint64_t *tmem_full = lr_empty + 1;                                  // both, per accumulator
  uint64_t *tmem_empty = tmem_full + 2;                                // even CTA, per accumulator
  uint64_t *drain = tmem_empty + 2;                                    // even CTA
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t h = dev::cluster_ctarank();
  const int G = p.K / 64;
  const int tiles_m = (p.ld_sa + 255) / 256;
  const int total = tiles_m * ((p.N + BN - 1) / BN);
  const int pair = static_cast<int>(dev::cluster_id_x()), num_pairs = static_cast<int>(dev::num_clusters_x());
  const int t_begin = static_cast<int>((static_cast<long long>(pair) * total) / num_pairs);
  const int t_end = static_cast<int>((static_cast<long long>(pair + 1) * total) / num_pairs);
  if (threadIdx.x == 0) {
    for (int s = 0; s < LSTAGES; ++s) {
      dev::mbar_init(&load_full[s], 1);
      dev::mbar_init(&load_empty[s], TEAM_WARPS);
    }
    for (int c = 0; c < CSTAGES; ++c) {
      dev::mbar_init(&conv_full[c], 2 * TEAM_WARPS);
      dev::mbar_init(&conv_empty[c], 1);
    }
    dev::mbar_init(lr_local, 1);
    dev::mbar_init(lr_pair, 2);
    dev::mbar_init(lr_empty, 1);
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(&tmem_full[b], 1);
      dev::mbar_init(&tmem_empty[b], 2 * 4);
    }
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
      int gi = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const PairTile pt = pair_tile(t, tiles_m, p.N);
        const int m0 = (2 * pt.m2 + static_cast<int>(h)) * 128, nb0 = weight_row0(pt, h);
        const bool a_live = m0 < p.ld_sa;    // the odd CTA of a last, half pair has no rows
        // weight rows past N read as zeros (the tensor map's bounds); their scales are not copied
        const int sb_bytes = pt.half ? SB / 2 : SB;
        for (int g = 0; g < G; ++g, ++gi) {
          const int s = gi % LSTAGES;
          if (!dev::mbar_wait(&load_empty[s], ((gi / LSTAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
            fail_wait();
            ok = false;
            break;
          }
          uint8_t *st = smem + LOAD_OFF + s * LSTAGE;
          // a CTA without rows loads no activation codes or scales: its converters use scale 0
          dev::mbar_arrive_expect_tx(&load_full[s], (a_live ? A4 + SA : 0) + B4 + sb_bytes);
          if (a_live) {
            dev::tma_load_2d(st, &maps.a, &load_full[s], g * 32, m0);
            dev::bulk_load(st + A4 + B4, p.a_scales + static_cast<size_t>(g) * p.ld_sa + m0, SA, &load_full[s]);
          }
          dev::tma_load_2d(st + A4, &maps.b, &load_full[s], g * 32, nb0);
          dev::bulk_load(st + A4 + B4 + SA, p.w_scales + static_cast<size_t>(g) * p.N + nb0, sb_bytes, &load_full[s]);
        }
      }
      // every copy issued lands before the block leaves
      for (int j = max(0, gi - LSTAGES); j < gi; ++j)
        dev::mbar_wait(&load_full[j % LSTAGES], (j / LSTAGES) & 1, p.limit_ns, nullptr);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ low-rank loader (both CTAs)
    if (lane == 0 && p.rank > 0) {
      int lt = 0;
      for (int t = t_begin; t < t_end; ++t, ++lt) {
        const PairTile pt = pair_tile(t, tiles_m, p.N);
        const int m0 = (2 * pt.m2 + static_cast<int>(h)) * 128, nb0 = weight_row0(pt, h);
        const bool a_live = m0 < p.ld_sa;
        if (!dev::mbar_wait(lr_empty, (lt & 1) ^ 1, p.limit_ns, abort_flag)) {
          fail_wait();
          break;
        }
        dev::mbar_arrive_expect_tx(lr_local, (a_live ? HALF16 : 0) + HALF16);
        if (a_live) dev::bulk_load(smem + LR_OFF, p.U + static_cast<size_t>(m0) * 128, HALF16, lr_local);
        dev::bulk_load(smem + LR_OFF + HALF16, p.l2t + static_cast<size_t>(nb0) * 128, HALF16, lr_local);
        if (!dev::mbar_wait(lr_local, lt & 1, p.limit_ns, abort_flag)) {
          fail_wait();
          dev::mbar_wait(lr_local, lt & 1, p.limit_ns, nullptr);   // the copies land before the block leaves
          break;
        }
        dev::mbar_arrive_cluster(dev::mapa(dev::smem_u32(lr_pair), 0));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (h == 0 && lane == 0) {
      bool ok = true, issued_any = false;
      int gi = 0, lt = 0;
      for (int t = t_begin; t < t_end && ok; ++t, ++lt) {
        const int b = lt & 1;
        const bool half = pair_tile(t, tiles_m, p.N).half;
        const uint32_t idesc_bf16 = half ? IDESC_BF16_HALF : IDESC_BF16, idesc_f16 = half ? IDESC_F16_HALF : IDESC_F16;
        if (!dev::mbar_wait_cluster(&tmem_empty[b], ((lt >> 1) & 1) ^ 1, p.limit_ns, abort_flag)) {
          fail_wait();
          break;
        }
        dev::tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(BN * b);
        uint32_t accumulate = 0;
        if (p.rank > 0) {
          if (!dev::mbar_wait_cluster(lr_pair, lt & 1, p.limit_ns, abort_flag)) {
            fail_wait();
            break;
          }
          dev::tc_fence_after();
          const uint32_t ua = dev::smem_u32(smem + LR_OFF), lb = ua + HALF16;
          for (int j = 0; j < p.rank / 16; ++j) {   // K = 16 bf16 = 32 bytes per MMA
            dev::umma_bf16_pair(acc, dev::desc_sw128(ua + 32 * j), dev::desc_sw128(lb + 32 * j), idesc_bf16,
                                accumulate);
            accumulate = 1;
          }
          issued_any = true;
          dev::tc_commit_pair_mc(lr_empty, 0x3);   // both CTAs may reload their low-rank rows
        }
        for (int g = 0; g < G; ++g, ++gi) {
          const int c = gi % CSTAGES;
          if (!dev::mbar_wait(&conv_full[c], (gi / CSTAGES) & 1, p.limit_ns, abort_flag)) {
            fail_wait();
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t sa = dev::smem_u32(smem + CONV_OFF + c * CSTAGE), sb = sa + HALF16;
          for (int j = 0; j < 4; ++j) {               // K = 16 fp16 = 32 bytes per MMA
            dev::umma_bf16_pair(acc, dev::desc_sw128(sa + 32 * j), dev::desc_sw128(sb + 32 * j), idesc_f16,
                                accumulate);
            accumulate = 1;
          }
          issued_any = true;
          dev::tc_commit_pair_mc(&conv_empty[c], 0x3);   // both CTAs' slot c is free once these MMAs have read it
        }
        if (ok) dev::tc_commit_pair_mc(&tmem_full[b], 0x3);
      }
      if (issued_any) {   // the tensor cores are idle before TMEM is freed
        dev::tc_commit_pair(drain);
        dev::mbar_wait(drain, 0, p.limit_ns, nullptr);
      }
    }
  } else if (warp >= CONV_WARP0 && warp < EPI_WARP0) {
    // ------------------------------------------------------------ converters (both CTAs)
    const int team = (warp - CONV_WARP0) / TEAM_WARPS;
    const int ct = ((warp - CONV_WARP0) % TEAM_WARPS) * 32 + lane;
    int gi = 0;
    bool ok = true;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const PairTile pt = pair_tile(t, tiles_m, p.N);
      const bool a_live = (2 * pt.m2 + static_cast<int>(h)) * 128 < p.ld_sa;
      for (int g = 0; g < G; ++g, ++gi) {
        if (gi % TEAMS != team) continue;            // the other teams' groups
        const int s = gi % LSTAGES, c = gi % CSTAGES;
        if (!dev::mbar_wait_warp(&load_full[s], (gi / LSTAGES) & 1, p.limit_ns, abort_flag) ||
            !dev::mbar_wait_warp(&conv_empty[c], ((gi / CSTAGES) & 1) ^ 1, p.limit_ns, abort_flag)) {
          fail_wait();
          ok = false;
          break;
        }
        const uint8_t *st = smem + LOAD_OFF + s * LSTAGE;
        const uint16_t *sc = reinterpret_cast<const uint16_t *>(st + A4 + B4);   // activation, then weight scales
        uint8_t *cv = smem + CONV_OFF + c * CSTAGE;
#pragma unroll
        for (int j = 0; j < HR_PER_THREAD; ++j) {
          // half row hr of the 256 rows (activations 0..127, weights 128..255): 32 codes, k 32 hh .. 32 hh + 31
          const int hr = ct + TEAM_WARPS * 32 * j, row = hr >> 1, hh = hr & 1;
          const uint4 q = *reinterpret_cast<const uint4 *>(st + row * 32 + hh * 16);
          const uint16_t sbits = (row < 128 && !a_live) ? 0 : sc[row];
          const __half s16 = __float2half_rn(__uint_as_float(static_cast<uint32_t>(sbits) << 16));
          const __half2 s2 = __halves2half2(s16, s16);
          const int r = row & 127;
          uint8_t *tile = cv + (row < 128 ? 0 : HALF16) + r * 128;
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
    }
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    int lt = 0;
    for (int t = t_begin; t < t_end; ++t, ++lt) {
      const PairTile pt = pair_tile(t, tiles_m, p.N);
      const int b = lt & 1;
      if (!dev::mbar_wait_warp(&tmem_full[b], (lt >> 1) & 1, p.limit_ns, abort_flag)) {
        fail_wait();
        break;
      }
      dev::tc_fence_after();
      const int m0 = (2 * pt.m2 + static_cast<int>(h)) * 128, n0 = pt.nt * BN;
      const int row = 32 * q + lane, grow = m0 + row;
      const int nchunk = pt.half ? BN / 64 : BN / 32;   // 32-column chunks of the tile
#pragma unroll 1
      for (int cb = 0; cb < nchunk; ++cb) {
        uint32_t v[32];
        dev::tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(BN * b + 32 * cb),
                                v);
        dev::tmem_wait_ld();
        if (cb == nchunk - 1) {                        // the accumulator is read: hand it back to the MMA thread
          dev::tc_fence_before();
          __syncwarp();
          if (lane == 0) dev::mbar_arrive_cluster(dev::mapa(dev::smem_u32(&tmem_empty[b]), 0));
        }
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

// Per device and epilogue kind, once: the shared-memory opt-in and the number
// of SM pairs that can hold one CTA each at that size.
template <int EPI>
int prepare_device(int *pairs_out) {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev_id = 0;
  if (cudaGetDevice(&dev_id) != cudaSuccess || dev_id < 0 || dev_id >= 64) {
    cudaGetLastError();
    return fail(SVDQ_ERR_CUDA, "svdq_linear_int4: no current device");
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev_id] == 0) {
    cudaError_t e =
        cudaFuncSetAttribute(int4_gemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_int4: ") + cudaGetErrorString(e));
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_id) != cudaSuccess || sms < 2) sms = 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, int4_gemm_tc_kernel<EPI>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = sms / 2;
    }
    cached[dev_id] = n;
  }
  *pairs_out = cached[dev_id];
  return SVDQ_OK;
}

template <int EPI>
int launch(const TcMaps &maps, const TcParams &p, cudaStream_t stream) {
  int resident = 0;
  const int rc = prepare_device<EPI>(&resident);
  if (rc != SVDQ_OK) return rc;
  const int tiles = (p.ld_sa + 255) / 256 * ((p.N + BN - 1) / BN);
  const int pairs = tiles < resident ? tiles : resident;
  DependentLaunch dl(dim3(2 * pairs), dim3(THREADS), SMEM_BYTES, stream);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, int4_gemm_tc_kernel<EPI>, maps, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("svdq_linear_int4 launch: ") + cudaGetErrorString(e));
  return ok();
}

}  // namespace

// The tcgen05 INT4 GEMM (N % 128 == 0); arguments already checked by svdq_linear_int4.
int launch_int4_tc(const uint8_t *a_codes, const void *a_scales, const void *U, const uint8_t *w_codes,
                   const void *w_scales, const void *l2t, const void *bias, int M, int N, int K, int rank, int epilogue,
                   int gelu_col_begin, void *Y, int ldy, unsigned int *status, cudaStream_t stream) {
  TcMaps maps;
  const int mp = (M + 127) / 128 * 128;
  int rc = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, static_cast<uint64_t>(K / 2),
                          static_cast<uint64_t>(mp), static_cast<uint64_t>(K / 2), 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc != SVDQ_OK) return rc;
  rc = encode_tmap_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, static_cast<uint64_t>(K / 2),
                      static_cast<uint64_t>(N), static_cast<uint64_t>(K / 2), 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
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
  switch (epilogue) {
    case SVDQ_EPILOGUE_GELU_ERF: return launch<SVDQ_EPILOGUE_GELU_ERF>(maps, p, stream);
    case SVDQ_EPILOGUE_GELU_TANH: return launch<SVDQ_EPILOGUE_GELU_TANH>(maps, p, stream);
    default: return launch<SVDQ_EPILOGUE_NONE>(maps, p, stream);
  }
}

}  // namespace svdq
