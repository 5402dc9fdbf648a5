// K2: W4A4 GEMM with the low-rank up-projection fused in.
//
// The pages fuse the 16-bit low-rank up-projection into the 4-bit GEMM so the
// correction branch does not eat the W4A4 gain (web page "Nunchaku Diffusers
// 支持降低显存占用，但硬件仍决定适用范围", remio.ai, section "SVDQuant 将棘手数值移出
// 4 位路径").  Per 256 x 256 output tile:
//   acc  = U_tile . L2T_tile^T                 tcgen05.mma kind::f16 (bf16)
//   acc += sum_k (qa sa)(qw sw)                tcgen05.mma kind::mxf4nvf4,
//                                               block16 ue4m3 scales in TMEM
//   Y    = bf16( epilogue( s_a s_w acc + bias ) )
// U arrives pre-divided by s_a s_w, so both branches share one fp32
// accumulator and one scale in the epilogue.
//
// SM pairs.  The kernel runs in clusters of two CTAs, one per SM of a TPC,
// and every MMA is a cta_group::2 MMA of 256 x 256 x 64: CTA h of the pair
// holds rows 128h..128h+127 of the activation tile and weight rows (output
// columns) 128h..128h+127 of the weight tile, and its TMEM receives its own
// 128 rows of the accumulator.  Each SM therefore loads its half of A and
// of B per k-stage (32 KB of codes) plus the scales: its 128 rows of A
// scales and the B scales of all 256 weight rows that both TMEMs need.
//
// Roles (one CTA per SM, persistent over pair tiles, 12 warps):
//   warp 0      producer in both CTAs: per stage four TMA copies into its
//               own shared memory - the A and B scales first, completing on
//               the even CTA's `sf_loaded` barrier, then the A and B code
//               halves, completing on its `full` barrier
//   warp 1      owns TMEM (pair allocation); in the even CTA it issues the
//               MMAs from one thread and commits each stage to both CTAs'
//               `empty` barriers
//   warp 2      even CTA: moves each stage's block scales from both CTAs'
//               shared memory into their TMEM (tcgen05.cp, cta_group::2) as
//               soon as `sf_loaded` completes; from its own warp the copies
//               overlap the MMAs and the codes' transfer
//   warps 4..11 epilogue in both CTAs: drain the CTA's 128 x 256 fp32
//               accumulator, hand TMEM back (to the even CTA's barrier),
//               then scale, add bias, GELU, round to bf16 into a
//               64-byte-swizzled 32 x 32 staging tile and write it with TMA
//               stores
// Pipeline: 4 stages of 50 KB per CTA; TMEM holds the accumulator (256
// columns) and 4 x 48 columns of block scales.
// This header holds the kernel template; gemm_w4a4.cu instantiates the plain
// GEMM and its entry point, gemm_w4a4_requant.cu the re-quantizing variant.  A pair walks a contiguous
// run of tiles, n fastest (one row block's A tiles stay hot in L2 while its
// output columns are swept).
// Measured limit: every tcgen05.cp of block scales takes ~115 cycles of the
// SM's copy engine whatever its size (a 512-byte 32x128b.warpx4 atom or a
// 4 KB 128x256b block alike).  The weight bundle therefore stores each B-scale
// atom four times over, the image of its warpx4 copy, so one 128x256b copy
// moves a k-block's scales for all 256 weight rows: a k-stage needs 8 copies
// (A: 1, B: 1 per k-block) instead of 12, against 4 MMAs of ~128 cycles.
// Every wait is bounded; a wait that runs out records SVDQ_ERR_TIMEOUT and
// raises the abort flag of both CTAs; in-flight work is drained, the pair
// meets at a cluster barrier and frees TMEM.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace w4a4 {

constexpr int BM = 128;                       // rows per CTA (256 per pair)
constexpr int BN = 256;                       // output columns per pair tile
constexpr int STAGES = 4;
constexpr int ROW = 2048;                     // bytes per row of the bundle tensor maps
constexpr int A_BYTES = BM * 144;             // activation tile: codes 16 KB + scales 2 KB
constexpr int SFA_OFF = BM * 128;
constexpr int A_CODE_BYTES = BM * 128;
constexpr int SFA_BYTES = BM * 16;
constexpr int B_OFF = A_BYTES;                // 18432, a multiple of 1024
constexpr int B_BYTES = 128 * 128;            // this CTA's 128 weight rows of codes
constexpr int SFB_OFF = B_OFF + B_BYTES;      // scales of all 256 weight rows, each atom 4 times
constexpr int SFB_BYTES = 4 * 4096;           // per k-block: [rows 0-127: 4 x 512 B][rows 128-255: 4 x 512 B]
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFB_BYTES;  // 51200
constexpr int LR_BYTES = 128 * 128;           // U (this CTA's rows) and L2T (its columns), 16 KB each
constexpr int EPI_WARPS = 8;
constexpr int EPI_TILE_BYTES = 32 * 64;       // 32 rows x 32 bf16, 64-byte swizzle
constexpr int EPI_OFF = STAGES * STAGE_BYTES;
constexpr int TAB_OFF = EPI_OFF + EPI_WARPS * EPI_TILE_BYTES;   // 128 floats: 1 / block scale, next layer
constexpr int BAR_OFF = TAB_OFF + 128 * 4;
constexpr int SMEM_BYTES = 1024 + BAR_OFF + 256;
constexpr int THREADS = (4 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL = 256;              // stage s: SFA at +48s (+4 kb), SFB at +48s+16 (+8 kb, +4 per row block)
static_assert(STAGE_BYTES % 1024 == 0 && B_OFF % 1024 == 0, "MMA operand tiles start on 1024-byte boundaries");
static_assert(A_CODE_BYTES % ROW == 0 && SFA_BYTES % ROW == 0 && B_BYTES % ROW == 0 && SFB_BYTES % ROW == 0 &&
                  LR_BYTES % ROW == 0,
              "copies are whole tensor-map rows");
static_assert(SF_COL + 48 * STAGES <= TMEM_COLS, "scale columns fit in TMEM");

// Instruction descriptors (tcgen05 instruction-descriptor bit fields):
// [4,6) accumulator format (1 = f32), [7,10) A format, [10,13) B format,
// [17,23) N >> 3, [24,29) M >> 4 (M = 256: the pair); block-scaled: [23]
// scale format (0 = ue4m3), scale-factor ids 0; A/B K-major (bits 15/16 = 0).
constexpr uint32_t IDESC_BF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((256 >> 4) << 24);
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((256 >> 4) << 24);

__device__ __forceinline__ uint32_t sfa_col(int s, int kb) { return SF_COL + 48 * s + 4 * kb; }
__device__ __forceinline__ uint32_t sfb_col(int s, int kb) { return SF_COL + 48 * s + 16 + 8 * kb; }

struct Params {
  int M, N, rank, epilogue, gelu_col_begin;
  int num_m2, num_n, num_tiles, k_stages, lr_stages, kb_total;
  const float *s_a, *s_w;
  const uint16_t *bias;
  unsigned int *status;
  unsigned long long limit_ns;
  int store_y;                  // 0: the bf16 output is not written (re-quantizing variant only)
  // Re-quantizing variant: the next layer, whose input is this layer's output (K_next = N).
  const float *nx_inv;          // [N] inv_lambda of the next layer
  const uint16_t *nx_l1t;       // [RQ][N] bf16: the next layer's L1^T
  const float *nx_s_a, *nx_s_w; // the next layer's tensor scales (device scalars)
  uint8_t *nx_bundle;           // the next layer's 128-row activation bundle
  float *nx_acc;                // [M][RQ] fp32 partial sums of the next layer's X^ . L1, zero at launch
  int nx_ks;                    // k-stages of the next bundle: ceil(N / 256)
};

struct Maps {
  CUtensorMap a, sfa, b, sfb, u, l2, y;
};

// One launch computes up to G independent GEMMs of the same epilogue kind
// (a grouped launch): their tiles form one sequence, problem after problem,
// which the persistent SM pairs split into contiguous runs.  A single GEMM is
// a group of one, compiled with G = 1 so that it carries no group lookup and
// the small parameter block of one problem.
constexpr int kMaxGroup = SVDQ_MAX_GROUP;
template <int G>
struct Group {
  Maps maps[G];
  Params p[G];
  int tile_end[G];              // prefix sums of the problems' tile counts
  int count;
  int total_tiles;
  unsigned int *status;
  unsigned long long limit_ns;
};

// Problem `pi` of tile `tile` of the group's sequence, and the tile's index inside it.
struct TileRef {
  int pi, m2, n_blk;            // problem, 256-row pair block, 256-column block
};
template <int G>
__device__ __forceinline__ TileRef locate_tile(const Group<G> &g, int tile) {
  int pi = 0;
  if constexpr (G > 1)
    while (pi + 1 < g.count && tile >= g.tile_end[pi]) ++pi;
  const int lt = tile - (pi > 0 ? g.tile_end[pi - 1] : 0);
  return TileRef{pi, lt / g.p[pi].num_n, lt % g.p[pi].num_n};
}


// Raises the abort flag of this CTA and of its partner, records the timeout.
__device__ __forceinline__ void abort_pair(volatile int *abort_flag, uint32_t peer_abort, unsigned int *status) {
  *abort_flag = 1;
  dev::st_cluster_u32(peer_abort, 1u);
  dev::report(status, SVDQ_ERR_TIMEOUT);
}

// EPI: the epilogue (SVDQ_EPILOGUE_*), a template parameter so that each
// instantiation holds only its own, fully unrolled epilogue: with both GELU
// forms behind runtime branches the kernel's code outgrew the instruction
// cache and every role stalled on instruction fetch.
//
// RQ: -1 for the plain GEMM; otherwise the re-quantizing variant, RQ being
// the next layer's rank (0..64).  That variant's epilogue turns the layer's
// output into the next layer's input operands instead of (or as well as)
// writing it: the pages fuse the input quantization with the low-rank
// down-projection, and a linear whose output feeds the next SVDQ linear (MLP
// fc1 -> fc2) can take that fusion one step further, so its bf16 output
// never travels through memory.  Per output element, in the next layer's own
// f32 steps: x^ = f32(bf16(y) * inv_lambda_next[n]); per 16 columns the
// ue4m3 block scale and the e2m1 codes, written straight into the next
// layer's 128-row bundle (the CTA's 128 x 256 tile is exactly one tile of it);
// and bf16(x^) . L1_next over the tile's 256 columns on mma.sync, added into
// an fp32 [M][RQ] buffer with vector atomics (a separate kernel turns the
// sums into the next layer's U once every column block is done).
template <int EPI, int RQ, int G>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_w4a4_kernel(const __grid_constant__ Group<G> grp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + BAR_OFF);  // even CTA: both CTAs' bytes
  uint64_t *sf_full = full + STAGES;                               // even CTA: scales in TMEM
  uint64_t *empty = sf_full + STAGES;                              // both CTAs: stage free again
  uint64_t *tmem_full = empty + STAGES;                            // both CTAs: accumulator ready
  uint64_t *tmem_empty = tmem_full + 1;                            // even CTA: both CTAs drained it
  uint64_t *drain_mma = tmem_empty + 1;
  uint64_t *drain_cp = drain_mma + 1;
  uint64_t *sf_loaded = drain_cp + 1;                              // even CTA: both CTAs' scale bytes
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(sf_loaded + STAGES);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t h = dev::cluster_ctarank();         // 0: even CTA (issues the MMAs), 1: odd
  const int pair = static_cast<int>(dev::cluster_id_x());
  const int num_pairs = static_cast<int>(dev::num_clusters_x());
  // this pair's tiles: a contiguous run of tile ids, n fastest
  const int t_begin = static_cast<int>((static_cast<long long>(pair) * grp.total_tiles) / num_pairs);
  const int t_end = static_cast<int>((static_cast<long long>(pair + 1) * grp.total_tiles) / num_pairs);
  const unsigned long long limit_ns = grp.limit_ns;
  unsigned int *const status = grp.status;
  const uint32_t peer_abort = dev::mapa(dev::smem_u32(const_cast<int *>(abort_flag)), h ^ 1u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      dev::mbar_init(&full[s], 1);            // the even CTA's producer arrival (+ the bytes of both CTAs)
      dev::mbar_init(&sf_full[s], 1);
      dev::mbar_init(&empty[s], 1);
      dev::mbar_init(&sf_loaded[s], 1);
    }
    dev::mbar_init(tmem_full, 1);
    dev::mbar_init(tmem_empty, 2 * EPI_WARPS);
    dev::mbar_init(drain_mma, 1);
    dev::mbar_init(drain_cp, 1);
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  if (warp == 1) {
    dev::tmem_alloc_pair(tmem_base_slot, TMEM_COLS);
    dev::tmem_relinquish_pair();
  }
  dev::tc_fence_before();
  __syncwarp();
  dev::cluster_sync();                        // both CTAs' barriers exist before anyone arrives remotely
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  dev::grid_dependency_wait();                // the operands written by the previous kernel are visible
  dev::grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      for (int q = 0; q < grp.count; ++q) {
        dev::prefetch_tmap(&grp.maps[q].a);
        dev::prefetch_tmap(&grp.maps[q].sfa);
        dev::prefetch_tmap(&grp.maps[q].b);
        dev::prefetch_tmap(&grp.maps[q].sfb);
        if (grp.p[q].lr_stages) {
          dev::prefetch_tmap(&grp.maps[q].u);
          dev::prefetch_tmap(&grp.maps[q].l2);
        }
      }
      int it = 0;
      bool ok = true;
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        const TileRef tr = locate_tile(grp, tile);
        const Params &p = grp.p[tr.pi];
        const Maps &maps = grp.maps[tr.pi];
        const int stages_per_tile = p.lr_stages + p.k_stages;
        const int m_blk = 2 * tr.m2 + static_cast<int>(h);  // this CTA's 128-row block
        const int n_blk = tr.n_blk;
        for (int st = 0; st < stages_per_tile; ++st, ++it) {
          const int s = it % STAGES;
          if (!dev::mbar_wait_cluster(&empty[s], ((it / STAGES) & 1) ^ 1, limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = dev::mapa(dev::smem_u32(&full[s]), 0);
          uint8_t *dst = smem + s * STAGE_BYTES;
          if (st < p.lr_stages) {
            if (h == 0) {
              dev::mbar_arrive(&sf_loaded[s]);    // no scales in the low-rank stage
              dev::mbar_arrive_expect_tx(&full[s], 2u * 2u * LR_BYTES);
            }
            dev::tma_load_2d_pair(dst, &maps.u, bar, 0, m_blk * (LR_BYTES / ROW));
            dev::tma_load_2d_pair(dst + B_OFF, &maps.l2, bar, 0, (2 * n_blk + static_cast<int>(h)) * (LR_BYTES / ROW));
          } else {
            const int ks = st - p.lr_stages;
            const int wrow = (n_blk * p.k_stages + ks) * ((2 * B_BYTES + SFB_BYTES) / ROW);
            const int arow = (m_blk * p.k_stages + ks) * (A_BYTES / ROW);
            const uint32_t sbar = dev::mapa(dev::smem_u32(&sf_loaded[s]), 0);
            if (h == 0) {
              dev::mbar_arrive_expect_tx(&sf_loaded[s], 2u * (SFA_BYTES + SFB_BYTES));
              dev::mbar_arrive_expect_tx(&full[s], 2u * (A_CODE_BYTES + B_BYTES));
            }
            // the scales first, on their own barrier: their copies into TMEM
            // then overlap the transfer of the codes
            dev::tma_load_2d_pair(dst + SFA_OFF, &maps.sfa, sbar, 0, arow + SFA_OFF / ROW);
            dev::tma_load_2d_pair(dst + SFB_OFF, &maps.sfb, sbar, 0, wrow + 2 * B_BYTES / ROW);
            dev::tma_load_2d_pair(dst, &maps.a, bar, 0, arow);
            dev::tma_load_2d_pair(dst + B_OFF, &maps.b, bar, 0, wrow + static_cast<int>(h) * (B_BYTES / ROW));
          }
        }
      }
      if (!ok) abort_pair(abort_flag, peer_abort, status);
      // Before the pair may leave: the even CTA waits for every stage it
      // armed to complete (that covers the odd CTA's copies as well).
      if (h == 0) {
        for (int j = max(0, it - STAGES); j < it; ++j) {
          dev::mbar_wait_cluster(&full[j % STAGES], (j / STAGES) & 1, limit_ns, nullptr);
          dev::mbar_wait_cluster(&sf_loaded[j % STAGES], (j / STAGES) & 1, limit_ns, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (h == 0 && lane == 0) {
      int it = 0, tcount = 0;
      bool ok = true, issued_any = false;
      for (int tile = t_begin; tile < t_end && ok; ++tile, ++tcount) {
        const Params &p = grp.p[locate_tile(grp, tile).pi];
        const int stages_per_tile = p.lr_stages + p.k_stages;
        if (!dev::mbar_wait_cluster(tmem_empty, (tcount & 1) ^ 1, limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        dev::tc_fence_after();
        uint32_t accumulate = 0;
        for (int st = 0; st < stages_per_tile; ++st, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!dev::mbar_wait(&sf_full[s], ph, limit_ns, abort_flag) ||
              !dev::mbar_wait_cluster(&full[s], ph, limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          dev::tc_fence_after();
          const uint32_t sa = dev::smem_u32(smem + s * STAGE_BYTES);
          const uint32_t sb = sa + B_OFF;
          if (st < p.lr_stages) {
            for (int j = 0; j < p.rank / 16; ++j) {  // K = 16 bf16 = 32 bytes per MMA
              dev::umma_bf16_pair(tmem, dev::desc_sw128(sa + 32 * j), dev::desc_sw128(sb + 32 * j), IDESC_BF16,
                                  accumulate);
              accumulate = 1;
            }
          } else {
            const int nkb = min(4, p.kb_total - 4 * (st - p.lr_stages));
            for (int kb = 0; kb < nkb; ++kb) {  // K = 64 e2m1 = 32 bytes per MMA
              dev::umma_nvfp4_pair(tmem, dev::desc_sw128(sa + 32 * kb), dev::desc_sw128(sb + 32 * kb), IDESC_NVFP4,
                                   tmem + sfa_col(s, kb), tmem + sfb_col(s, kb), accumulate);
              accumulate = 1;
            }
          }
          issued_any = true;
          dev::tc_commit_pair_mc(&empty[s], 0x3);  // both CTAs' stage s free once these MMAs finish
        }
        if (!ok) break;
        dev::tc_commit_pair_mc(tmem_full, 0x3);    // both halves of the accumulator ready
      }
      if (!ok) abort_pair(abort_flag, peer_abort, status);
      if (issued_any) {  // the tensor cores must be idle before TMEM is freed
        dev::tc_commit_pair(drain_mma);
        dev::mbar_wait(drain_mma, 0, limit_ns, nullptr);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale-factor copies (even CTA)
    if (h == 0 && lane == 0) {
      int it = 0;
      bool ok = true, issued_any = false;
      for (int tile = t_begin; tile < t_end && ok; ++tile) {
        const Params &p = grp.p[locate_tile(grp, tile).pi];
        const int stages_per_tile = p.lr_stages + p.k_stages;
        for (int st = 0; st < stages_per_tile; ++st, ++it) {
          const int s = it % STAGES;
          if (!dev::mbar_wait_cluster(&sf_loaded[s], (it / STAGES) & 1, limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          if (st >= p.lr_stages) {
            const int nkb = min(4, p.kb_total - 4 * (st - p.lr_stages));
            const uint32_t ssfa = dev::smem_u32(smem + s * STAGE_BYTES + SFA_OFF);
            const uint32_t ssfb = dev::smem_u32(smem + s * STAGE_BYTES + SFB_OFF);
            for (int kb = 0; kb < nkb; ++kb) {
              dev::tmem_cp_32x128b_x4_pair(tmem + sfa_col(s, kb), dev::desc_sf(ssfa + 512 * kb));
              // both 128-row halves of the B scales in one copy: the four replicas of an
              // atom fill the four lane quarters as one warpx4 copy of it would
              dev::tmem_cp_128x256b_pair(tmem + sfb_col(s, kb), dev::desc_sf_2x(ssfb + 4096 * kb));
            }
            issued_any = true;
          }
          dev::tc_commit_pair(&sf_full[s]);  // arrives once this stage's copies have landed
        }
      }
      if (!ok) abort_pair(abort_flag, peer_abort, status);
      if (issued_any) {
        dev::tc_commit_pair(drain_cp);
        dev::mbar_wait(drain_cp, 0, limit_ns, nullptr);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int e = warp - 4;
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int half = e >> 2;                // which 128 of the 256 columns
    uint8_t *stage_out = smem + EPI_OFF + e * EPI_TILE_BYTES;
    const uint32_t tmem_empty_even = dev::mapa(dev::smem_u32(tmem_empty), 0);
    float *rinv_tab = reinterpret_cast<float *>(smem + TAB_OFF);
    float d6n = 0.0f;
    if constexpr (RQ >= 0) {
      // 1 / (block scale of code c) of the next layer: f32(e4m3(c) * s_a_next), then f32(1 / that)
      const float s_an = __ldg(grp.p[0].nx_s_a);   // a re-quantizing launch holds one problem
      d6n = __fmul_rn(6.0f, s_an);
      if (e < 4) {
        const uint32_t c = static_cast<uint32_t>(e * 32 + lane);
        const float scale = c < 127u ? __fmul_rn(dev::e4m3_value(c), s_an) : 0.0f;
        rinv_tab[c] = scale == 0.0f ? 0.0f : __frcp_rn(scale);
      }
      dev::named_barrier(1, EPI_WARPS * 32);
    }
    int tcount = 0;
    for (int tile = t_begin; tile < t_end; ++tile, ++tcount) {
      const TileRef tr = locate_tile(grp, tile);
      const Params &p = grp.p[tr.pi];
      const Maps &maps = grp.maps[tr.pi];
      const int m_blk = 2 * tr.m2 + static_cast<int>(h);
      const int n_blk = tr.n_blk;
      const float alpha = __fmul_rn(__ldg(p.s_a), __ldg(p.s_w));
      if (!dev::mbar_wait_cluster(tmem_full, tcount & 1, limit_ns, abort_flag)) {
        abort_pair(abort_flag, peer_abort, status);
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
      if (lane == 0) dev::mbar_arrive_cluster(tmem_empty_even);  // the MMA thread may start the next tile

      const int row0 = m_blk * BM + 32 * q;
      const int col0 = n_blk * BN + half * 128;
      // re-quantizing variant: this 128-row block exists in the next bundle (rows past M are zero there)
      const bool rows_live = RQ >= 0 && m_blk * BM < p.M;
      const bool row_ok = row0 + lane < p.M;
      uint8_t *ntile = nullptr;
      uint32_t xb[4][16];                     // bf16(x^) pairs of the next layer, per 32-column chunk
      uint32_t sword[2] = {0u, 0u};           // the next layer's block scales of this row, per 64 columns
      if constexpr (RQ >= 0)
        ntile = p.nx_bundle + (static_cast<size_t>(m_blk) * p.nx_ks + n_blk) * static_cast<size_t>(BM * 144);
#pragma unroll
      for (int c = 0; c < 4; ++c) {           // four 32-column chunks
        uint32_t out[16];                     // bf16(y) pairs of the chunk
#pragma unroll
        for (int g = 0; g < 4; ++g) {         // 8 columns (16 bytes) at a time
          const int col = col0 + 32 * c + 8 * g;
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
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 yy = dev::fma2_rn(make_float2(alpha, alpha),
                                           make_float2(__uint_as_float(v[c][8 * g + 2 * j]),
                                                       __uint_as_float(v[c][8 * g + 2 * j + 1])),
                                           make_float2(b[2 * j], b[2 * j + 1]));
            float y0 = yy.x, y1 = yy.y;
            if constexpr (EPI != SVDQ_EPILOGUE_NONE) {
              // computed for every column and selected: straight-line code lets the
              // independent GELU chains of a chunk interleave (a branch per element
              // serialised them)
              const bool act0 = col + 2 * j >= p.gelu_col_begin, act1 = col + 2 * j + 1 >= p.gelu_col_begin;
              float g0, g1;
              if constexpr (EPI == SVDQ_EPILOGUE_GELU_ERF) {
                const float2 gg = dev::gelu_erf2(yy);
                g0 = gg.x;
                g1 = gg.y;
              } else {
                g0 = dev::gelu_tanh(y0);
                g1 = dev::gelu_tanh(y1);
              }
              y0 = act0 ? g0 : y0;
              y1 = act1 ? g1 : y1;
            }
            __nv_bfloat162 hv = __floats2bfloat162_rn(y0, y1);
            out[4 * g + j] = *reinterpret_cast<uint32_t *>(&hv);
          }
        }
        if (RQ < 0 || p.store_y) {
          if (lane == 0) dev::bulk_wait_group_read<0>();  // staging tile free again
          __syncwarp();
          // row `lane` of the 32 x 32 staging tile, 16-byte chunk g, 64-byte swizzle
#pragma unroll
          for (int g = 0; g < 4; ++g)
            *reinterpret_cast<uint4 *>(stage_out + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(out[4 * g], out[4 * g + 1], out[4 * g + 2], out[4 * g + 3]);
          dev::fence_proxy_async();  // make the generic writes visible to the TMA store
          __syncwarp();
          if (lane == 0 && row0 < p.M && col0 + 32 * c < p.N) {  // the TMA clips the ragged edges
            dev::tma_store_2d(&maps.y, stage_out, col0 + 32 * c, row0);
            dev::bulk_commit_group();
          }
        }
        if constexpr (RQ >= 0) {
          // x^ of the next layer: f32(bf16(y) * inv_lambda_next), 0 past M and past N (the
          // chunk lies wholly inside or outside N, N being a multiple of 64)
          float inv[32];
          const bool cols_ok = col0 + 32 * c < p.N;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 f = cols_ok ? __ldg(reinterpret_cast<const float4 *>(p.nx_inv + col0 + 32 * c) + i)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            inv[4 * i] = f.x;
            inv[4 * i + 1] = f.y;
            inv[4 * i + 2] = f.z;
            inv[4 * i + 3] = f.w;
          }
          float xh[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            xh[2 * i] = row_ok ? __fmul_rn(__uint_as_float(out[i] << 16), inv[2 * i]) : 0.0f;
            xh[2 * i + 1] = row_ok ? __fmul_rn(__uint_as_float(out[i] & 0xFFFF0000u), inv[2 * i + 1]) : 0.0f;
            __nv_bfloat162 hx = __floats2bfloat162_rn(xh[2 * i], xh[2 * i + 1]);
            xb[c][i] = *reinterpret_cast<uint32_t *>(&hx);
          }
          uint32_t code[4], sb[2];
#pragma unroll
          for (int bk = 0; bk < 2; ++bk) {   // two blocks of 16 along K_next
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(xh[16 * bk + i]));
            sb[bk] = dev::cvt_e4m3(__fdiv_rn(amax, d6n));
            const float rinv = rinv_tab[sb[bk]];
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              uint32_t word = 0;
#pragma unroll
              for (int bt = 0; bt < 4; ++bt) {
                const int i = 16 * bk + 8 * w + 2 * bt;
                word |= dev::cvt_e2m1x2(__fmul_rn(xh[i], rinv), __fmul_rn(xh[i + 1], rinv)) << (8 * bt);
              }
              code[2 * bk + w] = word;
            }
          }
          const int r = 32 * q + lane;        // row inside the next bundle's 128-row tile
          if (rows_live)
            *reinterpret_cast<uint4 *>(ntile + r * 128 + ((((4 * half + c) ^ r) & 7) << 4)) =
                make_uint4(code[0], code[1], code[2], code[3]);
          sword[c >> 1] |= (sb[0] | (sb[1] << 8)) << (16 * (c & 1));
        }
      }
      if constexpr (RQ >= 0) {
        if (rows_live) {
          // scale words: 16-blocks 8 half + 4 s .. + 3 of row r: atom (2 half + s), lane-row, quarter q
#pragma unroll
          for (int s = 0; s < 2; ++s)
            *reinterpret_cast<uint32_t *>(ntile + BM * 128 + (2 * half + s) * 512 + lane * 16 + q * 4) = sword[s];
        }
      }
      if constexpr (RQ > 0) {
        if (rows_live) {
          // bf16(x^) . L1_next over this warp's 128 columns: 32 rows x RQ, mma.sync m16n8k16
          constexpr int NT = RQ / 8;
          const int g8 = lane >> 2, t4 = lane & 3;
          float acc[2][NT][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (col0 + 32 * c >= p.N) break;   // warp-uniform; chunks past N hold zeros
            if (lane == 0) dev::bulk_wait_group_read<0>();
            __syncwarp();
#pragma unroll
            for (int g = 0; g < 4; ++g)
              *reinterpret_cast<uint4 *>(stage_out + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4)) =
                  make_uint4(xb[c][4 * g], xb[c][4 * g + 1], xb[c][4 * g + 2], xb[c][4 * g + 3]);
            __syncwarp();
            uint32_t a[2][2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
              for (int kt = 0; kt < 2; ++kt) {
                const int mi = lane >> 3;
                const int rr = 16 * mt + (mi & 1) * 8 + (lane & 7);
                const int gg = 2 * kt + (mi >> 1);
                dev::ldmatrix_x4(dev::smem_u32(stage_out + rr * 64 + ((gg ^ ((rr >> 1) & 3)) << 4)), a[mt][kt][0],
                                 a[mt][kt][1], a[mt][kt][2], a[mt][kt][3]);
              }
            __syncwarp();                      // the staging tile may be written again
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint16_t *l1 = p.nx_l1t + static_cast<size_t>(8 * nt + g8) * p.N + col0 + 32 * c + 2 * t4;
#pragma unroll
              for (int kt = 0; kt < 2; ++kt) {
                const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t *>(l1 + 16 * kt));
                const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t *>(l1 + 16 * kt + 8));
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) dev::mma_bf16_16816(acc[mt][nt], a[mt][kt], b0, b1);
              }
            }
          }
          // add the 32 rows x RQ partial sums into the next layer's accumulator (rows < M)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int ra = row0 + 16 * mt + g8, rb = ra + 8;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (ra < p.M)
                atomicAdd(reinterpret_cast<float2 *>(p.nx_acc + static_cast<size_t>(ra) * RQ + 8 * nt + 2 * t4),
                          make_float2(acc[mt][nt][0], acc[mt][nt][1]));
              if (rb < p.M)
                atomicAdd(reinterpret_cast<float2 *>(p.nx_acc + static_cast<size_t>(rb) * RQ + 8 * nt + 2 * t4),
                          make_float2(acc[mt][nt][2], acc[mt][nt][3]));
            }
          }
        }
      }
    }
    if (lane == 0) dev::bulk_wait_group<0>();
  }

  dev::tc_fence_before();
  __syncwarp();
  dev::cluster_sync();                        // no MMA or copy of the pair is still running
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}


// ---------------------------------------------------------------------------
// Host side shared by the entry points.

// Argument checks, tensor maps and launch parameters of one GEMM call.  Y may
// be null only when `y_optional` (then nothing is written through maps.y).
inline int setup_gemm(const char *fn, const uint8_t *a_bundle, const void *U, const float *s_a,
                      const uint8_t *w_bundle, const void *l2t, const float *s_w, const void *bias, int M, int N,
                      int K, int rank, int epilogue, int gelu_col_begin, void *Y, int ldy, bool y_optional,
                      Maps *maps, Params *p, DeviceState **st_out) {
  const std::string name(fn);
  if (!a_bundle || !s_a || !w_bundle || !s_w || (!Y && !y_optional) || (rank > 0 && (!U || !l2t)))
    return fail(SVDQ_ERR_INVALID_ARG, name + ": null pointer");
  if (epilogue < SVDQ_EPILOGUE_NONE || epilogue > SVDQ_EPILOGUE_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARG, name + ": unknown epilogue");
  if (M < 1 || K < 64 || K % 64 || N < 8 || N % 8 || (Y && (ldy < N || ldy % 8)))
    return fail(SVDQ_ERR_SHAPE, name + ": need M >= 1, K % 64 == 0, N % 8 == 0, ldy >= N, ldy % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, name + ": rank must be a multiple of 16 in [0, 64]");
  if (gelu_col_begin < 0 || gelu_col_begin > N) return fail(SVDQ_ERR_SHAPE, name + ": gelu_col_begin outside [0, N]");
  if (!aligned16(a_bundle) || !aligned16(w_bundle) || (Y && !aligned16(Y)) || (bias && !aligned16(bias)) ||
      (rank > 0 && (!aligned16(U) || !aligned16(l2t))))
    return fail(SVDQ_ERR_ALIGNMENT, name + ": pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  *st_out = st;

  *p = Params{};
  p->M = M;
  p->N = N;
  p->rank = rank;
  p->epilogue = epilogue;
  p->gelu_col_begin = gelu_col_begin;
  p->num_m2 = (M + 2 * BM - 1) / (2 * BM);
  p->num_n = (N + BN - 1) / BN;
  p->num_tiles = p->num_m2 * p->num_n;
  p->kb_total = K / 64;
  p->k_stages = bundle_ks(K);
  p->lr_stages = rank > 0 ? 1 : 0;
  p->s_a = s_a;
  p->s_w = s_w;
  p->bias = static_cast<const uint16_t *>(bias);
  p->status = st->status_word;
  p->limit_ns = kWaitLimitNs;
  p->store_y = Y != nullptr;

  // The bundles are read as rows of 2 KB (256 x 8-byte elements); a copy is
  // a box of whole rows.  Rows past the end of a buffer (the odd half of a
  // pair tile whose rows lie beyond M) read as zeros.
  const auto u64 = CU_TENSOR_MAP_DATA_TYPE_UINT64;
  const auto none = CU_TENSOR_MAP_SWIZZLE_NONE;
  const uint64_t a_rows = bundle_bytes(M, K, 128) / ROW, w_rows = bundle_bytes(N, K, 256) / ROW;
  int rc = encode_tmap_2d(&maps->a, u64, a_bundle, ROW / 8, a_rows, ROW, ROW / 8, A_CODE_BYTES / ROW, none);
  if (rc == SVDQ_OK)
    rc = encode_tmap_2d(&maps->sfa, u64, a_bundle, ROW / 8, a_rows, ROW, ROW / 8, SFA_BYTES / ROW, none);
  if (rc == SVDQ_OK) rc = encode_tmap_2d(&maps->b, u64, w_bundle, ROW / 8, w_rows, ROW, ROW / 8, B_BYTES / ROW, none);
  if (rc == SVDQ_OK)
    rc = encode_tmap_2d(&maps->sfb, u64, w_bundle, ROW / 8, w_rows, ROW, ROW / 8, SFB_BYTES / ROW, none);
  if (rc == SVDQ_OK && rank > 0) {
    rc = encode_tmap_2d(&maps->u, u64, U, ROW / 8, lowrank_bytes(M, 128) / ROW, ROW, ROW / 8, LR_BYTES / ROW, none);
    if (rc == SVDQ_OK)
      rc = encode_tmap_2d(&maps->l2, u64, l2t, ROW / 8, lowrank_bytes(N, 256) / ROW, ROW, ROW / 8, LR_BYTES / ROW,
                          none);
  } else {
    maps->u = maps->a;  // unused without the low-rank stage
    maps->l2 = maps->a;
  }
  if (rc == SVDQ_OK) {
    if (Y)
      rc = encode_tmap_2d(&maps->y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, static_cast<uint64_t>(N),
                          static_cast<uint64_t>(M), static_cast<uint64_t>(ldy) * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
    else
      maps->y = maps->a;  // never used: no bf16 output
  }
  return rc;
}

// Per device and kernel family (RQ), once: the shared-memory opt-in of the
// three epilogue instantiations and the number of SM pairs that can hold one
// CTA each at that size.
template <int RQ, int G>
int prepare_device(const char *fn, int sm_count, int *pairs_out) {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev_id = 0;
  if (cudaGetDevice(&dev_id) != cudaSuccess || dev_id < 0 || dev_id >= 64)
    return fail(SVDQ_ERR_CUDA, std::string(fn) + ": no current device");
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev_id] == 0) {
    cudaError_t e = cudaFuncSetAttribute(gemm_w4a4_kernel<SVDQ_EPILOGUE_NONE, RQ, G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_w4a4_kernel<SVDQ_EPILOGUE_GELU_ERF, RQ, G>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_w4a4_kernel<SVDQ_EPILOGUE_GELU_TANH, RQ, G>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + ": " + cudaGetErrorString(e));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sm_count & ~1), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_w4a4_kernel<SVDQ_EPILOGUE_NONE, RQ, G>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = sm_count / 2;
    }
    cached[dev_id] = n;
  }
  *pairs_out = cached[dev_id];
  return SVDQ_OK;
}

// A group of one problem.
inline Group<1> single_group(const Maps &maps, const Params &p) {
  Group<1> g{};
  g.maps[0] = maps;
  g.p[0] = p;
  g.tile_end[0] = p.num_tiles;
  g.count = 1;
  g.total_tiles = p.num_tiles;
  g.status = p.status;
  g.limit_ns = p.limit_ns;
  return g;
}

// Launches the instantiation of `epilogue` on min(tiles, resident) SM pairs.
template <int RQ, int G>
int launch_gemm(const char *fn, const Group<G> &g, int epilogue, int sm_count, cudaStream_t stream) {
  int resident = 0;
  int rc = prepare_device<RQ, G>(fn, sm_count, &resident);
  if (rc != SVDQ_OK) return rc;
  const int pairs = g.total_tiles < resident ? g.total_tiles : resident;
  DependentLaunch dl(dim3(2 * pairs), dim3(THREADS), SMEM_BYTES, stream);
  cudaError_t e = epilogue == SVDQ_EPILOGUE_GELU_ERF
                      ? cudaLaunchKernelEx(&dl.cfg, gemm_w4a4_kernel<SVDQ_EPILOGUE_GELU_ERF, RQ, G>, g)
                  : epilogue == SVDQ_EPILOGUE_GELU_TANH
                      ? cudaLaunchKernelEx(&dl.cfg, gemm_w4a4_kernel<SVDQ_EPILOGUE_GELU_TANH, RQ, G>, g)
                      : cudaLaunchKernelEx(&dl.cfg, gemm_w4a4_kernel<SVDQ_EPILOGUE_NONE, RQ, G>, g);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + " launch: " + cudaGetErrorString(e));
  return SVDQ_OK;
}
template <int RQ>
int launch_gemm(const char *fn, const Maps &maps, const Params &p, int sm_count, cudaStream_t stream) {
  return launch_gemm<RQ, 1>(fn, single_group(maps, p), p.epilogue, sm_count, stream);
}

}  // namespace w4a4
}  // namespace svdq
