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
//   * one CTA per 32 rows, 16 compute warps + 1 TMA warp + 1 store warp; a
//     ring of stages, each a [32 rows x 256 cols] bf16 tile of X, an
//     [r x 256] tile of L1^T (one 3-D TMA copy each, as four 64-column boxes
//     with the 128-byte swizzle), the stage's 256-float slice of inv_lambda
//     (a bulk copy) and a staging area for the stage's codes and scales;
//   * compute warp w owns the 16-column slice w of every stage for all 32
//     rows.  It loads the slice once, with ldmatrix, straight into the
//     m16n8k16 A-fragment layout: lane (g, t) holds columns 2t, 2t+1, 2t+8,
//     2t+9 of rows g + 8q, q = 0..3, i.e. a quarter of four 16-element blocks;
//   * from those registers: x^ = x * inv_lambda, the bf16 A fragments of the
//     down-projection (mma.sync into r/2 independent accumulators per lane),
//     and the block maxima, reduced over the 4 lanes of a row group by a
//     butterfly that leaves each lane owning one whole block.  That lane
//     takes the f32 division for the block scale and looks 1/scale up in a
//     per-CTA table of all 128 scale codes (the tensor scale is fixed per
//     call, so f32(1 / f32(e4m3 * s_a)) has only 128 values); the four
//     1/scale values come back by shuffles, every lane converts its 16
//     elements, and a second butterfly gathers each block's 8 code bytes in
//     its owner lane, which puts them (and the scale byte) into the staging
//     area in the bundle's byte order;
//   * the store warp copies each staged stage out with full-line stores (a
//     CTA's code rows are 4 KB of contiguous bundle) and frees the stage;
//   * warps never meet inside the loop: each waits for its stage with a
//     bounded mbarrier wait (decided warp-uniformly; a warp whose wait runs
//     out records SVDQ_ERR_TIMEOUT and leaves the loop) and signals the store
//     warp with one arrive.  At the end the 16 per-slice partial U tiles are added in
//     shared memory and written as 128-row swizzled tiles.
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
constexpr int CWARPS = 16;         // compute warps: one 16-column slice each
constexpr int THREADS = (CWARPS + 2) * 32;   // + TMA warp + store warp
constexpr int X_BOX = BM * 128;    // one [32 x 64] bf16 box, 128-byte rows
constexpr int X_STAGE = 4 * X_BOX;
constexpr int INV_BYTES = KC * 4;
constexpr int OUT_BYTES = 6144;   // inv_lambda slice (1 KB), code rows (4 KB), scale words (512 B), padded
constexpr int RING_BYTES = 224 * 1024;

struct Params {
  int M, K, KS;
  const float *inv_lambda;
  const float *s_a, *s_w;
  uint8_t *bundle;
  uint8_t *U;
  unsigned int *status;
  unsigned long long limit_ns;
};

// A grouped launch: up to G activations quantized by one grid, the CTAs of
// problem i after those of problems 0..i-1; each CTA reads its problem's
// tensor maps and parameters.  A single call is a group of one (G = 1).
constexpr int kMaxGroup = SVDQ_MAX_GROUP;
template <int G>
struct Group {
  CUtensorMap tx[G], tl[G];
  Params p[G];
  int blk_end[G];               // prefix sums of the problems' CTA counts
  int count;
};

template <int RANK>
__host__ __device__ constexpr int stage_bytes() {
  return X_STAGE + 4 * RANK * 128 + OUT_BYTES;
}
template <int RANK>
__host__ __device__ constexpr int num_stages() {
  return RING_BYTES / stage_bytes<RANK>() < 8 ? RING_BYTES / stage_bytes<RANK>() : 8;
}
template <int RANK>
__host__ __device__ constexpr int smem_bytes() {
  return 1024 + num_stages<RANK>() * stage_bytes<RANK>() + 128 * 4 + 512;
}
// the per-slice partial U tiles reuse the ring at the end
static_assert(CWARPS * BM * (64 + 4) * 4 <= num_stages<64>() * stage_bytes<64>(), "partials must fit the ring");

// Byte offset of the 16-byte chunk holding column c (0..63, multiple of 8) of
// row r inside a 128-byte-swizzled box of 128-byte rows.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ r) & 7) << 4));
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ float absmax4(float a, float b, float c, float d) {
  return fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d)));
}

template <int RANK, int G>
__global__ void __launch_bounds__(THREADS, 1)
    quant_act_kernel(const __grid_constant__ Group<G> grp) {
  constexpr int STAGES = num_stages<RANK>();
  constexpr int L1_BOX = RANK * 128;
  constexpr int STAGE = stage_bytes<RANK>();
  constexpr int INV_OFF = X_STAGE + 4 * L1_BOX;
  constexpr int CODE_OFF = INV_OFF + INV_BYTES;    // [32 rows x 128 B] code rows, bundle swizzle
  constexpr int SC_OFF = CODE_OFF + BM * 128;      // [4 boxes][32 rows] scale words
  constexpr int NT = RANK / 8;     // 8-column tiles of U

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *rinv_tab = reinterpret_cast<float *>(smem + STAGES * STAGE);   // [128]
  uint64_t *full = reinterpret_cast<uint64_t *>(rinv_tab + 128);
  uint64_t *empty = full + STAGES;   // the store warp has written the stage out
  uint64_t *done = empty + STAGES;   // the compute warps have staged the stage's codes and scales
  volatile int *abort_flag = reinterpret_cast<volatile int *>(done + STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int pi = 0;
  if constexpr (G > 1)
    while (pi + 1 < grp.count && static_cast<int>(blockIdx.x) >= grp.blk_end[pi]) ++pi;
  const CUtensorMap &tm_x = grp.tx[pi];
  const CUtensorMap &tm_l1 = grp.tl[pi];
  const Params &p = grp.p[pi];
  const int m0 = (static_cast<int>(blockIdx.x) - (pi > 0 ? grp.blk_end[pi - 1] : 0)) * BM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], 1);
      dev::mbar_init(&done[s], CWARPS);
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
        // the 3-D boxes always land whole (columns past K as zeros)
        dev::mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(X_STAGE + 4 * L1_BOX + nbox * 256));
        uint8_t *st = smem + s * STAGE;
        dev::tma_load_3d(st, &tm_x, &full[s], 0, m0, 4 * c);
        if (RANK > 0) dev::tma_load_3d(st + X_STAGE, &tm_l1, &full[s], 0, 0, 4 * c);
        dev::bulk_load(st + INV_OFF, p.inv_lambda + c * KC, static_cast<uint32_t>(nbox * 256), &full[s]);
        ++issued;
      }
      // every issued copy lands before the block leaves
      for (int c = max(0, issued - STAGES); c < issued; ++c)
        dev::mbar_wait(&full[c % STAGES], (c / STAGES) & 1, p.limit_ns, nullptr);
    }
    return;
  }

  const int m_blk = m0 / 128;
  if (warp == CWARPS + 1) {
    // ---------------------------------------------------------- store warp
    // copies each stage's staged code rows (4 KB, contiguous in the bundle
    // tile) and scale words out with full-line stores, then frees the stage
    const uint32_t qd = static_cast<uint32_t>((m0 % 128) >> 5);
    for (int c = 0; c < p.KS; ++c) {
      const int s = c % STAGES;
      if (!dev::mbar_wait_warp(&done[s], (c / STAGES) & 1, p.limit_ns, abort_flag)) {
        *abort_flag = 1;
        dev::report(p.status, SVDQ_ERR_TIMEOUT);
        break;
      }
      const uint8_t *st = smem + s * STAGE;
      uint8_t *tile = p.bundle + (static_cast<size_t>(m_blk) * p.KS + c) * bundle_tile_bytes(128);
      uint4 v[8];
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = *reinterpret_cast<const uint4 *>(st + CODE_OFF + (i * 32 + lane) * 16);
#pragma unroll
      for (int b = 0; b < 4; ++b) w[b] = *reinterpret_cast<const uint32_t *>(st + SC_OFF + (b * 32 + lane) * 4);
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&empty[s]);
      uint8_t *rows = tile + (m0 % 128) * 128;
#pragma unroll
      for (int i = 0; i < 8; ++i) *reinterpret_cast<uint4 *>(rows + (i * 32 + lane) * 16) = v[i];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        *reinterpret_cast<uint32_t *>(tile + 128 * 128 + b * 512 + lane * 16 + qd * 4) = w[b];
    }
    if (RANK > 0) dev::named_barrier(1, (CWARPS + 1) * 32);   // the ring may now hold the partials
    return;
  }

  // -------------------------------------------------------------- compute warps
  const int g = lane >> 2, t = lane & 3;
  const int bx = warp >> 2;                     // 64-column box of this warp's slice
  const int kc = (warp & 3) * 16;               // slice offset inside the box
  const bool o1 = (t & 1) != 0, o2 = (t & 2) != 0;
  // the block this lane owns after the butterflies: rows g + 8 q, q = 2 o1 + o2
  const int row_own = 8 * (2 * (t & 1) + ((t >> 1) & 1)) + g;
  // staged like the bundle tile: code chunk (warp >> 1) of the row, 128-byte swizzle on the row
  // inside the 128-row tile (m0 is a multiple of 32, so that row and row_own agree mod 8)
  const uint32_t code_off =
      static_cast<uint32_t>(CODE_OFF + row_own * 128 + ((((warp >> 1) ^ row_own) & 7) << 4) + 8 * (warp & 1));
  const uint32_t scale_off = static_cast<uint32_t>(SC_OFF + (bx * 32 + row_own) * 4 + (warp & 3));
  const float d6 = __fmul_rn(6.0f, s_a);
  // ldmatrix lane addresses: A rows (per 16-row half), B rows of L1^T (per pair of 8-column tiles)
  const uint32_t a_off0 = sw_off((lane & 7) + ((lane >> 3) & 1) * 8, kc + (lane >> 4) * 8);
  const uint32_t a_off1 = sw_off(16 + (lane & 7) + ((lane >> 3) & 1) * 8, kc + (lane >> 4) * 8);
  const int lsrc = lane & ~3;
  // prmt selectors of the code-byte gather (they depend on the lane's parity bits)
  const uint32_t sel_a = o1 ? 0x1504u : 0x5140u, sel_b = o1 ? 0x3726u : 0x7362u;
  const uint32_t sel_w0 = o2 ? 0x1054u : 0x5410u, sel_w1 = o2 ? 0x3276u : 0x7632u;

  float acc[2][NT > 0 ? NT : 1][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int n = 0; n < (NT > 0 ? NT : 1); ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][n][i] = 0.0f;
  bool failed = false;

  for (int c = 0; c < p.KS; ++c) {
    const int s = c % STAGES;
    if (!dev::mbar_wait_warp(&full[s], (c / STAGES) & 1, p.limit_ns, abort_flag)) {
      *abort_flag = 1;
      dev::report(p.status, SVDQ_ERR_TIMEOUT);
      failed = true;
      break;
    }
    const int nbox = min(4, (p.K - c * KC) / 64);
    uint8_t *st = smem + s * STAGE;
    // x^ of the lane's 16 elements: xs[q][0..3] = row g + 8q, columns 2t, 2t+1, 2t+8, 2t+9
    float xs[4][4];
    if (bx < nbox) {
      const uint32_t xbase = dev::smem_u32(st + bx * X_BOX);
      uint32_t a0[4], a1[4];
      dev::ldmatrix_x4(xbase + a_off0, a0[0], a0[1], a0[2], a0[3]);
      dev::ldmatrix_x4(xbase + a_off1, a1[0], a1[1], a1[2], a1[3]);
      const float *iv = reinterpret_cast<const float *>(st + INV_OFF) + bx * 64 + kc + 2 * t;
      const float2 i0 = *reinterpret_cast<const float2 *>(iv);
      const float2 i1 = *reinterpret_cast<const float2 *>(iv + 8);
      // fragment register h of half mt: rows g (h even) / g + 8 (h odd), columns 2t.. (h < 2) / 2t+8.. (h >= 2)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t lo = (q >> 1) ? a1[q & 1] : a0[q & 1];
        const uint32_t hi = (q >> 1) ? a1[2 + (q & 1)] : a0[2 + (q & 1)];
        const float2 p0 = dev::mul2_rn(make_float2(bf16_lo(lo), bf16_hi(lo)), i0);
        const float2 p1 = dev::mul2_rn(make_float2(bf16_lo(hi), bf16_hi(hi)), i1);
        xs[q][0] = p0.x;
        xs[q][1] = p0.y;
        xs[q][2] = p1.x;
        xs[q][3] = p1.y;
      }
      if (RANK > 0) {
        // down-projection of this slice: A = bf16(x^), B = L1^T rows (ldmatrix of 2 tiles x 2 k-halves)
        uint32_t af[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          af[mt][0] = bf16x2(xs[2 * mt][0], xs[2 * mt][1]);
          af[mt][1] = bf16x2(xs[2 * mt + 1][0], xs[2 * mt + 1][1]);
          af[mt][2] = bf16x2(xs[2 * mt][2], xs[2 * mt][3]);
          af[mt][3] = bf16x2(xs[2 * mt + 1][2], xs[2 * mt + 1][3]);
        }
        const uint32_t lbase = dev::smem_u32(st + X_STAGE + bx * L1_BOX);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t b[4];
          dev::ldmatrix_x4(lbase + sw_off(np * 16 + (lane >> 4) * 8 + (lane & 7), kc + ((lane >> 3) & 1) * 8), b[0],
                           b[1], b[2], b[3]);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            dev::mma_bf16_16816(acc[mt][2 * np], af[mt], b[0], b[1]);
            dev::mma_bf16_16816(acc[mt][2 * np + 1], af[mt], b[2], b[3]);
          }
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < 4; ++i) xs[q][i] = 0.0f;   // columns past K quantize as zeros
    }

    // block maxima: lane partials, then a butterfly over the row group's 4 lanes
    const float m0q = absmax4(xs[0][0], xs[0][1], xs[0][2], xs[0][3]);
    const float m1q = absmax4(xs[1][0], xs[1][1], xs[1][2], xs[1][3]);
    const float m2q = absmax4(xs[2][0], xs[2][1], xs[2][2], xs[2][3]);
    const float m3q = absmax4(xs[3][0], xs[3][1], xs[3][2], xs[3][3]);
    float ka = o1 ? m2q : m0q, kb = o1 ? m3q : m1q;       // keep blocks {2 o1, 2 o1 + 1}
    ka = fmaxf(ka, __shfl_xor_sync(0xFFFFFFFFu, o1 ? m0q : m2q, 1));
    kb = fmaxf(kb, __shfl_xor_sync(0xFFFFFFFFu, o1 ? m1q : m3q, 1));
    const float amax = fmaxf(o2 ? kb : ka, __shfl_xor_sync(0xFFFFFFFFu, o2 ? ka : kb, 2));   // block 2 o1 + o2
    const uint32_t sb = dev::cvt_e4m3(__fdiv_rn(amax, d6));
    const float rown = rinv_tab[sb];
    // 1/scale of blocks 0..3 from their owners (lanes t = 0, 2, 1, 3)
    float rq[4];
    rq[0] = __shfl_sync(0xFFFFFFFFu, rown, lsrc);
    rq[1] = __shfl_sync(0xFFFFFFFFu, rown, lsrc + 2);
    rq[2] = __shfl_sync(0xFFFFFFFFu, rown, lsrc + 1);
    rq[3] = __shfl_sync(0xFFFFFFFFu, rown, lsrc + 3);
    // code bytes t (columns 2t, 2t+1) and t + 4 (columns 2t+8, 2t+9) of each block
    uint32_t cq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
    {
      const float2 r2 = make_float2(rq[q], rq[q]);
      const float2 c0 = dev::mul2_rn(make_float2(xs[q][0], xs[q][1]), r2);
      const float2 c1 = dev::mul2_rn(make_float2(xs[q][2], xs[q][3]), r2);
      cq[q] = dev::cvt_e2m1x4(c0.x, c0.y, c1.x, c1.y);
    }
    // gather: after the xor-1 step a lane holds bytes {e, e+1, e+4, e+5} (e = t & 2) of its
    // two kept blocks, after the xor-2 step all 8 bytes of the block it owns
    const uint32_t keep = o1 ? (cq[2] | (cq[3] << 16)) : (cq[0] | (cq[1] << 16));
    const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, o1 ? (cq[0] | (cq[1] << 16)) : (cq[2] | (cq[3] << 16)), 1);
    const uint32_t da = prmt(keep, recv, sel_a), db = prmt(keep, recv, sel_b);
    const uint32_t mine = o2 ? db : da;
    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, o2 ? da : db, 2);
    *reinterpret_cast<uint2 *>(st + code_off) = make_uint2(prmt(mine, other, sel_w0), prmt(mine, other, sel_w1));
    st[scale_off] = static_cast<uint8_t>(sb);
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&done[s]);
  }

  // ---- U = (sum of the 16 slices' partial products) / (s_a s_w), bf16, 128-row tiles
  const int tid = threadIdx.x;  // 0..511
  constexpr int RS = RANK + 4;   // padded row of a partial tile
  if (RANK > 0) {
    dev::named_barrier(1, (CWARPS + 1) * 32);      // the ring is no longer read (store warp included)
    float *red = reinterpret_cast<float *>(smem) + warp * BM * RS;   // [CWARPS][BM][RS]
    if (!failed) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int n = 0; n < (NT > 0 ? NT : 1); ++n) {
          const int row = mt * 16 + g, col = n * 8 + 2 * t;
          *reinterpret_cast<float2 *>(red + row * RS + col) = make_float2(acc[mt][n][0], acc[mt][n][1]);
          *reinterpret_cast<float2 *>(red + (row + 8) * RS + col) = make_float2(acc[mt][n][2], acc[mt][n][3]);
        }
    }
    dev::named_barrier(2, CWARPS * 32);
  }
  // a wait that ran out anywhere leaves U zero (the status word carries the error)
  const bool any_failed = RANK > 0 && *abort_flag != 0;
  const float alpha = __fmul_rn(s_a, __ldg(p.s_w));
  // every thread: column pairs (2 cp, 2 cp + 1) of the CTA's rows, the 16 partials added in order
  for (int idx = tid; idx < BM * (SVDQ_LR_STRIDE / 2); idx += CWARPS * 32) {
    const int rr = idx / (SVDQ_LR_STRIDE / 2), cp = idx % (SVDQ_LR_STRIDE / 2);
    uint32_t o = 0;
    if (RANK > 0 && 2 * cp < RANK && !any_failed) {
      const float *red = reinterpret_cast<const float *>(smem) + rr * RS + 2 * cp;
      float2 sum = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int w = 0; w < CWARPS; ++w) {
        const float2 v = *reinterpret_cast<const float2 *>(red + w * BM * RS);
        sum.x += v.x;
        sum.y += v.y;
      }
      o = bf16x2(__fdiv_rn(sum.x, alpha), __fdiv_rn(sum.y, alpha));
    }
    *reinterpret_cast<uint32_t *>(p.U + lowrank_offset(m0 + rr, 2 * cp, 128)) = o;
  }
}

template <int RANK, int G>
int launch(const Group<G> &g, int grid, cudaStream_t stream, const char *fn) {
  const int smem = smem_bytes<RANK>();
  const int rc = smem_optin_once<quant_act_kernel<RANK, G>>(smem, fn);
  if (rc != SVDQ_OK) return rc;
  DependentLaunch dl(dim3(grid), dim3(THREADS), smem, stream);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, quant_act_kernel<RANK, G>, g);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + " launch: " + cudaGetErrorString(e));
  return ok();
}

// Checks one problem and fills its parameters; returns its CTA count in *grid.
int check_problem(const std::string &fn, const void *X, int M, int K, int ldx, const float *inv_lambda,
                  const void *l1t, int rank, const float *s_a, const float *s_w, uint8_t *a_bundle, void *U,
                  Params *p, int *grid) {
  if (!X || !inv_lambda || !s_a || !s_w || !a_bundle || !U || (rank > 0 && !l1t))
    return fail(SVDQ_ERR_INVALID_ARG, fn + ": null pointer");
  if (M < 1 || K < 64 || K % 64 || ldx < K || ldx % 8)
    return fail(SVDQ_ERR_SHAPE, fn + ": need M >= 1, K % 64 == 0, ldx >= K, ldx % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, fn + ": rank must be a multiple of 16 in [0, 64]");
  if (!aligned16(X) || !aligned16(inv_lambda) || !aligned16(a_bundle) || !aligned16(U) ||
      (rank > 0 && !aligned16(l1t)))
    return fail(SVDQ_ERR_ALIGNMENT, fn + ": pointers must be 16-byte aligned");
  p->M = M;
  p->K = K;
  p->KS = bundle_ks(K);
  p->inv_lambda = inv_lambda;
  p->s_a = s_a;
  p->s_w = s_w;
  p->bundle = a_bundle;
  p->U = static_cast<uint8_t *>(U);
  p->limit_ns = kWaitLimitNs;   // p->status: the caller's device
  *grid = (M + 127) / 128 * (128 / BM);   // every row of every 128-row tile
  return SVDQ_OK;
}

// The tensor maps of a checked problem: X as [K/64 boxes][M rows][64 columns] and L1^T as
// [K/64][rank][64], one copy per stage each.
int encode_problem(const void *X, int M, int K, int ldx, const void *l1t, int rank, CUtensorMap *tx,
                   CUtensorMap *tl) {
  const uint64_t kb = static_cast<uint64_t>(K / 64);
  int rc = encode_tmap_3d(tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, {64, static_cast<uint64_t>(M), kb},
                          {static_cast<uint64_t>(ldx) * 2, 128}, {64, BM, 4}, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != SVDQ_OK) return rc;
  if (rank > 0) {
    rc = encode_tmap_3d(tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, l1t, {64, static_cast<uint64_t>(rank), kb},
                        {static_cast<uint64_t>(K) * 2, 128}, {64, static_cast<uint32_t>(rank), 4},
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != SVDQ_OK) return rc;
  } else {
    *tl = *tx;
  }
  return SVDQ_OK;
}

template <int G>
int launch_rank(int rank, const Group<G> &g, int grid, cudaStream_t s, const char *fn) {
  switch (rank) {
    case 0: return launch<0, G>(g, grid, s, fn);
    case 16: return launch<16, G>(g, grid, s, fn);
    case 32: return launch<32, G>(g, grid, s, fn);
    case 48: return launch<48, G>(g, grid, s, fn);
    default: return launch<64, G>(g, grid, s, fn);
  }
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_quantize_act(const void *X, int M, int K, int ldx, const float *inv_lambda, const void *l1t,
                                 int rank, const float *s_a, const float *s_w, uint8_t *a_bundle, void *U,
                                 svdq_stream_t stream) {
  static const char *fn = "svdq_quantize_act";
  Group<1> g{};
  int grid = 0;
  int rc = check_problem(fn, X, M, K, ldx, inv_lambda, l1t, rank, s_a, s_w, a_bundle, U, &g.p[0], &grid);
  if (rc != SVDQ_OK) return rc;
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  g.p[0].status = st->status_word;
  rc = encode_problem(X, M, K, ldx, l1t, rank, &g.tx[0], &g.tl[0]);
  if (rc != SVDQ_OK) return rc;
  g.blk_end[0] = grid;
  g.count = 1;
  return launch_rank(rank, g, grid, reinterpret_cast<cudaStream_t>(stream), fn);
}

extern "C" int svdq_quantize_act_grouped(const svdq_quant_problem *problems, int count, int rank,
                                         svdq_stream_t stream) {
  static const char *fn = "svdq_quantize_act_grouped";
  if (!problems) return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": null problem list");
  if (count < 1 || count > kMaxGroup)
    return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": count must be in [1, " + std::to_string(kMaxGroup) + "]");
  Group<kMaxGroup> g{};
  int total = 0;
  for (int i = 0; i < count; ++i) {
    const svdq_quant_problem &q = problems[i];
    int grid = 0;
    const int rc = check_problem(std::string(fn) + " (problem " + std::to_string(i) + ")", q.X, q.M, q.K, q.ldx,
                                 q.inv_lambda, q.l1t, rank, q.s_a, q.s_w, q.a_bundle, q.U, &g.p[i], &grid);
    if (rc != SVDQ_OK) return rc;
    total += grid;
    g.blk_end[i] = total;
  }
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  for (int i = 0; i < count; ++i) {
    g.p[i].status = st->status_word;
    const svdq_quant_problem &q = problems[i];
    const int rc = encode_problem(q.X, q.M, q.K, q.ldx, q.l1t, rank, &g.tx[i], &g.tl[i]);
    if (rc != SVDQ_OK) return rc;
  }
  g.count = count;
  return launch_rank(rank, g, total, reinterpret_cast<cudaStream_t>(stream), fn);
}
