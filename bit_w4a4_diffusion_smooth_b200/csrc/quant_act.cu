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
//   * compute warp w owns rows 16 (w >> 3) .. +15 and the 32-column slice
//     w & 7 of every stage; lane l of it owns one whole 16-element block
//     (row 16 (w >> 3) + (l & 15), block l >> 4 of the slice), read as two
//     16-byte chunks of the swizzled box.  The lane alone forms x^ = x *
//     inv_lambda, the block maximum, the f32 division for the block scale,
//     1/scale from a per-CTA table of all 128 scale codes (the tensor scale
//     is fixed per call, so f32(1 / f32(e4m3 * s_a)) has only 128 values)
//     and the block's 8 code bytes, which it puts (with the scale byte)
//     into the staging area in the bundle's byte order: no shuffles;
//   * the lane writes bf16(x^) back over its x; the warp then loads its
//     16 x 32 tile of it with ldmatrix as m16n8k16 A fragments for the
//     down-projection (mma.sync into r/8 accumulators per lane, B = L1^T
//     rows by ldmatrix);
//   * the store warp copies each staged stage out with full-line stores (a
//     CTA's code rows are 4 KB of contiguous bundle) and frees the stage;
//   * warps never meet inside the loop: each waits for its stage with a
//     bounded mbarrier wait (decided warp-uniformly; a warp whose wait runs
//     out records SVDQ_ERR_TIMEOUT and leaves the loop) and signals the store
//     warp with one arrive.  At the end the 8 per-slice partial U tiles of
//     each 16-row half are added in shared memory and written as 128-row
//     swizzled tiles.
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
constexpr int CWARPS = 16;         // compute warps: 16 rows x one 32-column slice each
constexpr int THREADS = (CWARPS + 2) * 32;   // + TMA warp + store warp
constexpr int X_BOX = BM * 128;    // one [32 x 64] bf16 box, 128-byte rows
constexpr int X_STAGE = 4 * X_BOX;
constexpr int INV_BYTES = KC * 4;
constexpr int OUT_BYTES = 6144;   // inv_lambda slice (1 KB), code rows (4 KB), scale words (512 B), padded
constexpr int RING_BYTES = 224 * 1024;
// INT4 form: each compute warp's 16 row maxima of its two blocks, per stage parity, for the warp
// that holds the other half of the 64-column groups
constexpr int XCH_BYTES = 2 * 16 * 16 * 4;

struct Params {
  int M, K, KS;
  const float *inv_lambda;
  const float *s_a, *s_w;       // NVFP4 tensor scales (unused by the INT4 form)
  uint8_t *bundle;              // NVFP4 codes and scales
  uint8_t *codes4;              // INT4 form: codes [rows][K/2] and group scales [K/64][ld_s] (bf16)
  uint16_t *scales4;
  int ld_s;
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
  return 1024 + num_stages<RANK>() * stage_bytes<RANK>() + 128 * 4 + 512 + XCH_BYTES;
}
// the per-slice partial U tiles reuse the ring at the end
static_assert(CWARPS * 16 * (64 + 4) * 4 <= num_stages<64>() * stage_bytes<64>(), "partials must fit the ring");

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
// Named barrier over nthreads threads that also ORs a predicate across them: every
// participant gets the same answer (used to leave a loop together).
__device__ __forceinline__ bool barrier_or(int id, int nthreads, bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, %2, %3, q;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(r)
               : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
               : "memory");
  return r != 0;
}
__device__ __forceinline__ float absmax4(float a, float b, float c, float d) {
  return fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d)));
}

// INT4: the form of the INT4 W4A4 variant (groups of 64 along K, bf16 group scales, codes in
// plain rows); otherwise NVFP4 into the operand bundle.
template <int RANK, int G, bool INT4>
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
  float *xch = reinterpret_cast<float *>(smem + STAGES * STAGE + 1024);   // [2][CWARPS][16]

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
  const float s_a = INT4 ? 1.0f : __ldg(p.s_a);
  if (!INT4 && threadIdx.x < 128) {
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
      if constexpr (INT4) {
        // code rows: 32 rows x 8 chunks of 16 bytes (staged with the chunk index xor the row);
        // scales: 4 groups x 32 rows of bf16.  Only the stage's groups inside K are written.
        const int ngrp = min(4, (p.K - c * KC) / 64);
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = i * 32 + lane, r = j >> 3, ch = j & 7;
          v[i] = *reinterpret_cast<const uint4 *>(st + CODE_OFF + r * 128 + (((ch ^ r) & 7) << 4));
        }
        const uint2 sc = *reinterpret_cast<const uint2 *>(st + SC_OFF + ((lane >> 3) * 32 + 4 * (lane & 7)) * 2);
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&empty[s]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = i * 32 + lane, r = j >> 3, ch = j & 7;
          if (ch < 2 * ngrp)
            *reinterpret_cast<uint4 *>(p.codes4 + static_cast<size_t>(m0 + r) * (p.K / 2) + c * (KC / 2) + ch * 16) = v[i];
        }
        if ((lane >> 3) < ngrp)
          *reinterpret_cast<uint2 *>(p.scales4 + static_cast<size_t>(4 * c + (lane >> 3)) * p.ld_s + m0 +
                                     4 * (lane & 7)) = sc;
        continue;
      }
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
  // warp w: rows 16 (w >> 3) .. +15 of the CTA and the 32-column slice w & 7 of every stage;
  // lane l: row 16 (w >> 3) + (l & 15) and the 16-column block l >> 4 of that slice, which it
  // quantizes on its own
  const int rh = warp >> 3, cs = warp & 7;
  const int bx = cs >> 1;                                   // 64-column box of the slice
  const int row = 16 * rh + (lane & 15), blk = lane >> 4;
  const int col = 32 * (cs & 1) + 16 * blk;                 // the block's first column inside the box
  const uint32_t x_off0 = sw_off(row, col), x_off1 = sw_off(row, col + 8);
  // staged like the bundle tile: 16-byte code chunk cs of the row, half blk; scale byte 2 cs + blk
  // of the row's 16 (m0 is a multiple of 32, so row and the bundle row agree mod 8)
  const uint32_t code_off = static_cast<uint32_t>(CODE_OFF + row * 128 + (((cs ^ row) & 7) << 4) + 8 * blk);
  const uint32_t scale_off = static_cast<uint32_t>(SC_OFF + (bx * 32 + row) * 4 + ((2 * cs + blk) & 3));
  const float d6 = __fmul_rn(6.0f, s_a);
  // ldmatrix lane addresses of the down-projection: A = the warp's 16 rows of bf16(x^) (written
  // back in place), B = rows of L1^T (per pair of 8-column tiles), each per k16 step kk
  const int arow = 16 * rh + (lane & 15);
  const int acol = 32 * (cs & 1) + 8 * (lane >> 4);
  const int brow = (lane >> 4) * 8 + (lane & 7), bcol = 32 * (cs & 1) + ((lane >> 3) & 1) * 8;

  float acc[NT > 0 ? NT : 1][4];
#pragma unroll
  for (int n = 0; n < (NT > 0 ? NT : 1); ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;
  bool failed = false;

  if constexpr (INT4) {
    // A 64-column group is box bx of the stage: this lane's block and the other block of the
    // same row in this warp (lane ^ 16), and the two blocks of the row in the pair warp w ^ 1.
    // The pair exchanges its row maxima through shared memory at a barrier of its own (ids
    // 3..10), whose OR-reduced predicate also carries a wait that ran out, so both warps of the
    // pair leave the loop together.
    const int pair_bar = 3 + (warp >> 1);
    for (int c = 0; c < p.KS; ++c) {
      const int s = c % STAGES;
      const bool got = dev::mbar_wait_warp(&full[s], (c / STAGES) & 1, p.limit_ns, abort_flag);
      if (!got) {
        *abort_flag = 1;
        dev::report(p.status, SVDQ_ERR_TIMEOUT);
      }
      const int nbox = min(4, (p.K - c * KC) / 64);
      uint8_t *st = smem + s * STAGE;
      uint8_t *xb = st + bx * X_BOX;
      const bool live = got && bx < nbox;   // warp-uniform: groups past K quantize as zeros
      float xs[16];
      float bmax = 0.0f;
      if (live) {
        const uint4 w0 = *reinterpret_cast<const uint4 *>(xb + x_off0);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(xb + x_off1);
        const float4 *iv = reinterpret_cast<const float4 *>(st + INV_OFF) + (bx * 64 + col) / 4;
        const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 v = iv[i];
          const float2 p0 = dev::mul2_rn(make_float2(bf16_lo(wv[2 * i]), bf16_hi(wv[2 * i])), make_float2(v.x, v.y));
          const float2 p1 =
              dev::mul2_rn(make_float2(bf16_lo(wv[2 * i + 1]), bf16_hi(wv[2 * i + 1])), make_float2(v.z, v.w));
          xs[4 * i] = p0.x;
          xs[4 * i + 1] = p0.y;
          xs[4 * i + 2] = p1.x;
          xs[4 * i + 3] = p1.y;
        }
        bmax = absmax4(xs[0], xs[1], xs[2], xs[3]);
        bmax = fmaxf(bmax, absmax4(xs[4], xs[5], xs[6], xs[7]));
        bmax = fmaxf(bmax, absmax4(xs[8], xs[9], xs[10], xs[11]));
        bmax = fmaxf(bmax, absmax4(xs[12], xs[13], xs[14], xs[15]));
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) xs[i] = 0.0f;
      }
      bmax = fmaxf(bmax, __shfl_xor_sync(0xFFFFFFFFu, bmax, 16));
      float *xw = xch + (c & 1) * CWARPS * 16;
      if (lane < 16) xw[warp * 16 + lane] = bmax;
      if (barrier_or(pair_bar, 64, !got || *abort_flag != 0)) {
        failed = true;
        break;
      }
      const float gmax = fmaxf(bmax, xw[(warp ^ 1) * 16 + (lane & 15)]);
      // s = bf16(f32(gmax / 7)) (0 below 2^-120), q = clamp(rne(f32(x^ * f32(1 / s))), -8, 7)
      const float sv = gmax < 0x1.0p-120f ? 0.0f : __bfloat162float(__float2bfloat16_rn(__fdiv_rn(gmax, 7.0f)));
      const float rcp = sv == 0.0f ? 0.0f : __frcp_rn(sv);
      uint32_t cw[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int q = min(7, max(-8, __float2int_rn(__fmul_rn(xs[i], rcp))));
        cw[i >> 3] |= (static_cast<uint32_t>(q) & 0xFu) << (4 * (i & 7));
      }
      *reinterpret_cast<uint2 *>(st + code_off) = make_uint2(cw[0], cw[1]);
      if ((cs & 1) == 0 && blk == 0)   // one writer per row and group
        reinterpret_cast<uint16_t *>(st + SC_OFF)[bx * 32 + row] = __bfloat16_as_ushort(__float2bfloat16_rn(sv));
      if (RANK > 0 && live) {
        // bf16(x^) back in place of x, as the A operand of the down-projection
        *reinterpret_cast<uint4 *>(xb + x_off0) =
            make_uint4(bf16x2(xs[0], xs[1]), bf16x2(xs[2], xs[3]), bf16x2(xs[4], xs[5]), bf16x2(xs[6], xs[7]));
        *reinterpret_cast<uint4 *>(xb + x_off1) =
            make_uint4(bf16x2(xs[8], xs[9]), bf16x2(xs[10], xs[11]), bf16x2(xs[12], xs[13]), bf16x2(xs[14], xs[15]));
        __syncwarp();
        const uint32_t xbase = dev::smem_u32(xb);
        const uint32_t lbase = dev::smem_u32(st + X_STAGE + bx * L1_BOX);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          uint32_t af[4];
          dev::ldmatrix_x4(xbase + sw_off(arow, acol + 16 * kk), af[0], af[1], af[2], af[3]);
#pragma unroll
          for (int np = 0; np < NT / 2; ++np) {
            uint32_t bq[4];
            dev::ldmatrix_x4(lbase + sw_off(np * 16 + brow, bcol + 16 * kk), bq[0], bq[1], bq[2], bq[3]);
            dev::mma_bf16_16816(acc[2 * np], af, bq[0], bq[1]);
            dev::mma_bf16_16816(acc[2 * np + 1], af, bq[2], bq[3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&done[s]);
    }
  } else {
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
      uint32_t sb = 0, code0 = 0, code1 = 0;
      if (bx < nbox) {   // warp-uniform: columns past K quantize as zeros (code and scale 0)
        uint8_t *xb = st + bx * X_BOX;
        const uint4 w0 = *reinterpret_cast<const uint4 *>(xb + x_off0);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(xb + x_off1);
        const float4 *iv = reinterpret_cast<const float4 *>(st + INV_OFF) + (bx * 64 + col) / 4;
        const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        // x^ of the block's 16 elements, in column order
        float xs[16];
  #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 v = iv[i];
          const float2 p0 = dev::mul2_rn(make_float2(bf16_lo(wv[2 * i]), bf16_hi(wv[2 * i])), make_float2(v.x, v.y));
          const float2 p1 = dev::mul2_rn(make_float2(bf16_lo(wv[2 * i + 1]), bf16_hi(wv[2 * i + 1])), make_float2(v.z, v.w));
          xs[4 * i] = p0.x;
          xs[4 * i + 1] = p0.y;
          xs[4 * i + 2] = p1.x;
          xs[4 * i + 3] = p1.y;
        }
        float amax = absmax4(xs[0], xs[1], xs[2], xs[3]);
        amax = fmaxf(amax, absmax4(xs[4], xs[5], xs[6], xs[7]));
        amax = fmaxf(amax, absmax4(xs[8], xs[9], xs[10], xs[11]));
        amax = fmaxf(amax, absmax4(xs[12], xs[13], xs[14], xs[15]));
        sb = dev::cvt_e4m3(__fdiv_rn(amax, d6));
        const float rinv = rinv_tab[sb];
        const float2 r2 = make_float2(rinv, rinv);
        uint32_t cw[4];
  #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 c0 = dev::mul2_rn(make_float2(xs[4 * i], xs[4 * i + 1]), r2);
          const float2 c1 = dev::mul2_rn(make_float2(xs[4 * i + 2], xs[4 * i + 3]), r2);
          cw[i] = dev::cvt_e2m1x4(c0.x, c0.y, c1.x, c1.y);     // code bytes 2i, 2i + 1
        }
        code0 = cw[0] | (cw[1] << 16);
        code1 = cw[2] | (cw[3] << 16);
        if (RANK > 0) {
          // bf16(x^) back in place of x, as the A operand of the down-projection
          *reinterpret_cast<uint4 *>(xb + x_off0) =
              make_uint4(bf16x2(xs[0], xs[1]), bf16x2(xs[2], xs[3]), bf16x2(xs[4], xs[5]), bf16x2(xs[6], xs[7]));
          *reinterpret_cast<uint4 *>(xb + x_off1) =
              make_uint4(bf16x2(xs[8], xs[9]), bf16x2(xs[10], xs[11]), bf16x2(xs[12], xs[13]), bf16x2(xs[14], xs[15]));
          __syncwarp();
          const uint32_t xbase = dev::smem_u32(xb);
          const uint32_t lbase = dev::smem_u32(st + X_STAGE + bx * L1_BOX);
  #pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            uint32_t af[4];
            dev::ldmatrix_x4(xbase + sw_off(arow, acol + 16 * kk), af[0], af[1], af[2], af[3]);
  #pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
              uint32_t bq[4];
              dev::ldmatrix_x4(lbase + sw_off(np * 16 + brow, bcol + 16 * kk), bq[0], bq[1], bq[2], bq[3]);
              dev::mma_bf16_16816(acc[2 * np], af, bq[0], bq[1]);
              dev::mma_bf16_16816(acc[2 * np + 1], af, bq[2], bq[3]);
            }
          }
        }
      }
      *reinterpret_cast<uint2 *>(st + code_off) = make_uint2(code0, code1);
      st[scale_off] = static_cast<uint8_t>(sb);
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&done[s]);
    }
  }

  // ---- U = (sum of the 8 slices' partial products of each row half) / (s_a s_w), bf16, 128-row tiles
  const int tid = threadIdx.x;  // 0..511
  constexpr int RS = RANK + 4;   // padded row of a partial tile
  constexpr int SLICES = CWARPS / 2;
  if (RANK > 0) {
    dev::named_barrier(1, (CWARPS + 1) * 32);      // the ring is no longer read (store warp included)
    float *red = reinterpret_cast<float *>(smem) + warp * 16 * RS;   // [CWARPS][16][RS]
    if (!failed) {
      const int g = lane >> 2, t = lane & 3;
#pragma unroll
      for (int n = 0; n < (NT > 0 ? NT : 1); ++n) {
        const int cc = n * 8 + 2 * t;
        *reinterpret_cast<float2 *>(red + g * RS + cc) = make_float2(acc[n][0], acc[n][1]);
        *reinterpret_cast<float2 *>(red + (g + 8) * RS + cc) = make_float2(acc[n][2], acc[n][3]);
      }
    }
    dev::named_barrier(2, CWARPS * 32);
  }
  // a wait that ran out anywhere leaves U zero (the status word carries the error)
  const bool any_failed = RANK > 0 && *abort_flag != 0;
  const float alpha = INT4 ? 1.0f : __fmul_rn(s_a, __ldg(p.s_w));
  // every thread: column pairs (2 cp, 2 cp + 1) of the CTA's rows, the slices' partials added in order
  for (int idx = tid; idx < BM * (SVDQ_LR_STRIDE / 2); idx += CWARPS * 32) {
    const int rr = idx / (SVDQ_LR_STRIDE / 2), cp = idx % (SVDQ_LR_STRIDE / 2);
    uint32_t o = 0;
    if (RANK > 0 && 2 * cp < RANK && !any_failed) {
      const float *red = reinterpret_cast<const float *>(smem) + ((rr >> 4) * SLICES * 16 + (rr & 15)) * RS + 2 * cp;
      float2 sum = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int w = 0; w < SLICES; ++w) {
        const float2 v = *reinterpret_cast<const float2 *>(red + w * 16 * RS);
        sum.x += v.x;
        sum.y += v.y;
      }
      o = bf16x2(__fdiv_rn(sum.x, alpha), __fdiv_rn(sum.y, alpha));
    }
    *reinterpret_cast<uint32_t *>(p.U + lowrank_offset(m0 + rr, 2 * cp, 128)) = o;
  }
}

template <int RANK, int G, bool INT4>
int launch(const Group<G> &g, int grid, cudaStream_t stream, const char *fn) {
  const int smem = smem_bytes<RANK>();
  const int rc = smem_optin_once<quant_act_kernel<RANK, G, INT4>>(smem, fn);
  if (rc != SVDQ_OK) return rc;
  DependentLaunch dl(dim3(grid), dim3(THREADS), smem, stream);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, quant_act_kernel<RANK, G, INT4>, g);
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

template <int G, bool INT4 = false>
int launch_rank(int rank, const Group<G> &g, int grid, cudaStream_t s, const char *fn) {
  switch (rank) {
    case 0: return launch<0, G, INT4>(g, grid, s, fn);
    case 16: return launch<16, G, INT4>(g, grid, s, fn);
    case 32: return launch<32, G, INT4>(g, grid, s, fn);
    case 48: return launch<48, G, INT4>(g, grid, s, fn);
    default: return launch<64, G, INT4>(g, grid, s, fn);
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

extern "C" int svdq_quantize_act_int4(const void *X, int M, int K, int ldx, const float *inv_lambda, const void *l1t,
                                      int rank, uint8_t *a_codes, void *a_scales, void *U, svdq_stream_t stream) {
  static const char *fn = "svdq_quantize_act_int4";
  if (!X || !inv_lambda || !a_codes || !a_scales || !U || (rank > 0 && !l1t))
    return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": null pointer");
  if (M < 1 || K < 64 || K % 64 || ldx < K || ldx % 8)
    return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": need M >= 1, K % 64 == 0, ldx >= K, ldx % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": rank must be a multiple of 16 in [0, 64]");
  if (!aligned16(X) || !aligned16(inv_lambda) || !aligned16(a_codes) || !aligned16(a_scales) || !aligned16(U) ||
      (rank > 0 && !aligned16(l1t)))
    return fail(SVDQ_ERR_ALIGNMENT, std::string(fn) + ": pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  Group<1> g{};
  Params &p = g.p[0];
  p.M = M;
  p.K = K;
  p.KS = bundle_ks(K);
  p.inv_lambda = inv_lambda;
  p.codes4 = a_codes;
  p.scales4 = static_cast<uint16_t *>(a_scales);
  p.ld_s = (M + 127) / 128 * 128;
  p.U = static_cast<uint8_t *>(U);
  p.status = st->status_word;
  p.limit_ns = kWaitLimitNs;
  const int rc = encode_problem(X, M, K, ldx, l1t, rank, &g.tx[0], &g.tl[0]);
  if (rc != SVDQ_OK) return rc;
  const int grid = (M + 127) / 128 * (128 / BM);
  g.blk_end[0] = grid;
  g.count = 1;
  return launch_rank<1, true>(rank, g, grid, reinterpret_cast<cudaStream_t>(stream), fn);
}
