// K3: AWQ W4A16 projection for small row counts (modulation / adaLN layers).
//
// The pages give these precision-sensitive, low-compute projections 4-bit
// weights and 16-bit activations (web page "Nunchaku Diffusers 支持降低显存占用，
// 但硬件仍决定适用范围", remio.ai, section "Nunchaku Diffusers 支持改变了加载路径").
// With up to 16 rows the layer is one pass over the weights and the kernel
// is bound by how many weight bytes are in flight:
//   * one CTA of 8 warps per quad of 64 output columns, two CTAs per SM (at
//     the adaLN widths every CTA of the grid is resident at once).  A quad's
//     weights are contiguous (quad-major layout), so one thread requests them
//     at the start with bulk copies into a shared-memory ring of chunks of 8
//     groups of 64 along K (16 KB of codes + 1 KB of scales + 1 KB of zero
//     points each, 6 chunks = K 3072 in flight per CTA, ~200 KB per SM);
//     longer K refills a chunk once all 8 warps have consumed it;
//   * warp w takes group w of every chunk, reading its four 16-column blocks
//     (512 bytes each, lane-contiguous) from shared memory as soon as the
//     chunk's barrier completes;
//   * the products run on the tensor cores as Y^T = W^T . X^T (mma.sync
//     m16n8k16: 16 output columns x 16 k per instruction, the rows of X in
//     the 8-wide slot); X^ = f32(x * inv_awq) is split into bf16 hi + lo
//     parts (hi + lo carries ~16 significant bits).  Up to 4 rows, the hi
//     parts fill slots 0..3 and the lo parts slots 4..7 of one MMA, added
//     at the end; more rows take one MMA per part;
//   * dequantization in registers: two nibbles at a time become a bf16 pair
//     (128 + q) by one mask-and-or.  With one block of rows the zero point
//     leaves the inner loop: an MMA with an all-ones A fragment gives
//     sum_k b per row, and the group's sum of (q - z) b is
//     sum (128 + q) b - (128 + z) sum b, one f32 fma per output; two row
//     blocks subtract 128 + z from every pair (bf16x2, exact) instead;
//   * per group the fp32 partial is scaled by s in registers; the warps'
//     partials are added through shared memory (the ring, once drained).
// More than 16 rows (a batch of modulation vectors) run as blocks of 16 rows
// on the grid's second dimension; each block is one more pass over the
// weights, mostly from L2.
// A grouped launch runs several projections of the same input shape (the
// modulation layers of a DiT step all read the same conditioning vector):
// their quads form one sequence on the grid's first dimension, problem after
// problem, and each CTA finds its problem by a binary search over the prefix
// sums of the quad counts.  A single call is a group of one (no search).
// The weight layout (qweight) is the MMA fragment order; see svdq.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <string>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }
// bf16 (128 + q) for the two nibbles at bits [0, 4) and [16, 20) of w.
__device__ __forceinline__ uint32_t nib_pair(uint32_t w) { return (w & 0x000F000Fu) | 0x43004300u; }

// (q - z) as bf16 pairs, exact: (128 + q) - (128 + z) for the two nibbles of nib_pair(w).
__device__ __forceinline__ uint32_t minus_zero(uint32_t a128, uint32_t z128) {
  __nv_bfloat162 d = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&a128), *reinterpret_cast<__nv_bfloat162 *>(&z128));
  return *reinterpret_cast<uint32_t *>(&d);
}
// bf16 1.0 in both halves: the all-ones A fragment that sums B over k
constexpr uint32_t kOnes = 0x3F803F80u;

struct Params {
  int M, K, N, ldx, ldy, G;
  const uint16_t *X;
  const float *inv;
  const uint4 *qw;
  const uint16_t *scales, *zeros, *bias;
  uint16_t *Y;
  unsigned int *status;
  unsigned long long limit_ns;
};

// Up to C problems of the same M and K in one launch; quad_end holds the prefix sums of
// their quad counts (N / 64).
constexpr int kAwqMaxGroup = SVDQ_AWQ_MAX_GROUP;
template <int C>
struct AwqGroup {
  Params p[C];
  int quad_end[C];
  int count;
};

// The raw X words and inv_awq pairs a lane needs for the four k16 steps of
// one group (rows nt*8+g, columns 16j+2t, +1, +8, +9): fetched in one go,
// before the group's weights have landed, so that their latency overlaps
// the wait instead of stalling every k16 step.
template <int NT>
struct XRaw {
  uint32_t w[4][NT][2];
  float2 iv[4][2];
};
// row(nt): the row of X whose words lane slot nt carries (rows past M read as zeros).
template <int NT, typename RowOf>
__device__ __forceinline__ void fetch_x(const Params &p, int k0, RowOf row, int j0, int j1, XRaw<NT> &r) {
#pragma unroll
  for (int j = j0; j < j1; ++j) {
    const int k = k0 + 16 * j;
    r.iv[j][0] = p.inv ? __ldg(reinterpret_cast<const float2 *>(p.inv + k)) : make_float2(1.f, 1.f);
    r.iv[j][1] = p.inv ? __ldg(reinterpret_cast<const float2 *>(p.inv + k + 8)) : make_float2(1.f, 1.f);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = row(nt);
      r.w[j][nt][0] = m < p.M ? __ldg(reinterpret_cast<const uint32_t *>(p.X + static_cast<size_t>(m) * p.ldx + k)) : 0u;
      r.w[j][nt][1] =
          m < p.M ? __ldg(reinterpret_cast<const uint32_t *>(p.X + static_cast<size_t>(m) * p.ldx + k + 8)) : 0u;
    }
  }
}
// B fragments (hi and lo bf16 parts of X^ = f32(x * inv_awq)) of k16 step j.
template <int NT>
__device__ __forceinline__ void split_x(const XRaw<NT> &r, int j, uint32_t (&bh)[NT][2], uint32_t (&bl)[NT][2]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const uint32_t w0 = r.w[j][nt][0], w1 = r.w[j][nt][1];
    float x[4];
    x[0] = __fmul_rn(__uint_as_float(w0 << 16), r.iv[j][0].x);
    x[1] = __fmul_rn(__uint_as_float(w0 & 0xFFFF0000u), r.iv[j][0].y);
    x[2] = __fmul_rn(__uint_as_float(w1 << 16), r.iv[j][1].x);
    x[3] = __fmul_rn(__uint_as_float(w1 & 0xFFFF0000u), r.iv[j][1].y);
    float h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
      l[i] = x[i] - h[i];  // exact
    }
    bh[nt][0] = pack_bf16x2(h[0], h[1]);
    bh[nt][1] = pack_bf16x2(h[2], h[3]);
    bl[nt][0] = pack_bf16x2(l[0], l[1]);
    bl[nt][1] = pack_bf16x2(l[2], l[3]);
  }
}

// B fragments of k16 step j with the hi and lo parts in one MMA (up to 4
// rows): lane (g, t) carries part g >> 2 (0: hi, 1: lo) of row g & 3, so n
// slots 0..3 hold the rows' hi parts and 4..7 their lo parts.  lo_sel is 0
// on hi lanes and -1 on lo lanes: x^ + lo_sel f32(bf16(x^)) is x^ itself or
// the exact remainder x^ - hi, then rounded to bf16 like the hi part.
__device__ __forceinline__ void split_x_merged(const XRaw<1> &r, int j, float lo_sel, uint32_t (&b)[2]) {
  const uint32_t w0 = r.w[j][0][0], w1 = r.w[j][0][1];
  const float2 x01 = dev::mul2_rn(make_float2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xFFFF0000u)),
                                  r.iv[j][0]);
  const float2 x23 = dev::mul2_rn(make_float2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xFFFF0000u)),
                                  r.iv[j][1]);
  const uint32_t h01 = pack_bf16x2(x01.x, x01.y), h23 = pack_bf16x2(x23.x, x23.y);
  const float2 sel = make_float2(lo_sel, lo_sel);
  const float2 v01 = dev::fma2_rn(make_float2(bf16_bits_to_float(h01 & 0xFFFFu), bf16_bits_to_float(h01 >> 16)), sel, x01);
  const float2 v23 = dev::fma2_rn(make_float2(bf16_bits_to_float(h23 & 0xFFFFu), bf16_bits_to_float(h23 >> 16)), sel, x23);
  b[0] = pack_bf16x2(v01.x, v01.y);
  b[1] = pack_bf16x2(v23.x, v23.y);
}

// ===========================================================================
// One CTA per quad (64 output columns) and block of 8 NT rows.
constexpr int S_THREADS = 256;
constexpr int S_WARPS = S_THREADS / 32;
constexpr int CHUNK_G = S_WARPS;                 // groups per chunk: one per warp
constexpr int CHUNK_QW = CHUNK_G * 2048;         // codes: 2 KB per group (four 16-column blocks)
constexpr int CHUNK_SZ = CHUNK_G * 128;          // scales (and zero points): 64 bf16 per group
constexpr int CHUNK_BYTES = CHUNK_QW + 2 * CHUNK_SZ;
constexpr int RING = 6;
constexpr int BAR_OFF = RING * CHUNK_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 2 * RING * 8 + 16;
static_assert(S_WARPS * 4 * 2 * 32 * 4 * 4 <= BAR_OFF, "the partial sums fit the drained ring");

// MERGED: up to 4 rows, the hi and lo parts of X^ in one MMA (NT = 1).
template <int NT, bool MERGED, int C>
__global__ void __launch_bounds__(S_THREADS, 2) awq_gemv_kernel(const __grid_constant__ AwqGroup<C> grp) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + BAR_OFF);
  uint64_t *empty = full + RING;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + RING);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t = lane & 3;
  int pi = 0;                                     // this CTA's problem
  if constexpr (C > 1) {
    int lo = 0, hi = grp.count - 1;
    while (lo < hi) {                             // the first problem whose quads end past blockIdx.x
      const int mid = (lo + hi) >> 1;
      if (static_cast<int>(blockIdx.x) < grp.quad_end[mid]) hi = mid; else lo = mid + 1;
    }
    pi = lo;
  }
  Params p = grp.p[pi];
  const int quad = static_cast<int>(blockIdx.x) - (pi > 0 ? grp.quad_end[pi - 1] : 0);
  const int nchunks = (p.G + CHUNK_G - 1) / CHUNK_G;
  {  // this CTA's block of 8 NT rows
    const int r0 = static_cast<int>(blockIdx.y) * 8 * NT;
    p.X += static_cast<size_t>(r0) * p.ldx;
    p.Y += static_cast<size_t>(r0) * p.ldy;
    p.M = min(8 * NT, p.M - r0);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      dev::mbar_init(&full[s], 1);
      dev::mbar_init(&empty[s], S_WARPS);
    }
    *abort_flag = 0;
    dev::fence_mbar_init();
  }
  __syncthreads();
  dev::grid_dependency_wait();
  dev::grid_launch_dependents();

  // chunk c: groups 8c .. 8c+7 of the quad, into ring slot c % RING
  auto issue = [&](int c) {
    uint8_t *dst = smem + (c % RING) * CHUNK_BYTES;
    const int g0 = c * CHUNK_G, ng = min(CHUNK_G, p.G - g0);
    const size_t blk = static_cast<size_t>(quad) * p.G + g0;
    uint64_t *bar = &full[c % RING];
    dev::mbar_arrive_expect_tx(bar, static_cast<uint32_t>(ng * (2048 + 2 * 128)));
    dev::bulk_load(dst, p.qw + blk * 128, static_cast<uint32_t>(ng * 2048), bar);
    dev::bulk_load(dst + CHUNK_QW, p.scales + blk * 64, static_cast<uint32_t>(ng * 128), bar);
    dev::bulk_load(dst + CHUNK_QW + CHUNK_SZ, p.zeros + blk * 64, static_cast<uint32_t>(ng * 128), bar);
  };
  int issued = 0;
  if (threadIdx.x == 0)
    for (; issued < min(RING, nchunks); ++issued) issue(issued);

  float tot[4][NT][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < NT; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) tot[a][b][e] = 0.0f;

  static_assert(!MERGED || NT == 1, "the merged form carries one block of 4 rows");
  constexpr bool FOLD = NT == 1;
  // the row of X a lane's B slot nt carries
  auto row_of = [&](int nt) { return MERGED ? (g8 & 3) : nt * 8 + g8; };
  const float lo_sel = MERGED && g8 >= 4 ? -1.0f : 0.0f;
  const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};

#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int slot = c % RING;
    const int grp = c * CHUNK_G + warp;
    XRaw<NT> xr;
    // one row block (the modulation layers): all four steps' X up front; two row blocks would
    // hold twice the registers, so those fetch each step's X where it is used
    if (NT == 1 && grp < p.G) fetch_x<NT>(p, grp * 64 + 2 * t, row_of, 0, 4, xr);
    if (!dev::mbar_wait_warp(&full[slot], (c / RING) & 1, p.limit_ns, abort_flag)) {
      *abort_flag = 1;
      dev::report(p.status, SVDQ_ERR_TIMEOUT);
      break;
    }
    if (grp < p.G) {
      const uint8_t *src = smem + slot * CHUNK_BYTES;
      uint4 wq[4];
      uint32_t sp[4], zp[4];  // bf16 s and z of columns g (low half) and g + 8 (high half) of each block
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        wq[cb] = reinterpret_cast<const uint4 *>(src + warp * 2048)[cb * 32 + lane];
        const uint16_t *sc = reinterpret_cast<const uint16_t *>(src + CHUNK_QW + warp * 128) + cb * 16 + g8;
        const uint16_t *zc = reinterpret_cast<const uint16_t *>(src + CHUNK_QW + CHUNK_SZ + warp * 128) + cb * 16 + g8;
        sp[cb] = static_cast<uint32_t>(sc[0]) | (static_cast<uint32_t>(sc[8]) << 16);
        zp[cb] = static_cast<uint32_t>(zc[0]) | (static_cast<uint32_t>(zc[8]) << 16);
      }
      // one row block (FOLD): acc = sum_k (128 + q) b and sx = sum_k b over the group's 64 k, and
      // sum_k (q - z) b = acc - (128 + z) sx, taken once per group in f32; two row blocks
      // (registers for sx would spill) subtract 128 + z from every pair instead
      uint32_t z128[4][2];
      if constexpr (!FOLD) {
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          const float zl = 128.0f + bf16_bits_to_float(zp[cb] & 0xFFFFu), zh = 128.0f + bf16_bits_to_float(zp[cb] >> 16);
          z128[cb][0] = pack_bf16x2(zl, zl);
          z128[cb][1] = pack_bf16x2(zh, zh);
        }
      }
      float acc[4][NT][4], sx[NT][4];
#pragma unroll
      for (int b = 0; b < NT; ++b)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sx[b][e] = 0.0f;
#pragma unroll
          for (int a = 0; a < 4; ++a) acc[a][b][e] = 0.0f;
        }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t bh[NT][2], bl[NT][2];
        if constexpr (MERGED) {
          split_x_merged(xr, j, lo_sel, bh[0]);
        } else {
          if (NT > 1) fetch_x<NT>(p, grp * 64 + 2 * t, row_of, j, j + 1, xr);
          split_x<NT>(xr, j, bh, bl);
        }
        if constexpr (FOLD) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            dev::mma_bf16_16816(sx[nt], ones, bh[nt][0], bh[nt][1]);
            if (!MERGED) dev::mma_bf16_16816(sx[nt], ones, bl[nt][0], bl[nt][1]);
          }
        }
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          const uint32_t w = j == 0 ? wq[cb].x : j == 1 ? wq[cb].y : j == 2 ? wq[cb].z : wq[cb].w;
          // (128 + q) as bf16 pairs: columns g / g + 8 at k 2t, 2t+1 (a0 / a1) and 2t+8, 2t+9 (a2 / a3)
          uint32_t a[4] = {nib_pair(w), nib_pair(w >> 4), nib_pair(w >> 8), nib_pair(w >> 12)};
          if constexpr (!FOLD) {
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = minus_zero(a[i], z128[cb][i & 1]);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            dev::mma_bf16_16816(acc[cb][nt], a, bh[nt][0], bh[nt][1]);
            if (!MERGED) dev::mma_bf16_16816(acc[cb][nt], a, bl[nt][0], bl[nt][1]);
          }
        }
      }
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        // C rows g (e < 2) and g + 8 (e >= 2) are the block's columns g and g + 8
        const float s_lo = bf16_bits_to_float(sp[cb] & 0xFFFFu), s_hi = bf16_bits_to_float(sp[cb] >> 16);
        const float z_lo = 128.0f + bf16_bits_to_float(zp[cb] & 0xFFFFu), z_hi = 128.0f + bf16_bits_to_float(zp[cb] >> 16);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            tot[cb][nt][e] = __fmaf_rn(
                e < 2 ? s_lo : s_hi,
                FOLD ? __fmaf_rn(-(e < 2 ? z_lo : z_hi), sx[nt][e], acc[cb][nt][e]) : acc[cb][nt][e], tot[cb][nt][e]);
      }
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[slot]);
    // a longer K: refill this slot with chunk c + RING once every warp has read it
    if (threadIdx.x == 0 && issued < nchunks) {
      if (!dev::mbar_wait(&empty[slot], (c / RING) & 1, p.limit_ns, abort_flag)) {
        *abort_flag = 1;
        dev::report(p.status, SVDQ_ERR_TIMEOUT);
      } else {
        issue(issued++);
      }
    }
  }
  // every copy this CTA issued has landed before its shared memory is reused or released
  if (threadIdx.x == 0)
    for (int c = max(0, issued - RING); c < issued; ++c)
      dev::mbar_wait(&full[c % RING], (c / RING) & 1, p.limit_ns, nullptr);
  __syncthreads();

  if constexpr (MERGED) {
    // n slots 4..7 (lanes t = 2, 3) hold the lo parts of the rows in slots 0..3 (lanes t = 0, 1)
#pragma unroll
    for (int cb = 0; cb < 4; ++cb)
#pragma unroll
      for (int e = 0; e < 4; ++e) tot[cb][0][e] += __shfl_xor_sync(0xFFFFFFFFu, tot[cb][0][e], 2);
  }
  float *red = reinterpret_cast<float *>(smem);  // [WARPS][4][NT][32][4]
#pragma unroll
  for (int cb = 0; cb < 4; ++cb)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) red[(((warp * 4 + cb) * NT + nt) * 32 + lane) * 4 + e] = tot[cb][nt][e];
  __syncthreads();
  if (*abort_flag) return;                        // Y is left as it was; the status word has the error

  constexpr int SLOTS = 4 * NT * 32 * 4;
  for (int slot = threadIdx.x; slot < SLOTS; slot += S_THREADS) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < S_WARPS; ++w) v += red[w * SLOTS + slot];
    const int e = slot & 3, ln = (slot >> 2) & 31, nt = (slot >> 7) % NT, cb = (slot >> 7) / NT;
    const int n = quad * 64 + cb * 16 + (ln >> 2) + (e >= 2 ? 8 : 0);
    const int m = nt * 8 + 2 * (ln & 3) + (e & 1);
    if (m < p.M) {
      if (p.bias) v += bf16_bits_to_float(p.bias[n]);
      __nv_bfloat16 h = __float2bfloat16_rn(v);
      p.Y[static_cast<size_t>(m) * p.ldy + n] = *reinterpret_cast<uint16_t *>(&h);
    }
  }
}

template <int NT, bool MERGED, int C>
int launch(const AwqGroup<C> &g, int total_quads, int M, cudaStream_t stream, const char *fn) {
  const int rc = smem_optin_once<awq_gemv_kernel<NT, MERGED, C>>(SMEM_BYTES, fn);
  if (rc != SVDQ_OK) return rc;
  DependentLaunch dl(dim3(total_quads, (M + 8 * NT - 1) / (8 * NT)), dim3(S_THREADS), SMEM_BYTES, stream);
  cudaError_t e = cudaLaunchKernelEx(&dl.cfg, awq_gemv_kernel<NT, MERGED, C>, g);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + " launch: " + cudaGetErrorString(e));
  return ok();
}

// up to 4 rows: hi and lo parts in one MMA; up to 8: one block of rows; more: blocks of 16
// rows, one pass over the weights each
template <int C>
int launch_rows(const AwqGroup<C> &g, int total_quads, int M, cudaStream_t s, const char *fn) {
  if (M <= 4) return launch<1, true, C>(g, total_quads, M, s, fn);
  return M > 8 ? launch<2, false, C>(g, total_quads, M, s, fn) : launch<1, false, C>(g, total_quads, M, s, fn);
}

// Checks one problem and fills its parameter block (all but the status word).
int make_problem(const char *fn, const void *X, int M, int K, int ldx, const float *inv_awq, const uint32_t *qweight,
                 const void *scales, const void *zeros, const void *bias, int N, void *Y, int ldy, Params *p) {
  const std::string name(fn);
  if (!X || !qweight || !scales || !zeros || !Y) return fail(SVDQ_ERR_INVALID_ARG, name + ": null pointer");
  if (M < 1 || M > 65535 * 16 || K < 64 || K % 64 || N < 64 || N % 64 || ldx < K || ldx % 8 || ldy < N ||
      ldy % 8)
    return fail(SVDQ_ERR_SHAPE, name + ": need 1 <= M <= 1048560, K % 64 == 0, N % 64 == 0, ldx >= K, "
                                       "ldy >= N, ldx/ldy % 8 == 0");
  if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
      (inv_awq && !aligned16(inv_awq)) || !aligned16(Y))
    return fail(SVDQ_ERR_ALIGNMENT, name + ": pointers must be 16-byte aligned");
  *p = Params{};
  p->M = M;
  p->K = K;
  p->N = N;
  p->ldx = ldx;
  p->ldy = ldy;
  p->G = K / 64;
  p->X = static_cast<const uint16_t *>(X);
  p->inv = inv_awq;
  p->qw = reinterpret_cast<const uint4 *>(qweight);
  p->scales = static_cast<const uint16_t *>(scales);
  p->zeros = static_cast<const uint16_t *>(zeros);
  p->bias = static_cast<const uint16_t *>(bias);
  p->Y = static_cast<uint16_t *>(Y);
  p->limit_ns = kWaitLimitNs;
  return SVDQ_OK;
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int awq_linear_w4a16(const void *X, int M, int K, int ldx, const float *inv_awq, const uint32_t *qweight,
                                const void *scales, const void *zeros, int group, const void *bias, int N, void *Y,
                                int ldy, svdq_stream_t stream) {
  const char *fn = "awq_linear_w4a16";
  if (!X || !qweight || !scales || !zeros || !Y) return fail(SVDQ_ERR_INVALID_ARG, "awq_linear_w4a16: null pointer");
  if (group != 64) return fail(SVDQ_ERR_SHAPE, "awq_linear_w4a16: group must be 64");
  AwqGroup<1> g;
  // shapes and alignment first (no device needed), then the device state
  int rc = make_problem(fn, X, M, K, ldx, inv_awq, qweight, scales, zeros, bias, N, Y, ldy, &g.p[0]);
  if (rc != SVDQ_OK) return rc;
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  g.p[0].status = st->status_word;
  g.quad_end[0] = N / 64;
  g.count = 1;
  return launch_rows<1>(g, N / 64, M, reinterpret_cast<cudaStream_t>(stream), fn);
}

extern "C" int awq_linear_w4a16_grouped(const awq_problem_t *problems, int count, int M, int K, int group,
                                        svdq_stream_t stream) {
  const char *fn = "awq_linear_w4a16_grouped";
  if (!problems || count < 1 || count > kAwqMaxGroup)
    return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": need 1 <= count <= " + std::to_string(kAwqMaxGroup));
  if (group != 64) return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": group must be 64");
  static thread_local AwqGroup<kAwqMaxGroup> g;   // ~13 KB: kept off the stack
  int total = 0;
  for (int i = 0; i < count; ++i) {
    const awq_problem_t &q = problems[i];
    const int rc = make_problem(fn, q.X, M, K, q.ldx, q.inv_awq, q.qweight, q.scales, q.zeros, q.bias, q.N, q.Y,
                                q.ldy, &g.p[i]);
    if (rc != SVDQ_OK) return rc;
    if (total > (1 << 30) - q.N / 64) return fail(SVDQ_ERR_SHAPE, std::string(fn) + ": too many columns in one launch");
    total += q.N / 64;
    g.quad_end[i] = total;
  }
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  for (int i = 0; i < count; ++i) g.p[i].status = st->status_word;
  for (int i = count; i < kAwqMaxGroup; ++i) g.quad_end[i] = total;
  g.count = count;
  return launch_rows<kAwqMaxGroup>(g, total, M, reinterpret_cast<cudaStream_t>(stream), fn);
}
