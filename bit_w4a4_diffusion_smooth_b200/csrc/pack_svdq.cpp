// Offline (host) quantization of one SVDQuant layer: smoothing, top-r SVD
// branch, residual, NVFP4 packing.
//
// Follows the layer as the pages describe it (web page "Nunchaku Diffusers
// 支持降低显存占用，但硬件仍决定适用范围", remio.ai, section "SVDQuant 将棘手数值移出
// 4 位路径": activation outliers are moved into the weight, a small 16-bit
// low-rank branch holds the hardest part, the residual runs in 4 bits) and
// the quantize step of the offline workflow ("Diffusers × Nunchaku 4-bit",
// donmalab.com, section "自行量化模型的流程").
//
// Arithmetic: float64 for smoothing, SVD and residual; float32 with one IEEE
// rounding per operation for the NVFP4 decisions (built with
// -ffp-contract=off so no multiply-add is fused).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <functional>
#include <random>
#include <thread>
#include <vector>

#include "svdq_internal.h"

namespace svdq {
namespace {

float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round a double to the nearest bf16 (ties to even) in one step and return
// its bit pattern.  The spacing of bf16 around |v| is 2^(e-7) (8 significant
// bits), floored at the subnormal spacing 2^-133.
uint16_t bf16_bits_from_double(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  int e2;
  std::frexp(a, &e2);  // a = f * 2^e2, f in [0.5, 1)
  int e = std::max(e2 - 1, -126);
  double quantum = std::ldexp(1.0, e - 7);
  double r = std::nearbyint(a / quantum) * quantum;  // default rounding: ties to even
  float f = static_cast<float>(std::copysign(r, v));  // exact: r has <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16);
}

// e2m1 magnitudes by code, from the format: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
const float kE2m1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

// Nearest e2m1 code (ties to the even code), saturating at 6; the sign bit
// follows the sign of the input, zero included.
uint8_t e2m1_code(float y) {
  uint8_t s = std::signbit(y) ? 8 : 0;
  float a = std::fabs(y);
  if (!(a < 6.0f)) return s | 7;
  int best = 0;
  float bd = a;
  for (int c = 1; c < 8; ++c) {
    float d = std::fabs(a - kE2m1Mag[c]);
    if (d < bd || (d == bd && (c & 1) == 0)) {
      bd = d;
      best = c;
    }
  }
  return static_cast<uint8_t>(s | best);
}

// Table of the 127 finite non-negative e4m3 values, increasing with the code.
struct E4m3Table {
  float v[127];
  E4m3Table() {
    for (int c = 0; c < 127; ++c) {
      int e = c >> 3, m = c & 7;
      v[c] = e == 0 ? std::ldexp(static_cast<float>(m), -9)
                    : std::ldexp(1.0f + static_cast<float>(m) / 8.0f, e - 7);
    }
  }
};
const E4m3Table kE4m3;

// Nearest finite e4m3 code of x >= 0 (ties to the even code), saturating at 448.
uint8_t ue4m3_code(float x) {
  if (!(x < 448.0f)) return 126;
  const float *lo = std::upper_bound(kE4m3.v, kE4m3.v + 127, x);
  int hi_c = static_cast<int>(lo - kE4m3.v);  // first code with value > x
  if (hi_c == 0) return 0;
  int lo_c = hi_c - 1;
  if (hi_c > 126) return 126;
  float dl = x - kE4m3.v[lo_c], dh = kE4m3.v[hi_c] - x;
  if (dl < dh) return static_cast<uint8_t>(lo_c);
  if (dh < dl) return static_cast<uint8_t>(hi_c);
  return static_cast<uint8_t>((lo_c & 1) == 0 ? lo_c : hi_c);
}

float tensor_scale(float amax) { return amax == 0.0f ? 1.0f : amax / 2688.0f; }

void parallel_for(int n, int threads, const std::function<void(int, int)> &fn);

}  // namespace

// ---------------------------------------------------------------------------
// Threading helper
namespace {
void parallel_for(int n, int threads, const std::function<void(int, int)> &fn) {
  if (threads <= 1 || n < 2) {
    fn(0, n);
    return;
  }
  threads = std::min(threads, n);
  std::vector<std::thread> pool;
  int chunk = (n + threads - 1) / threads;
  for (int t = 0; t < threads; ++t) {
    int b = t * chunk, e = std::min(n, b + chunk);
    if (b >= e) break;
    pool.emplace_back([=, &fn] { fn(b, e); });
  }
  for (auto &th : pool) th.join();
}

// Dense row-major helpers.  A is [rows][cols].
// Y[rows][p] = A . X, X [cols][p].  Four rows of A share each pass over X;
// every output still sums its terms in order j = 0, 1, ...
void mul_a_x(const double *A, int rows, int cols, const double *X, int p, double *Y, int threads) {
  parallel_for((rows + 3) / 4, threads, [&](int b, int e) {
    std::vector<double> acc(4 * static_cast<size_t>(p));
    for (int i0 = 4 * b; i0 < std::min(rows, 4 * e); i0 += 4) {
      const int nr = std::min(4, rows - i0);
      std::fill(acc.begin(), acc.end(), 0.0);
      const double *a = A + static_cast<size_t>(i0) * cols;
      for (int j = 0; j < cols; ++j) {
        const double *x = X + static_cast<size_t>(j) * p;
        for (int r = 0; r < nr; ++r) {
          const double arj = a[static_cast<size_t>(r) * cols + j];
          double *ac = acc.data() + static_cast<size_t>(r) * p;
          for (int t = 0; t < p; ++t) ac[t] += arj * x[t];
        }
      }
      for (int r = 0; r < nr; ++r)
        std::copy(acc.begin() + static_cast<size_t>(r) * p, acc.begin() + static_cast<size_t>(r + 1) * p,
                  Y + static_cast<size_t>(i0 + r) * p);
    }
  });
}
// Z[cols][p] = A^T . Q, Q [rows][p]
void mul_at_q(const double *A, int rows, int cols, const double *Q, int p, double *Z, int threads) {
  const int tile = 256;
  int ntiles = (cols + tile - 1) / tile;
  parallel_for(ntiles, threads, [&](int b, int e) {
    for (int tt = b; tt < e; ++tt) {
      int c0 = tt * tile, c1 = std::min(cols, c0 + tile);
      double *z = Z + static_cast<size_t>(c0) * p;
      std::fill(z, z + static_cast<size_t>(c1 - c0) * p, 0.0);
      for (int i = 0; i < rows; ++i) {
        const double *a = A + static_cast<size_t>(i) * cols;
        const double *q = Q + static_cast<size_t>(i) * p;
        for (int c = c0; c < c1; ++c) {
          double aic = a[c];
          double *zc = Z + static_cast<size_t>(c) * p;
          for (int t = 0; t < p; ++t) zc[t] += aic * q[t];
        }
      }
    }
  });
}

// Orthonormalize the p columns of Y [rows][p] in place (modified Gram-Schmidt,
// applied twice for stability).  Columns that vanish are left zero.  The
// columns are worked on in a column-major copy, so that every dot product and
// update streams contiguous memory (the sums run over rows in the same order).
void orthonormalize(double *Y, int rows, int p) {
  std::vector<double> colmaj(static_cast<size_t>(rows) * p);
  for (int i = 0; i < rows; ++i)
    for (int c = 0; c < p; ++c) colmaj[static_cast<size_t>(c) * rows + i] = Y[static_cast<size_t>(i) * p + c];
  for (int pass = 0; pass < 2; ++pass) {
    for (int c = 0; c < p; ++c) {
      double *yc = colmaj.data() + static_cast<size_t>(c) * rows;
      for (int d = 0; d < c; ++d) {
        const double *yd = colmaj.data() + static_cast<size_t>(d) * rows;
        double dot = 0.0;
        for (int i = 0; i < rows; ++i) dot += yc[i] * yd[i];
        for (int i = 0; i < rows; ++i) yc[i] -= dot * yd[i];
      }
      double nrm = 0.0;
      for (int i = 0; i < rows; ++i) nrm += yc[i] * yc[i];
      nrm = std::sqrt(nrm);
      double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
      for (int i = 0; i < rows; ++i) yc[i] *= inv;
    }
  }
  for (int i = 0; i < rows; ++i)
    for (int c = 0; c < p; ++c) Y[static_cast<size_t>(i) * p + c] = colmaj[static_cast<size_t>(c) * rows + i];
}

}  // namespace

// Eigen-decomposition of the symmetric p x p matrix C (row-major) by cyclic
// Jacobi rotations.  On return the eigenvalues are on C's diagonal and the
// eigenvectors are the columns of V.
void jacobi_eigen(std::vector<double> &C, int p, std::vector<double> &V) {
  V.assign(static_cast<size_t>(p) * p, 0.0);
  for (int i = 0; i < p; ++i) V[static_cast<size_t>(i) * p + i] = 1.0;
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < p; ++i)
      for (int j = 0; j < p; ++j)
        (i == j ? diag : off) += C[static_cast<size_t>(i) * p + j] * C[static_cast<size_t>(i) * p + j];
    if (off <= 1e-30 * diag || off == 0.0) break;
    for (int a = 0; a < p - 1; ++a) {
      for (int b = a + 1; b < p; ++b) {
        double cab = C[static_cast<size_t>(a) * p + b];
        if (cab == 0.0) continue;
        double caa = C[static_cast<size_t>(a) * p + a], cbb = C[static_cast<size_t>(b) * p + b];
        double theta = (cbb - caa) / (2.0 * cab);
        double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < p; ++k) {  // C <- C J (columns a, b)
          double cka = C[static_cast<size_t>(k) * p + a], ckb = C[static_cast<size_t>(k) * p + b];
          C[static_cast<size_t>(k) * p + a] = c * cka - s * ckb;
          C[static_cast<size_t>(k) * p + b] = s * cka + c * ckb;
        }
        for (int k = 0; k < p; ++k) {  // C <- J^T C (rows a, b)
          double cak = C[static_cast<size_t>(a) * p + k], cbk = C[static_cast<size_t>(b) * p + k];
          C[static_cast<size_t>(a) * p + k] = c * cak - s * cbk;
          C[static_cast<size_t>(b) * p + k] = s * cak + c * cbk;
        }
        for (int k = 0; k < p; ++k) {
          double vka = V[static_cast<size_t>(k) * p + a], vkb = V[static_cast<size_t>(k) * p + b];
          V[static_cast<size_t>(k) * p + a] = c * vka - s * vkb;
          V[static_cast<size_t>(k) * p + b] = s * vka + c * vkb;
        }
      }
    }
  }
}

namespace {

// Standard normal draws from a fully specified engine (mt19937_64) through
// Box-Muller, so the pack is reproducible across C++ libraries.
void gaussian_fill(double *x, size_t n, uint64_t seed) {
  std::mt19937_64 eng(seed);
  const double two_pi = 6.283185307179586;
  for (size_t i = 0; i < n; i += 2) {
    double u1 = (static_cast<double>(eng() >> 11) + 1.0) * 0x1.0p-53;  // (0, 1]
    double u2 = static_cast<double>(eng() >> 11) * 0x1.0p-53;          // [0, 1)
    double r = std::sqrt(-2.0 * std::log(u1));
    x[i] = r * std::cos(two_pi * u2);
    if (i + 1 < n) x[i + 1] = r * std::sin(two_pi * u2);
  }
}

// Orthonormal basis Ur [K][r] of the dominant r-dimensional column space of
// Wp [K][N]: randomized subspace iteration with oversampling 48 and 10 power
// iterations, then a Rayleigh-Ritz step (eigen-decomposition of B B^T with
// B = Q^T Wp) to pick the top r directions.
void top_r_basis(const double *Wp, int K, int N, int r, int threads, uint64_t seed,
                 std::vector<double> &Ur) {
  int p = std::min(std::min(K, N), r + 48);
  std::vector<double> omega(static_cast<size_t>(N) * p), Y(static_cast<size_t>(K) * p),
      Z(static_cast<size_t>(N) * p);
  gaussian_fill(omega.data(), omega.size(), seed);
  mul_a_x(Wp, K, N, omega.data(), p, Y.data(), threads);
  orthonormalize(Y.data(), K, p);
  for (int it = 0; it < 10; ++it) {
    mul_at_q(Wp, K, N, Y.data(), p, Z.data(), threads);
    orthonormalize(Z.data(), N, p);
    mul_a_x(Wp, K, N, Z.data(), p, Y.data(), threads);
    orthonormalize(Y.data(), K, p);
  }
  // B^T = Wp^T Q  [N][p];  C = B B^T = (B^T)^T (B^T)  [p][p]
  mul_at_q(Wp, K, N, Y.data(), p, Z.data(), threads);
  std::vector<double> C(static_cast<size_t>(p) * p, 0.0), V;
  for (int n = 0; n < N; ++n) {
    const double *z = Z.data() + static_cast<size_t>(n) * p;
    for (int a = 0; a < p; ++a)
      for (int b = 0; b < p; ++b) C[static_cast<size_t>(a) * p + b] += z[a] * z[b];
  }
  jacobi_eigen(C, p, V);
  std::vector<int> order(p);
  for (int i = 0; i < p; ++i) order[i] = i;
  std::sort(order.begin(), order.end(), [&](int a, int b) {
    return C[static_cast<size_t>(a) * p + a] > C[static_cast<size_t>(b) * p + b];
  });
  Ur.assign(static_cast<size_t>(K) * r, 0.0);
  for (int j = 0; j < K; ++j)
    for (int i = 0; i < r; ++i) {
      double acc = 0.0;
      int col = order[i];
      for (int t = 0; t < p; ++t) acc += Y[static_cast<size_t>(j) * p + t] * V[static_cast<size_t>(t) * p + col];
      Ur[static_cast<size_t>(j) * r + i] = acc;
    }
}
}  // namespace

// NVFP4 quantization of float32 rows into a bundle of tile height th (see svdq.h).
static void quantize_rows_f32(const float *T, int rows, int K, float s_t, int th, uint8_t *bundle, int threads) {
  const float d = 6.0f * s_t;
  std::memset(bundle, 0, bundle_bytes(rows, K, th));
  parallel_for(rows, threads, [&](int b, int e) {
    for (int m = b; m < e; ++m) {
      const float *t = T + static_cast<size_t>(m) * K;
      for (int kb = 0; kb < K / 16; ++kb) {
        float amax = 0.0f;
        for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(t[kb * 16 + i]));
        uint8_t sb = ue4m3_code(amax / d);
        float scale = kE4m3.v[sb] * s_t;
        float inv = scale == 0.0f ? 0.0f : 1.0f / scale;
        for (int i = 0; i < 16; i += 2) {
          const int k = kb * 16 + i;
          uint8_t lo = e2m1_code(t[k] * inv);
          uint8_t hi = e2m1_code(t[k + 1] * inv);
          bundle[bundle_code_offset(m, k, K, th)] = static_cast<uint8_t>(lo | (hi << 4));
        }
        for (int rep = 0; rep < bundle_scale_replicas(th); ++rep) bundle[bundle_scale_offset(m, kb * 16, K, th, rep)] = sb;
      }
    }
  });
}

static int default_threads(int t) {
  if (t > 0) return t;
  unsigned h = std::thread::hardware_concurrency();
  return h == 0 ? 1 : static_cast<int>(h);
}

}  // namespace svdq

using namespace svdq;

extern "C" int svdq_quantize_host(const float *T, int rows, int K, float s_t, int tile_rows, uint8_t *bundle) {
  if (!T || !bundle) return fail(SVDQ_ERR_INVALID_ARG, "svdq_quantize_host: null pointer");
  if (rows < 1 || K < 64 || K % 64) return fail(SVDQ_ERR_SHAPE, "svdq_quantize_host: need rows >= 1, K % 64 == 0");
  if (tile_rows != 128 && tile_rows != 256) return fail(SVDQ_ERR_SHAPE, "svdq_quantize_host: tile_rows must be 128 or 256");
  if (!(s_t > 0.0f) || !std::isfinite(s_t)) return fail(SVDQ_ERR_INVALID_ARG, "svdq_quantize_host: s_t must be > 0");
  quantize_rows_f32(T, rows, K, s_t, tile_rows, bundle, default_threads(0));
  return ok();
}

extern "C" int svdq_pack_weights(const uint16_t *W, int K, int N, const float *act_absmax, int rank,
                                 int num_threads, uint64_t seed, float *inv_lambda, uint16_t *l1t,
                                 uint8_t *l2t, uint8_t *w_bundle, float *s_w, float *s_a, float *residual) {
  if (!W || !act_absmax || !inv_lambda || !l2t || !w_bundle || !s_w || !s_a ||
      (rank > 0 && !l1t))
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_pack_weights: null pointer");
  if (K < 64 || K % 64 || N < 8 || N % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_pack_weights: need K % 64 == 0 and N % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16 || rank > std::min(K, N))
    return fail(SVDQ_ERR_SHAPE, "svdq_pack_weights: rank must be a multiple of 16 in [0, 64]");
  const int threads = default_threads(num_threads);
  const size_t KN = static_cast<size_t>(K) * N;

  // 1. Smoothing: lambda_j = sqrt(absmaxX_j / absmaxW_j), inv_lambda = f32(1/lambda).
  std::vector<double> Wp(KN);
  for (int j = 0; j < K; ++j) {
    double aw = 0.0;
    for (int n = 0; n < N; ++n) aw = std::max(aw, std::fabs(static_cast<double>(bf16_to_float(W[static_cast<size_t>(j) * N + n]))));
    double ax = static_cast<double>(act_absmax[j]);
    double lam = (ax > 0.0 && aw > 0.0) ? std::sqrt(ax / aw) : 1.0;
    inv_lambda[j] = static_cast<float>(1.0 / lam);
    const double inv = static_cast<double>(inv_lambda[j]);
    for (int n = 0; n < N; ++n)
      Wp[static_cast<size_t>(j) * N + n] = static_cast<double>(bf16_to_float(W[static_cast<size_t>(j) * N + n])) / inv;
  }

  // 2. Low-rank branch: L1 = U_r Sigma_r, L2 = V_r^T with U_r from the top-r
  //    basis and Sigma_r V_r^T = U_r^T W'; both rounded to bf16.
  std::vector<double> L1(static_cast<size_t>(K) * rank), L2(static_cast<size_t>(rank) * N);
  if (rank > 0) {
    std::vector<double> Ur;
    top_r_basis(Wp.data(), K, N, rank, threads, seed, Ur);
    std::vector<double> Gt(static_cast<size_t>(N) * rank);  // (U_r^T W')^T  [N][r]
    mul_at_q(Wp.data(), K, N, Ur.data(), rank, Gt.data(), threads);
    for (int i = 0; i < rank; ++i) {
      double nrm = 0.0;
      for (int n = 0; n < N; ++n) nrm += Gt[static_cast<size_t>(n) * rank + i] * Gt[static_cast<size_t>(n) * rank + i];
      double sigma = std::sqrt(nrm);
      double inv_sigma = sigma > 0.0 ? 1.0 / sigma : 0.0;
      for (int j = 0; j < K; ++j) {
        uint16_t b = bf16_bits_from_double(Ur[static_cast<size_t>(j) * rank + i] * sigma);
        l1t[static_cast<size_t>(i) * K + j] = b;
        L1[static_cast<size_t>(j) * rank + i] = static_cast<double>(bf16_to_float(b));
      }
      for (int n = 0; n < N; ++n) {
        uint16_t b = bf16_bits_from_double(Gt[static_cast<size_t>(n) * rank + i] * inv_sigma);
        L2[static_cast<size_t>(i) * N + n] = static_cast<double>(bf16_to_float(b));
      }
    }
  }
  std::memset(l2t, 0, lowrank_bytes(N, 256));
  for (int n = 0; n < N; ++n)
    for (int i = 0; i < rank; ++i) {
      float f = static_cast<float>(L2[static_cast<size_t>(i) * N + n]);
      uint32_t u;
      std::memcpy(&u, &f, 4);
      const uint16_t b = static_cast<uint16_t>(u >> 16);
      std::memcpy(l2t + lowrank_offset(n, i, 256), &b, 2);
    }

  // 3. Residual R = W' - L1 L2 in float64, rounded to float32, stored K-major
  //    per output column (R^T) for the blocks along K.
  std::vector<float> Rt(KN);
  float amax = 0.0f;
  {
    std::vector<float> colmax(N, 0.0f);
    parallel_for(N, threads, [&](int b, int e) {
      for (int n = b; n < e; ++n) {
        float cm = 0.0f;
        for (int j = 0; j < K; ++j) {
          double acc = Wp[static_cast<size_t>(j) * N + n];
          for (int i = 0; i < rank; ++i) acc -= L1[static_cast<size_t>(j) * rank + i] * L2[static_cast<size_t>(i) * N + n];
          float f = static_cast<float>(acc);
          Rt[static_cast<size_t>(n) * K + j] = f;
          cm = std::max(cm, std::fabs(f));
        }
        colmax[n] = cm;
      }
    });
    for (int n = 0; n < N; ++n) amax = std::max(amax, colmax[n]);
  }
  if (residual) {
    for (int j = 0; j < K; ++j)
      for (int n = 0; n < N; ++n) residual[static_cast<size_t>(j) * N + n] = Rt[static_cast<size_t>(n) * K + j];
  }

  // 4. NVFP4 of R (blocks of 16 along K for each output column).
  *s_w = tensor_scale(amax);
  quantize_rows_f32(Rt.data(), N, K, *s_w, 256, w_bundle, threads);

  // 5. Static activation scale from the calibration maxima.
  float xa = 0.0f;
  for (int j = 0; j < K; ++j) xa = std::max(xa, act_absmax[j] * inv_lambda[j]);
  *s_a = tensor_scale(xa);
  return ok();
}

extern "C" int svdq_weight_sizes(int K, int N, int rank, size_t *inv_lambda_bytes, size_t *l1t_bytes,
                                 size_t *l2t_bytes, size_t *w_bundle_bytes) {
  if (K < 64 || K % 64 || N < 8 || N % 8)
    return fail(SVDQ_ERR_SHAPE, "svdq_weight_sizes: need K % 64 == 0 and N % 8 == 0");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_weight_sizes: rank must be a multiple of 16 in [0, 64]");
  if (inv_lambda_bytes) *inv_lambda_bytes = static_cast<size_t>(K) * 4;
  if (l1t_bytes) *l1t_bytes = static_cast<size_t>(rank) * K * 2;
  if (l2t_bytes) *l2t_bytes = lowrank_bytes(N, 256);
  if (w_bundle_bytes) *w_bundle_bytes = bundle_bytes(N, K, 256);
  return ok();
}

extern "C" int svdq_act_sizes(int M, int K, size_t *a_bundle_bytes, size_t *u_bytes) {
  if (M < 1 || K < 64 || K % 64) return fail(SVDQ_ERR_SHAPE, "svdq_act_sizes: need M >= 1 and K % 64 == 0");
  if (a_bundle_bytes) *a_bundle_bytes = bundle_bytes(M, K, 128);
  if (u_bytes) *u_bytes = lowrank_bytes(M, 128);
  return ok();
}
