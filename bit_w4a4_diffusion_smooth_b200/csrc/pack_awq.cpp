// Offline (host) AWQ INT4 packing for the W4A16 projection.
//
// The pages use AWQ W4A16 (4-bit weights, 16-bit activations) for the
// precision-sensitive, low-compute modulation and adaptive-norm projections
// (web page "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定适用范围", remio.ai,
// section "Nunchaku Diffusers 支持改变了加载路径").  Group size and layout are
// not on the pages; this library takes asymmetric INT4 in groups of 64 along
// K with bf16 scales and integer zero points (see svdq.h).
// float64 arithmetic, one rounding per operation (-ffp-contract=off).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "svdq_internal.h"

namespace {

uint16_t bf16_bits_of_exact(double v) {
  float f = static_cast<float>(v);
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16);
}

double bf16_round(double v) {
  if (v == 0.0) return v;
  double a = std::fabs(v);
  int e2;
  std::frexp(a, &e2);
  int e = std::max(e2 - 1, -126);
  double quantum = std::ldexp(1.0, e - 7);
  return std::copysign(std::nearbyint(a / quantum) * quantum, v);
}

double bf16_value(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// Position of weight (output column n, input k) in the packed qweight array:
// the fragment order of the W4A16 kernel.  Columns come in quads of 64 (four
// blocks of 16) and K in groups of 64; the quads follow each other, and
// inside a quad the groups, so that the four blocks of one group are 2 KB of
// contiguous memory.  Each (quad, group, block) holds 32 lanes x 4 words,
// word j of a lane covering k16-step j of the group.  Lane = 4 g + t and the
// 8 nibbles of a word hold, with c = column within the block and kq = k
// within the step:
//   nibble 0 / 4: c = g,     kq = 2t / 2t+1
//   nibble 1 / 5: c = g + 8, kq = 2t / 2t+1
//   nibble 2 / 6: c = g,     kq = 2t+8 / 2t+9
//   nibble 3 / 7: c = g + 8, kq = 2t+8 / 2t+9
size_t awq_word_index(int n, int k, int G) {
  const int quad = n / 64, blk = (n / 16) % 4, c = n % 16, grp = k / 64, j = (k % 64) / 16, kq = k % 16;
  const int lane = (c % 8) * 4 + (kq % 8) / 2;
  return (((static_cast<size_t>(quad) * G + grp) * 4 + blk) * 32 + lane) * 4 + j;
}
// Position of the scale / zero point of (output column n, group g): the 64
// values of one (quad, group) are contiguous.
size_t awq_group_index(int n, int g, int G) {
  return (static_cast<size_t>(n / 64) * G + g) * 64 + n % 64;
}
int awq_nibble_index(int n, int k) {
  const int c = n % 16, kq = k % 16;
  return (c / 8) + 2 * (kq / 8) + 4 * (kq % 2);
}

}  // namespace

using namespace svdq;

extern "C" int awq_pack_weights(const uint16_t *W, int K, int N, const float *awq_scale, int group,
                                uint32_t *qweight, uint16_t *scales, uint16_t *zeros, float *inv_awq) {
  if (!W || !awq_scale || !qweight || !scales || !zeros || !inv_awq)
    return fail(SVDQ_ERR_INVALID_ARG, "awq_pack_weights: null pointer");
  if (group != 64) return fail(SVDQ_ERR_SHAPE, "awq_pack_weights: group must be 64");
  if (K < group || K % group || N < 64 || N % 64)
    return fail(SVDQ_ERR_SHAPE, "awq_pack_weights: need K % 64 == 0 and N % 64 == 0");
  for (int k = 0; k < K; ++k)
    if (!(awq_scale[k] > 0.0f) || !std::isfinite(awq_scale[k]))
      return fail(SVDQ_ERR_INVALID_ARG, "awq_pack_weights: AWQ scales must be finite and > 0");
  const int G = K / group;
  std::memset(qweight, 0, static_cast<size_t>(N) * (K / 8) * 4);
  std::vector<double> wa(group);
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      double lo = 0.0, hi = 0.0;
      for (int i = 0; i < group; ++i) {
        int k = g * group + i;
        wa[i] = static_cast<double>(awq_scale[k]) * bf16_value(W[static_cast<size_t>(k) * N + n]);
        lo = std::min(lo, wa[i]);
        hi = std::max(hi, wa[i]);
      }
      double s = bf16_round((hi - lo) / 15.0);
      double z = 0.0;
      if (s == 0.0) {
        s = 1.0;
      } else {
        z = std::min(15.0, std::max(0.0, std::nearbyint(-lo / s)));
      }
      scales[awq_group_index(n, g, G)] = bf16_bits_of_exact(s);
      zeros[awq_group_index(n, g, G)] = bf16_bits_of_exact(z);
      for (int i = 0; i < group; ++i) {
        int k = g * group + i;
        double q = std::min(15.0, std::max(0.0, std::nearbyint(wa[i] / s) + z));
        qweight[awq_word_index(n, k, G)] |= static_cast<uint32_t>(q) << (4 * awq_nibble_index(n, k));
      }
    }
  }
  for (int k = 0; k < K; ++k) inv_awq[k] = 1.0f / awq_scale[k];
  return ok();
}

extern "C" int awq_packed_sizes(int K, int N, int group, size_t *qweight_bytes, size_t *scales_bytes,
                                size_t *zeros_bytes, size_t *inv_awq_bytes) {
  using svdq::fail;
  if (!qweight_bytes || !scales_bytes || !zeros_bytes || !inv_awq_bytes)
    return fail(SVDQ_ERR_INVALID_ARG, "awq_packed_sizes: null pointer");
  if (group != 64 || K < 64 || K % 64 || N < 64 || N % 64)
    return fail(SVDQ_ERR_SHAPE, "awq_packed_sizes: need group == 64, K % 64 == 0, N % 64 == 0");
  const size_t k = static_cast<size_t>(K), n = static_cast<size_t>(N);
  *qweight_bytes = n * k / 2;
  *scales_bytes = n * (k / 64) * 2;
  *zeros_bytes = n * (k / 64) * 2;
  *inv_awq_bytes = k * 4;
  return svdq::ok();
}
