// Host side of the INT4 W4A4 variant: group quantization of float32 rows and
// the byte sizes of the INT4 operands (no GPU).
//
// The pages ship an INT4 W4A4 checkpoint beside NVFP4 for GPUs without NVFP4
// (web page "Diffusers × Nunchaku 4-bit", donmalab.com, section
// "實務上的影響與硬體要求").  The layer is the NVFP4 layer with its 4-bit branch
// in signed integers: groups of 64 along K, one bf16 scale per row and group,
//   s = bf16(f32(amax / 7)),  q = clamp(rne(f32(v * f32(1 / s))), -8, 7),
// s = 0 and q = 0 for a group whose amax is below 2^-120.  Every step is one
// IEEE float32 operation (no contraction), so the codes match the device
// quantizer's and the reference's bit for bit.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "svdq_internal.h"

namespace svdq {
namespace {

constexpr int kGroup = 64;

uint16_t bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return static_cast<uint16_t>(u >> 16);   // not reached: f is finite
  const uint32_t lsb = (u >> 16) & 1u;
  return static_cast<uint16_t>((u + 0x7FFFu + lsb) >> 16);
}

float bf16_value(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

void quantize_rows(const float *T, int r0, int r1, int K, int ld_s, uint8_t *codes, uint16_t *scales) {
  const float tiny = std::ldexp(1.0f, -120);
  for (int r = r0; r < r1; ++r) {
    const float *t = T + static_cast<size_t>(r) * K;
    uint8_t *c = codes + static_cast<size_t>(r) * (K / 2);
    for (int g = 0; g < K / kGroup; ++g) {
      float amax = 0.0f;
      for (int i = 0; i < kGroup; ++i) amax = std::max(amax, std::fabs(t[g * kGroup + i]));
      const uint16_t sb = amax < tiny ? 0 : bf16_rne(amax / 7.0f);
      const float s = bf16_value(sb);
      const float inv = s == 0.0f ? 0.0f : 1.0f / s;
      scales[static_cast<size_t>(g) * ld_s + r] = sb;
      for (int i = 0; i < kGroup; i += 2) {
        int q[2];
        for (int j = 0; j < 2; ++j) {
          const float p = t[g * kGroup + i + j] * inv;
          q[j] = static_cast<int>(std::min(7.0f, std::max(-8.0f, std::nearbyint(p))));
        }
        c[(g * kGroup + i) / 2] = static_cast<uint8_t>((q[0] & 0xF) | ((q[1] & 0xF) << 4));
      }
    }
  }
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" int svdq_quantize_int4_host(const float *T, int rows, int K, int ld_s, uint8_t *codes, uint16_t *scales) {
  if (!T || !codes || !scales) return fail(SVDQ_ERR_INVALID_ARG, "svdq_quantize_int4_host: null pointer");
  if (rows < 1 || K < kGroup || K % kGroup || ld_s < rows)
    return fail(SVDQ_ERR_SHAPE, "svdq_quantize_int4_host: need rows >= 1, K % 64 == 0, ld_s >= rows");
  unsigned h = std::thread::hardware_concurrency();
  const int threads = static_cast<int>(std::max(1u, std::min(h == 0 ? 1u : h, 64u)));
  const int per = (rows + threads - 1) / threads;
  std::vector<std::thread> pool;
  for (int b = 0; b < rows; b += per) pool.emplace_back(quantize_rows, T, b, std::min(rows, b + per), K, ld_s, codes, scales);
  for (auto &th : pool) th.join();
  return ok();
}

extern "C" int svdq_int4_weight_sizes(int K, int N, size_t *codes_bytes, size_t *scales_bytes) {
  if (K < kGroup || K % kGroup || N < 128 || N % 128)
    return fail(SVDQ_ERR_SHAPE, "svdq_int4_weight_sizes: need K % 64 == 0 and N % 128 == 0");
  if (codes_bytes) *codes_bytes = static_cast<size_t>(N) * (K / 2);
  if (scales_bytes) *scales_bytes = static_cast<size_t>(K / kGroup) * N * 2;
  return ok();
}

extern "C" int svdq_int4_act_sizes(int M, int K, size_t *codes_bytes, size_t *scales_bytes) {
  if (M < 1 || K < kGroup || K % kGroup) return fail(SVDQ_ERR_SHAPE, "svdq_int4_act_sizes: need M >= 1 and K % 64 == 0");
  const size_t mp = (static_cast<size_t>(M) + 127) / 128 * 128;
  if (codes_bytes) *codes_bytes = mp * (K / 2);
  if (scales_bytes) *scales_bytes = static_cast<size_t>(K / kGroup) * mp * 2;
  return ok();
}
