// Host-side internals shared by the translation units of the library.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>

#include <cuda.h>

#include "../../include/svdq.h"

namespace svdq {

// Records `msg` as the calling thread's last error and returns `status`.
int fail(int status, const std::string &msg);
// Clears the calling thread's last error and returns SVDQ_OK.
int ok();

#ifdef __CUDACC__
#define SVDQ_HD __host__ __device__ __forceinline__
#else
#define SVDQ_HD inline
#endif

// Byte offset of block scale (row m, 16-block kb) in the tcgen05 scale-factor
// tile order used for every NVFP4 scale buffer of this library: atoms of
// 128 rows x 4 scales (512 bytes), atoms ordered K-fastest; inside an atom
// row m sits at (m % 32) * 16 + ((m % 128) / 32) * 4 and block kb at kb % 4.
// This is the order in which tcgen05.cp (32x128b, warpx4) moves one atom into
// four TMEM columns: lane m % 32, column (m % 128) / 32, byte kb % 4.
SVDQ_HD size_t sf_offset(int m, int kb, int K) {
  return (static_cast<size_t>(m >> 7) * static_cast<size_t>(K >> 6) + static_cast<size_t>(kb >> 2)) * 512u +
         static_cast<size_t>(m & 31) * 16u + static_cast<size_t>((m >> 5) & 3) * 4u +
         static_cast<size_t>(kb & 3);
}
SVDQ_HD size_t sf_bytes(int rows, int K) {
  return static_cast<size_t>((rows + 127) / 128) * 128u * static_cast<size_t>(K / 16);
}

// Per-device state filled by svdq_init.
struct DeviceState {
  bool initialized = false;
  int sm_count = 0;
  int max_smem_optin = 0;
  unsigned int *status_word = nullptr;  // device address of the status word
};
// State of the current device, or nullptr (after recording an error) if the
// current device was not initialized.
DeviceState *current_device_state();

// Bounded-wait limit handed to every kernel, in nanoseconds.
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;

bool aligned16(const void *p);

// Encodes a 2-D TMA descriptor (tiled, zero fill out of bounds) for a
// row-major tensor of `outer` rows x `inner` elements with the given row
// stride in bytes.  Returns SVDQ_OK or an error status (message recorded).
int encode_tmap_2d(CUtensorMap *out, CUtensorMapDataType dtype, const void *base, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle);

}  // namespace svdq
