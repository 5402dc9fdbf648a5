// Host-side internals shared by the translation units of the library.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

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

// ---------------------------------------------------------------------------
// Operand bundles: the layout in which NVFP4 operands (codes + block scales)
// live in memory, built so that one GEMM pipeline stage is one contiguous copy.
//
// A matrix of `rows` x K elements is cut into tiles of TH rows (128 for
// activations, 256 for weights) by 256 K-elements.  Tile (tr, ks) starts at
//   (tr * KS + ks) * TH * 144 bytes,   KS = ceil(K / 256),
// and holds
//   * TH rows x 128 bytes of e2m1 codes, element k of row r in byte k/2 of
//     the row (low nibble for even k), rows 128 bytes apart, the 16-byte
//     chunks of a row permuted by the 128-byte swizzle: chunk c of row r at
//     r*128 + ((c ^ (r % 8)) * 16) - the shared-memory image a tcgen05 MMA
//     reads with a SWIZZLE_128B K-major descriptor;
//   * then TH/128 x 4 atoms of 512 bytes of ue4m3 block scales: the scale of
//     (row r, 16-block j of the tile) at TH*128 + (j/4)*(TH/128)*512*RP +
//     (r/128)*512*RP + (r%32)*16 + ((r%128)/32)*4 + j%4, in each of RP
//     replicas 512 bytes apart.  One 512-byte atom (128 rows x one k-block)
//     is the image of a tcgen05.cp 32x128b.warpx4 copy; four replicas of it
//     are the image of the same columns written by one 128x256b copy, and the
//     two 128-row halves of a 256-row tile side by side fill its 8 columns.
//     RP = 1 for 128-row tiles (activations), 4 for 256-row tiles (weights).
// Rows past `rows` and elements past K are zero (codes and scales).
constexpr int kStageK = 256;

SVDQ_HD int bundle_ks(int K) { return (K + kStageK - 1) / kStageK; }
SVDQ_HD int bundle_scale_replicas(int th) { return th == 256 ? 4 : 1; }
SVDQ_HD size_t bundle_tile_bytes(int th) {
  return static_cast<size_t>(th) * 128u + static_cast<size_t>(th / 128) * 2048u * bundle_scale_replicas(th);
}
SVDQ_HD size_t bundle_bytes(int rows, int K, int th) {
  return static_cast<size_t>((rows + th - 1) / th) * static_cast<size_t>(bundle_ks(K)) * bundle_tile_bytes(th);
}
SVDQ_HD size_t bundle_tile_offset(int m, int k, int K, int th) {
  return (static_cast<size_t>(m / th) * static_cast<size_t>(bundle_ks(K)) + static_cast<size_t>(k / kStageK)) *
         bundle_tile_bytes(th);
}
// Byte holding the code of element (m, k); the low nibble for even k.
SVDQ_HD size_t bundle_code_offset(int m, int k, int K, int th) {
  const int r = m % th, kb = (k % kStageK) / 2;
  return bundle_tile_offset(m, k, K, th) + static_cast<size_t>(r) * 128u +
         static_cast<size_t>((((kb >> 4) ^ r) & 7) << 4) + static_cast<size_t>(kb & 15);
}
// Byte holding the block scale of element (m, k) in replica `rep`.
SVDQ_HD size_t bundle_scale_offset(int m, int k, int K, int th, int rep = 0) {
  const int r = m % th, j = (k % kStageK) / 16;
  const size_t atom = 512u * static_cast<size_t>(bundle_scale_replicas(th));
  return bundle_tile_offset(m, k, K, th) + static_cast<size_t>(th) * 128u +
         static_cast<size_t>(j >> 2) * static_cast<size_t>(th / 128) * atom + static_cast<size_t>(r >> 7) * atom +
         static_cast<size_t>(rep) * 512u + static_cast<size_t>(r & 31) * 16u + static_cast<size_t>((r >> 5) & 3) * 4u +
         static_cast<size_t>(j & 3);
}

// Low-rank operands: tiles of TH rows x 64 bf16 (TH = 128 for U, 256 for
// L2T), 128-byte rows with the 128-byte swizzle; element (m, j) at
//   (m/TH)*TH*128 + (m%TH)*128 + (((j/8) ^ (m%8)) * 16) + (j%8)*2.
SVDQ_HD size_t lowrank_bytes(int rows, int th) {
  return static_cast<size_t>((rows + th - 1) / th) * static_cast<size_t>(th) * 128u;
}
SVDQ_HD size_t lowrank_offset(int m, int j, int th) {
  const int r = m % th;
  return static_cast<size_t>(m / th) * static_cast<size_t>(th) * 128u + static_cast<size_t>(r) * 128u +
         static_cast<size_t>((((j >> 3) ^ r) & 7) << 4) + static_cast<size_t>(j & 7) * 2u;
}

// Eigen-decomposition of the symmetric p x p matrix C (row-major, float64) by
// cyclic Jacobi rotations: eigenvalues on C's diagonal, eigenvectors in the
// columns of V (host; used by the host and the device packs).
void jacobi_eigen(std::vector<double> &C, int p, std::vector<double> &V);

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

#ifdef __CUDACC__
// Launch configuration for the hot-path kernels: programmatic stream
// serialization lets a kernel start while its predecessor finishes (each
// kernel waits for its predecessors before touching global memory).
struct DependentLaunch {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg;
  DependentLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t stream) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
};
#endif

#ifdef __CUDACC__
// Raises a kernel's dynamic shared-memory limit to `bytes`, once per device
// (a host call that need not be repeated on every launch).
template <auto Kernel>
int smem_optin_once(int bytes, const char *fn) {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return fail(SVDQ_ERR_CUDA, std::string(fn) + ": no current device");
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string(fn) + ": " + cudaGetErrorString(e));
    done[dev] = true;
  }
  return SVDQ_OK;
}
#endif

// Bounded-wait limit handed to every kernel, in nanoseconds.
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;

bool aligned16(const void *p);

// Encodes a 2-D TMA descriptor (tiled, zero fill out of bounds) for a
// row-major tensor of `outer` rows x `inner` elements with the given row
// stride in bytes.  Returns SVDQ_OK or an error status (message recorded).
int encode_tmap_2d(CUtensorMap *out, CUtensorMapDataType dtype, const void *base, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swizzle);

// Encodes a 3-D TMA descriptor (tiled, zero fill out of bounds): dims[0] is
// contiguous, strides[0] / strides[1] are the byte strides of dims 1 and 2
// (any order, multiples of 16).
int encode_tmap_3d(CUtensorMap *out, CUtensorMapDataType dtype, const void *base, const uint64_t (&dims)[3],
                   const uint64_t (&strides)[2], const uint32_t (&box)[3], CUtensorMapSwizzle swizzle);

// The INT4 W4A4 GEMM on tcgen05 (int4_gemm_tc.cu), for N % 128 == 0; svdq_linear_int4 checks the
// arguments and dispatches here.
int launch_int4_tc(const uint8_t *a_codes, const void *a_scales, const void *U, const uint8_t *w_codes,
                   const void *w_scales, const void *l2t, const void *bias, int M, int N, int K, int rank, int epilogue,
                   int gelu_col_begin, void *Y, int ldy, unsigned int *status, cudaStream_t stream);

}  // namespace svdq
