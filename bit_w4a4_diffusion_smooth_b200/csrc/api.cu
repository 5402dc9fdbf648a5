// C ABI plumbing: device selection and validation, per-thread error text,
// the per-device status word written by bounded waits, and two probes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "device_common.cuh"
#include "svdq_internal.h"

namespace svdq {

namespace {
thread_local std::string g_last_error;
std::mutex g_state_mutex;
std::vector<DeviceState> g_states;
}  // namespace

int fail(int status, const std::string &msg) {
  g_last_error = msg;
  return status;
}
int ok() {
  g_last_error.clear();
  return SVDQ_OK;
}
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// One status word per device: the first error code a kernel's bounded wait
// recorded since the last svdq_check_status.
__device__ unsigned int g_status_word;

DeviceState *current_device_state() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    fail(SVDQ_ERR_CUDA, "cudaGetDevice failed");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_state_mutex);
  if (dev < 0 || dev >= static_cast<int>(g_states.size()) || !g_states[dev].initialized) {
    fail(SVDQ_ERR_NOT_INITIALIZED, "svdq_init() was not called for device " + std::to_string(dev));
    return nullptr;
  }
  return &g_states[dev];
}

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      p = nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}
}  // namespace

namespace {
// Encoded tensor maps, cached by every argument of the encode: a map is a pure
// function of them (base address, extents, strides, box, swizzle, element
// type), so a hit returns exactly what the driver would encode again.  The
// per-call cost of a layer's GEMM (seven maps) and activation kernel (two)
// then shrinks to lookups once its buffers have been seen.  Direct-mapped; a
// colliding entry is simply replaced.
struct TmapKey {
  uint64_t dims[3], strides[2];
  const void *base;
  uint32_t box[3];
  int dtype, rank, swizzle;
};
struct TmapEntry {
  CUtensorMap map;
  TmapKey key;
  bool valid;
};
constexpr size_t kTmapCacheSize = 1024;
std::mutex g_tmap_mutex;
TmapEntry g_tmap_cache[kTmapCacheSize];

TmapKey make_key(int rank, CUtensorMapDataType dtype, const void *base, const uint64_t *dims, const uint64_t *strides,
                 const uint32_t *box, CUtensorMapSwizzle swizzle) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));   // padding bytes take part in the comparison
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
  k.base = base;
  k.dtype = static_cast<int>(dtype);
  k.rank = rank;
  k.swizzle = static_cast<int>(swizzle);
  return k;
}

size_t key_slot(const TmapKey &k) {
  uint64_t h = 1469598103934665603ull;   // FNV-1a over the key's bytes
  const unsigned char *b = reinterpret_cast<const unsigned char *>(&k);
  for (size_t i = 0; i < sizeof(k); ++i) h = (h ^ b[i]) * 1099511628211ull;
  return static_cast<size_t>(h % kTmapCacheSize);
}

int encode_tiled(int rank, CUtensorMap *out, CUtensorMapDataType dtype, const void *base, const uint64_t *dims,
                 const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swizzle) {
  const TmapKey key = make_key(rank, dtype, base, dims, strides, box, swizzle);
  const size_t slot = key_slot(key);
  {
    std::lock_guard<std::mutex> lock(g_tmap_mutex);
    const TmapEntry &e = g_tmap_cache[slot];
    if (e.valid && std::memcmp(&e.key, &key, sizeof(key)) == 0) {
      *out = e.map;
      return SVDQ_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t d[3] = {0, 0, 0}, st[2] = {0, 0};
  cuuint32_t bx[3] = {0, 0, 0}, estride[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  CUresult r = fn(out, dtype, static_cast<cuuint32_t>(rank), const_cast<void *>(base), d, st, bx, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (" + std::to_string(rank) + "-D) failed (code " +
                                   std::to_string(static_cast<int>(r)) + ")");
  std::lock_guard<std::mutex> lock(g_tmap_mutex);
  TmapEntry &e = g_tmap_cache[slot];
  e.map = *out;
  e.key = key;
  e.valid = true;
  return SVDQ_OK;
}
}  // namespace

int encode_tmap_2d(CUtensorMap *out, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                   uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  const uint64_t dims[2] = {inner, outer}, strides[1] = {row_stride_bytes};
  const uint32_t box[2] = {box_inner, box_outer};
  return encode_tiled(2, out, dtype, base, dims, strides, box, swizzle);
}

int encode_tmap_3d(CUtensorMap *out, CUtensorMapDataType dtype, const void *base, const uint64_t (&dims)[3],
                   const uint64_t (&strides)[2], const uint32_t (&box)[3], CUtensorMapSwizzle swizzle) {
  return encode_tiled(3, out, dtype, base, dims, strides, box, swizzle);
}

namespace {
__global__ void wait_timeout_kernel(unsigned long long limit_ns, unsigned int *status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    dev::mbar_init(&bar, 1);
    dev::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the wait has to run out.
    if (!dev::mbar_wait(&bar, 0, limit_ns, nullptr)) dev::report(status, SVDQ_ERR_TIMEOUT);
  }
  __syncthreads();
}

__global__ void convert_probe_kernel(const float *in, int n, uint8_t *e2m1_out, uint8_t *e4m3_out) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) e4m3_out[i] = static_cast<uint8_t>(dev::cvt_e4m3(in[i]));
  if (i < n / 2) e2m1_out[i] = static_cast<uint8_t>(dev::cvt_e2m1x2(in[2 * i], in[2 * i + 1]));
}
}  // namespace

}  // namespace svdq

using namespace svdq;

extern "C" int svdq_version(void) { return 10000; }

extern "C" const char *svdq_last_error_string(void) { return g_last_error.c_str(); }

extern "C" const char *svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_SHAPE: return "SVDQ_ERR_SHAPE";
    case SVDQ_ERR_ALIGNMENT: return "SVDQ_ERR_ALIGNMENT";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "SVDQ_ERR_UNSUPPORTED_DEVICE";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT";
    case SVDQ_ERR_NOT_INITIALIZED: return "SVDQ_ERR_NOT_INITIALIZED";
    default: return "SVDQ_ERR_UNKNOWN";
  }
}

extern "C" int svdq_init(int device) {
  int count = 0;
  cudaError_t e = cudaGetDeviceCount(&count);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(SVDQ_ERR_CUDA, std::string("cudaGetDeviceCount: ") + cudaGetErrorString(e));
  }
  if (device < 0 || device >= count) return fail(SVDQ_ERR_INVALID_ARG, "svdq_init: no such device");
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("cudaGetDeviceProperties: ") + cudaGetErrorString(e));
  if (prop.major != 10 || prop.minor != 0)
    return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "svdq_init: device " + std::to_string(device) + " (" + prop.name +
                                                 ") has compute capability " + std::to_string(prop.major) + "." +
                                                 std::to_string(prop.minor) + "; this library runs on 10.0 (B200) only");
  e = cudaSetDevice(device);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("cudaSetDevice: ") + cudaGetErrorString(e));
  void *status = nullptr;
  e = cudaGetSymbolAddress(&status, g_status_word);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
  std::lock_guard<std::mutex> lock(g_state_mutex);
  if (static_cast<int>(g_states.size()) < count) g_states.resize(count);
  DeviceState &st = g_states[device];
  st.sm_count = prop.multiProcessorCount;
  st.max_smem_optin = static_cast<int>(prop.sharedMemPerBlockOptin);
  st.status_word = static_cast<unsigned int *>(status);
  st.initialized = true;
  return ok();
}

extern "C" int svdq_check_status(svdq_stream_t stream) {
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("stream failed: ") + cudaGetErrorString(e));
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word));
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("reading status: ") + cudaGetErrorString(e));
  unsigned int zero = 0;
  e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("clearing status: ") + cudaGetErrorString(e));
  if (word != 0) return fail(static_cast<int>(word), "a kernel's bounded wait ran out");
  return ok();
}

extern "C" int svdq_debug_wait_timeout(uint64_t limit_ns, svdq_stream_t stream) {
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  if (limit_ns > 10ull * 1000 * 1000 * 1000) return fail(SVDQ_ERR_INVALID_ARG, "limit above 10 s");
  wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns, st->status_word);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return ok();
}

namespace svdq {
namespace {
__global__ void gelu_probe_kernel(const float *in, int n, int kind, float *out) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = kind == SVDQ_EPILOGUE_GELU_TANH ? dev::gelu_tanh(in[i]) : dev::gelu_erf2(make_float2(in[i], 0.0f)).x;
}
}  // namespace
}  // namespace svdq

extern "C" int svdq_debug_gelu(const float *in, int n, int kind, float *out, svdq_stream_t stream) {
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  if (!in || !out) return fail(SVDQ_ERR_INVALID_ARG, "svdq_debug_gelu: null pointer");
  if (kind != SVDQ_EPILOGUE_GELU_ERF && kind != SVDQ_EPILOGUE_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_debug_gelu: kind must be a GELU epilogue");
  if (n < 1) return fail(SVDQ_ERR_SHAPE, "svdq_debug_gelu: n must be >= 1");
  gelu_probe_kernel<<<(n + 255) / 256, 256, 0, stream>>>(in, n, kind, out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return ok();
}

extern "C" int svdq_debug_convert(const float *in, int n, uint8_t *e2m1_out, uint8_t *e4m3_out,
                                  svdq_stream_t stream) {
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  if (!in || !e2m1_out || !e4m3_out) return fail(SVDQ_ERR_INVALID_ARG, "svdq_debug_convert: null pointer");
  if (n < 2 || n % 2) return fail(SVDQ_ERR_SHAPE, "svdq_debug_convert: n must be even and >= 2");
  convert_probe_kernel<<<(n + 255) / 256, 256, 0, stream>>>(in, n, e2m1_out, e4m3_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SVDQ_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return ok();
}
