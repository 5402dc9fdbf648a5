// K2: the W4A4 GEMM with the low-rank up-projection fused in - entry point
// of the plain variant (the kernel itself is in gemm_w4a4_kernel.cuh).
#include "gemm_w4a4_kernel.cuh"

using namespace svdq;
using namespace svdq::w4a4;

extern "C" int svdq_linear_w4a4(const uint8_t *a_bundle, const void *U, const float *s_a, const uint8_t *w_bundle,
                                const void *l2t, const float *s_w, const void *bias, int M, int N, int K, int rank,
                                int epilogue, int gelu_col_begin, void *Y, int ldy, svdq_stream_t stream) {
  Maps maps;
  Params p;
  DeviceState *st = nullptr;
  int rc = setup_gemm("svdq_linear_w4a4", a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, epilogue,
                      gelu_col_begin, Y, ldy, false, &maps, &p, &st);
  if (rc != SVDQ_OK) return rc;
  rc = launch_gemm<-1>("svdq_linear_w4a4", maps, p, st->sm_count, reinterpret_cast<cudaStream_t>(stream));
  return rc == SVDQ_OK ? ok() : rc;
}
