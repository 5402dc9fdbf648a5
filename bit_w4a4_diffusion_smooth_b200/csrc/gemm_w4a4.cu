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

extern "C" int svdq_linear_w4a4_grouped(const svdq_w4a4_problem *problems, int count, int rank, int epilogue,
                                        svdq_stream_t stream) {
  static const char *fn = "svdq_linear_w4a4_grouped";
  if (!problems) return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": null problem list");
  if (count < 1 || count > kMaxGroup)
    return fail(SVDQ_ERR_INVALID_ARG, std::string(fn) + ": count must be in [1, " + std::to_string(kMaxGroup) + "]");
  Group<kMaxGroup> g{};
  DeviceState *st = nullptr;
  int tiles = 0;
  for (int i = 0; i < count; ++i) {
    const svdq_w4a4_problem &q = problems[i];
    const std::string name = std::string(fn) + " (problem " + std::to_string(i) + ")";
    int rc = setup_gemm(name.c_str(), q.a_bundle, q.U, q.s_a, q.w_bundle, q.l2t, q.s_w, q.bias, q.M, q.N, q.K, rank,
                        epilogue, q.gelu_col_begin, q.Y, q.ldy, false, &g.maps[i], &g.p[i], &st);
    if (rc != SVDQ_OK) return rc;
    tiles += g.p[i].num_tiles;
    g.tile_end[i] = tiles;
  }
  g.count = count;
  g.total_tiles = tiles;
  g.status = g.p[0].status;
  g.limit_ns = g.p[0].limit_ns;
  const int rc = launch_gemm<-1, kMaxGroup>(fn, g, epilogue, st->sm_count, reinterpret_cast<cudaStream_t>(stream));
  return rc == SVDQ_OK ? ok() : rc;
}
