// INT4 W4A4 GEMM with the low-rank up-projection, bias and GELU fused in: the
// C-ABI entry point (argument checks) in front of the tcgen05 kernel of
// int4_gemm_tc.cu.
//
// The pages ship an INT4 W4A4 variant beside NVFP4 for GPUs without NVFP4
// tensor cores (web page "Diffusers × Nunchaku 4-bit", donmalab.com, section
// "實務上的影響與硬體要求"); its 4-bit branch is, in this library's reading,
// symmetric INT4 in groups of 64 along K with one bf16 scale per row or output
// column and group:
//   Y = epilogue( sum_g (s_a[m,g] s_w[n,g]) sum_{k in g} q_a[m,k] q_w[n,k]
//                 + U . L2 + bias )
// B200's tensor cores have no 4-bit integer MMA (the warp-level s4 MMA
// measured 40 times slower than the 8-bit one: it is emulated), and an 8-bit
// integer MMA leaves a per-group rescale of every output to the CUDA cores;
// the kernel instead multiplies exact fp16 operands q * s made from the codes
// (int4_gemm_tc.cu), for every width this entry point accepts.
#include <cuda_runtime.h>

#include <string>

#include "svdq_internal.h"

using namespace svdq;

extern "C" int svdq_linear_int4(const uint8_t *a_codes, const void *a_scales, const void *U, const uint8_t *w_codes,
                                const void *w_scales, const void *l2t, const void *bias, int M, int N, int K, int rank,
                                int epilogue, int gelu_col_begin, void *Y, int ldy, svdq_stream_t stream) {
  if (!a_codes || !a_scales || !w_codes || !w_scales || !Y || (rank > 0 && (!U || !l2t)))
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_int4: null pointer");
  if (epilogue < SVDQ_EPILOGUE_NONE || epilogue > SVDQ_EPILOGUE_GELU_TANH)
    return fail(SVDQ_ERR_INVALID_ARG, "svdq_linear_int4: unknown epilogue");
  if (M < 1 || K < 64 || K % 64 || N < 128 || N % 128 || ldy < N || ldy % 8 || gelu_col_begin < 0 ||
      gelu_col_begin > N)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_int4: need M >= 1, K % 64 == 0, N % 128 == 0, ldy >= N, ldy % 8 == 0, "
                                "0 <= gelu_col_begin <= N");
  if (rank < 0 || rank > SVDQ_LR_STRIDE || rank % 16)
    return fail(SVDQ_ERR_SHAPE, "svdq_linear_int4: rank must be a multiple of 16 in [0, 64]");
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (rank > 0 && (!aligned16(U) || !aligned16(l2t))))
    return fail(SVDQ_ERR_ALIGNMENT, "svdq_linear_int4: pointers must be 16-byte aligned");
  DeviceState *st = current_device_state();
  if (!st) return SVDQ_ERR_NOT_INITIALIZED;
  return launch_int4_tc(a_codes, a_scales, U, w_codes, w_scales, l2t, bias, M, N, K, rank, epilogue, gelu_col_begin,
                        Y, ldy, st->status_word, reinterpret_cast<cudaStream_t>(stream));
}
