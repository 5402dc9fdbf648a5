/*
 * svdq.h - C ABI of the B200 (sm_100a) SVDQuant W4A4 linear layer and the AWQ
 * W4A16 projection.
 *
 * The layer (web page "Nunchaku Diffusers 支持降低显存占用，但硬件仍决定适用范围",
 * remio.ai, section "SVDQuant 将棘手数值移出 4 位路径"; and "Diffusers × Nunchaku
 * 4-bit", donmalab.com, section "量化的核心挑戰：為什麼 4-bit 很難？"):
 *
 *     Y = (X^ . L1) . L2 + Q(X^) . Q(R) + b,   X^ = X . diag(lambda)^-1,
 *     W' = diag(lambda) . W,  L1 . L2 = top-r SVD of W',  R = W' - L1 . L2
 *
 * with Q() the NVFP4 format (e2m1 elements, one e4m3 scale per 16 elements
 * along K, one fp32 scale per tensor).  The same pages assign 4-bit-weight,
 * 16-bit-activation AWQ layers to the modulation / adaptive-norm projections
 * (remio.ai, section "Nunchaku Diffusers 支持改变了加载路径").
 *
 * Conventions for every call
 *   - Return value: an svdq_status.  On failure svdq_last_error_string()
 *     (per calling thread) describes the first problem found.  Argument checks
 *     happen on the host before anything is enqueued; a failed check enqueues
 *     nothing.
 *   - Device calls take device pointers and are asynchronous on the caller's
 *     CUDA stream (cudaStream_t passed as svdq_stream_t; NULL = legacy default
 *     stream).  They never synchronize and never allocate device memory.
 *   - Host calls (the *_pack_* and *_sizes calls) take host pointers and run
 *     on the calling thread; they need no GPU.
 *   - The caller owns every buffer.  Buffers must not overlap unless stated.
 *   - bf16 tensors are passed as raw 16-bit patterns (uint16_t / void*).
 *   - Every device pointer must be 16-byte aligned and every row stride a
 *     multiple of 16 bytes (SVDQ_ERR_ALIGNMENT otherwise).
 *   - Device waits inside the kernels are bounded (about one second); a wait
 *     that runs out records SVDQ_ERR_TIMEOUT in a per-device status word that
 *     svdq_check_status() returns.  Kernels never trap.
 *
 * Packed layouts (all produced by this library; documented so callers can
 * move them around as opaque bytes):
 *   bundle  NVFP4 operand (e2m1 codes + ue4m3 block scales), cut into tiles
 *           of TH rows x 256 K-elements (TH = 128 for activations, 256 for
 *           weights).  Tile (tr, ks) starts at (tr * ceil(K/256) + ks) * T
 *           bytes, T = TH*144 for TH = 128 and TH*192 for TH = 256, and holds
 *           TH rows x 128 bytes of codes (element k of row r in
 *           byte k/2 of the row, low nibble for even k; code = sign bit 3 |
 *           e2m1 magnitude 0..7; the 16-byte chunks of a row permuted by the
 *           128-byte swizzle: chunk c of row r at r*128 + ((c ^ (r%8)) * 16)),
 *           then 4 x TH/128 x RP atoms of 512 bytes of block scales (RP = 1 for
 *           TH = 128, 4 for TH = 256): the scale of row r, 16-block j of the
 *           tile is at TH*128 + (j/4)*(TH/128)*512*RP + (r/128)*512*RP +
 *           q*512 + (r%32)*16 + ((r%128)/32)*4 + j%4 for every replica q < RP
 *           (the weight scales are stored four times over: the shared-memory
 *           image of one wide tensor-memory copy).  Rows past the matrix and
 *           elements past K are zero.  Each tile is the shared-memory image of
 *           one GEMM pipeline stage, so a stage is one contiguous copy.
 *   L1T     low-rank down-projection, transposed: [rank][K] bf16, row-major.
 *   U, L2T  low-rank activations (M rows) and up-projection (N rows) as tiles
 *           of TH rows x 64 bf16 (TH = 128 for U, 256 for L2T), 128-byte rows
 *           with the 128-byte swizzle: element (m, j) at (m/TH)*TH*128 +
 *           (m%TH)*128 + (((j/8) ^ (m%8)) * 16) + (j%8)*2; columns >= rank are 0.
 *   AWQ     qweight: N*K/8 uint32 words in the fragment order of the W4A16
 *           kernel's tensor-core tiles.  Columns go in quads of 64 = four
 *           blocks of 16, K in groups of 64; quad Q, group G, block b owns
 *           words [((Q*(K/64)+G)*4+b)*128, +128) - the four blocks of one
 *           group of one quad are 2 KB of contiguous memory:
 *           32 lanes x 4 words, word j of lane 4g+t covering k = 64G+16j+kq.
 *           Its nibbles (bits 4i..4i+3) hold, for column c of the block:
 *             i = 0 / 4: c = g,   kq = 2t / 2t+1;   i = 1 / 5: c = g+8, kq = 2t / 2t+1
 *             i = 2 / 6: c = g,   kq = 2t+8/2t+9;   i = 3 / 7: c = g+8, kq = 2t+8/2t+9
 *           scales, zeros: N*K/64 bf16 each (zeros are integers 0..15), the
 *           value of column n and group G at (((n/64)*(K/64)+G)*64 + n%64).
 */
#ifndef SVDQ_B200_H
#define SVDQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *svdq_stream_t; /* identical to cudaStream_t */

enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size */
  SVDQ_ERR_SHAPE = 2,             /* a shape rule below is violated */
  SVDQ_ERR_ALIGNMENT = 3,         /* pointer or stride not 16-byte aligned */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 4,/* not a compute capability 10.0 GPU */
  SVDQ_ERR_CUDA = 5,              /* a CUDA runtime / driver call failed */
  SVDQ_ERR_TIMEOUT = 6,           /* a bounded device wait ran out */
  SVDQ_ERR_NOT_INITIALIZED = 7    /* svdq_init() was not called for the device */
};

enum svdq_epilogue {
  SVDQ_EPILOGUE_NONE = 0,
  SVDQ_EPILOGUE_GELU_ERF = 1,     /* 0.5 y (1 + erf(y / sqrt 2)) */
  SVDQ_EPILOGUE_GELU_TANH = 2     /* 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))) */
};

#define SVDQ_LR_STRIDE 64  /* row stride (elements) of U and L2T; max rank */
#define SVDQ_GROUP 16      /* NVFP4 block size along K */
#define SVDQ_AMAX_WORKSPACE_BYTES 256  /* workspace of svdq_act_amax */
#define SVDQ_MAX_GROUP 4   /* problems per grouped launch */

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int svdq_version(void);

/* Text of the last error raised on the calling thread ("" if none). */
const char *svdq_last_error_string(void);

/* Name of a status code. */
const char *svdq_status_string(int status);

/*
 * Select and validate a GPU.  The pages require that an unsupported
 * GPU / kernel combination is reported as an error instead of running
 * silently (remio.ai, section "硬件支持划分了最快路径与最广泛路径"); here that
 * means anything but compute capability 10.0 (sm_100a: B200) returns
 * SVDQ_ERR_UNSUPPORTED_DEVICE.  Makes `device` current on the calling thread
 * and caches its properties.  Must precede the device calls below for that
 * device.  Idempotent.
 */
int svdq_init(int device);

/*
 * Byte sizes of the packed buffers of one SVDQ layer (host, no GPU).
 * Rules: K % 64 == 0, N % 8 == 0, 0 <= rank <= 64, rank % 16 == 0.
 *   inv_lambda [K] f32, L1T [rank][K] bf16, L2T (256-row tiles),
 *   w_bundle (256-row tiles).
 */
int svdq_weight_sizes(int K, int N, int rank, size_t *inv_lambda_bytes, size_t *l1t_bytes,
                      size_t *l2t_bytes, size_t *w_bundle_bytes);

/* Byte sizes of the activation-side buffers: a_bundle (128-row tiles) and U
 * (128-row tiles).  Rules: M >= 1, K % 64 == 0. */
int svdq_act_sizes(int M, int K, size_t *a_bundle_bytes, size_t *u_bytes);

/*
 * Offline quantization of one layer on the host (the pages' quantize step:
 * "diffuse-compressor" turns the weights into 4 bits and produces the
 * low-rank branch; donmalab.com, section "自行量化模型的流程").
 *
 *   W          [K][N] bf16, host.  Input features by output features.
 *   act_absmax [K] f32, host: per-input-channel max |X| over calibration
 *              data (the pages: calibration samples decide the scales and
 *              the low-rank correction, remio.ai, section
 *              "基准测试展示了性能提升，但并非普遍结论").
 *   rank       0..64, multiple of 16.
 *   num_threads host threads for the SVD (<= 0: all cores).
 * Outputs (host buffers of the sizes from svdq_weight_sizes):
 *   inv_lambda [K]  f32(1 / lambda_j), lambda_j = sqrt(absmaxX_j / absmaxW_j)
 *                   (1 when either is 0);
 *   l1t        [rank][K] bf16 = (U_r Sigma_r)^T of W' = W / inv_lambda;
 *   l2t        V_r (rows of V_r^T, transposed) as 256-row low-rank tiles;
 *   w_bundle   NVFP4 of R = W' - L1 L2 (f32-rounded), blocks along K, as a
 *              256-row bundle (output column n = row n);
 *   s_w        fp32 tensor scale of R: f32(max|R|) / 2688 (1 if R == 0);
 *   s_a        static activation tensor scale:
 *              max_j f32(absmaxX_j * inv_lambda_j) / 2688.
 *   residual   optional [K][N] f32 copy of f32(R) (NULL to skip).
 * The top-r SVD is a seeded randomized subspace iteration (deterministic for
 * a given seed and thread count).
 */
int svdq_pack_weights(const uint16_t *W, int K, int N, const float *act_absmax, int rank,
                      int num_threads, uint64_t seed, float *inv_lambda, uint16_t *l1t,
                      uint8_t *l2t, uint8_t *w_bundle, float *s_w, float *s_a, float *residual);

/*
 * Calibration on the GPU: act_absmax[k] = max(act_absmax[k], max_m |X[m][k]|)
 * for k < K (device buffers; act_absmax accumulates over calls: zero it
 * before the first batch).  The pages' offline quantize step derives the
 * scales from calibration data (remio.ai, section
 * "基准测试展示了性能提升，但并非普遍结论"); the result is svdq_pack_weights' /
 * svdq_pack_weights_device's act_absmax.
 * Rules: M >= 1, K % 8 == 0, ldx >= K, ldx % 8 == 0.
 */
int svdq_calibrate_absmax(const void *X, int M, int K, int ldx, float *act_absmax, svdq_stream_t stream);

/* Bytes of the device workspace svdq_pack_weights_device needs (host, no GPU):
 * the float64 W' [K][N] plus the subspace iteration's blocks. */
int svdq_pack_device_workspace_size(int K, int N, int rank, size_t *bytes);

/*
 * The offline pack of svdq_pack_weights, on the GPU (donmalab.com, section
 * "自行量化模型的流程": quantize the weights to 4 bits and produce the low-rank
 * branch).  Same arguments and results, in device memory, except:
 *   - the top-r subspace comes from the same randomized subspace iteration
 *     (oversampling 48, 10 power iterations, float64) with a counter-based
 *     random test matrix, so L1, L2 (and therefore R and its codes) differ
 *     from the host pack's within the freedom of the SVD; inv_lambda and s_a
 *     are identical;
 *   - residual is NULL or [K][N] f32 (device); workspace is a device buffer
 *     of svdq_pack_device_workspace_size bytes.
 * The float64 products run on cuBLAS; the small p x p factorizations between
 * them on the host, so the call synchronizes `stream` (an offline step, not
 * the hot path).  Rules: those of svdq_pack_weights; rank <= min(K, N).
 */
int svdq_pack_weights_device(const void *W, int K, int N, const float *act_absmax, int rank, uint64_t seed,
                             float *inv_lambda, void *l1t, uint8_t *l2t, uint8_t *w_bundle, float *s_w,
                             float *s_a, float *residual, void *workspace, svdq_stream_t stream);

/*
 * NVFP4 quantization of a host float32 matrix T [rows][K] (host, no GPU),
 * blocks of 16 along K under tensor scale s_t, into a bundle of tile height
 * tile_rows (128 or 256; bundle_bytes from the layout above).  Used by the
 * pack; exposed for tooling and tests.
 */
int svdq_quantize_host(const float *T, int rows, int K, float s_t, int tile_rows, uint8_t *bundle);

/*
 * Activation side of one SVDQ layer (the first fused kernel on the pages:
 * the low-rank down-projection combined with the quantization of the input,
 * remio.ai, section "SVDQuant 将棘手数值移出 4 位路径").  One pass over X:
 *   x^      = f32(x * inv_lambda[k])
 *   per block of 16 along K:  sb = e4m3_rne_sat(f32(amax|x^|) / f32(6 s_a)),
 *                             q  = e2m1_rne_sat(x^ * f32(1 / f32(sb * s_a)))
 *   U[m][j] = bf16( sum_k bf16(x^[m][k]) * L1T[j][k] / f32(s_a * s_w) )
 * Args: X [M][ldx] bf16 (device), ldx >= K; inv_lambda [K] f32; l1t
 * [rank][K] bf16 (ignored when rank == 0); s_a, s_w device scalars (f32);
 * outputs a_bundle (128-row bundle, padding rows and columns written as 0)
 * and U (128-row low-rank tiles, columns rank..63 and padding rows 0).
 * Rules: K % 64 == 0, ldx % 8 == 0, 0 <= rank <= 64, rank % 16 == 0, M >= 1.
 */
int svdq_quantize_act(const void *X, int M, int K, int ldx, const float *inv_lambda,
                      const void *l1t, int rank, const float *s_a, const float *s_w,
                      uint8_t *a_bundle, void *U, svdq_stream_t stream);

/*
 * Dynamic activation scale (optional pre-pass of svdq_quantize_act).  The
 * pages say calibration decides the quantization scales (remio.ai, section
 * "基准测试展示了性能提升，但并非普遍结论"); svdq_pack_weights calibrates a static
 * s_a once, this call takes it from the tensor being quantized instead:
 *   s_a = f32(max_{m,k} |f32(x[m][k] * inv_lambda[k])|) / 2688   (1 if that max is 0)
 * written to the device scalar *s_a, in the f32 steps svdq_quantize_act uses;
 * pass the same scalar to svdq_quantize_act and svdq_linear_w4a4.
 * Args: X [M][ldx] bf16, inv_lambda [K] f32, workspace: device buffer of
 * SVDQ_AMAX_WORKSPACE_BYTES (cleared and used by the call; free again when
 * the call's stream work is done), s_a: one f32 (device).  Enqueues a memset
 * of the workspace and one kernel.
 * Rules: M >= 1, K % 64 == 0, ldx >= K, ldx % 8 == 0.
 */
int svdq_act_amax(const void *X, int M, int K, int ldx, const float *inv_lambda, void *workspace, float *s_a,
                  svdq_stream_t stream);

/*
 * The W4A4 GEMM with the low-rank up-projection fused in (the second fused
 * kernel on the pages, remio.ai, section "SVDQuant 将棘手数值移出 4 位路径"):
 *   acc = U . L2T^T + sum_k qa sa qw sw     (tcgen05 block-scaled FP4, fp32)
 *   Y   = bf16( epilogue( f32(s_a s_w) * acc + bias ) )
 * epilogue: svdq_epilogue; GELU applies to output columns >= gelu_col_begin
 * only (a fused QKV + MLP-in projection activates just its MLP part).
 * Args: a_bundle and U from svdq_quantize_act; w_bundle, L2T and the
 * scalars from svdq_pack_weights (uploaded); bias [N] bf16 or NULL;
 * Y [M][ldy] bf16, ldy >= N.
 * Rules: K % 64 == 0, N % 8 == 0, ldy % 8 == 0, 0 <= rank <= 64,
 * rank % 16 == 0, M >= 1, 0 <= gelu_col_begin <= N.
 */
int svdq_linear_w4a4(const uint8_t *a_bundle, const void *U, const float *s_a,
                     const uint8_t *w_bundle, const void *l2t, const float *s_w, const void *bias,
                     int M, int N, int K, int rank, int epilogue, int gelu_col_begin, void *Y,
                     int ldy, svdq_stream_t stream);

/*
 * Grouped launches: several independent layers of the same kind in one
 * launch, for a step that runs the same projection on streams of different
 * lengths (a dual-stream DiT block's image tokens and text tokens).  The
 * pages' pipeline runs each projection on both streams; one launch over both
 * keeps the whole GPU busy where the short stream alone would fill a few
 * SMs.  No counterpart on the pages beyond that: the arithmetic of every
 * problem is exactly that of the single call with the same arguments.
 * `problems` is a HOST array of `count` (1..SVDQ_MAX_GROUP) descriptors,
 * read during the call; each problem's fields follow the single call's
 * arguments, meaning and rules.  Errors name the first bad problem.
 */
typedef struct svdq_quant_problem {
  const void *X;                /* [M][ldx] bf16 */
  int M, K, ldx;
  const float *inv_lambda;      /* [K] f32 */
  const void *l1t;              /* [rank][K] bf16 */
  const float *s_a, *s_w;       /* device scalars */
  uint8_t *a_bundle;            /* out */
  void *U;                      /* out */
} svdq_quant_problem;

typedef struct svdq_w4a4_problem {
  const uint8_t *a_bundle;
  const void *U;
  const float *s_a;
  const uint8_t *w_bundle;
  const void *l2t;
  const float *s_w;
  const void *bias;             /* [N] bf16 or NULL */
  int M, N, K;
  int gelu_col_begin;
  void *Y;                      /* [M][ldy] bf16 */
  int ldy;
} svdq_w4a4_problem;

/* svdq_quantize_act on every problem; all problems share `rank`. */
int svdq_quantize_act_grouped(const svdq_quant_problem *problems, int count, int rank, svdq_stream_t stream);

/* svdq_linear_w4a4 on every problem; all share `rank` and `epilogue`.  The
 * persistent SM pairs take the problems' 256 x 256 tiles as one sequence. */
int svdq_linear_w4a4_grouped(const svdq_w4a4_problem *problems, int count, int rank, int epilogue,
                             svdq_stream_t stream);

/*
 * The W4A4 GEMM of a layer whose output is the input of the next SVDQ layer
 * (MLP fc1 -> fc2), re-quantizing its output for that layer in the same
 * kernel.  The pages fuse the quantization of a layer's input with its
 * low-rank down-projection (remio.ai, section "SVDQuant 将棘手数值移出 4 位路径");
 * this call moves that fusion into the epilogue of the producing GEMM, so the
 * 16-bit activation between the two layers is never written out and the next
 * layer needs no svdq_quantize_act.  With y = the layer's output (after the
 * epilogue, as svdq_linear_w4a4 computes it), for the next layer:
 *   x^      = f32(bf16(y) * next_inv_lambda[n])          (n < N; K_next = N)
 *   next_a_bundle, next_U = exactly what svdq_quantize_act would write for an
 *             input X = bf16(y) with next_inv_lambda, next_l1t, next_rank,
 *             next_s_a and next_s_w (codes and block scales bit-identical;
 *             U's fp32 sum is formed in another order, so it may differ in
 *             the last bit of its bf16 rounding).
 * Args: the first fifteen as svdq_linear_w4a4, except that Y may be NULL (the
 * bf16 output is then not written at all, ldy ignored).  next_inv_lambda [N]
 * f32, next_l1t [next_rank][N] bf16, next_s_a / next_s_w device scalars of
 * the next layer; next_a_bundle (128-row bundle of M x N, size from
 * svdq_act_sizes(M, N)), next_U (128-row low-rank tiles); workspace: device
 * buffer of svdq_requant_workspace_size(M, next_rank) bytes (fp32 partial
 * sums), cleared and used by the call, free again when the call's stream
 * work is done; next_l1t, next_U and workspace may be NULL when next_rank
 * is 0.  The call enqueues a memset of the workspace, the GEMM and one small
 * kernel that turns the sums into next_U.
 * Rules: those of svdq_linear_w4a4, plus N % 64 == 0 and next_rank a
 * multiple of 16 in [0, 64].
 */
int svdq_linear_w4a4_requant(const uint8_t *a_bundle, const void *U, const float *s_a,
                             const uint8_t *w_bundle, const void *l2t, const float *s_w, const void *bias,
                             int M, int N, int K, int rank, int epilogue, int gelu_col_begin, void *Y,
                             int ldy, const float *next_inv_lambda, const void *next_l1t, int next_rank,
                             const float *next_s_a, const float *next_s_w, uint8_t *next_a_bundle,
                             void *next_U, float *workspace, svdq_stream_t stream);

/*
 * svdq_linear_w4a4_requant without the workspace argument, for callers that
 * cannot allocate device memory: a plugin of an inference engine whose
 * interface hands over only a layer's inputs and outputs, or code that must
 * not call cudaMalloc between kernels (the call can synchronize the device)
 * and keeps no memory pool of its own.  No counterpart on the pages: it is an
 * interface variant of this library, the arithmetic is that of
 * svdq_linear_w4a4_requant.
 * The fp32 partial sums live in one fixed array in the library's device image
 * (1 MiB, every GPU that loads the library holds it until the process exits):
 * M * next_rank must be at most 262144, else SVDQ_ERR_SHAPE.  Every call on a
 * device shares that array and the call clears it first, so calls whose
 * stream work overlaps on the GPU (other streams, other threads) race on it;
 * serialize them.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  It allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 */
int svdq_linear_w4a4_requant_noalloc(const uint8_t *a_bundle, const void *U, const float *s_a,
                                     const uint8_t *w_bundle, const void *l2t, const float *s_w,
                                     const void *bias, int M, int N, int K, int rank, int epilogue,
                                     int gelu_col_begin, void *Y, int ldy, const float *next_inv_lambda,
                                     const void *next_l1t, int next_rank, const float *next_s_a,
                                     const float *next_s_w, uint8_t *next_a_bundle, void *next_U,
                                     svdq_stream_t stream);

/* Bytes of the workspace svdq_linear_w4a4_requant needs: M * next_rank * 4
 * (host, no GPU).  Rules: M >= 1, next_rank a multiple of 16 in [0, 64]. */
int svdq_requant_workspace_size(int M, int next_rank, size_t *bytes);

/*
 * Offline AWQ quantization on the host (asymmetric INT4 per group along K):
 *   W_a = diag(awq_scale) W;  per group and output column:
 *   lo = min(0, min W_a), hi = max(0, max W_a), s = bf16((hi - lo) / 15),
 *   z = clamp(rne(-lo / s), 0, 15), q = clamp(rne(W_a / s) + z, 0, 15);
 *   an all-zero group takes s = 1, z = 0.  inv_awq[k] = f32(1 / awq_scale[k]).
 * Args: W [K][N] bf16 host; awq_scale [K] f32 (> 0); group 64 (K % group == 0);
 * N % 64 == 0; outputs qweight (N*K/8 u32, fragment order above),
 * scales/zeros (N*K/group bf16 each, layout above), inv_awq [K].
 */
int awq_pack_weights(const uint16_t *W, int K, int N, const float *awq_scale, int group,
                     uint32_t *qweight, uint16_t *scales, uint16_t *zeros, float *inv_awq);

/*
 * Byte sizes of the packed AWQ buffers of a K x N weight (host, no GPU):
 * qweight N*K/2, scales and zeros N*K/group*2 each, inv_awq K*4.
 * Rules: group == 64, K % 64 == 0, N % 64 == 0.
 */
int awq_packed_sizes(int K, int N, int group, size_t *qweight_bytes, size_t *scales_bytes,
                     size_t *zeros_bytes, size_t *inv_awq_bytes);

/*
 * AWQ W4A16 projection for small row counts (the modulation / adaLN layers):
 *   Y[m][n] = bf16( sum_g s(n,g) * sum_{k in g} f32(x[m][k] inv_awq[k]) (q - z(n,g)) + bias[n] )
 * in fp32.  X [M][ldx] bf16; inv_awq [K] f32 or NULL (= 1); bias [N] or NULL.
 * The products run on tensor cores with X^ split into bf16 hi + lo parts
 * (relative error of the split ~2^-17).
 * Rules: 1 <= M <= 1048560, group == 64, K % 64 == 0, N % 64 == 0, ldx >= K,
 * ldy >= N, ldx % 8 == 0, ldy % 8 == 0.  Up to 16 rows are one pass over
 * the weights; more rows run as blocks of 16, one pass each (from L2).
 */
int awq_linear_w4a16(const void *X, int M, int K, int ldx, const float *inv_awq,
                     const uint32_t *qweight, const void *scales, const void *zeros, int group,
                     const void *bias, int N, void *Y, int ldy, svdq_stream_t stream);

/*
 * Several AWQ projections of the same input shape in one launch (the
 * modulation / adaLN layers of a DiT step all read the same conditioning
 * vector).  Each problem is computed exactly as awq_linear_w4a16 computes it
 * (the same kernel per 64-column quad; outputs bit-identical to separate
 * calls); the problems' quads form one grid, problem after problem.
 * `problems` is a HOST array of `count` (1..SVDQ_AWQ_MAX_GROUP) descriptors,
 * read during the call; M, K and group are shared; every descriptor obeys the
 * rules of awq_linear_w4a16 (its own X, ldx, inv_awq, weights, bias, N, Y,
 * ldy).  Errors as awq_linear_w4a16, checked for every problem before
 * anything is launched; SVDQ_ERR_INVALID_ARG for count outside the range.
 */
#define SVDQ_AWQ_MAX_GROUP 128
typedef struct awq_problem {
  const void *X;              /* [M][ldx] bf16 */
  int ldx;
  const float *inv_awq;       /* [K] f32 or NULL */
  const uint32_t *qweight;    /* N*K/2 bytes, layout of awq_pack_weights */
  const void *scales;         /* bf16 */
  const void *zeros;          /* bf16 */
  const void *bias;           /* [N] bf16 or NULL */
  int N;
  void *Y;                    /* [M][ldy] bf16 */
  int ldy;
} awq_problem_t;
int awq_linear_w4a16_grouped(const awq_problem_t *problems, int count, int M, int K, int group,
                             svdq_stream_t stream);

/*
 * AWQ W4A16 for many rows (the GEMM path; awq_linear_w4a16 reads the packed
 * weights once per block of 16 rows, which suits the few rows of a
 * modulation layer).  Same result definition as awq_linear_w4a16,
 *   Y = (X diag(inv_awq)) deq(W) + bias,
 * computed as: w = f32(inv_awq[k] (q - z) s) expanded into two bf16 matrices
 * W_hi = bf16(w), W_lo = bf16(w - W_hi) (together ~16 significant bits),
 * D = X . W_hi + X . W_lo in fp32 (two bf16 GEMMs through cuBLASLt), then
 * Y = bf16(D + bias).  The pages have no counterpart beyond the W4A16
 * projection itself.
 * workspace: device scratch of awq_gemm_workspace_size(M, K, N) bytes
 * (4 K N for W_hi and W_lo, then 4 M N for D), 16-byte aligned; its contents
 * do not matter and are overwritten.
 * Args and rules: those of awq_linear_w4a16 (any M >= 1), plus workspace and a
 * 16-byte aligned bias when given.
 */
int awq_gemm_workspace_size(int M, int K, int N, size_t *bytes);
/* The two halves of awq_linear_w4a16_gemm, for a layer called many times:
 * awq_expand_weights writes W_hi and W_lo into the first 4 K N bytes of the
 * workspace (its arguments and rules as in awq_linear_w4a16_gemm); as long as
 * the caller keeps those bytes, awq_linear_w4a16_expanded computes Y from them
 * (the workspace of awq_gemm_workspace_size(M, K, N) bytes: the expansion,
 * then D). */
int awq_expand_weights(const float *inv_awq, const uint32_t *qweight, const void *scales, const void *zeros,
                       int K, int N, int group, void *workspace, svdq_stream_t stream);
int awq_linear_w4a16_expanded(const void *X, int M, int K, int ldx, const void *bias, int N, void *Y, int ldy,
                              void *workspace, svdq_stream_t stream);
int awq_linear_w4a16_gemm(const void *X, int M, int K, int ldx, const float *inv_awq,
                          const uint32_t *qweight, const void *scales, const void *zeros, int group,
                          const void *bias, int N, void *Y, int ldy, void *workspace, svdq_stream_t stream);

/*
 * Waits for `stream`, then returns and clears the device status word of the
 * current device: SVDQ_OK, or SVDQ_ERR_TIMEOUT if a kernel's bounded wait ran
 * out since the last check (SVDQ_ERR_CUDA if the stream itself failed).
 * There is one status word per device, shared by the kernels of every stream:
 * a check synchronizes only `stream`, so a timeout recorded by a kernel still
 * running on another stream may be reported by a later check, or cleared by
 * this one if it lands between the read and the clear.  Callers that use
 * several streams and need an exact attribution synchronize the device first.
 */
int svdq_check_status(svdq_stream_t stream);

/* ------------------------------------------------------------- INT4 W4A4
 * The pages ship an INT4 W4A4 variant beside NVFP4 for GPUs without NVFP4
 * (donmalab.com, "Diffusers × Nunchaku 4-bit", section "實務上的影響與硬體要求";
 * remio.ai, section "硬件支持划分了最快路径与最广泛路径") and give no layout.
 * This library's reading: the NVFP4 layer (smoothing, low-rank branch,
 * residual; svdq_pack_weights) with its 4-bit branch in signed integers,
 * groups of 64 along K, one bf16 scale per row (activations) or output column
 * (weights) and group:
 *   s = bf16(f32(amax / 7)),   q = clamp(rne(f32(v * f32(1 / s))), -8, 7)
 * with s = 0 and q = 0 for a group whose amax is below 2^-120.
 * Layouts: codes [rows][K/2] bytes, element k in byte k/2 (low nibble for
 * even k), two's complement; scales [K/64][ld] bf16 (group-major), ld = N for
 * weights and the activation rows rounded up to 128 for activations.  U and
 * L2T keep the low-rank tile layouts of the NVFP4 calls.
 */

/* Byte sizes of the INT4 weight codes and scales.  Rules: K % 64 == 0, N % 128 == 0. */
int svdq_int4_weight_sizes(int K, int N, size_t *codes_bytes, size_t *scales_bytes);

/* Byte sizes of the INT4 activation codes and scales (rows rounded up to 128).
 * Rules: M >= 1, K % 64 == 0. */
int svdq_int4_act_sizes(int M, int K, size_t *codes_bytes, size_t *scales_bytes);

/*
 * Group quantization of host float32 rows T [rows][K] (host, no GPU) into
 * codes [rows][K/2] and scales [K/64][ld_s] (ld_s >= rows): the weight side of
 * the INT4 pack, applied to the transposed residual R^T [N][K] that
 * svdq_pack_weights returns.  Rules: rows >= 1, K % 64 == 0, ld_s >= rows.
 */
int svdq_quantize_int4_host(const float *T, int rows, int K, int ld_s, uint8_t *codes, uint16_t *scales);

/*
 * Activation side of the INT4 layer, one pass over X like svdq_quantize_act:
 *   x^ = f32(x * inv_lambda[k]);  codes and scales of x^ as above;
 *   U[m][j] = bf16( sum_k bf16(x^[m][k]) * L1T[j][k] )   (no tensor scale)
 * Args: X [M][ldx] bf16 (device); inv_lambda [K] f32; l1t [rank][K] bf16
 * (ignored when rank == 0); outputs a_codes, a_scales (sizes from
 * svdq_int4_act_sizes; padding rows written as 0) and U (128-row low-rank
 * tiles).  Rules: those of svdq_quantize_act.
 */
int svdq_quantize_act_int4(const void *X, int M, int K, int ldx, const float *inv_lambda, const void *l1t,
                           int rank, uint8_t *a_codes, void *a_scales, void *U, svdq_stream_t stream);

/*
 * The INT4 GEMM with the low-rank up-projection fused in:
 *   Y = bf16( epilogue( sum_g (s_a[m,g] s_w[n,g]) sum_{k in g} q_a q_w
 *                       + U . L2T^T + bias ) )
 * B200 has no 4-bit integer MMA.  The codes become exact fp16 operands q * s
 * (4 + 8 significant bits fit fp16's 11; exact while |q s| lies in fp16's
 * normal range, i.e. activation and weight magnitudes below ~57,000 and group
 * scales above 2^-14) multiplied on the tensor cores (tcgen05 kind::f16, fp32
 * accumulation, no per-group rescale) by persistent SM pairs over 256 x 256
 * tiles, with a last tile of 128 columns when N % 256 == 128.
 * Args: a_codes, a_scales, U from svdq_quantize_act_int4; w_codes,
 * w_scales from svdq_quantize_int4_host, l2t from svdq_pack_weights
 * (uploaded); bias [N] bf16 or NULL; Y [M][ldy] bf16.
 * Rules: M >= 1, K % 64 == 0, N % 128 == 0, ldy >= N, ldy % 8 == 0,
 * 0 <= rank <= 64, rank % 16 == 0, 0 <= gelu_col_begin <= N.
 */
int svdq_linear_int4(const uint8_t *a_codes, const void *a_scales, const void *U, const uint8_t *w_codes,
                     const void *w_scales, const void *l2t, const void *bias, int M, int N, int K, int rank,
                     int epilogue, int gelu_col_begin, void *Y, int ldy, svdq_stream_t stream);

/*
 * Self-test of the bounded wait used by every kernel: launches one block that
 * waits on a shared-memory barrier nothing will ever complete, with a limit
 * of `limit_ns` nanoseconds.  The status word then holds SVDQ_ERR_TIMEOUT.
 * Exists so that the timeout path can be tested without a fault.
 */
int svdq_debug_wait_timeout(uint64_t limit_ns, svdq_stream_t stream);

/*
 * Conversion probe (device buffers, n even):
 *   e2m1_out[i] = e2m1(in[2i+1]) << 4 | e2m1(in[2i])   for i < n/2
 *   e4m3_out[i] = e4m3(in[i])                           for i < n
 * both round-to-nearest-even with saturation, through the same conversion
 * instructions the kernels use.  Lets the tests check those conversions
 * against the format definitions.
 */
int svdq_debug_convert(const float *in, int n, uint8_t *e2m1_out, uint8_t *e4m3_out,
                       svdq_stream_t stream);

/*
 * GELU probe (device buffers): out[i] = GELU(in[i]) for i < n through the
 * device function the W4A4 epilogue applies, kind = SVDQ_EPILOGUE_GELU_ERF
 * (erf form, erf by Abramowitz & Stegun 7.1.26) or SVDQ_EPILOGUE_GELU_TANH.
 * Lets the tests bound that function's error against the definition.
 */
int svdq_debug_gelu(const float *in, int n, int kind, float *out, svdq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_B200_H */
