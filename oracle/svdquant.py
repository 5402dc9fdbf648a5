"""SVDQuant linear layer: smoothing, low-rank 16-bit branch, NVFP4 residual.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

What the layer computes, after [Remio] "SVDQuant 将棘手数值移出 4 位路径" and
[Donmalab] "量化的核心挑戰：為什麼 4-bit 很難？":

  1. Smoothing moves activation outliers into the weight:
        X^ = X . diag(lambda)^-1,      W' = diag(lambda) . W
  2. A small 16-bit low-rank branch holds the hardest part of W':
        L1 . L2 = top-r SVD of W'      (L1 = U_r Sigma_r, L2 = V_r^T, bf16)
  3. The rest is quantized to 4 bits, activations and weights alike:
        R = W' - L1 . L2
  4. The two branches are added:
        Y = (X^ . L1) . L2 + Q(X^) . Q(R) + b

W is [K, N] (input features by output features); X is [M, K].

Readings where the pages are silent (each also in the design notes):
  * lambda_j = sqrt(amaxX_j / amaxW_j) (migration strength 1/2), lambda_j = 1
    if either maximum is 0; the kernels receive inv_lambda = f32(1/lambda).
  * W' divides by the float32 inv_lambda (float64 division), so that
    X^ . W' equals X . W whenever X^ = X . inv_lambda.
  * The activation tensor scale is static: calibrated from the per-channel
    absolute maxima of X (the pages: calibration samples decide the scales,
    section "基准测试展示了性能提升，但并非普遍结论").
  * The low-rank branch is a small 16-bit branch ([Remio], section "SVDQuant
    将棘手数值移出 4 位路径"): its input
    is the smoothed activation rounded to bf16 (RNE of the float32 X^), its
    factors are bf16; products and sums are exact here (float64).
  * The low-rank up-projection enters the 4-bit GEMM's accumulator divided by
    alpha = f32(s_A * s_W), the epilogue multiplies by alpha (the fusion of the
    up-projection into the 4-bit GEMM, section "SVDQuant 将棘手数值移出 4 位路径").
  * GELU is the erf form unless the tanh form is asked for.
"""
import math

import numpy as np
from scipy.special import erf

from . import formats, nvfp4

F32 = np.float32

EPILOGUE_NONE = 0
EPILOGUE_GELU_ERF = 1
EPILOGUE_GELU_TANH = 2


def smooth(amax_x, amax_w):
    """inv_lambda_j = f32(1 / sqrt(amaxX_j / amaxW_j)) per input channel j."""
    ax = np.asarray(amax_x, dtype=np.float64)
    aw = np.asarray(amax_w, dtype=np.float64)
    lam = np.ones_like(ax)
    ok = (ax > 0) & (aw > 0)
    lam[ok] = np.sqrt(ax[ok] / aw[ok])
    return (1.0 / lam).astype(F32)


def smoothed_weight(w, inv_lambda):
    """W'_{jn} = W_{jn} / inv_lambda_j in float64."""
    return np.asarray(w, dtype=np.float64) / np.asarray(inv_lambda, dtype=np.float64)[:, None]


def low_rank(w_prime, rank, round_bf16=True):
    """Top-r SVD branch: L1 = U_r Sigma_r [K, r], L2 = V_r^T [r, N].

    With round_bf16 the factors are rounded to bf16 (the 16-bit branch).
    Singular vectors are only defined up to sign, so callers compare L1.L2.
    """
    k, n = w_prime.shape
    if rank == 0:
        return np.zeros((k, 0)), np.zeros((0, n))
    u, s, vt = np.linalg.svd(w_prime, full_matrices=False)
    l1 = u[:, :rank] * s[:rank]
    l2 = vt[:rank, :]
    if round_bf16:
        l1 = formats.bf16_round(l1)
        l2 = formats.bf16_round(l2)
    return l1, l2


def activation_tensor_scale(amax_x, inv_lambda):
    """s_A from per-channel calibration maxima: amax_j f32(amaxX_j * inv_j) / 2688."""
    prod = (np.asarray(amax_x, dtype=F32) * np.asarray(inv_lambda, dtype=F32)).astype(F32)
    return nvfp4.tensor_scale(np.max(prod) if prod.size else F32(0.0))


def dynamic_activation_scale(x, inv_lambda):
    """s_A of one activation tensor, taken from that tensor itself: f32(max |X^|) / 2688 with
    X^ = f32(x * inv_lambda), 1 when that maximum is 0.

    The static reading calibrates s_A once from calibration data; the pages only say that
    calibration decides the scales ([Remio] "基准测试展示了性能提升，但并非普遍结论"), so the
    per-call (dynamic) scale is the other reading, offered as an optional pre-pass.  Calibrated on
    the same tensor, the two agree: f32 multiplication by inv_j >= 0 is monotonic, so the largest
    f32(|x_mj| inv_j) of a column is f32(max_m |x_mj| inv_j).
    """
    x = np.asarray(x, dtype=np.float64)
    inv = np.asarray(inv_lambda, dtype=F32)
    x_hat32 = (x.astype(F32) * inv[None, :]).astype(F32)
    return nvfp4.tensor_scale(np.max(np.abs(x_hat32)) if x_hat32.size else F32(0.0))


def pack(w, amax_x, rank, round_bf16=True):
    """Offline quantization of one layer ([Donmalab] "自行量化模型的流程": quantize
    the weights to 4 bits and produce the low-rank branch).

    w: float64 [K, N] holding bf16 values; amax_x: float32 [K] calibration
    maxima of |X| per input channel.
    """
    w = np.asarray(w, dtype=np.float64)
    amax_w = np.max(np.abs(w), axis=1)
    inv_lambda = smooth(amax_x, amax_w)
    w_prime = smoothed_weight(w, inv_lambda)
    l1, l2 = low_rank(w_prime, rank, round_bf16)
    r = w_prime - l1 @ l2
    r32 = r.astype(F32)
    s_w = nvfp4.tensor_scale(np.max(np.abs(r32)) if r32.size else 0.0)
    w_codes, w_sf = nvfp4.quantize_blocks(r32.T, s_w)      # blocks along K per column
    s_a = activation_tensor_scale(amax_x, inv_lambda)
    return dict(inv_lambda=inv_lambda, w_prime=w_prime, l1=l1, l2=l2, residual=r,
                s_w=s_w, w_codes=w_codes, w_sf=w_sf, s_a=s_a)


def alpha(s_a, s_w):
    return F32(F32(s_a) * F32(s_w))


def quantize_act(x, inv_lambda, l1, s_a, s_w):
    """Activation side ([Remio]: input quantization fused with the low-rank
    down-projection).

    x: float64 [M, K] holding bf16 values.  Returns NVFP4 codes [M, K] and
    scales [M, K/16] of X^ = f32(x * inv_lambda), and U = (bf16(X^) . L1) /
    alpha in float64 (the 16-bit branch takes X^ in bf16).
    """
    x = np.asarray(x, dtype=np.float64)
    inv = np.asarray(inv_lambda, dtype=F32)
    x_hat32 = (x.astype(F32) * inv[None, :]).astype(F32)
    codes, sf = nvfp4.quantize_blocks(x_hat32, s_a)
    x_hat16 = formats.bf16_round(x_hat32.astype(np.float64))
    u = (x_hat16 @ np.asarray(l1, dtype=np.float64)) / np.float64(alpha(s_a, s_w))
    return codes, sf, u


def gelu(y, kind):
    if kind == EPILOGUE_GELU_ERF:
        return 0.5 * y * (1.0 + erf(y / math.sqrt(2.0)))
    if kind == EPILOGUE_GELU_TANH:
        return 0.5 * y * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (y + 0.044715 * y ** 3)))
    raise ValueError("unknown GELU kind")


def w4a4_linear(a_codes, a_sf, s_a, w_codes, w_sf, s_w, u_over_alpha, l2, bias=None,
                epilogue=EPILOGUE_NONE, gelu_col_begin=0):
    """Y = alpha * (U/alpha) . L2 + deq(A) . deq(W)^T + b, then optional GELU on
    columns >= gelu_col_begin.  float64 [M, N].

    a_codes [M, K], a_sf [M, K/16], w_codes [N, K], w_sf [N, K/16];
    u_over_alpha [M, r]; l2 [r, N]; bias [N] or None.
    """
    a = nvfp4.dequantize(a_codes, a_sf, s_a)
    b = nvfp4.dequantize(w_codes, w_sf, s_w)
    y = a @ b.T
    l2 = np.asarray(l2, dtype=np.float64)
    if l2.shape[0]:
        y = y + np.float64(alpha(s_a, s_w)) * (np.asarray(u_over_alpha, dtype=np.float64) @ l2)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    if epilogue != EPILOGUE_NONE:
        y = y.copy()
        y[:, gelu_col_begin:] = gelu(y[:, gelu_col_begin:], epilogue)
    return y


def forward(x, packed, bias=None, epilogue=EPILOGUE_NONE, gelu_col_begin=0):
    """The whole layer on one activation: quantize_act then w4a4_linear."""
    codes, sf, u = quantize_act(x, packed["inv_lambda"], packed["l1"], packed["s_a"],
                                packed["s_w"])
    return w4a4_linear(codes, sf, packed["s_a"], packed["w_codes"], packed["w_sf"],
                       packed["s_w"], u, packed["l2"], bias, epilogue, gelu_col_begin)
