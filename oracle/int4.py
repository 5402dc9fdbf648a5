"""INT4 W4A4 variant of the SVDQuant layer: the 4-bit branch in signed integers.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The pages ship an INT4 W4A4 variant beside NVFP4, for the GPUs that have no
NVFP4 (web page "Diffusers × Nunchaku 4-bit", donmalab.com, section
"實務上的影響與硬體要求"; remio.ai, section "硬件支持划分了最快路径与最广泛路径").
They give no layout for it.  Readings (each also in the design notes):

  * smoothing, the low-rank branch and the residual R are those of the NVFP4
    layer (svdquant.pack): only the 4-bit branch changes;
  * the 4-bit branch quantizes along K in groups of 64 (the group size the
    pages' AWQ W4A16 layers use), symmetric signed integers, one scale per
    row (activations) or output column (weights) and group:
        s = bf16(f32(amax / 7))                 RNE; amax over the group
        q = clamp(rne(f32(v * f32(1 / s))), -8, 7)
    v is the f32 value (X^ = f32(x * inv_lambda) for activations, f32(R) for
    weights); like the NVFP4 quantizer it multiplies by the f32 reciprocal.
    A group whose amax is below 2^-120 has s = 0 and q = 0 (the reciprocal
    would overflow);
  * the GEMM: Y = sum_g (s_a[m,g] s_w[n,g]) sum_{k in g} qa[m,k] qw[n,k]
    + U . L2 + b, U = bf16(X^) . L1 (no tensor scale to divide out; U is
    stored in bf16), then the optional GELU, as in svdquant.w4a4_linear.
"""
import numpy as np

from . import formats, svdquant

F32 = np.float32
GROUP = 64
QMIN, QMAX = -8, 7
TINY = np.float32(2.0 ** -120)


def group_scales(v):
    """v: float32 [rows, K] (K a multiple of 64) -> scales as float64 [rows, K/64] (bf16 values)."""
    v = np.asarray(v, dtype=F32)
    rows, k = v.shape
    amax = np.max(np.abs(v.reshape(rows, k // GROUP, GROUP)), axis=2).astype(F32)
    s = formats.bf16_round((amax / F32(7.0)).astype(F32).astype(np.float64))
    return np.where(amax < TINY, 0.0, s)


def quantize_groups(v):
    """v: float32 [rows, K] -> (q int8 [rows, K] in [-8, 7], s float64 [rows, K/64])."""
    v = np.asarray(v, dtype=F32)
    rows, k = v.shape
    s = group_scales(v)
    s32 = s.astype(F32)
    with np.errstate(divide="ignore"):
        r = np.where(s32 > 0, F32(1.0) / np.where(s32 > 0, s32, F32(1.0)), F32(0.0)).astype(F32)
    prod = (v.reshape(rows, k // GROUP, GROUP) * r[:, :, None]).astype(F32)
    q = np.clip(np.rint(prod), QMIN, QMAX).astype(np.int8).reshape(rows, k)
    return q, s


def dequantize(q, s):
    rows, k = q.shape
    return (q.reshape(rows, k // GROUP, GROUP).astype(np.float64) * s[:, :, None]).reshape(rows, k)


def pack(w, amax_x, rank, round_bf16=True):
    """Offline quantization of one layer: the NVFP4 pack's smoothing, low-rank
    branch and residual, with the residual in INT4 groups along K per output
    column.  w: float64 [K, N] (bf16 values); amax_x: float32 [K]."""
    p = svdquant.pack(w, amax_x, rank, round_bf16)
    qw, sw = quantize_groups(p["residual"].astype(F32).T)      # [N, K], [N, K/64]
    return dict(inv_lambda=p["inv_lambda"], l1=p["l1"], l2=p["l2"], residual=p["residual"], qw=qw, sw=sw)


def quantize_act(x, inv_lambda, l1):
    """x: float64 [M, K] (bf16 values) -> (qa int8 [M, K], sa [M, K/64], U float64 [M, r])."""
    x = np.asarray(x, dtype=np.float64)
    inv = np.asarray(inv_lambda, dtype=F32)
    x_hat32 = (x.astype(F32) * inv[None, :]).astype(F32)
    qa, sa = quantize_groups(x_hat32)
    x_hat16 = formats.bf16_round(x_hat32.astype(np.float64))
    u = x_hat16 @ np.asarray(l1, dtype=np.float64)
    return qa, sa, u


def int4_linear(qa, sa, qw, sw, u, l2, bias=None, epilogue=svdquant.EPILOGUE_NONE, gelu_col_begin=0):
    """Y = sum over groups of (sa sw) (qa . qw^T restricted to the group) + U . L2 + b, then the
    optional GELU on columns >= gelu_col_begin.  float64 [M, N].

    qa [M, K], sa [M, K/64]; qw [N, K], sw [N, K/64]; u [M, r]; l2 [r, N]; bias [N] or None."""
    m, k = qa.shape
    n = qw.shape[0]
    y = np.zeros((m, n), dtype=np.float64)
    for g in range(k // GROUP):
        sl = slice(GROUP * g, GROUP * (g + 1))
        p = qa[:, sl].astype(np.int64) @ qw[:, sl].astype(np.int64).T       # exact integer partials
        y += (sa[:, g][:, None] * sw[:, g][None, :]) * p.astype(np.float64)
    l2 = np.asarray(l2, dtype=np.float64)
    if l2.shape[0]:
        y = y + np.asarray(u, dtype=np.float64) @ l2
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    if epilogue != svdquant.EPILOGUE_NONE:
        y = y.copy()
        y[:, gelu_col_begin:] = svdquant.gelu(y[:, gelu_col_begin:], epilogue)
    return y


def forward(x, packed, bias=None, epilogue=svdquant.EPILOGUE_NONE, gelu_col_begin=0):
    """The whole layer on one activation: quantize_act then int4_linear (U in bf16, as stored)."""
    qa, sa, u = quantize_act(x, packed["inv_lambda"], packed["l1"])
    return int4_linear(qa, sa, packed["qw"], packed["sw"], formats.bf16_round(u), packed["l2"], bias, epilogue,
                       gelu_col_begin)
