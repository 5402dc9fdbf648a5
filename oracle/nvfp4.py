"""Two-level NVFP4 quantization of a 2-D tensor along its last axis.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The pages say that the residual weight and the smoothed activation both run
in 4 bits and that Blackwell uses the NVFP4 format ([Remio] "SVDQuant
将棘手数值移出 4 位路径" and "硬件支持划分了最快路径与最广泛路径"; [Donmalab]
"實務上的影響與硬體要求").  The format itself: e2m1 elements, one ue4m3 scale
per 16 consecutive elements along K, one fp32 scale per tensor.

Steps, each in float32 with one IEEE rounding per operation (the precision
that decides the codes, shared with the kernels):

  s_T   = f32(amax(|T|)) / 2688            (2688 = 6 * 448: the largest block
                                             scale lands on the largest e4m3)
  d     = 6 * s_T
  sb    = ue4m3( f32(amax_block) / d )      per block of 16, RNE, satfinite
  scale = sb * s_T
  inv   = 1 / scale                         (0 when scale is 0)
  q     = e2m1( x * inv )                   per element, RNE, satfinite

Readings where the pages are silent: the tensor scale divides by 6*448; the
element is multiplied by the reciprocal of its block scale (one division per
block, not per element); a block whose scale rounds to 0 gives all-zero
codes of the input's sign; an all-zero tensor takes s_T = 1.
"""
import numpy as np

from . import formats

BLOCK = 16
F32 = np.float32


def tensor_scale(amax):
    """fp32 per-tensor scale from the tensor's absolute maximum."""
    a = F32(amax)
    if a == F32(0.0):
        return F32(1.0)
    return F32(a / F32(2688.0))


def quantize_blocks(t, s_t):
    """Quantize float32 rows ``t`` [rows, K] (K % 16 == 0) under tensor scale s_t.

    Returns (codes uint8 [rows, K] with values 0..15, sf uint8 [rows, K/16]
    holding ue4m3 bit patterns).
    """
    t = np.asarray(t, dtype=F32)
    rows, k = t.shape
    if k % BLOCK:
        raise ValueError("K must be a multiple of 16")
    s_t = F32(s_t)
    blocks = t.reshape(rows, k // BLOCK, BLOCK)
    amax_b = np.max(np.abs(blocks), axis=2)                 # exact in f32
    d = F32(F32(6.0) * s_t)
    sb_code = formats.ue4m3_encode((amax_b / d).astype(F32))
    sb = formats.ue4m3_decode(sb_code).astype(F32)           # exact in f32
    scale = (sb * s_t).astype(F32)
    with np.errstate(divide="ignore"):
        inv = np.where(scale == 0, F32(0.0), (F32(1.0) / scale)).astype(F32)
    scaled = (blocks * inv[:, :, None]).astype(F32)
    codes = formats.e2m1_encode(scaled).reshape(rows, k)
    return codes, sb_code


def dequantize(codes, sf, s_t):
    """float64 value of NVFP4 data: e2m1(q) * sb * s_T."""
    codes = np.asarray(codes)
    rows, k = codes.shape
    vals = formats.e2m1_decode(codes).reshape(rows, k // BLOCK, BLOCK)
    sb = formats.ue4m3_decode(sf).astype(np.float64)
    return (vals * sb[:, :, None] * np.float64(F32(s_t))).reshape(rows, k)
