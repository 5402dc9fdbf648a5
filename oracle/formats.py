"""Element formats of the 4-bit path, written from their definitions.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

* e2m1 (the NVFP4 element, OCP MX FP4): 1 sign, 2 exponent (bias 1), 1 mantissa
  bit.  Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign.
* ue4m3 (the NVFP4 block scale): FP8 E4M3 with the sign bit 0, bias 7, 3
  mantissa bits, subnormal quantum 2^-9, largest finite 448 (the all-ones
  pattern is NaN and never produced).
* bf16: 1 sign, 8 exponent, 7 mantissa bits.

Rounding everywhere is round-to-nearest, ties to even, with saturation to the
largest finite magnitude (the "satfinite" behaviour), the plainest reading of
quantization to these formats; the pages name the formats (NVFP4 on
Blackwell, [Remio] "硬件支持划分了最快路径与最广泛路径") but not a rounding rule.
"""
import numpy as np

# Magnitude of each e2m1 code 0..7, straight from the bit definition:
# code = e1 e0 m; e == 0 -> subnormal 0.5*m; else 2^(e-1) * (1 + m/2).
E2M1_MAGNITUDE = np.array(
    [0.5 * (c & 1) if (c >> 1) == 0 else 2.0 ** ((c >> 1) - 1) * (1.0 + 0.5 * (c & 1))
     for c in range(8)], dtype=np.float64)
E2M1_VALUE = np.concatenate([E2M1_MAGNITUDE, -E2M1_MAGNITUDE])  # code 0..15
E2M1_MAX = 6.0
UE4M3_MAX = 448.0


def e2m1_encode(x):
    """Round float32 values to the nearest e2m1 code, ties to even, saturating.

    The thresholds are the midpoints of the grid; at a midpoint the code with
    mantissa bit 0 wins (0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4,
    5->4).  The sign of the input is kept, so a negative value that rounds to
    zero gives code 8 (negative zero).
    """
    x = np.asarray(x, dtype=np.float32)
    if np.isnan(x).any():
        raise ValueError("e2m1_encode: NaN input")
    a = np.abs(x).astype(np.float64)
    mag = np.zeros(a.shape, dtype=np.uint8)
    mag[(a > 0.25) & (a < 0.75)] = 1
    mag[(a >= 0.75) & (a <= 1.25)] = 2
    mag[(a > 1.25) & (a < 1.75)] = 3
    mag[(a >= 1.75) & (a <= 2.5)] = 4
    mag[(a > 2.5) & (a < 3.5)] = 5
    mag[(a >= 3.5) & (a <= 5.0)] = 6
    mag[a > 5.0] = 7
    sign = np.signbit(x).astype(np.uint8) << 3
    return (mag | sign).astype(np.uint8)


def e2m1_decode(codes):
    return E2M1_VALUE[np.asarray(codes, dtype=np.int64) & 15]


def ue4m3_decode(codes):
    """Value of each ue4m3 bit pattern (0..126; 127 is NaN and rejected)."""
    c = np.asarray(codes, dtype=np.int64)
    if (c < 0).any() or (c > 126).any():
        raise ValueError("ue4m3_decode: code out of the finite positive range")
    e = c >> 3
    m = c & 7
    sub = m * 2.0 ** -9
    nrm = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    return np.where(e == 0, sub, nrm)


def ue4m3_encode(v):
    """Round non-negative float32 values to the nearest ue4m3 code (RNE, satfinite).

    Values at or above 448 give 448; values at or below 2^-10 (half the
    smallest subnormal) give 0, the tie going to the even code 0.
    """
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    if np.isnan(v).any() or (v < 0).any():
        raise ValueError("ue4m3_encode: needs finite non-negative input")
    _, e2 = np.frexp(v)                      # v = f * 2^e2, f in [0.5, 1)
    e = e2.astype(np.int64) - 1              # v in [2^e, 2^(e+1))
    # Spacing of the e4m3 grid around v: 2^(e-3) for normals, 2^-9 below 2^-6.
    quantum = np.exp2(np.maximum(e, -6) - 3.0)
    val = np.rint(v / quantum) * quantum     # division by a power of two is exact
    val = np.minimum(val, UE4M3_MAX)         # satfinite
    # Bit pattern of the rounded value.
    _, e2r = np.frexp(val)
    er = e2r.astype(np.int64) - 1
    is_sub = val < 2.0 ** -6
    m_sub = np.rint(val / 2.0 ** -9)
    m_nrm = np.rint((val / np.exp2(er.astype(np.float64)) - 1.0) * 8.0)
    code = np.where(is_sub, m_sub, (er + 7) * 8 + m_nrm)
    code = np.where(val == 0.0, 0, code)
    return code.astype(np.uint8)


def bf16_round(x):
    """Round float64 values to the nearest bf16 value (RNE), returned as float64.

    One rounding, straight from float64 (no detour through float32, which
    could round twice).  Overflow is not expected in this path and raises.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e2 = np.frexp(a)
    e = e2.astype(np.int64) - 1
    quantum = np.exp2(np.maximum(e, -126) - 7.0)   # 8 significant bits
    r = np.rint(a / quantum) * quantum
    if (r > 3.3895313892515355e38).any():
        raise OverflowError("bf16_round: overflow")
    return np.where(a == 0.0, x, np.copysign(r, x))


def bf16_bits_to_float(bits):
    """Exact value of bf16 bit patterns (uint16) as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def float_to_bf16_bits(x):
    """Bit patterns of float64 values that are already exact bf16 values."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    if not np.array_equal(f.astype(np.float64), x, equal_nan=True):
        raise ValueError("float_to_bf16_bits: value is not a float32")
    u = f.view(np.uint32)
    if (u & 0xFFFF).any():
        raise ValueError("float_to_bf16_bits: value is not a bf16")
    return (u >> 16).astype(np.uint16)
