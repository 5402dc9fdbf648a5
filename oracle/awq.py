"""AWQ W4A16 projection: 4-bit weights, 16-bit activations.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The pages assign AWQ W4A16 to the precision-sensitive, low-compute modulation
and adaptive-norm projections ([Remio] "Nunchaku Diffusers 支持改变了加载路径";
[Donmalab] "Nunchaku Lite：讓高效量化變得簡單").  They fix neither the group size
nor the integer layout; the reading used here is the usual AWQ recipe:

  W_a = diag(a) . W                       per-input-channel AWQ scale a
  per group of 64 rows (along K) and per output column n:
      lo = min(0, min W_a),  hi = max(0, max W_a)
      s  = bf16((hi - lo) / 15)           (s = 1, z = 0 for an all-zero group)
      z  = clamp(rne(-lo / s), 0, 15)
      q  = clamp(rne(W_a / s) + z, 0, 15)
  y = (x . inv_a) . ((q - z) . s) + b,    inv_a = f32(1 / a)

All pack arithmetic is float64 with one rounding per operation.
"""
import numpy as np

from . import formats

F32 = np.float32


def pack(w, a, group=64):
    """w: float64 [K, N]; a: float32 [K] -> dict(q [K,N] u8, s, z [K/group, N] f64, inv_a)."""
    w = np.asarray(w, dtype=np.float64)
    k, n = w.shape
    if k % group:
        raise ValueError("K must be a multiple of the group size")
    a64 = np.asarray(a, dtype=F32).astype(np.float64)
    wa = a64[:, None] * w
    g = wa.reshape(k // group, group, n)
    lo = np.minimum(0.0, g.min(axis=1))
    hi = np.maximum(0.0, g.max(axis=1))
    s = formats.bf16_round((hi - lo) / 15.0)
    zero_group = s == 0.0
    s = np.where(zero_group, 1.0, s)
    z = np.clip(np.rint(-lo / s), 0, 15)
    z = np.where(zero_group, 0.0, z)
    q = np.clip(np.rint(g / s[:, None, :]) + z[:, None, :], 0, 15)
    inv_a = (F32(1.0) / np.asarray(a, dtype=F32)).astype(F32)
    return dict(q=q.reshape(k, n).astype(np.uint8), s=s, z=z, inv_a=inv_a, w_a=wa)


def dequantize(q, s, z, group=64):
    q = np.asarray(q, dtype=np.float64)
    k, n = q.shape
    g = q.reshape(k // group, group, n)
    return ((g - z[:, None, :]) * s[:, None, :]).reshape(k, n)


def linear(x, inv_a, q, s, z, bias=None, group=64):
    """y = (x . inv_a) . deq(W_a) + b in float64.  x: float64 [M, K] bf16 values."""
    x_hat = np.asarray(x, dtype=np.float64) * np.asarray(inv_a, dtype=F32).astype(np.float64)[None, :]
    y = x_hat @ dequantize(q, s, z, group)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y
