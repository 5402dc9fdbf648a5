"""The host side of the INT4 W4A4 variant against the oracle (CPU only).

svdq_quantize_int4_host must give the oracle's codes and scales bit for bit
(both take the same float32 steps: amax / 7, bf16 rounding, the float32
reciprocal, the product, round-half-even, the clamp), over ragged magnitudes,
all-zero groups, groups below the 2^-120 cut and exact halves; and the INT4
pack must quantize the residual of svdq_pack_weights exactly so.
"""
import numpy as np
import pytest

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import formats, int4


def _unpack(codes, rows, k):
    lo = (codes & 0xF).astype(np.int8)
    hi = (codes >> 4).astype(np.int8)
    q = np.empty((rows, k), np.int8)
    q[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    q[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return q


def _scales(sbits, rows):
    return (sbits[:, :rows].astype(np.uint32) << 16).view(np.float32).T.astype(np.float64)


@pytest.mark.parametrize("rows,k,seed", [(1, 64, 1), (37, 192, 2), (300, 640, 3)])
def test_host_quantizer_matches_oracle(rows, k, seed):
    rng = np.random.default_rng(seed)
    t = (rng.standard_normal((rows, k)) * np.exp(rng.uniform(-30, 30, (rows, 1)))).astype(np.float32)
    t[0, :64] = 0.0                                                  # an all-zero group
    if rows > 5:
        t[5, :64] = 1e-40                                            # below the 2^-120 cut
        t[4, :64] = np.float32(7.0) * np.arange(-32, 32, dtype=np.float32) / 64   # s = 1: halves and exact steps
        t[4, 0] = 7.0
    codes, sbits = lib.svdq_quantize_int4_host(t, ld_s=rows + 3)
    q, s = int4.quantize_groups(t)
    np.testing.assert_array_equal(_unpack(codes, rows, k), q)
    np.testing.assert_array_equal(_scales(sbits, rows), s)


def test_int4_pack_quantizes_its_residual_as_the_oracle():
    k, n, rank = 512, 384, 32
    xb, _ = synthetic.activation(64, k, 9, synthetic.count(0.01, k), 50.0)
    wb, _ = synthetic.weight(k, n, 9, 0.02, synthetic.count(0.005, k), 8.0)
    amax = np.max(np.abs(formats.bf16_bits_to_float(xb)), axis=0).astype(np.float32)
    p = lib.svdq_pack_weights_int4(wb, amax, rank)
    q, s = int4.quantize_groups(p["residual"].T)
    np.testing.assert_array_equal(_unpack(p["w_codes"], n, k), q)
    np.testing.assert_array_equal(_scales(p["w_scales"], n), s)
    assert p["w_codes"].shape == (n, k // 2) and p["w_scales"].shape == (k // 64, n)
