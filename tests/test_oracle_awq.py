"""Pins for the oracle's AWQ W4A16 projection (CPU only)."""
from fractions import Fraction

import numpy as np

from oracle import awq, formats
from bit_w4a4_diffusion_smooth_b200 import synthetic

F32 = np.float32


def _weights(k=128, n=40, seed=3):
    wb, _ = synthetic.weight(k, n, seed, 0.02)
    return formats.bf16_bits_to_float(wb), synthetic.awq_scales(k, seed)


def test_codes_and_zeros_are_in_range_and_scales_are_bf16():
    w, a = _weights()
    p = awq.pack(w, a)
    assert p["q"].min() >= 0 and p["q"].max() <= 15
    assert ((p["z"] >= 0) & (p["z"] <= 15) & (p["z"] == np.rint(p["z"]))).all()
    formats.float_to_bf16_bits(p["s"])


def test_dequantization_error_is_at_most_half_a_step():
    w, a = _weights()
    p = awq.pack(w, a)
    deq = awq.dequantize(p["q"], p["s"], p["z"])
    step = np.repeat(p["s"], 64, axis=0)
    err = np.abs(p["w_a"] - deq)
    # the bf16 rounding of s can stretch the last step by 15 * 2^-9 of a step
    assert (err <= step * (0.5 + 15 * 2.0 ** -8)).all()


def test_group_range_maps_to_end_codes():
    """Each group's minimum (if below 0) lands near code 0 and its maximum (if
    above 0) near code 15; the group is cut along K, not N."""
    w, a = _weights()
    p = awq.pack(w, a)
    g = p["w_a"].reshape(2, 64, -1)
    q = p["q"].reshape(2, 64, -1).astype(int)
    lo = np.take_along_axis(q, g.argmin(axis=1)[:, None, :], axis=1)[:, 0, :]
    hi = np.take_along_axis(q, g.argmax(axis=1)[:, None, :], axis=1)[:, 0, :]
    assert (lo[g.min(axis=1) < 0] <= 1).all()
    assert (hi[g.max(axis=1) > 0] >= 14).all()


def test_grid_weights_are_exact():
    """W_a already of the form (q - z) * s with s a bf16 value is reproduced exactly."""
    rng = np.random.default_rng(4)
    k, n = 128, 8
    s = formats.bf16_round(rng.uniform(0.01, 0.1, (2, n)))
    z = rng.integers(3, 12, (2, n)).astype(np.float64)
    q = rng.integers(0, 16, (k, n))
    q[0, :] = 0
    q[64, :] = 0
    q[1, :] = 15
    q[65, :] = 15
    w_a = ((q.reshape(2, 64, n) - z[:, None, :]) * s[:, None, :]).reshape(k, n)
    p = awq.pack(w_a, np.ones(k, F32))
    np.testing.assert_array_equal(p["s"], s)
    np.testing.assert_array_equal(p["z"], z)
    np.testing.assert_array_equal(p["q"], q)


def test_all_zero_group():
    w = np.zeros((64, 3))
    w[:, 2] = 0.5
    p = awq.pack(w, np.ones(64, F32))
    assert p["s"][0, 0] == 1.0 and p["z"][0, 0] == 0 and (p["q"][:, 0] == 0).all()
    # a one-signed group keeps zero exactly representable (range includes 0)
    assert p["z"][0, 2] == 0 and (p["q"][:, 2] == 15).all()


def test_awq_scale_is_compensated_on_the_input():
    """(x . inv_a) . (a . W) == x . W before quantization, to float64 rounding."""
    w, a = _weights()
    xb, _ = synthetic.activation(2, 128, 3)
    x = formats.bf16_bits_to_float(xb)
    p = awq.pack(w, a)
    lhs = (x * p["inv_a"].astype(np.float64)[None, :]) @ p["w_a"]
    np.testing.assert_allclose(lhs, x @ w, rtol=1e-6, atol=1e-9)


def test_linear_brute_force():
    w, a = _weights(k=64, n=5)
    xb, _ = synthetic.activation(2, 64, 9)
    x = formats.bf16_bits_to_float(xb)
    b = np.arange(5) * 0.01
    p = awq.pack(w, a)
    y = awq.linear(x, p["inv_a"], p["q"], p["s"], p["z"], b)
    for i in range(2):
        for j in range(5):
            acc = Fraction(float(b[j]))
            for t in range(64):
                acc += (Fraction(float(x[i, t])) * Fraction(float(p["inv_a"][t]))
                        * (int(p["q"][t, j]) - Fraction(float(p["z"][0, j])))
                        * Fraction(float(p["s"][0, j])))
            assert abs(y[i, j] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))
    # and the quantized layer stays close to the unquantized one
    ref = x @ w + b
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.5
