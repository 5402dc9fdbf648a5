"""Pins for the oracle's SVDQuant layer (CPU only).

Pinned against closed forms and invariants the method fixes: smoothing leaves
the exact product unchanged, the low-rank branch obeys Eckart-Young with the
spectrum taken from an independent eigen-solver, an exactly rank-r weight
leaves no residual, r = 0 reduces to a plain dequantize-then-multiply GEMM
(brute-forced with exact rationals), and grid-valued operands with unit
scales give the exact product.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats, nvfp4, svdquant
from bit_w4a4_diffusion_smooth_b200 import synthetic

F32 = np.float32


def _case(m=32, k=128, n=96, seed=0, outliers=3):
    xb, _ = synthetic.activation(m, k, seed, outliers, 30.0)
    wb, _ = synthetic.weight(k, n, seed, 0.02, 2, 8.0)
    bb = synthetic.bias(n, seed)
    x = formats.bf16_bits_to_float(xb)
    w = formats.bf16_bits_to_float(wb)
    b = formats.bf16_bits_to_float(bb)
    return x, w, b


def test_lambda_closed_form():
    inv = svdquant.smooth([50.0, 2.0, 0.0, 3.0], [2.0, 8.0, 1.0, 0.0])
    assert inv[0] == F32(0.2) and inv[1] == F32(2.0)
    assert inv[2] == F32(1.0) and inv[3] == F32(1.0)     # guards


def test_smoothing_keeps_exact_product():
    x, w, _ = _case()
    amax_x = np.max(np.abs(x), axis=0)
    inv = svdquant.smooth(amax_x, np.max(np.abs(w), axis=1))
    wp = svdquant.smoothed_weight(w, inv)
    x_hat = x * inv.astype(np.float64)[None, :]
    ref = x @ w
    np.testing.assert_allclose(x_hat @ wp, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    # smoothing evens out the channel ranges of the activation
    assert np.max(np.abs(x_hat), axis=0).std() < np.max(np.abs(x), axis=0).std()


def test_low_rank_eckart_young_against_eigensolver():
    _, w, _ = _case(k=96, n=160)
    for r in (0, 1, 8, 16):
        l1, l2 = svdquant.low_rank(w, r, round_bf16=False)
        err = np.sum((w - l1 @ l2) ** 2)
        ev = np.sort(np.linalg.eigvalsh(w.T @ w))[::-1]     # sigma^2, another routine
        tail = np.sum(np.clip(ev[r:], 0, None))
        assert abs(err - tail) <= 1e-9 * np.sum(ev), r


def test_low_rank_reconstructs_full_rank():
    _, w, _ = _case(k=64, n=80)
    l1, l2 = svdquant.low_rank(w, 64, round_bf16=False)
    np.testing.assert_allclose(l1 @ l2, w, atol=1e-13)
    # L2 rows are orthonormal (L2 = V^T); L1 columns are orthogonal
    np.testing.assert_allclose(l2 @ l2.T, np.eye(64), atol=1e-12)
    g = l1.T @ l1
    np.testing.assert_allclose(g - np.diag(np.diag(g)), 0, atol=1e-12)


def test_low_rank_bf16_factors_are_bf16():
    _, w, _ = _case()
    l1, l2 = svdquant.low_rank(w, 8)
    formats.float_to_bf16_bits(l1)
    formats.float_to_bf16_bits(l2)


def test_exact_rank_r_weight_leaves_only_low_rank_branch():
    rng = np.random.default_rng(5)
    k, n, r, m = 128, 64, 8, 16
    w = rng.standard_normal((k, r)) @ rng.standard_normal((r, n)) * 0.02
    xb, _ = synthetic.activation(m, k, 5, 2, 20.0)
    x = formats.bf16_bits_to_float(xb)
    p = svdquant.pack(w, np.max(np.abs(x), axis=0).astype(F32), r, round_bf16=False)
    assert np.abs(p["residual"]).max() <= 1e-12 * np.abs(p["w_prime"]).max()
    y = svdquant.forward(x, p)
    x_hat32 = (x.astype(F32) * p["inv_lambda"][None, :]).astype(F32).astype(np.float64)
    low = (formats.bf16_round(x_hat32) @ p["l1"]) @ p["l2"]
    np.testing.assert_allclose(y, low, rtol=0, atol=1e-9 * np.abs(low).max())
    # the only departure from X W is the bf16 input of the 16-bit branch
    np.testing.assert_allclose(y, x @ w, rtol=0, atol=2.0 ** -7 * np.abs(low).max())


def _brute_gemm(a_codes, a_sf, s_a, w_codes, w_sf, s_w, bias):
    """Dequantize-then-multiply with exact rationals, element by element."""
    m, k = a_codes.shape
    n = w_codes.shape[0]
    fa = [Fraction(float(v)) for v in formats.E2M1_VALUE]
    sa, sw = Fraction(float(F32(s_a))), Fraction(float(F32(s_w)))
    out = np.zeros((m, n))
    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for kk in range(k):
                qa = fa[a_codes[i, kk]] * Fraction(float(formats.ue4m3_decode(a_sf[i, kk // 16]))) * sa
                qw = fa[w_codes[j, kk]] * Fraction(float(formats.ue4m3_decode(w_sf[j, kk // 16]))) * sw
                acc += qa * qw
            out[i, j] = float(acc + Fraction(float(bias[j])))
    return out


def test_rank_zero_reduces_to_plain_w4a4_gemm():
    rng = np.random.default_rng(6)
    m, k, n = 3, 32, 4
    a_codes = rng.integers(0, 16, (m, k)).astype(np.uint8)
    w_codes = rng.integers(0, 16, (n, k)).astype(np.uint8)
    a_sf = rng.integers(20, 90, (m, k // 16)).astype(np.uint8)
    w_sf = rng.integers(20, 90, (n, k // 16)).astype(np.uint8)
    s_a, s_w = F32(0.37), F32(1.9)
    bias = rng.standard_normal(n)
    y = svdquant.w4a4_linear(a_codes, a_sf, s_a, w_codes, w_sf, s_w,
                             np.zeros((m, 0)), np.zeros((0, n)), bias)
    np.testing.assert_allclose(y, _brute_gemm(a_codes, a_sf, s_a, w_codes, w_sf, s_w, bias),
                               rtol=1e-13, atol=1e-13)


def test_grid_operands_with_unit_scales_give_exact_product():
    rng = np.random.default_rng(7)
    m, k, n = 4, 64, 5
    a_codes = rng.integers(0, 16, (m, k)).astype(np.uint8)
    w_codes = rng.integers(0, 16, (n, k)).astype(np.uint8)
    ones_a = np.full((m, k // 16), 0x38, np.uint8)
    ones_w = np.full((n, k // 16), 0x38, np.uint8)
    y = svdquant.w4a4_linear(a_codes, ones_a, 1.0, w_codes, ones_w, 1.0,
                             np.zeros((m, 0)), np.zeros((0, n)))
    # products of grid values are multiples of 1/4 and small: exact in float64
    av = formats.e2m1_decode(a_codes)
    wv = formats.e2m1_decode(w_codes)
    for i in range(m):
        for j in range(n):
            assert y[i, j] == sum(Fraction(float(av[i, t])) * Fraction(float(wv[j, t]))
                                  for t in range(k))


def test_low_rank_branch_is_added_with_alpha():
    """U enters divided by alpha and leaves multiplied by it: with zero codes
    the output is exactly U.L2 + b."""
    rng = np.random.default_rng(8)
    m, k, n, r = 5, 32, 6, 4
    u = rng.standard_normal((m, r))
    l2 = rng.standard_normal((r, n))
    s_a, s_w = F32(0.5), F32(0.25)
    y = svdquant.w4a4_linear(np.zeros((m, k), np.uint8), np.zeros((m, 2), np.uint8), s_a,
                             np.zeros((n, k), np.uint8), np.zeros((n, 2), np.uint8), s_w,
                             u / 0.125, l2)
    np.testing.assert_allclose(y, u @ l2, rtol=1e-14, atol=1e-14)


def test_quantize_act_on_grid_activation():
    """X = G . diag(lambda) with G on the e2m1 grid and lambda powers of two:
    X^ = G exactly, so the codes are G's and U = G.L1 / alpha."""
    rng = np.random.default_rng(9)
    m, k, r = 4, 64, 3
    g = rng.choice([0, 0.5, 1, 1.5, 2, 3, 4, 6], (m, k)) * rng.choice([-1, 1], (m, k))
    g.reshape(m, k // 16, 16)[:, :, 3] = 6.0
    lam = np.exp2(rng.integers(-3, 4, k)).astype(np.float64)
    x = g * lam[None, :]
    inv = (1.0 / lam).astype(F32)
    l1 = rng.standard_normal((k, r))
    s_a, s_w = F32(1.0), F32(0.5)
    codes, sf, u = svdquant.quantize_act(x, inv, l1, s_a, s_w)
    assert (sf == 0x38).all()
    np.testing.assert_array_equal(formats.e2m1_decode(codes), np.where(g == 0, 0, g))
    np.testing.assert_allclose(u, (g @ l1) / 0.5, rtol=1e-13)   # G is exact in bf16


def test_low_rank_input_is_bf16():
    """The 16-bit branch sees X^ rounded to bf16: a value that bf16 cannot hold
    moves U by exactly its rounding error times L1."""
    k = 16
    x = np.zeros((1, k))
    x[0, 0] = 1.0 + 2.0 ** -7           # exact in bf16
    x[0, 1] = 1.0
    inv = np.ones(k, F32)
    inv[1] = F32(1.0 + 2.0 ** -9)         # X^[1] = 1 + 2^-9 rounds to 1 in bf16 (tie -> even)
    l1 = np.eye(k)[:, :2]
    _, _, u = svdquant.quantize_act(x, inv, l1, F32(1.0), F32(1.0))
    assert u[0, 0] == 1.0 + 2.0 ** -7 and u[0, 1] == 1.0


def test_gelu_forms():
    y = np.array([-3.0, -1.0, 0.0, 0.5, 2.0])
    e = svdquant.gelu(y, svdquant.EPILOGUE_GELU_ERF)
    # GELU(0) = 0, GELU(y) - GELU(-y) = y (erf is odd)
    assert e[2] == 0.0
    np.testing.assert_allclose(svdquant.gelu(y, 1) - svdquant.gelu(-y, 1), y, atol=1e-15)
    t = svdquant.gelu(y, svdquant.EPILOGUE_GELU_TANH)
    np.testing.assert_allclose(t, e, atol=2e-3)       # the tanh form approximates erf
    # only the chosen column range is activated
    rng = np.random.default_rng(10)
    m, k, n = 2, 16, 6
    yy = svdquant.w4a4_linear(np.zeros((m, k), np.uint8), np.zeros((m, 1), np.uint8), 1.0,
                              np.zeros((n, k), np.uint8), np.zeros((n, 1), np.uint8), 1.0,
                              np.zeros((m, 0)), np.zeros((0, n)), rng.standard_normal(n),
                              svdquant.EPILOGUE_GELU_ERF, gelu_col_begin=4)
    raw = svdquant.w4a4_linear(np.zeros((m, k), np.uint8), np.zeros((m, 1), np.uint8), 1.0,
                               np.zeros((n, k), np.uint8), np.zeros((n, 1), np.uint8), 1.0,
                               np.zeros((m, 0)), np.zeros((0, n)),
                               np.random.default_rng(10).standard_normal(n))
    np.testing.assert_array_equal(yy[:, :4], raw[:, :4])
    np.testing.assert_allclose(yy[:, 4:], svdquant.gelu(raw[:, 4:], 1))


def test_activation_scale_from_calibration_maxima():
    x, w, _ = _case()
    amax_x = np.max(np.abs(x), axis=0).astype(F32)
    inv = svdquant.smooth(amax_x, np.max(np.abs(w), axis=1))
    s_a = svdquant.activation_tensor_scale(amax_x, inv)
    x_hat32 = (x.astype(F32) * inv[None, :]).astype(F32)
    assert s_a == nvfp4.tensor_scale(np.max(np.abs(x_hat32)))
    codes, sf, _ = svdquant.quantize_act(x, inv, np.zeros((x.shape[1], 0)), s_a, F32(1.0))
    assert formats.ue4m3_decode(sf).max() == 448.0     # the largest block hits 448


def test_forward_is_close_to_unquantized_layer():
    """Information only in spirit (the pages print no accuracy figure), but a
    gross error in any step would blow this far past 10 %."""
    x, w, b = _case(m=64, k=256, n=128, seed=3, outliers=4)
    amax_x = np.max(np.abs(x), axis=0).astype(F32)
    p = svdquant.pack(w, amax_x, 16)
    y = svdquant.forward(x, p, b)
    ref = x @ w + b
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.1
    # and the low-rank branch helps: r = 0 does worse on outlier-heavy inputs
    p0 = svdquant.pack(w, amax_x, 0)
    rel0 = np.linalg.norm(svdquant.forward(x, p0, b) - ref) / np.linalg.norm(ref)
    assert rel <= rel0 * 1.05


def test_dynamic_activation_scale_pins():
    """The per-tensor (dynamic) activation scale: brute force over every element of a small input,
    the all-zero tensor (scale 1), and agreement with the static scale calibrated on the same
    tensor's per-channel maxima (a different formulation of the same maximum)."""
    from oracle import nvfp4
    rng = np.random.default_rng(11)
    x = formats.bf16_round(rng.standard_normal((7, 48)) * np.exp(rng.uniform(-3, 3, 48)))
    x[3, 5] = -x[3, 5] * 40.0                    # a negative outlier decides the maximum
    x = formats.bf16_round(x)
    inv = np.exp(rng.uniform(-2, 2, 48)).astype(np.float32)
    best = np.float32(0.0)
    for i in range(x.shape[0]):
        for j in range(x.shape[1]):
            v = abs(np.float32(np.float32(x[i, j]) * inv[j]))
            best = max(best, v)
    assert svdquant.dynamic_activation_scale(x, inv) == np.float32(best / np.float32(2688.0))
    amax = np.max(np.abs(x), axis=0).astype(np.float32)
    assert svdquant.dynamic_activation_scale(x, inv) == svdquant.activation_tensor_scale(amax, inv)
    assert svdquant.dynamic_activation_scale(np.zeros((3, 16)), np.ones(16, np.float32)) == np.float32(1.0)
    # a tensor whose largest |x^| is 2688 has scale exactly 1 (the largest block scale then lands on 448)
    z = np.zeros((2, 16))
    z[1, 7] = -2688.0
    assert svdquant.dynamic_activation_scale(z, np.ones(16, np.float32)) == np.float32(1.0)
    codes, sf = nvfp4.quantize_blocks(z.astype(np.float32), np.float32(1.0))
    assert sf[1, 0] == 0x7E and codes[1, 7] == 0xF   # e4m3 448, e2m1 -6
