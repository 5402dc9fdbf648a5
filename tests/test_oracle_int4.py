"""Pins of the INT4 W4A4 oracle (oracle/int4.py) against what the format and
the mathematics fix, independent of the oracle's own formulas:

  * exact reconstruction on a grid: a group whose values are integer
    multiples of a bf16-exact step, with amax = 7 steps, quantizes to those
    integers;
  * round-half-even on exact halves, and no code outside [-7, 7] (the scale
    is amax/7 rounded to bf16, so |v|/s <= 7 (1 + 2^-8));
  * the quantization error is at most half a step wherever nothing clips;
  * groups are independent (a group's codes depend on its own values only)
    and an all-zero group has scale 0 and codes 0;
  * the grouped GEMM equals the matrix product of the dequantized operands
    (a library matmul over whole rows), and with zero codes the layer reduces
    to the plain low-rank product plus bias;
  * end to end, the layer approximates X . W, better with the low-rank branch
    than without it.
"""
import numpy as np
import pytest

from bit_w4a4_diffusion_smooth_b200 import synthetic
from oracle import formats, int4, svdquant

F32 = np.float32


def test_grid_values_reconstruct_exactly():
    step = 2.0 ** -5
    ks = np.array([7, -7, 3, -2, 0, 5, -6, 1] * 8, dtype=np.float64)     # one group of 64, amax = 7 steps
    v = (ks * step).astype(F32)[None, :]
    q, s = int4.quantize_groups(v)
    assert s[0, 0] == 7 * step / 7
    np.testing.assert_array_equal(q[0], ks.astype(np.int8))


def test_round_half_even_and_range():
    # amax 7 -> s = 1 exactly; halves round to even
    v = np.zeros((1, 64), dtype=F32)
    v[0, :8] = [7.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5]
    q, s = int4.quantize_groups(v)
    assert s[0, 0] == 1.0
    np.testing.assert_array_equal(q[0, :8], [7, 2, 4, -2, -4, 0, 0, 2])
    rng = np.random.default_rng(3)
    big = (rng.standard_normal((64, 512)) * np.exp(rng.uniform(-20, 20, (64, 1)))).astype(F32)
    qb, sb = int4.quantize_groups(big)
    assert qb.min() >= -7 and qb.max() <= 7
    assert np.all(sb == formats.bf16_round(sb))                            # scales are bf16 values


def test_error_is_at_most_half_a_step():
    rng = np.random.default_rng(4)
    v = (rng.standard_normal((32, 256)) * rng.uniform(0.01, 50, (32, 1))).astype(F32)
    q, s = int4.quantize_groups(v)
    err = np.abs(v.astype(np.float64) - int4.dequantize(q, s))
    step = np.repeat(s, 64, axis=1)
    assert np.all(err <= 0.5 * step * (1 + 2.0 ** -20) + 1e-300)


def test_groups_are_independent_and_zero_groups_vanish():
    rng = np.random.default_rng(5)
    v = rng.standard_normal((4, 256)).astype(F32)
    v[1, 64:128] = 0.0
    q, s = int4.quantize_groups(v)
    assert s[1, 1] == 0.0 and not q[1, 64:128].any()
    w = v.copy()
    w[:, 128:192] *= F32(100.0)                                            # changes group 2 only
    q2, s2 = int4.quantize_groups(w)
    keep = np.r_[0:128, 192:256]
    np.testing.assert_array_equal(q2[:, keep], q[:, keep])
    np.testing.assert_array_equal(np.delete(s2, 2, axis=1), np.delete(s, 2, axis=1))


def test_grouped_gemm_equals_product_of_dequantized_operands():
    rng = np.random.default_rng(6)
    m, k, n = 9, 320, 12
    qa = rng.integers(-8, 8, (m, k)).astype(np.int8)
    qw = rng.integers(-8, 8, (n, k)).astype(np.int8)
    sa = formats.bf16_round(rng.uniform(0.01, 2.0, (m, k // 64)))
    sw = formats.bf16_round(rng.uniform(0.01, 2.0, (n, k // 64)))
    y = int4.int4_linear(qa, sa, qw, sw, np.zeros((m, 0)), np.zeros((0, n)))
    want = np.matmul(int4.dequantize(qa, sa), int4.dequantize(qw, sw).T)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_zero_codes_leave_the_low_rank_branch_and_bias():
    rng = np.random.default_rng(7)
    m, k, n, r = 5, 128, 16, 8
    u = formats.bf16_round(rng.standard_normal((m, r)))
    l2 = formats.bf16_round(rng.standard_normal((r, n)))
    b = formats.bf16_round(rng.standard_normal(n))
    y = int4.int4_linear(np.zeros((m, k), np.int8), np.ones((m, 2)), np.zeros((n, k), np.int8), np.ones((n, 2)),
                         u, l2, b)
    np.testing.assert_allclose(y, np.matmul(u, l2) + b[None, :], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("epilogue", [svdquant.EPILOGUE_NONE, svdquant.EPILOGUE_GELU_ERF])
def test_layer_approximates_the_float_layer(epilogue):
    m, k, n = 64, 512, 192
    xb, _ = synthetic.activation(m, k, 8, synthetic.count(0.01, k), 50.0)
    wb, _ = synthetic.weight(k, n, 8, 0.02, synthetic.count(0.005, k), 8.0)
    x = formats.bf16_bits_to_float(xb)
    w = formats.bf16_bits_to_float(wb)
    amax = np.max(np.abs(x), axis=0).astype(F32)
    ref = x @ w
    if epilogue != svdquant.EPILOGUE_NONE:
        ref = svdquant.gelu(ref, epilogue)
    errs = []
    for rank in (0, 32):
        y = int4.forward(x, int4.pack(w, amax, rank), epilogue=epilogue)
        errs.append(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    assert errs[1] < 0.08 and errs[1] < errs[0]
