"""Pins for the oracle's two-level NVFP4 block quantizer (CPU only)."""
from fractions import Fraction

import numpy as np

from oracle import formats, nvfp4

F32 = np.float32
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def _grid_blocks(rng, rows, k):
    """Rows of e2m1 grid values (random signs) whose every block holds a +-6."""
    v = rng.choice(GRID, size=(rows, k)) * rng.choice([-1.0, 1.0], size=(rows, k))
    v = v.reshape(rows, k // 16, 16)
    v[:, :, 0] = 6.0 * rng.choice([-1.0, 1.0], size=(rows, k // 16))
    return v.reshape(rows, k)


def test_tensor_scale_closed_forms():
    assert nvfp4.tensor_scale(2688.0) == F32(1.0)
    assert nvfp4.tensor_scale(0.0) == F32(1.0)
    assert nvfp4.tensor_scale(5376.0) == F32(2.0)


def test_grid_values_with_unit_scales_are_exact():
    rng = np.random.default_rng(0)
    t = _grid_blocks(rng, 8, 64)
    codes, sf = nvfp4.quantize_blocks(t.astype(F32), F32(1.0))
    assert (sf == 0x38).all()                      # every block scale is 1.0
    np.testing.assert_array_equal(formats.e2m1_decode(codes), t)
    np.testing.assert_array_equal(nvfp4.dequantize(codes, sf, 1.0), t)


def test_grid_values_with_power_of_two_scales_are_exact():
    rng = np.random.default_rng(1)
    t = _grid_blocks(rng, 4, 128)
    # Block j scaled by 2^(j-4): the block scales are exact e4m3 powers of two.
    pw = np.exp2(np.arange(8) - 4.0)
    ts = (t.reshape(4, 8, 16) * pw[None, :, None]).reshape(4, 128)
    s_t = F32(0.25)
    ts_scaled = ts * 0.25
    codes, sf = nvfp4.quantize_blocks(ts_scaled.astype(F32), s_t)
    np.testing.assert_array_equal(formats.ue4m3_decode(sf), np.broadcast_to(pw, (4, 8)))
    np.testing.assert_array_equal(nvfp4.dequantize(codes, sf, s_t), ts_scaled)


def test_block_maximum_maps_to_six():
    """With the block scale in the e4m3 normal range its rounding error is at
    most 1/16, so the largest element lands in [5.65, 6.4] before rounding and
    must take the code of +-6."""
    rng = np.random.default_rng(2)
    t = rng.standard_normal((64, 256)).astype(F32) * F32(3.0)
    s_t = nvfp4.tensor_scale(np.max(np.abs(t)))
    codes, sf = nvfp4.quantize_blocks(t, s_t)
    blocks = t.reshape(64, 16, 16)
    c = codes.reshape(64, 16, 16)
    arg = np.argmax(np.abs(blocks), axis=2)
    normal = formats.ue4m3_decode(sf) >= 2.0 ** -6
    top = np.take_along_axis(c, arg[:, :, None], axis=2)[:, :, 0]
    assert normal.mean() > 0.99
    assert ((top[normal] & 7) == 7).all()
    # and the sign of the largest element is kept
    sgn = np.take_along_axis(blocks, arg[:, :, None], axis=2)[:, :, 0] < 0
    assert (((top[normal] >> 3) == 1) == sgn[normal]).all()


def test_elements_round_to_nearest_grid_point_of_their_block():
    """Each code is the nearest grid point (ties to even) of x * (1/scale),
    checked with exact rationals on the float32 product the rule prescribes."""
    rng = np.random.default_rng(3)
    t = (rng.standard_normal((16, 64)) * np.exp2(rng.integers(-6, 6, (16, 1)))).astype(F32)
    s_t = nvfp4.tensor_scale(np.max(np.abs(t)))
    codes, sf = nvfp4.quantize_blocks(t, s_t)
    scale = (formats.ue4m3_decode(sf).astype(F32) * s_t).astype(F32)
    for r in range(16):
        for j in range(64):
            sc = scale[r, j // 16]
            inv = F32(1.0) / sc if sc != 0 else F32(0.0)
            y = Fraction(float(F32(t[r, j] * inv)))
            mags = [Fraction(g) for g in GRID]
            d = [abs(abs(y) - m) for m in mags]
            best = min(range(8), key=lambda i: (d[i], i % 2))
            if abs(y) >= 6:
                best = 7
            assert codes[r, j] & 7 == best, (r, j)


def test_dequantization_error_bound():
    """|x - deq| <= half the local grid spacing times the block scale (the
    widest gap, between 4 and 6, gives 1 * scale)."""
    rng = np.random.default_rng(4)
    t = rng.standard_normal((32, 512)).astype(F32)
    s_t = nvfp4.tensor_scale(np.max(np.abs(t)))
    codes, sf = nvfp4.quantize_blocks(t, s_t)
    deq = nvfp4.dequantize(codes, sf, s_t)
    scale = np.repeat(formats.ue4m3_decode(sf) * float(s_t), 16, axis=1)
    err = np.abs(t.astype(np.float64) - deq)
    assert (err <= 1.0 * scale * (1 + 1e-6)).all()
    # On average the error is far below the worst case.
    assert err.mean() < 0.3 * scale.mean()


def test_zero_blocks_and_zero_tensor():
    t = np.zeros((2, 32), dtype=F32)
    t[1, :16] = -0.0
    t[1, 16:] = np.linspace(-1, 1, 16)
    s_t = nvfp4.tensor_scale(np.max(np.abs(t)))
    codes, sf = nvfp4.quantize_blocks(t, s_t)
    assert (sf[0] == 0).all() and (codes[0] == 0).all()
    assert sf[1, 0] == 0 and (codes[1, :16] == 8).all()    # -0 keeps its sign
    codes0, sf0 = nvfp4.quantize_blocks(np.zeros((1, 16), F32), nvfp4.tensor_scale(0.0))
    assert (codes0 == 0).all() and (sf0 == 0).all()


def test_block_index_runs_along_k():
    """A single large element only changes its own block's scale."""
    t = np.ones((3, 64), dtype=F32)
    t[1, 37] = 100.0
    codes, sf = nvfp4.quantize_blocks(t, nvfp4.tensor_scale(100.0))
    assert sf[1, 2] != sf[1, 0] and sf[1, 0] == sf[1, 1] == sf[1, 3] == sf[0, 2] == sf[2, 2]
