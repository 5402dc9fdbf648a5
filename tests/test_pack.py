"""Host pack of the library (C++) against the oracle (CPU only).

Bit-exact where the method fixes the result: inverse smoothing factors,
activation scale, and - stage-wise - the NVFP4 codes and scales of the
pack's own residual, and every AWQ code, scale and zero point.  The top-r SVD
is checked by Eckart-Young against the oracle's exact spectrum (singular
vectors are not unique, so the factors themselves are not compared).
"""
import numpy as np
import pytest

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import awq as oawq
from oracle import formats, nvfp4, svdquant
from tests import layouts

F32 = np.float32


def _case(m, k, n, seed, x_out=4, x_fac=30.0, w_out=2, w_fac=8.0):
    xb, _ = synthetic.activation(m, k, seed, x_out, x_fac)
    wb, _ = synthetic.weight(k, n, seed, 0.02, w_out, w_fac)
    x = formats.bf16_bits_to_float(xb)
    amax = np.max(np.abs(x), axis=0).astype(F32)
    return xb, wb, x, amax


@pytest.mark.parametrize("k,n,rank", [(256, 256, 16), (128, 64, 0), (192, 128, 32), (320, 264, 16)])
def test_pack_matches_oracle(k, n, rank):
    xb, wb, x, amax = _case(64, k, n, seed=k + n + rank)
    p = lib.svdq_pack_weights(wb, amax, rank, want_residual=True)
    w = formats.bf16_bits_to_float(wb)
    o = svdquant.pack(w, amax, rank)
    np.testing.assert_array_equal(p["inv_lambda"], o["inv_lambda"])
    assert p["s_a"][0] == o["s_a"]
    # stage-wise: the oracle quantizes the pack's own residual
    r32 = p["residual"]
    s_w = nvfp4.tensor_scale(np.max(np.abs(r32)))
    assert p["s_w"][0] == s_w
    codes, sf = nvfp4.quantize_blocks(r32.T, s_w)
    gc, gsf = layouts.bundle_unpack(p["w_bundle"], n, k, 256)
    assert layouts.scale_replicas_agree(p["w_bundle"], n, k, 256)
    np.testing.assert_array_equal(gc, codes)
    np.testing.assert_array_equal(gsf, sf)
    assert layouts.bundle_padding_is_zero(p["w_bundle"], n, k, 256)
    # the residual is W' - L1 L2 with the pack's bf16 factors
    l1 = layouts.bf16_bits_to_f64(p["l1t"]).T
    l2bits = layouts.lowrank_unpack(p["l2t"], n, 256)
    l2 = layouts.bf16_bits_to_f64(l2bits)[:, :rank].T
    assert (l2bits[:, rank:] == 0).all()
    np.testing.assert_allclose(r32, (o["w_prime"] - l1 @ l2).astype(F32), rtol=0, atol=1e-6)
    # L1 L2 itself is not compared with the oracle's: with a nearly flat tail
    # of the spectrum the top-r subspace is not unique (see the Eckart-Young
    # test for what is).


@pytest.mark.parametrize("k,n,rank,tol", [(256, 256, 16, 1e-3), (512, 1536, 32, 1e-3)])
def test_pack_svd_eckart_young(k, n, rank, tol):
    xb, wb, x, amax = _case(64, k, n, seed=3, x_out=max(1, k // 64), x_fac=50.0, w_out=max(1, k // 200))
    _check_eckart_young(wb, amax, rank, tol)


@pytest.mark.slow
def test_pack_svd_eckart_young_full_size_qkv():
    """The pack the benchmark uses: the attention-QKV weight 3072 x 9216 at rank 32, calibrated
    on its 4608-row activation, against the exact spectrum of W'."""
    c = synthetic.QKV
    xb, wb, _ = c.make()
    amax = np.max(np.abs(formats.bf16_bits_to_float(xb)), axis=0).astype(F32)
    _check_eckart_young(wb, amax, c.rank, 1e-3)


def _check_eckart_young(wb, amax, rank, tol):
    w = formats.bf16_bits_to_float(wb)
    p = lib.svdq_pack_weights(wb, amax, rank, want_residual=True)
    wp = svdquant.smoothed_weight(w, p["inv_lambda"])
    sig = np.linalg.svd(wp, compute_uv=False)
    optimal = np.sum(sig[rank:] ** 2)
    # the pack's factors before bf16 rounding would reach the optimum; with
    # bf16 factors the residual grows by at most the rounding of L1 L2
    got = np.sum(p["residual"].astype(np.float64) ** 2)
    assert got >= optimal * (1 - 1e-9)
    assert got <= optimal * (1 + tol) + np.sum(sig[:rank] ** 2) * 2 ** -14, (got / optimal - 1)


def test_pack_is_deterministic():
    xb, wb, x, amax = _case(32, 128, 64, seed=5)
    a = lib.svdq_pack_weights(wb, amax, 16, num_threads=3, seed=7)
    b = lib.svdq_pack_weights(wb, amax, 16, num_threads=3, seed=7)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])


def test_host_quantizer_matches_oracle_bit_exactly():
    rng = np.random.default_rng(0)
    t = (rng.standard_normal((70, 320)) * np.exp2(rng.integers(-8, 8, (70, 1)))).astype(F32)
    # plant exact ties of the e2m1 grid and of the e4m3 scale
    t[3, :16] = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -5, -0.25, 0, -0.0, 4, 3, 2, 1], F32)
    t[5, 16:32] = 0.0
    s_t = nvfp4.tensor_scale(np.max(np.abs(t)))
    oc, osf = nvfp4.quantize_blocks(t, s_t)
    for th in (128, 256):
        bundle = lib.svdq_quantize_host(t, s_t, th)
        gc, gsf = layouts.bundle_unpack(bundle, 70, 320, th)
        np.testing.assert_array_equal(gc, oc)
        np.testing.assert_array_equal(gsf, osf)
        assert layouts.scale_replicas_agree(bundle, 70, 320, th)
        assert layouts.bundle_padding_is_zero(bundle, 70, 320, th)
    oc1, osf1 = nvfp4.quantize_blocks(t[3:4], F32(1.0))
    c1, _ = layouts.bundle_unpack(lib.svdq_quantize_host(t[3:4].copy(), 1.0), 1, 320, 128)
    np.testing.assert_array_equal(c1, oc1)


@pytest.mark.parametrize("rows,k,th", [(130, 320, 128), (300, 576, 256)])
def test_bundle_layout_reader_round_trip(rows, k, th):
    """The test-side reader inverts a bundle written by hand from the header text."""
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 16, (rows, k)).astype(np.uint8)
    sf = rng.integers(0, 127, (rows, k // 16)).astype(np.uint8)
    tile_bytes = th * 144 if th == 128 else th * 192
    rp = 1 if th == 128 else 4
    buf = np.zeros(((rows + th - 1) // th) * ((k + 255) // 256) * tile_bytes, np.uint8)
    for m in range(rows):
        for kk in range(0, k, 2):
            tile = ((m // th) * ((k + 255) // 256) + kk // 256) * tile_bytes
            r, byte = m % th, (kk % 256) // 2
            buf[tile + r * 128 + (((byte // 16) ^ (r % 8)) * 16) + byte % 16] = codes[m, kk] | (codes[m, kk + 1] << 4)
        for j16 in range(k // 16):
            kk = j16 * 16
            tile = ((m // th) * ((k + 255) // 256) + kk // 256) * tile_bytes
            r, j = m % th, (kk % 256) // 16
            for q in range(rp):
                buf[tile + th * 128 + (j // 4) * (th // 128) * 512 * rp + (r // 128) * 512 * rp + q * 512
                    + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4] = sf[m, j16]
    gc, gsf = layouts.bundle_unpack(buf, rows, k, th)
    np.testing.assert_array_equal(gc, codes)
    np.testing.assert_array_equal(gsf, sf)
    np.testing.assert_array_equal(layouts.bundle_pack(codes, sf, rows, k, th), buf)


@pytest.mark.parametrize("k,n", [(64, 64), (192, 128), (3072, 64)])
def test_awq_pack_matches_oracle(k, n):
    wb, _ = synthetic.weight(k, n, 11, 0.02)
    a = synthetic.awq_scales(k, 11)
    p = lib.awq_pack_weights(wb, a)
    o = oawq.pack(formats.bf16_bits_to_float(wb), a)
    np.testing.assert_array_equal(layouts.awq_unpack(p["qweight"], k, n), o["q"])
    np.testing.assert_array_equal(layouts.awq_group_unpack(layouts.bf16_bits_to_f64(p["scales"]), k, n), o["s"])
    np.testing.assert_array_equal(layouts.awq_group_unpack(layouts.bf16_bits_to_f64(p["zeros"]), k, n), o["z"])
    np.testing.assert_array_equal(p["inv_awq"], o["inv_a"])


def test_awq_layout_reader_round_trip():
    """The test-side reader inverts a layout written by hand from the header text."""
    k, n = 128, 128
    G = k // 64
    q = np.random.default_rng(1).integers(0, 16, (k, n)).astype(np.uint8)
    words = np.zeros(n * k // 8, np.uint32)
    for kk in range(k):
        for c in range(n):
            quad, blk, cc = c // 64, (c // 16) % 4, c % 16
            grp, j, kq = kk // 64, (kk % 64) // 16, kk % 16
            lane = (cc % 8) * 4 + (kq % 8) // 2
            i = (cc // 8) + 2 * (kq // 8) + 4 * (kq % 2)
            words[(((quad * G + grp) * 4 + blk) * 32 + lane) * 4 + j] |= np.uint32(q[kk, c]) << np.uint32(4 * i)
    np.testing.assert_array_equal(layouts.awq_unpack(words, k, n), q)
    np.testing.assert_array_equal(layouts.awq_pack(q), words)


def test_awq_group_layout_from_header_text():
    """Scale / zero position of (column n, group g) = ((n/64)*G + g)*64 + n%64, written by
    hand; the test-side reader and writer agree with it."""
    k, n = 192, 128
    g_n = k // 64
    v = np.random.default_rng(2).integers(0, 1000, (g_n, n))
    flat = np.zeros(g_n * n, np.int64)
    for g in range(g_n):
        for c in range(n):
            flat[((c // 64) * g_n + g) * 64 + c % 64] = v[g, c]
    np.testing.assert_array_equal(layouts.awq_group_unpack(flat, k, n), v)
    np.testing.assert_array_equal(layouts.awq_group_pack(v), flat)
