"""GPU-side calibration and pack (svdq_calibrate_absmax, svdq_pack_weights_device)
against the oracle.

* Calibration: the per-channel maxima over two accumulated batches equal
  numpy's maximum of |X| exactly.
* Pack: inv_lambda and s_a bit-exact against the oracle's smoothing and
  activation scale; stage-wise, the oracle quantizes the device pack's own
  f32 residual and must find the same codes, block scales (all four
  replicas) and s_w; the residual is W' - L1 L2 for the pack's own bf16
  factors; and the top-r subspace is checked by Eckart-Young against the
  exact spectrum of W' (singular vectors are not unique, so the factors are
  not compared with the oracle's).
* The device-packed layer runs through K1 and K2 and matches the oracle's
  layer built from the same packed values (the pack's output is the layer's
  weight input, as in the stage-wise checks).
"""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import formats, nvfp4, svdquant
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu
F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def test_calibrate_absmax_accumulates_exactly():
    k = 320
    xa, _ = synthetic.activation(300, k, 1, 5, 40.0)
    xb, _ = synthetic.activation(77, k, 2, 3, 60.0)
    amax = torch.zeros(k, dtype=torch.float32, device=G.DEV)
    lib.svdq_calibrate_absmax(G.bf16_dev(xa), amax)
    lib.svdq_calibrate_absmax(G.bf16_dev(xb), amax)
    G.check_ok()
    want = np.maximum(np.max(np.abs(formats.bf16_bits_to_float(xa)), axis=0),
                      np.max(np.abs(formats.bf16_bits_to_float(xb)), axis=0)).astype(F32)
    np.testing.assert_array_equal(amax.cpu().numpy(), want)


def _pack(k, n, rank, seed, m=64, x_out=4, x_fac=30.0, w_out=2):
    xb, _ = synthetic.activation(m, k, seed, x_out, x_fac)
    wb, _ = synthetic.weight(k, n, seed, 0.02, w_out, 8.0)
    amax = torch.zeros(k, dtype=torch.float32, device=G.DEV)
    lib.svdq_calibrate_absmax(G.bf16_dev(xb), amax)
    d = lib.svdq_pack_weights_device(G.bf16_dev(wb), amax, rank, seed=seed, want_residual=True)
    G.check_ok()
    return xb, wb, amax.cpu().numpy(), d


@pytest.mark.parametrize("k,n,rank,tol", [(256, 256, 16, 1e-3), (320, 264, 16, 1e-3), (512, 1536, 32, 1e-3),
                                          (192, 128, 0, 0.0), (3072, 9216, 32, 1e-3)])
def test_device_pack_against_the_oracle(k, n, rank, tol):
    xb, wb, amax, d = _pack(k, n, rank, seed=k + n + rank)
    w = formats.bf16_bits_to_float(wb)
    o_inv = svdquant.smooth(amax, np.max(np.abs(w), axis=1))
    np.testing.assert_array_equal(d["inv_lambda"].cpu().numpy(), o_inv)
    assert d["s_a"].cpu().numpy()[0] == svdquant.activation_tensor_scale(amax, o_inv)
    # stage-wise NVFP4 of the pack's own residual
    r32 = d["residual"].cpu().numpy()
    s_w = nvfp4.tensor_scale(np.max(np.abs(r32)))
    assert d["s_w"].cpu().numpy()[0] == s_w
    codes, sf = nvfp4.quantize_blocks(r32.T, s_w)
    wbundle = G.u8(d["w_bundle"])
    gc, gsf = L.bundle_unpack(wbundle, n, k, 256)
    np.testing.assert_array_equal(gc, codes)
    np.testing.assert_array_equal(gsf, sf)
    assert L.scale_replicas_agree(wbundle, n, k, 256)
    assert L.bundle_padding_is_zero(wbundle, n, k, 256)
    # R = W' - L1 L2 with the pack's bf16 factors; Eckart-Young for the subspace
    wp = svdquant.smoothed_weight(w, o_inv)
    l2bits = L.lowrank_unpack(G.u8(d["l2t"]), n, 256)
    assert (l2bits[:, rank:] == 0).all()
    if rank:
        l1 = d["l1t"].float().cpu().numpy().astype(np.float64).T
        l2 = L.bf16_bits_to_f64(l2bits)[:, :rank].T
        np.testing.assert_allclose(r32, (wp - l1 @ l2).astype(F32), rtol=0, atol=2e-6)
        sig = np.linalg.svd(wp, compute_uv=False)
        optimal = np.sum(sig[rank:] ** 2)
        got = np.sum(r32.astype(np.float64) ** 2)
        assert got >= optimal * (1 - 1e-6)
        assert got <= optimal * (1 + tol) + np.sum(sig[:rank] ** 2) * 2 ** -14, (got / optimal - 1)
    else:
        np.testing.assert_array_equal(r32, wp.astype(F32))


def test_device_packed_layer_runs_through_the_kernels():
    """K1 + K2 on the device pack, against the oracle's layer built from the same packed values."""
    m, k, n, rank = 200, 768, 384, 32
    xb, wb, amax, d = _pack(k, n, rank, seed=5, m=m)
    x = formats.bf16_bits_to_float(xb)
    bb = synthetic.bias(n, 5)
    sz = lib.svdq_act_sizes(m, k)
    a = G.poisoned_u8(sz["a_bundle"])
    u = G.poisoned_u8(sz["u"])
    lib.svdq_quantize_act(G.bf16_dev(xb), d["inv_lambda"], d["l1t"], rank, d["s_a"], d["s_w"], a, u)
    Y = G.poisoned_bf16(m, n)
    lib.svdq_linear_w4a4(a, u, d["s_a"], d["w_bundle"], d["l2t"], d["s_w"], G.bf16_dev(bb), m, n, k, rank,
                         lib.EPILOGUE_GELU_ERF, 0, Y)
    G.check_ok()
    inv = d["inv_lambda"].cpu().numpy()
    l1 = d["l1t"].float().cpu().numpy().astype(np.float64).T
    l2 = L.bf16_bits_to_f64(L.lowrank_unpack(G.u8(d["l2t"]), n, 256))[:, :rank].T
    wc, wsf = L.bundle_unpack(G.u8(d["w_bundle"]), n, k, 256)
    s_a, s_w = d["s_a"].cpu().numpy()[0], d["s_w"].cpu().numpy()[0]
    oc, osf, ou = svdquant.quantize_act(x, inv, l1, s_a, s_w)
    gc, gsf, gu = G.unpack_act(a, u, m, k)
    np.testing.assert_array_equal(gc, oc)
    np.testing.assert_array_equal(gsf, osf)
    G.parity("device-packed layer U", L.bf16_bits_to_f64(gu[:, :rank]), ou)
    want = svdquant.w4a4_linear(oc, osf, s_a, wc, wsf, s_w, formats.bf16_round(ou), l2,
                                formats.bf16_bits_to_float(bb), svdquant.EPILOGUE_GELU_ERF)
    G.parity("device-packed layer Y", G.bf16_host(Y), want)
