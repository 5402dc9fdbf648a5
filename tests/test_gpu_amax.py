"""GPU parity of the dynamic activation-scale pass (svdq_act_amax) against the
oracle's dynamic_activation_scale, bit for bit, and of the dynamic-scale layer
it enables: svdq_quantize_act fed that device scalar must write the codes and
block scales the oracle derives with the same scale."""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import formats, svdquant
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def _amax(xb, inv, ldx=None):
    m, k = xb.shape
    X = G.bf16_dev(xb)
    if ldx is not None:
        Xp = torch.zeros((m, ldx), dtype=torch.bfloat16, device=G.DEV)
        Xp[:, :k] = X
        Xp[:, k:] = 1e4                      # outside the view: must not count
        X = Xp[:, :k]
    ws = torch.full((lib.AMAX_WORKSPACE_BYTES,), 0xA5, dtype=torch.uint8, device=G.DEV)
    s_a = torch.full((1,), float("nan"), dtype=torch.float32, device=G.DEV)
    lib.svdq_act_amax(X, G.dev(inv), ws, s_a)
    G.check_ok()
    return s_a


@pytest.mark.parametrize("m,k,seed,ldx", [(1, 64, 0, None), (37, 320, 1, None), (200, 1024, 2, 1040),
                                          (4608, 3072, 3, None), (512, 12288, 4, None)])
def test_act_amax_bit_exact(m, k, seed, ldx):
    xb, _ = synthetic.activation(m, k, seed, synthetic.count(0.01, k), 50.0)
    inv = synthetic.awq_scales(k, seed)                 # any positive f32 per channel
    s_a = _amax(xb, inv, ldx)
    want = svdquant.dynamic_activation_scale(formats.bf16_bits_to_float(xb), inv)
    assert s_a.cpu().numpy()[0] == want
    # twice in a row: the workspace is cleared by each call
    assert _amax(xb, inv, ldx).cpu().numpy()[0] == want


def test_act_amax_zero_tensor_gives_unit_scale():
    s_a = _amax(np.zeros((3, 128), np.uint16), np.ones(128, np.float32))
    assert s_a.cpu().numpy()[0] == np.float32(1.0)


def test_dynamic_scale_layer_codes_bit_exact():
    """svdq_act_amax -> svdq_quantize_act with that scalar: codes, block scales bit-exact and U
    within the parity bar against the oracle with the dynamic scale."""
    m, k, rank = 300, 768, 32
    xb, _ = synthetic.activation(m, k, 9, 8, 50.0)
    wb, _ = synthetic.weight(k, 256, 9, 0.02, 4, 8.0)
    x = formats.bf16_bits_to_float(xb)
    # a pack calibrated on other data: the dynamic scale replaces its static s_a
    xcal, _ = synthetic.activation(64, k, 10, 8, 20.0)
    p = svdquant.pack(formats.bf16_bits_to_float(wb), np.max(np.abs(formats.bf16_bits_to_float(xcal)), axis=0)
                      .astype(np.float32), rank)
    d = G.weights_dev(p, rank)
    s_dyn = _amax(xb, p["inv_lambda"])
    want_s = svdquant.dynamic_activation_scale(x, p["inv_lambda"])
    assert s_dyn.cpu().numpy()[0] == want_s
    d["s_a"] = s_dyn
    bundle, U = G.run_k1(xb, m, k, rank, d)
    oc, osf, ou = svdquant.quantize_act(x, p["inv_lambda"], p["l1"], want_s, p["s_w"])
    gc, gsf, gu = G.unpack_act(bundle, U, m, k)
    np.testing.assert_array_equal(gc, oc)
    np.testing.assert_array_equal(gsf, osf)
    assert osf.max() == 0x7E                           # the dynamic scale puts the largest block at 448
    G.parity("U with the dynamic scale", L.bf16_bits_to_f64(gu[:, :rank]), ou)
