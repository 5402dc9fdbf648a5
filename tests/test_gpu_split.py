"""The fused-projection adapter (layer.SplitProjection): a checkpoint packed as
one fused projection [W_q | W_k | W_v] (or QKV + MLP-in) mapped onto split
modules.

Every part's output must equal the fused layer's output columns bit for bit
(the parts are views of the fused layer's packed buffers and run the same
tile arithmetic), and must match the oracle on the layer's own packed values
within the parity tolerance.  Cases: three equal parts without GELU, and
unequal parts under a GELU that starts inside one part.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from bit_w4a4_diffusion_smooth_b200.layer import SplitProjection, SVDQLinear
from oracle import formats, svdquant
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def _fused(m, k, sizes, rank, epilogue, begin, seed):
    n = sum(sizes)
    xb, _ = synthetic.activation(m, k, seed, synthetic.count(0.01, k), 50.0)
    wb, _ = synthetic.weight(k, n, seed, 0.02, synthetic.count(0.005, k), 8.0)
    bb = synthetic.bias(n, seed)
    amax = np.max(np.abs(formats.bf16_bits_to_float(xb)), axis=0).astype(np.float32)
    layer = SVDQLinear.from_weight(wb, amax, rank, bias_bits=bb, epilogue=epilogue, gelu_col_begin=begin,
                                   device=G.DEV, seed=seed)
    return xb, bb, layer


def _oracle_rows(layer, xb, bb, rows, epilogue, begin):
    """The oracle's layer output on the fused layer's own packed values, for the given rows."""
    k, n, r = layer.K, layer.N, layer.rank
    x = formats.bf16_bits_to_float(xb)[rows]
    inv = layer.inv_lambda.cpu().numpy()
    l1 = layer.l1t.float().cpu().numpy().astype(np.float64).T
    l2 = L.bf16_bits_to_f64(L.lowrank_unpack(G.u8(layer.l2t), n, 256))[:, :r].T
    wc, wsf = L.bundle_unpack(G.u8(layer.w_bundle), n, k, 256)
    s_a, s_w = layer.s_a.cpu().numpy()[0], layer.s_w.cpu().numpy()[0]
    oc, osf, ou = svdquant.quantize_act(x, inv, l1, s_a, s_w)
    return svdquant.w4a4_linear(oc, osf, s_a, wc, wsf, s_w, formats.bf16_round(ou), l2,
                                formats.bf16_bits_to_float(bb), epilogue, begin)


@pytest.mark.parametrize("m,k,sizes,epilogue,begin", [
    (300, 768, (256, 256, 256), lib.EPILOGUE_NONE, 0),           # Q | K | V
    (200, 512, (512, 256, 768), lib.EPILOGUE_GELU_ERF, 640),      # QKV + MLP-in, GELU from inside part 1
])
def test_split_parts_equal_fused_columns_and_oracle(m, k, sizes, epilogue, begin):
    rank = 32
    xb, bb, layer = _fused(m, k, sizes, rank, epilogue, begin, seed=m + k)
    X = G.bf16_dev(xb)
    Yf = layer(X)
    split = SplitProjection(layer, sizes, names=[f"p{i}" for i in range(len(sizes))])
    parts = split(X)
    G.check_ok()
    rows = np.sort(np.random.default_rng(1).choice(m, 24, replace=False))
    want = _oracle_rows(layer, xb, bb, rows, epilogue, begin)
    n0 = 0
    for i, sz in enumerate(sizes):
        y = parts[f"p{i}"]
        assert torch.equal(y, Yf[:, n0:n0 + sz])
        G.parity(f"split part {i} ({sz} columns)", G.bf16_host(y)[rows], want[:, n0:n0 + sz], TOL)
        n0 += sz


def test_split_rejects_unaligned_parts():
    xb, bb, layer = _fused(64, 256, (256, 256), 16, lib.EPILOGUE_NONE, 0, seed=3)
    with pytest.raises(ValueError):
        SplitProjection(layer, (128, 384))
    with pytest.raises(ValueError):
        SplitProjection(layer, (256,))
