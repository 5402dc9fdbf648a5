"""The many-row AWQ W4A16 path (awq_linear_w4a16_gemm, and its two halves
awq_expand_weights + awq_linear_w4a16_expanded: the weights expanded into a
bf16 hi/lo workspace, then bf16 GEMMs) against the oracle, through the C ABI.

Same definition and bar as the GEMV path (the largest error in a row beyond
the bf16 rounding of the output, over the oracle row's RMS, <= 1e-2).  The
expanded weights keep ~16 significant bits (a bf16 hi + lo split), so the
GEMM cases are also held to 1e-3: a single bf16 copy of the weights reached
9e-3 on the same cases.  Cases:
ragged M around the GEMV/GEMM boundary, long K, wide N, no bias, strided X
and Y, and the user-facing layer choosing the path by row count.  The
workspace is poisoned first, so its old contents cannot leak into Y.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import awq as oawq
from oracle import formats
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def _pack(k, n, seed):
    wb, _ = synthetic.weight(k, n, seed, 0.02)
    a = synthetic.awq_scales(k, seed)
    p = oawq.pack(formats.bf16_bits_to_float(wb), a)
    dev = dict(inv=G.dev(p["inv_a"]), q=G.dev(L.awq_pack(p["q"])),
               s=G.bf16_dev(L.bf16_bits(L.awq_group_pack(p["s"]))), z=G.bf16_dev(L.bf16_bits(L.awq_group_pack(p["z"]))))
    return wb, a, p, dev


def _run(m, k, n, seed, with_bias=True, ldx=None, ldy=None):
    xb, _ = synthetic.activation(m, k, seed, synthetic.count(0.01, k), 20.0)
    wb, a, p, d = _pack(k, n, seed)
    bb = synthetic.bias(n, seed)
    X = G.bf16_dev(xb)
    if ldx is not None:
        Xp = torch.zeros((m, ldx), dtype=torch.bfloat16, device=G.DEV)
        Xp[:, :k] = X
        X = Xp[:, :k]
    Yfull = G.poisoned_bf16(m, ldy or n)
    Y = Yfull[:, :n]
    ws = torch.full((lib.awq_gemm_workspace_size(m, k, n),), 0xFF, dtype=torch.uint8, device=G.DEV)
    lib.awq_linear_w4a16_gemm(X, d["inv"], d["q"], d["s"], d["z"], G.bf16_dev(bb) if with_bias else None, n, Y, ws)
    G.check_ok()
    want = oawq.linear(formats.bf16_bits_to_float(xb), p["inv_a"], p["q"], p["s"], p["z"],
                       formats.bf16_bits_to_float(bb) if with_bias else None)
    if ldy is not None:
        assert torch.isnan(Yfull[:, n:].float()).all()      # columns past N untouched
    return G.parity(f"AWQ GEMM {m}x{k}->{n}", G.bf16_host(Y), want)[0]


@pytest.mark.parametrize("m,k,n", [(17, 256, 64), (65, 3072, 512), (300, 1024, 1280), (1000, 3072, 192),
                                   (4096, 512, 256), (129, 6144, 128)])
def test_awq_gemm_parity(m, k, n):
    assert _run(m, k, n, seed=m + k + n) <= 1e-3


def test_awq_gemm_strided_without_bias():
    assert _run(70, 512, 192, 31, with_bias=False, ldx=520, ldy=200) <= 1e-3


def test_awq_gemm_full_width_adaln_batch():
    """A batch of 256 modulation vectors through the 3072 -> 18432 adaLN projection."""
    assert _run(256, 3072, 18432, 41) <= 1e-3


def test_awq_layer_picks_the_path_by_rows():
    from bit_w4a4_diffusion_smooth_b200.layer import AWQLinear
    k, n = 512, 256
    wb, a, p, _ = _pack(k, n, 51)
    bb = synthetic.bias(n, 51)
    layer = AWQLinear.from_weight(wb, a, bb)
    for m in (layer.gemm_rows, layer.gemm_rows + 37):
        xb, _ = synthetic.activation(m, k, 52 + m)
        y = G.bf16_host(layer(G.bf16_dev(xb)))
        want = oawq.linear(formats.bf16_bits_to_float(xb), p["inv_a"], p["q"], p["s"], p["z"],
                           formats.bf16_bits_to_float(bb))
        G.parity(f"AWQ layer, M={m}", y, want)
    assert getattr(layer, "_workspace", None) is not None      # the second call took the GEMM path


def test_expanded_weights_serve_several_calls():
    """awq_expand_weights once, then awq_linear_w4a16_expanded on two inputs of different row counts."""
    k, n = 1024, 320
    wb, a, p, d = _pack(k, n, 61)
    bb = synthetic.bias(n, 61)
    ws = torch.full((lib.awq_gemm_workspace_size(300, k, n),), 0xFF, dtype=torch.uint8, device=G.DEV)
    lib.awq_expand_weights(d["inv"], d["q"], d["s"], d["z"], k, n, ws)
    for m in (300, 150):
        xb, _ = synthetic.activation(m, k, 62 + m)
        Y = G.poisoned_bf16(m, n)
        lib.awq_linear_w4a16_expanded(G.bf16_dev(xb), G.bf16_dev(bb), n, Y, ws)
        G.check_ok()
        want = oawq.linear(formats.bf16_bits_to_float(xb), p["inv_a"], p["q"], p["s"], p["z"],
                           formats.bf16_bits_to_float(bb))
        assert G.parity(f"expanded AWQ, M={m}", G.bf16_host(Y), want)[0] <= 1e-3
