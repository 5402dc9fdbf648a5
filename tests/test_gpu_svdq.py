"""GPU parity of the SVDQ path (K1 activation kernel, K2 W4A4 GEMM) against
the oracle, through the C ABI.

Every input comes from the seeded generators or from the oracle (its pack of
the weight, its quantization of the activation); test-side writers put them in
the library's layouts.  Nothing computed by the GPU is fed back to the oracle.

Bar: NVFP4 codes and block scales bit-exact; U and Y within 1e-2 of the
oracle, measured as the largest error in a row beyond the rounding of the
result to its bf16 output type, divided by the RMS of the oracle's row
(gpu_util.excess_error); the raw largest error over the row RMS
(gpu_util.row_rms_error) is recorded beside it for every comparison.  K2 is run on the oracle's own quantized operands
(identical on both sides; U enters as the bf16 buffer K1 writes).  Sizes span several tiles plus ragged tails in M, N and K; the
full-size workloads are checked on sampled rows.
"""
import functools

import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import formats, svdquant
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


@functools.lru_cache(maxsize=None)
def _case(m, k, n, rank, seed, x_out, x_fac, w_out, w_fac):
    """Seeded X, W, bias and the oracle's pack of W."""
    xb, _ = synthetic.activation(m, k, seed, x_out, x_fac)
    wb, _ = synthetic.weight(k, n, seed, 0.02, w_out, w_fac)
    bb = synthetic.bias(n, seed)
    x = formats.bf16_bits_to_float(xb)
    w = formats.bf16_bits_to_float(wb)
    amax = np.max(np.abs(x), axis=0).astype(np.float32)
    return xb, x, bb, svdquant.pack(w, amax, rank)


_weights_dev = G.weights_dev
_run_k1 = G.run_k1
_run_k2 = G.run_k2


def _check_k1(x, p, rank, bundle, U, rows=None):
    M, k = x.shape
    xs = x if rows is None else x[rows]
    oc, osf, ou = svdquant.quantize_act(xs, p["inv_lambda"], p["l1"], p["s_a"], p["s_w"])
    gc, gsf, gubits = G.unpack_act(bundle, U, M, k)
    if rows is not None:
        gc, gsf, gubits = gc[rows], gsf[rows], gubits[rows]
    np.testing.assert_array_equal(gc, oc)
    np.testing.assert_array_equal(gsf, osf)
    assert L.bundle_padding_is_zero(G.u8(bundle), M, k, 128)
    assert (gubits[:, rank:] == 0).all()
    pad = L.lowrank_unpack(G.u8(U), (M + 127) // 128 * 128, 128)[M:]
    assert (pad == 0).all()
    if rank:
        G.parity("U", L.bf16_bits_to_f64(gubits[:, :rank]), ou, TOL)


K1_CASES = [
    # m, k, n, rank, seed, x_out, x_fac, w_out, w_fac
    (64, 256, 256, 16, 0, 4, 30.0, 0, 1.0),      # the tiny workload
    (200, 320, 64, 32, 5, 3, 50.0, 1, 8.0),      # ragged M and K (K % 256 != 0)
    (130, 512, 64, 0, 6, 5, 50.0, 0, 1.0),       # no low-rank branch
    (33, 1024, 128, 64, 7, 10, 50.0, 2, 8.0),    # largest rank
    (1, 64, 16, 16, 8, 1, 10.0, 0, 1.0),         # single row, single scale atom
    (96, 768, 96, 48, 9, 8, 50.0, 4, 8.0),
]


@pytest.mark.parametrize("case", K1_CASES)
def test_quantize_act_parity(case):
    m, k, n, rank = case[:4]
    xb, x, bb, p = _case(*case)
    bundle, U = _run_k1(xb, m, k, rank, _weights_dev(p, rank))
    _check_k1(x, p, rank, bundle, U)


def test_quantize_act_strided_rows():
    case = (100, 256, 64, 16, 10, 2, 30.0, 0, 1.0)
    xb, x, bb, p = _case(*case)
    bundle, U = _run_k1(xb, 100, 256, 16, _weights_dev(p, 16), ldx=264)
    _check_k1(x, p, 16, bundle, U)


def _oracle_operands(x, p, rank, rows=None):
    """The oracle's activation operands: codes, scales, U/alpha rounded to bf16."""
    xs = x if rows is None else x[rows]
    oc, osf, ou = svdquant.quantize_act(xs, p["inv_lambda"], p["l1"], p["s_a"], p["s_w"])
    return oc, osf, formats.bf16_round(ou)


def _want_k2(oc, osf, ou, p, bias_bits, epilogue, begin):
    bias = formats.bf16_bits_to_float(bias_bits) if bias_bits is not None else None
    return svdquant.w4a4_linear(oc, osf, p["s_a"], p["w_codes"], p["w_sf"], p["s_w"], ou, p["l2"], bias,
                                epilogue, begin)


GEMM_CASES = [
    # (m, k, n, rank, seed, x_out, x_fac, w_out, w_fac), epilogue, gelu_begin, bias
    ((64, 256, 256, 16, 0, 4, 30.0, 0, 1.0), lib.EPILOGUE_NONE, 0, True),
    ((200, 320, 136, 32, 5, 3, 50.0, 1, 8.0), lib.EPILOGUE_GELU_ERF, 64, True),   # ragged M, N, K
    ((129, 512, 512, 0, 6, 5, 50.0, 0, 1.0), lib.EPILOGUE_GELU_TANH, 0, False),
    ((1, 64, 64, 16, 8, 1, 10.0, 0, 1.0), lib.EPILOGUE_NONE, 0, True),
    ((300, 1024, 1032, 64, 11, 10, 50.0, 5, 8.0), lib.EPILOGUE_GELU_ERF, 1000, True),
    ((512, 2048, 768, 32, 12, 20, 50.0, 10, 8.0), lib.EPILOGUE_NONE, 0, True),     # 8 K stages, 4x3 tiles
    ((384, 1536, 2304, 48, 13, 15, 50.0, 8, 8.0), lib.EPILOGUE_GELU_ERF, 768, True),  # > 1 tile per CTA
]


@pytest.mark.parametrize("case,epilogue,begin,with_bias", GEMM_CASES)
def test_linear_w4a4_parity(case, epilogue, begin, with_bias):
    m, k, n, rank = case[:4]
    xb, x, bb, p = _case(*case)
    d = _weights_dev(p, rank)
    oc, osf, ou = _oracle_operands(x, p, rank)
    bias = bb if with_bias else None
    Y, _ = _run_k2(oc, osf, ou, d, bias, m, n, k, rank, epilogue, begin)
    G.parity("Y", G.bf16_host(Y), _want_k2(oc, osf, ou, p, bias, epilogue, begin), TOL)


def test_linear_w4a4_strided_output_and_repeat():
    case = (64, 256, 256, 16, 0, 4, 30.0, 0, 1.0)
    xb, x, bb, p = _case(*case)
    d = _weights_dev(p, 16)
    oc, osf, ou = _oracle_operands(x, p, 16)
    Y1, full1 = _run_k2(oc, osf, ou, d, bb, 64, 256, 256, 16, 0, 0, ldy=272)
    Y2, _ = _run_k2(oc, osf, ou, d, bb, 64, 256, 256, 16, 0, 0, ldy=272)
    assert torch.equal(Y1, Y2)                            # deterministic
    assert torch.isnan(full1[:, 256:].float()).all()       # padding columns untouched
    G.parity("Y", G.bf16_host(Y1), _want_k2(oc, osf, ou, p, bb, 0, 0), TOL)


def _sample_rows(m, count=192, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(m, size=count - 4, replace=False).tolist()) | {0, 1, m - 2, m - 1}
    return np.array(sorted(rows))


def _full_case(c):
    return _case(c.m, c.k, c.n, c.rank, c.seed, c.x_outlier_channels, c.x_factor, c.w_outlier_rows, c.w_factor)


def test_full_size_qkv_sampled():
    """The attention-QKV workload at full size (4608 x 3072 -> 9216, r = 32):
    K1 on the whole input, checked on sampled rows; K2 on the oracle's
    operands for all rows, checked on sampled rows; then the GPU's own K1 -> K2
    chain against the oracle's whole layer."""
    c = synthetic.QKV
    xb, x, bb, p = _full_case(c)
    d = _weights_dev(p, c.rank)
    bundle, U = _run_k1(xb, c.m, c.k, c.rank, d)
    rows = _sample_rows(c.m)
    _check_k1(x, p, c.rank, bundle, U, rows=rows)

    oc, osf, ou = _oracle_operands(x, p, c.rank)
    Y, _ = _run_k2(oc, osf, ou, d, bb, c.m, c.n, c.k, c.rank, 0, 0)
    assert not torch.isnan(Y.float()).any()
    want = _want_k2(oc[rows], osf[rows], ou[rows], p, bb, 0, 0)
    G.parity("Y on oracle operands", G.bf16_host(Y)[rows], want, TOL)

    Y2 = G.poisoned_bf16(c.m, c.n)
    lib.svdq_linear_w4a4(bundle, U, d["s_a"], d["w_bundle"], d["l2t"], d["s_w"], G.bf16_dev(bb),
                         c.m, c.n, c.k, c.rank, 0, 0, Y2)
    G.check_ok()
    G.parity("Y of the GPU's K1 -> K2 chain", G.bf16_host(Y2)[rows], want, TOL)


def test_full_size_mlp_pair_sampled():
    """fc1 (3072 -> 12288 with GELU) then fc2 (12288 -> 3072), 4608 tokens.
    fc2 takes fc1's GELU output; its smoothing and static activation scale are
    calibrated from the oracle's fc1 output, and its parity inputs are the
    oracle's fc1 output rounded to bf16 (the GPU's fc1 output is compared, not
    reused)."""
    c1, c2 = synthetic.MLP_FC1, synthetic.MLP_FC2
    xb, x, bb1, p1 = _full_case(c1)
    d1 = _weights_dev(p1, c1.rank)
    rows = _sample_rows(c1.m, 96, seed=1)
    # fc1 through the GPU's own chain, compared with the oracle's layer
    bundle, U = _run_k1(xb, c1.m, c1.k, c1.rank, d1)
    H = G.poisoned_bf16(c1.m, c1.n)
    lib.svdq_linear_w4a4(bundle, U, d1["s_a"], d1["w_bundle"], d1["l2t"], d1["s_w"], G.bf16_dev(bb1),
                         c1.m, c1.n, c1.k, c1.rank, lib.EPILOGUE_GELU_ERF, 0, H)
    G.check_ok()
    oc1, osf1, ou1 = _oracle_operands(x, p1, c1.rank)
    h_oracle = _want_k2(oc1, osf1, ou1, p1, bb1, lib.EPILOGUE_GELU_ERF, 0)
    G.parity("fc1 H", G.bf16_host(H)[rows], h_oracle[rows], TOL)
    # fc2 on the oracle's fc1 output (rounded to bf16, the layer's output type)
    h = formats.bf16_round(h_oracle)
    hb = L.bf16_bits(h)
    wb2, _ = synthetic.weight(c2.k, c2.n, c2.seed, 0.02, c2.w_outlier_rows, c2.w_factor)
    bb2 = synthetic.bias(c2.n, c2.seed + 100)
    p2 = svdquant.pack(formats.bf16_bits_to_float(wb2), np.max(np.abs(h), axis=0).astype(np.float32), c2.rank)
    d2 = _weights_dev(p2, c2.rank)
    bundle2, U2 = _run_k1(hb, c2.m, c2.k, c2.rank, d2)
    _check_k1(h, p2, c2.rank, bundle2, U2, rows=rows)
    Y = G.poisoned_bf16(c2.m, c2.n)
    lib.svdq_linear_w4a4(bundle2, U2, d2["s_a"], d2["w_bundle"], d2["l2t"], d2["s_w"], G.bf16_dev(bb2),
                         c2.m, c2.n, c2.k, c2.rank, 0, 0, Y)
    G.check_ok()
    oc2, osf2, ou2 = _oracle_operands(h, p2, c2.rank, rows)
    want = _want_k2(oc2, osf2, ou2, p2, bb2, 0, 0)
    G.parity("fc2 Y", G.bf16_host(Y)[rows], want, TOL)


def test_layer_tracks_unquantized_product():
    """Information on top of parity: the quantized layer (host pack + K1 + K2)
    stays near X W + b on the tiny workload (the pages print no accuracy
    figure to pin)."""
    from bit_w4a4_diffusion_smooth_b200.layer import SVDQLinear
    c = synthetic.TINY
    xb, wb, bb = c.make()
    x = formats.bf16_bits_to_float(xb)
    w = formats.bf16_bits_to_float(wb)
    layer = SVDQLinear.from_weight(wb, np.max(np.abs(x), axis=0).astype(np.float32), c.rank, bb)
    y = G.bf16_host(layer(G.bf16_dev(xb)))
    ref = x @ w + formats.bf16_bits_to_float(bb)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.1


def test_layer_and_binding_reject_mismatched_buffers():
    """A short buffer or a wrong input width raises on the host before anything is launched."""
    from bit_w4a4_diffusion_smooth_b200.layer import SVDQLinear
    c = synthetic.TINY
    xb, wb, bb = c.make()
    x = formats.bf16_bits_to_float(xb)
    layer = SVDQLinear.from_weight(wb, np.max(np.abs(x), axis=0).astype(np.float32), c.rank, bb)
    X = G.bf16_dev(xb)
    with pytest.raises(ValueError):
        layer(X[:, : c.k - 64].contiguous())            # narrower than the layer's K
    with pytest.raises(ValueError):
        layer(X, Y=torch.empty((c.m, c.n - 8), dtype=torch.bfloat16, device=G.DEV))
    b = layer.buffers(c.m)
    with pytest.raises(ValueError):
        lib.svdq_quantize_act(X, layer.inv_lambda, layer.l1t, c.rank, layer.s_a, layer.s_w,
                              b["a_bundle"][:-16], b["U"])
    with pytest.raises(ValueError):
        lib.svdq_linear_w4a4(b["a_bundle"], b["U"], layer.s_a, layer.w_bundle[:-16], layer.l2t, layer.s_w,
                             layer.bias, c.m, c.n, c.k, c.rank, 0, 0,
                             torch.empty((c.m, c.n), dtype=torch.bfloat16, device=G.DEV))
    G.check_ok()


def test_layer_repeated_calls_match_checked_path():
    """A layer's later calls on the same buffers (pointers, shapes, strides, stream) go straight to
    the C entry points with the arguments marshalled on the first call: their outputs are bit-identical
    to those of the fully checked path on the same inputs, also after X's contents change in place
    and for another row count (a new set of buffers)."""
    from bit_w4a4_diffusion_smooth_b200.layer import SVDQLinear
    c = synthetic.TINY
    xb, wb, bb = c.make()
    x = formats.bf16_bits_to_float(xb)
    amax = np.max(np.abs(x), axis=0).astype(np.float32)
    layer = SVDQLinear.from_weight(wb, amax, c.rank, bb, epilogue=lib.EPILOGUE_GELU_ERF)
    fresh = lambda: SVDQLinear.from_weight(wb, amax, c.rank, bb, epilogue=lib.EPILOGUE_GELU_ERF)
    X = G.bf16_dev(xb)
    Y = torch.empty((c.m, c.n), dtype=torch.bfloat16, device=G.DEV)
    y1 = G.bf16_host(layer(X, Y))                        # first call: checked path, plan recorded
    xb2 = synthetic.activation(c.m, c.k, c.seed + 7, synthetic.count(0.01, c.k), 50.0)[0]
    X.copy_(G.bf16_dev(xb2))                             # same buffer, new contents
    y2 = G.bf16_host(layer(X, Y))                        # repeated call: the recorded plan
    G.check_ok()
    np.testing.assert_array_equal(y1, G.bf16_host(fresh()(G.bf16_dev(xb))))
    np.testing.assert_array_equal(y2, G.bf16_host(fresh()(G.bf16_dev(xb2))))
    m2 = c.m - 5                                         # another row count: new buffers, new plan
    Y2 = torch.empty((m2, c.n), dtype=torch.bfloat16, device=G.DEV)
    y3 = G.bf16_host(layer(X[:m2], Y2))
    y4 = G.bf16_host(layer(X[:m2], Y2))
    G.check_ok()
    np.testing.assert_array_equal(y3, G.bf16_host(fresh()(G.bf16_dev(xb2[:m2]))))
    np.testing.assert_array_equal(y4, y3)
