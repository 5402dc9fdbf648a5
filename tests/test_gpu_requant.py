"""GPU parity of the re-quantizing W4A4 GEMM (svdq_linear_w4a4_requant): the
MLP fc1 GEMM whose epilogue writes fc2's NVFP4 input operands (codes, block
scales) and fc2's low-rank activations instead of its bf16 output.

The oracle side composes functions that are already pinned: fc1's output is
oracle.svdquant.w4a4_linear, rounded to bf16 (the layer's output type), and
fc2's operands are oracle.svdquant.quantize_act of that.

* Exact case: every fc1 operand is on the e2m1 grid with power-of-two block
  scales and small-integer low-rank factors, so fc1's fp32 accumulation is
  exact in any order; then the GPU's bf16 output equals the oracle's bit for
  bit and so must every fc2 code and block scale.  U_next is compared within
  the parity tolerance (its fp32 sum is formed in another order).
* Full-size MLP pair (4608 x 3072 -> 12288 with GELU, then 12288 -> 3072):
  fc1's GPU result and the oracle's differ by float rounding, so a bf16
  output can land on the other side of a rounding boundary; the codes and
  scales are compared by their mismatch rate, and fc2's output on the fused
  operands against the oracle's unfused chain within the parity tolerance.
"""
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


def _grid_operands(rng, rows, k):
    """e2m1 codes and ue4m3 scales in {0.5, 1, 2}: products of two such values are exact."""
    codes = rng.integers(0, 16, (rows, k)).astype(np.uint8)
    sf = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (rows, k // 16))
    return codes, sf


def _next_layer(rng, n, next_rank, h):
    """The next layer's smoothing, L1 and scales, calibrated on its input h (float64 bf16 values)."""
    inv = np.exp(rng.uniform(np.log(0.25), np.log(4.0), n)).astype(np.float32)
    l1 = formats.bf16_round(rng.standard_normal((n, next_rank)) * 0.05)
    amax = np.max(np.abs(h), axis=0).astype(np.float32)
    s_a = svdquant.activation_tensor_scale(amax, inv)
    s_w = np.float32(0.0123)
    return inv, l1, s_a, s_w


def _run_requant(oc, osf, ou, l2, wc, wsf, bb, m, n, k, rank, epilogue, inv, l1, next_rank, s_a2, s_w2,
                 want_y=False):
    d = dict(s_a=G.dev(np.array([1.0], np.float32)), s_w=G.dev(np.array([1.0], np.float32)))
    nsz = lib.svdq_act_sizes(m, n)
    nb = G.poisoned_u8(nsz["a_bundle"])
    nu = G.poisoned_u8(nsz["u"])
    ws = torch.full((max(1, lib.svdq_requant_workspace_size(m, next_rank) // 4),), float("nan"),
                    dtype=torch.float32, device=G.DEV)
    Y = G.poisoned_bf16(m, n) if want_y else None
    lib.svdq_linear_w4a4_requant(
        G.dev(L.bundle_pack(oc, osf, m, k, 128)), G.dev(L.lowrank_pack(L.bf16_bits(ou), 128)) if rank else None,
        d["s_a"], G.dev(L.bundle_pack(wc, wsf, n, k, 256)),
        G.dev(L.lowrank_pack(L.bf16_bits(l2.T), 256)) if rank else None, d["s_w"], G.bf16_dev(bb), m, n, k, rank,
        epilogue, 0, Y, G.dev(inv), G.bf16_dev(L.bf16_bits(l1.T)) if next_rank else None, next_rank,
        G.dev(np.array([s_a2], np.float32)), G.dev(np.array([s_w2], np.float32)), nb,
        nu if next_rank else None, ws if next_rank else None)
    G.check_ok()
    return nb, nu, Y


@pytest.mark.parametrize("m,k,n,rank,next_rank", [
    (200, 512, 320, 16, 16),     # ragged M (two row tiles, the second partial); N % 256 != 0
    (64, 256, 256, 0, 32),       # no low-rank branch in fc1
    (300, 768, 576, 32, 64),     # several tiles per SM pair, the largest next rank
    (129, 256, 128, 16, 0),      # no low-rank branch in the next layer
])
def test_requant_exact_operands_bit_exact(m, k, n, rank, next_rank):
    rng = np.random.default_rng(m + k + n + rank)
    oc, osf = _grid_operands(rng, m, k)
    wc, wsf = _grid_operands(rng, n, k)
    ou = rng.integers(-4, 5, (m, rank)).astype(np.float64)
    l2 = rng.integers(-2, 3, (rank, n)).astype(np.float64)
    bias = rng.integers(-32, 33, n) * 0.25
    bb = L.bf16_bits(bias)
    one = np.float32(1.0)
    y = svdquant.w4a4_linear(oc, osf, one, wc, wsf, one, ou, l2, bias)     # exact in float64 and in fp32
    h = formats.bf16_round(y)
    inv, l1, s_a2, s_w2 = _next_layer(rng, n, next_rank, h)
    nb, nu, Y = _run_requant(oc, osf, ou, l2, wc, wsf, bb, m, n, k, rank, lib.EPILOGUE_NONE, inv, l1, next_rank,
                             s_a2, s_w2, want_y=True)
    np.testing.assert_array_equal(G.bf16_host(Y), h)                      # the optional bf16 output
    c2, sf2, u2 = svdquant.quantize_act(h, inv, l1, s_a2, s_w2)
    gc, gsf = L.bundle_unpack(G.u8(nb), m, n, 128)
    np.testing.assert_array_equal(gc, c2)
    np.testing.assert_array_equal(gsf, sf2)
    assert L.bundle_padding_is_zero(G.u8(nb), m, n, 128)
    if next_rank:
        gu = L.lowrank_unpack(G.u8(nu), (m + 127) // 128 * 128, 128)
        assert (gu[:, next_rank:] == 0).all() and (gu[m:] == 0).all()
        G.parity("next U", L.bf16_bits_to_f64(gu[:m, :next_rank]), u2, TOL)


def test_requant_gelu_without_output():
    """GELU (tanh form) epilogue and no bf16 output: the next layer's operands still match the
    oracle's quantization of the oracle's GELU output, except where the two GELU evaluations
    round to different bf16 values."""
    rng = np.random.default_rng(7)
    m, k, n, rank, next_rank = 160, 512, 384, 16, 32
    oc, osf = _grid_operands(rng, m, k)
    wc, wsf = _grid_operands(rng, n, k)
    ou = rng.integers(-4, 5, (m, rank)).astype(np.float64)
    l2 = rng.integers(-2, 3, (rank, n)).astype(np.float64)
    bias = rng.integers(-32, 33, n) * 0.25
    one = np.float32(1.0)
    h = formats.bf16_round(svdquant.w4a4_linear(oc, osf, one, wc, wsf, one, ou, l2, bias,
                                                svdquant.EPILOGUE_GELU_TANH))
    inv, l1, s_a2, s_w2 = _next_layer(rng, n, next_rank, h)
    nb, nu, _ = _run_requant(oc, osf, ou, l2, wc, wsf, L.bf16_bits(bias), m, n, k, rank, lib.EPILOGUE_GELU_TANH,
                             inv, l1, next_rank, s_a2, s_w2)
    c2, sf2, u2 = svdquant.quantize_act(h, inv, l1, s_a2, s_w2)
    gc, gsf = L.bundle_unpack(G.u8(nb), m, n, 128)
    assert np.mean(gsf != sf2) < 1e-2 and np.mean(gc != c2) < 1e-2
    assert L.bundle_padding_is_zero(G.u8(nb), m, n, 128)
    gu = L.lowrank_unpack(G.u8(nu), (m + 127) // 128 * 128, 128)
    G.parity("next U", L.bf16_bits_to_f64(gu[:m, :next_rank]), u2, TOL)


def test_requant_full_size_mlp_pair():
    """The MLP pair at full size: fc1 (4608 x 3072 -> 12288, GELU) re-quantized for fc2
    (12288 -> 3072) inside fc1's GEMM, then fc2's GEMM on those operands, against the oracle's
    unfused chain (fc1 output rounded to bf16, fc2's quantize_act and GEMM)."""
    c1, c2 = synthetic.MLP_FC1, synthetic.MLP_FC2
    xb, wb, bb1 = c1.make()
    x = formats.bf16_bits_to_float(xb)
    p1 = svdquant.pack(formats.bf16_bits_to_float(wb), np.max(np.abs(x), axis=0).astype(np.float32), c1.rank)
    d1 = G.weights_dev(p1, c1.rank)
    bias1 = formats.bf16_bits_to_float(bb1)
    oc1, osf1, ou1 = svdquant.quantize_act(x, p1["inv_lambda"], p1["l1"], p1["s_a"], p1["s_w"])
    h = formats.bf16_round(svdquant.w4a4_linear(oc1, osf1, p1["s_a"], p1["w_codes"], p1["w_sf"], p1["s_w"],
                                                formats.bf16_round(ou1), p1["l2"], bias1, svdquant.EPILOGUE_GELU_ERF))
    wb2, _ = synthetic.weight(c2.k, c2.n, c2.seed, 0.02, c2.w_outlier_rows, c2.w_factor)
    bb2 = synthetic.bias(c2.n, c2.seed + 100)
    p2 = svdquant.pack(formats.bf16_bits_to_float(wb2), np.max(np.abs(h), axis=0).astype(np.float32), c2.rank)
    d2 = G.weights_dev(p2, c2.rank)

    # GPU: fc1's K1, the re-quantizing fc1 GEMM (no bf16 output), fc2's GEMM
    bundle, U = G.run_k1(xb, c1.m, c1.k, c1.rank, d1)
    nsz = lib.svdq_act_sizes(c1.m, c1.n)
    nb = G.poisoned_u8(nsz["a_bundle"])
    nu = G.poisoned_u8(nsz["u"])
    ws = torch.empty(lib.svdq_requant_workspace_size(c1.m, c2.rank) // 4, dtype=torch.float32, device=G.DEV)
    lib.svdq_linear_w4a4_requant(bundle, U, d1["s_a"], d1["w_bundle"], d1["l2t"], d1["s_w"], G.bf16_dev(bb1),
                                 c1.m, c1.n, c1.k, c1.rank, lib.EPILOGUE_GELU_ERF, 0, None,
                                 d2["inv_lambda"], d2["l1t"], c2.rank, d2["s_a"], d2["s_w"], nb, nu, ws)
    G.check_ok()
    Y = G.poisoned_bf16(c2.m, c2.n)
    lib.svdq_linear_w4a4(nb, nu, d2["s_a"], d2["w_bundle"], d2["l2t"], d2["s_w"], G.bf16_dev(bb2),
                         c2.m, c2.n, c2.k, c2.rank, lib.EPILOGUE_NONE, 0, Y)
    G.check_ok()

    oc2, osf2, ou2 = svdquant.quantize_act(h, p2["inv_lambda"], p2["l1"], p2["s_a"], p2["s_w"])
    gc, gsf = L.bundle_unpack(G.u8(nb), c1.m, c1.n, 128)
    code_mis, scale_mis = float(np.mean(gc != oc2)), float(np.mean(gsf != osf2))
    print(f"fused fc2 operands vs the oracle's: code mismatch {code_mis:.2e}, scale mismatch {scale_mis:.2e}")
    assert code_mis < 1e-3 and scale_mis < 1e-3
    gu = L.lowrank_unpack(G.u8(nu), c1.m, 128)
    G.parity("fc2 U from the fused epilogue", L.bf16_bits_to_f64(gu[:, :c2.rank]), ou2, TOL)
    rows = np.unique(np.r_[np.random.default_rng(3).choice(c2.m, 124, replace=False), [0, 1, c2.m - 2, c2.m - 1]])
    want = svdquant.w4a4_linear(oc2[rows], osf2[rows], p2["s_a"], p2["w_codes"], p2["w_sf"], p2["s_w"],
                                formats.bf16_round(ou2[rows]), p2["l2"], formats.bf16_bits_to_float(bb2))
    G.parity("fc2 Y on the fused operands vs the unfused oracle chain", G.bf16_host(Y)[rows], want, TOL)
