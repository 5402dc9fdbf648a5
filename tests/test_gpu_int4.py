"""GPU parity of the INT4 W4A4 variant (svdq_quantize_act_int4, svdq_linear_int4)
against the oracle (oracle/int4.py), through the C ABI.

  * Activation side: codes and group scales bit-exact (both sides take the same
    float32 steps), padding rows zero, U within the parity bar; ragged M and K,
    ranks 0..64, strided X.
  * GEMM on the oracle's own operands (uploaded in the test-side layouts of
    tests/layouts.py): Y within the parity bar (excess error over the row RMS
    <= 1e-2, as for the NVFP4 GEMM); ragged M, K up to 3072, GELU from inside
    the output, no bias, rank 0, widths with a last block of 128 columns.
  * The chain K1 -> K2 at full size on the MLP fc1 (4608 x 3072 -> 12288, erf
    GELU), the single block's fused QKV + MLP-in (-> 21504, GELU from column
    9216) and its output projection (K = 15360), with the library's host pack:
    codes and scales of sampled rows bit-exact, and Y of those rows against the
    oracle on the GPU's own operands.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import formats, int4, svdquant
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def _data(m, k, n, seed):
    xb, _ = synthetic.activation(m, k, seed, synthetic.count(0.01, k), 50.0)
    wb, _ = synthetic.weight(k, n, seed, 0.02, synthetic.count(0.005, k), 8.0)
    x = formats.bf16_bits_to_float(xb)
    amax = np.max(np.abs(x), axis=0).astype(np.float32)
    return xb, x, wb, amax


def _k1(xb, m, k, rank, inv_lambda, l1, ldx=None):
    sz = lib.svdq_int4_act_sizes(m, k)
    X = G.bf16_dev(xb)
    if ldx is not None:
        Xp = torch.zeros((m, ldx), dtype=torch.bfloat16, device=G.DEV)
        Xp[:, :k] = X
        X = Xp[:, :k]
    codes = G.poisoned_u8(sz["codes"])
    scales = G.poisoned_u8(sz["scales"])
    U = G.poisoned_u8(lib.svdq_act_sizes(m, k)["u"])
    l1t = G.bf16_dev(L.bf16_bits(l1.T)) if rank else None
    lib.svdq_quantize_act_int4(X, G.dev(np.asarray(inv_lambda, np.float32)), l1t, rank, codes, scales, U, M=m, K=k)
    G.check_ok()
    return codes, scales, U


def _unpack_k1(codes, scales, U, m, k):
    mp = (m + 127) // 128 * 128
    c = G.u8(codes)
    q = L.int4_unpack(c, mp, k)
    s = L.int4_scales_unpack(G.u8(scales).view(np.uint16), mp, k // 64, mp)
    u = L.lowrank_unpack(G.u8(U), m, 128)
    return q, s, u


@pytest.mark.parametrize("m,k,rank,ldx", [(200, 320, 32, None), (4, 768, 0, None), (300, 3072, 16, 3080),
                                          (64, 256, 64, None), (129, 1024, 48, None)])
def test_int4_quantize_act_matches_oracle(m, k, rank, ldx):
    xb, x, wb, amax = _data(m, k, 128, m + k)
    p = int4.pack(formats.bf16_bits_to_float(wb), amax, rank)
    codes, scales, U = _k1(xb, m, k, rank, p["inv_lambda"], p["l1"], ldx)
    q, s, u = _unpack_k1(codes, scales, U, m, k)
    oq, osf, ou = int4.quantize_act(x, p["inv_lambda"], p["l1"])
    np.testing.assert_array_equal(q[:m], oq)
    np.testing.assert_array_equal(s[:m], osf)
    assert not q[m:].any() and not s[m:].any()                      # padding rows quantize to zero
    if rank:
        G.parity(f"INT4 K1 U, M={m} K={k} r={rank}", L.bf16_bits_to_f64(u[:, :rank]), ou, TOL)


def _k2(qa, sa, u_bits, qw, sw, l2, bias_bits, m, n, k, rank, epilogue, begin):
    mp = (m + 127) // 128 * 128
    qa_p = np.zeros((mp, k), np.int8)
    qa_p[:m] = qa
    sa_p = np.zeros((mp, k // 64))
    sa_p[:m] = sa
    Y = G.poisoned_bf16(m, n)
    U = G.dev(L.lowrank_pack(u_bits, 128)) if rank else None
    l2t = G.dev(L.lowrank_pack(L.bf16_bits(l2.T), 256)) if rank else None
    lib.svdq_linear_int4(G.dev(L.int4_pack(qa_p)), G.dev(L.int4_scales_pack(sa_p, mp)), U,
                         G.dev(L.int4_pack(qw)), G.dev(L.int4_scales_pack(sw, n)), l2t,
                         G.bf16_dev(bias_bits) if bias_bits is not None else None, m, n, k, rank, epilogue, begin, Y)
    G.check_ok()
    return G.bf16_host(Y)


@pytest.mark.parametrize("m,k,n,rank,epilogue,begin,with_bias", [
    (200, 320, 256, 32, svdquant.EPILOGUE_NONE, 0, True),
    (37, 1024, 384, 16, svdquant.EPILOGUE_GELU_ERF, 136, True),
    (129, 3072, 512, 0, svdquant.EPILOGUE_NONE, 0, False),
    (64, 512, 128, 64, svdquant.EPILOGUE_GELU_TANH, 0, True),
    (1, 256, 256, 32, svdquant.EPILOGUE_GELU_ERF, 0, True)])
def test_int4_gemm_matches_oracle(m, k, n, rank, epilogue, begin, with_bias):
    xb, x, wb, amax = _data(m, k, n, 7 * m + k)
    p = int4.pack(formats.bf16_bits_to_float(wb), amax, rank)
    qa, sa, u = int4.quantize_act(x, p["inv_lambda"], p["l1"])
    ub = formats.bf16_round(u)
    bb = synthetic.bias(n, m + n) if with_bias else None
    y = _k2(qa, sa, L.bf16_bits(ub), p["qw"], p["sw"], p["l2"], bb, m, n, k, rank, epilogue, begin)
    want = int4.int4_linear(qa, sa, p["qw"], p["sw"], ub, p["l2"],
                            formats.bf16_bits_to_float(bb) if with_bias else None, epilogue, begin)
    G.parity(f"INT4 K2 Y, M={m} K={k} N={n} r={rank}", y, want, TOL)


def test_int4_gemm_many_tiles_sampled():
    """Several 256 x 256 tiles per SM pair (both accumulators in turn), a last half pair, a last column
    block of 128 (N % 256 == 128), rank 16, tanh GELU from column 1000: sampled rows against the oracle
    on the same operands."""
    m, k, n, rank = 4480, 1024, 5248, 16
    xb, x, wb, amax = _data(m, k, n, 55)
    p = int4.pack(formats.bf16_bits_to_float(wb), amax, rank)
    qa, sa, u = int4.quantize_act(x, p["inv_lambda"], p["l1"])
    ub = formats.bf16_round(u)
    bb = synthetic.bias(n, 56)
    y = _k2(qa, sa, L.bf16_bits(ub), p["qw"], p["sw"], p["l2"], bb, m, n, k, rank, svdquant.EPILOGUE_GELU_TANH, 1000)
    rows = np.sort(np.random.default_rng(57).choice(m, 24, replace=False))
    rows[-1] = m - 1                                                 # a row of the last, half pair
    want = int4.int4_linear(qa[rows], sa[rows], p["qw"], p["sw"], ub[rows], p["l2"],
                            formats.bf16_bits_to_float(bb), svdquant.EPILOGUE_GELU_TANH, 1000)
    G.parity("INT4 K2 Y many tiles (sampled rows)", y[rows], want, TOL)


@pytest.mark.parametrize("name,m,k,n,epilogue,begin,seed", [
    ("mlp fc1", 4608, 3072, 12288, svdquant.EPILOGUE_GELU_ERF, 0, 90),
    ("single qkv_mlp", 4608, 3072, 21504, svdquant.EPILOGUE_GELU_ERF, 9216, 93),
    ("single out", 4608, 15360, 3072, svdquant.EPILOGUE_NONE, 0, 96)])
def test_int4_chain_full_size(name, m, k, n, epilogue, begin, seed):
    """The layer shapes of a 12B-class DiT at full size (the MLP fc1 with the erf GELU; the single
    block's fused QKV + MLP-in with GELU on columns 9216.. only; its output projection at K =
    15360): the library's host pack, K1 then K2 on the GPU, in the benchmark's launch
    configuration.  Codes and scales of sampled rows bit-exact, Y of those rows against the oracle
    on the GPU's own operands."""
    rank = 32
    xb, x, wb, amax = _data(m, k, n, seed)
    pk = lib.svdq_pack_weights_int4(wb, amax, rank)
    bb = synthetic.bias(n, seed + 1)
    l1 = L.bf16_bits_to_f64(pk["l1t"]).T
    codes, scales, U = _k1(xb, m, k, rank, pk["inv_lambda"], l1)
    Y = G.poisoned_bf16(m, n)
    lib.svdq_linear_int4(codes, scales, U, G.dev(pk["w_codes"]), G.dev(pk["w_scales"]), G.dev(pk["l2t"]),
                         G.bf16_dev(bb), m, n, k, rank, epilogue, begin, Y)
    G.check_ok()
    rows = np.sort(np.random.default_rng(seed + 2).choice(m, 24, replace=False))
    rows[0], rows[-1] = 0, m - 1
    q, s, u = _unpack_k1(codes, scales, U, m, k)
    oq, osf, ou = int4.quantize_act(x[rows], pk["inv_lambda"], l1)
    np.testing.assert_array_equal(q[rows], oq)
    np.testing.assert_array_equal(s[rows], osf)
    G.parity(f"INT4 {name} U", L.bf16_bits_to_f64(u[rows, :rank]), ou, TOL)
    qw = L.int4_unpack(pk["w_codes"], n, k)
    sw = L.int4_scales_unpack(pk["w_scales"], n, k // 64, n)
    l2 = L.bf16_bits_to_f64(L.lowrank_unpack(pk["l2t"], n, 256))[:, :rank].T
    want = int4.int4_linear(q[rows], s[rows], qw, sw, L.bf16_bits_to_f64(u[rows, :rank]), l2,
                            formats.bf16_bits_to_float(bb), epilogue, begin)
    G.parity(f"INT4 {name} Y (GPU operands)", G.bf16_host(Y)[rows], want, TOL)


def test_int4_layer_from_weight():
    """The user-facing INT4 layer (host pack, K1, GEMM) against the oracle on the layer's own packed values."""
    from bit_w4a4_diffusion_smooth_b200.layer import SVDQLinearInt4
    m, k, n, rank = 130, 512, 256, 32
    xb, x, wb, amax = _data(m, k, n, 77)
    bb = synthetic.bias(n, 78)
    layer = SVDQLinearInt4.from_weight(wb, amax, rank, bias_bits=bb, epilogue=svdquant.EPILOGUE_GELU_ERF)
    y = G.bf16_host(layer(G.bf16_dev(xb)))
    G.check_ok()
    pk = lib.svdq_pack_weights_int4(wb, amax, rank)
    l1 = L.bf16_bits_to_f64(pk["l1t"]).T
    qa, sa, u = int4.quantize_act(x, pk["inv_lambda"], l1)
    want = int4.int4_linear(qa, sa, L.int4_unpack(pk["w_codes"], n, k),
                            L.int4_scales_unpack(pk["w_scales"], n, k // 64, n), formats.bf16_round(u),
                            L.bf16_bits_to_f64(L.lowrank_unpack(pk["l2t"], n, 256))[:, :rank].T,
                            formats.bf16_bits_to_float(bb), svdquant.EPILOGUE_GELU_ERF, 0)
    G.parity("INT4 layer", y, want, TOL)
