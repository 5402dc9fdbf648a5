"""Grouped launches (svdq_quantize_act_grouped, svdq_linear_w4a4_grouped)
against the oracle and against the single calls, through the C ABI.

A grouped launch runs up to four independent problems in one grid.  Each
problem's outputs must be what the oracle gives for it (the same bars as the
single calls: codes and block scales bit-exact, U and Y within 1e-2 excess
error), and identical byte for byte to the single call with the same
arguments (the same kernel arithmetic per tile, in the same order).  The
problems differ in M (ragged tails), N, K, GELU column begin and weights;
the full-size case is a dual-stream DiT projection: 4096 image tokens and
512 text tokens of 3072 -> 9216, which one launch covers with all SM pairs.
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
def _case(m, k, n, rank, seed):
    xb, _ = synthetic.activation(m, k, seed, synthetic.count(0.01, k), 50.0)
    wb, _ = synthetic.weight(k, n, seed, 0.02, synthetic.count(0.005, k), 8.0)
    bb = synthetic.bias(n, seed)
    x = formats.bf16_bits_to_float(xb)
    w = formats.bf16_bits_to_float(wb)
    amax = np.max(np.abs(x), axis=0).astype(np.float32)
    return xb, x, bb, svdquant.pack(w, amax, rank)


def _k1_problem(xb, m, k, d):
    sz = lib.svdq_act_sizes(m, k)
    return dict(X=G.bf16_dev(xb), inv_lambda=d["inv_lambda"], l1t=d["l1t"], s_a=d["s_a"], s_w=d["s_w"],
                a_bundle=G.poisoned_u8(sz["a_bundle"]), U=G.poisoned_u8(sz["u"]), M=m, K=k)


# (m, k, n, seed): ragged M and K, three different shapes in one group
K1_GROUP = [(200, 320, 64, 1), (4, 768, 64, 2), (300, 3072, 64, 3)]


@pytest.mark.parametrize("rank", [0, 32])
def test_grouped_quantize_matches_oracle_and_single_calls(rank):
    cases = [(m, k, n, rank, seed) for m, k, n, seed in K1_GROUP]
    packs = [_case(*c) for c in cases]
    devs = [G.weights_dev(p, rank) for _, _, _, p in packs]
    probs = [_k1_problem(xb, c[0], c[1], d) for c, (xb, _, _, _), d in zip(cases, packs, devs)]
    lib.svdq_quantize_act_grouped(probs, rank)
    G.check_ok()
    for c, (xb, x, _, p), d, q in zip(cases, packs, devs, probs):
        m, k = c[0], c[1]
        oc, osf, ou = svdquant.quantize_act(x, p["inv_lambda"], p["l1"], p["s_a"], p["s_w"])
        gc, gsf, gu = G.unpack_act(q["a_bundle"], q["U"], m, k)
        np.testing.assert_array_equal(gc, oc)
        np.testing.assert_array_equal(gsf, osf)
        assert L.bundle_padding_is_zero(G.u8(q["a_bundle"]), m, k, 128)
        if rank:
            G.parity(f"grouped K1 U, M={m} K={k}", L.bf16_bits_to_f64(gu[:, :rank]), ou, TOL)
        b1, u1 = G.run_k1(xb, m, k, rank, d)
        assert torch.equal(b1, q["a_bundle"]) and torch.equal(u1, q["U"])


def _k2_problem(oc, osf, ou, d, bias_bits, m, n, k, begin):
    Y = G.poisoned_bf16(m, n)
    return dict(a_bundle=G.dev(L.bundle_pack(oc, osf, m, k, 128)), U=G.dev(L.lowrank_pack(L.bf16_bits(ou), 128)),
                s_a=d["s_a"], w_bundle=d["w_bundle"], l2t=d["l2t"], s_w=d["s_w"],
                bias=G.bf16_dev(bias_bits), M=m, N=n, K=k, gelu_col_begin=begin, Y=Y)


# (m, k, n, seed, gelu_col_begin): ragged M, N and K; different K per problem
K2_GROUP = [(200, 320, 136, 4, 64), (37, 1024, 520, 5, 0), (300, 512, 256, 6, 256), (513, 768, 264, 7, 100)]


@pytest.mark.parametrize("epilogue,rank", [(lib.EPILOGUE_GELU_ERF, 32), (lib.EPILOGUE_NONE, 16)])
def test_grouped_gemm_matches_oracle_and_single_calls(epilogue, rank):
    probs, want, single = [], [], []
    for m, k, n, seed, begin in K2_GROUP:
        xb, x, bb, p = _case(m, k, n, rank, seed)
        d = G.weights_dev(p, rank)
        oc, osf, ou = svdquant.quantize_act(x, p["inv_lambda"], p["l1"], p["s_a"], p["s_w"])
        ou = formats.bf16_round(ou)
        probs.append(_k2_problem(oc, osf, ou, d, bb, m, n, k, begin))
        want.append(svdquant.w4a4_linear(oc, osf, p["s_a"], p["w_codes"], p["w_sf"], p["s_w"], ou, p["l2"],
                                         formats.bf16_bits_to_float(bb), epilogue, begin))
        single.append((oc, osf, ou, d, bb, m, n, k, begin))
    lib.svdq_linear_w4a4_grouped(probs, rank, epilogue)
    G.check_ok()
    for q, w, s in zip(probs, want, single):
        G.parity(f"grouped K2 Y, M={q['M']} N={q['N']} K={q['K']}", G.bf16_host(q["Y"]), w, TOL)
        oc, osf, ou, d, bb, m, n, k, begin = s
        y1, _ = G.run_k2(oc, osf, ou, d, bb, m, n, k, rank, epilogue, begin)
        assert torch.equal(y1, q["Y"])


def test_grouped_dual_stream_projection_full_size():
    """Image (4096) and text (512) tokens of one 3072 -> 9216 projection in one K1 and one K2 launch:
    the GPU chain against the oracle on sampled rows of both streams, and against the single calls."""
    rank, k, n = 32, 3072, 9216
    wb, _ = synthetic.weight(k, n, 40, 0.02, synthetic.count(0.005, k), 8.0)
    streams = []
    for m, seed in ((4096, 41), (512, 42)):
        xb, _ = synthetic.activation(m, k, seed, synthetic.count(0.01, k), 50.0)
        streams.append((m, xb, formats.bf16_bits_to_float(xb)))
    amax = np.max(np.abs(np.concatenate([s[2] for s in streams])), axis=0).astype(np.float32)
    p = svdquant.pack(formats.bf16_bits_to_float(wb), amax, rank)
    d = G.weights_dev(p, rank)
    bb = synthetic.bias(n, 43)
    k1p = [_k1_problem(xb, m, k, d) for m, xb, _ in streams]
    lib.svdq_quantize_act_grouped(k1p, rank)
    k2p = [dict(a_bundle=q["a_bundle"], U=q["U"], s_a=d["s_a"], w_bundle=d["w_bundle"], l2t=d["l2t"], s_w=d["s_w"],
                bias=G.bf16_dev(bb), M=m, N=n, K=k, gelu_col_begin=0, Y=G.poisoned_bf16(m, n))
           for q, (m, _, _) in zip(k1p, streams)]
    lib.svdq_linear_w4a4_grouped(k2p, rank, lib.EPILOGUE_NONE)
    G.check_ok()
    rng = np.random.default_rng(44)
    for (m, xb, x), q1, q2 in zip(streams, k1p, k2p):
        rows = np.sort(rng.choice(m, 24, replace=False))
        oc, osf, ou = svdquant.quantize_act(x[rows], p["inv_lambda"], p["l1"], p["s_a"], p["s_w"])
        gc, gsf, gu = G.unpack_act(q1["a_bundle"], q1["U"], m, k)
        np.testing.assert_array_equal(gc[rows], oc)
        np.testing.assert_array_equal(gsf[rows], osf)
        G.parity(f"dual-stream U, M={m}", L.bf16_bits_to_f64(gu[rows, :rank]), ou, TOL)
        # Y on the GPU's own operands against the oracle on the same (bit-identical) operands
        ub = L.bf16_bits_to_f64(gu[rows, :rank])
        want = svdquant.w4a4_linear(oc, osf, p["s_a"], p["w_codes"], p["w_sf"], p["s_w"], ub, p["l2"],
                                    formats.bf16_bits_to_float(bb), lib.EPILOGUE_NONE, 0)
        G.parity(f"dual-stream Y, M={m}", G.bf16_host(q2["Y"])[rows], want, TOL)
        b1, u1 = G.run_k1(xb, m, k, rank, d)
        assert torch.equal(b1, q1["a_bundle"]) and torch.equal(u1, q1["U"])
        y1 = G.poisoned_bf16(m, n)
        lib.svdq_linear_w4a4(b1, u1, d["s_a"], d["w_bundle"], d["l2t"], d["s_w"], G.bf16_dev(bb), m, n, k, rank,
                             lib.EPILOGUE_NONE, 0, y1)
        G.check_ok()
        assert torch.equal(y1, q2["Y"])


def test_grouped_calls_reject_bad_lists():
    xb, x, bb, p = _case(64, 256, 64, 16, 9)
    d = G.weights_dev(p, 16)
    good = _k1_problem(xb, 64, 256, d)
    with pytest.raises(lib.SvdqError) as e:
        lib.svdq_quantize_act_grouped([good] * (lib.MAX_GROUP + 1), 16)
    assert e.value.status == lib.ERR_INVALID_ARG
    with pytest.raises(lib.SvdqError) as e:
        lib.svdq_quantize_act_grouped([], 16)
    assert e.value.status == lib.ERR_INVALID_ARG
