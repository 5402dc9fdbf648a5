"""GPU parity of the AWQ W4A16 projection (K3) against the oracle, through the
C ABI.  The weights are the oracle's AWQ pack, put in the library's fragment
layout by the test-side writer; bar: the largest error in a row beyond the
rounding to the bf16 output, over the RMS of the oracle's row, <= 1e-2
(gpu_util.excess_error)."""
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


def _run(m, k, n, seed, with_bias=True, use_inv=True):
    xb, _ = synthetic.activation(m, k, seed)
    wb, _ = synthetic.weight(k, n, seed, 0.02)
    a = synthetic.awq_scales(k, seed) if use_inv else np.ones(k, np.float32)
    bb = synthetic.bias(n, seed)
    p = oawq.pack(formats.bf16_bits_to_float(wb), a)
    Y = G.poisoned_bf16(m, n)
    lib.awq_linear_w4a16(G.bf16_dev(xb), G.dev(p["inv_a"]) if use_inv else None, G.dev(L.awq_pack(p["q"])),
                         G.bf16_dev(L.bf16_bits(L.awq_group_pack(p["s"]))), G.bf16_dev(L.bf16_bits(L.awq_group_pack(p["z"]))),
                         G.bf16_dev(bb) if with_bias else None, n, Y)
    G.check_ok()
    x = formats.bf16_bits_to_float(xb)
    want = oawq.linear(x, p["inv_a"], p["q"], p["s"], p["z"], formats.bf16_bits_to_float(bb) if with_bias else None)
    return G.parity(f"{m}x{k}->{n}", G.bf16_host(Y), want)[0]


@pytest.mark.parametrize("m,k,n", [
    # ring kernel (M <= 8): one stage per quad, partial last stage, several stages per quad,
    # groups past K, more 64-column quads than SMs, 2-3 ring stages when X^ is large
    (1, 64, 64), (2, 192, 128), (5, 1024, 320), (8, 512, 64), (2, 2048, 128), (4, 4096, 192),
    (2, 6144, 64), (7, 1600, 256), (8, 1024, 12800), (8, 12288, 128),
    # direct kernel (M > 8), and blocks of 16 rows beyond 16 (a full and a ragged last block)
    (9, 256, 192), (16, 3072, 512), (12, 4096, 128), (32, 1024, 256), (45, 3072, 192)])
def test_awq_parity(m, k, n):
    assert _run(m, k, n, seed=m + k + n) <= 1e-2


def test_awq_without_bias_and_scales():
    assert _run(4, 256, 64, 21, with_bias=False, use_inv=False) <= 1e-2


def test_awq_full_size_adaln():
    """The modulation workload: 2 x 3072 -> 18432 (6 x 3072 adaLN outputs)."""
    c = synthetic.AWQ
    assert _run(c.m, c.k, c.n, c.seed) <= 1e-2


def test_awq_layer_from_host_pack():
    """The user-facing layer (library host pack + K3) against the oracle."""
    from bit_w4a4_diffusion_smooth_b200.layer import AWQLinear
    xb, wb, bb, a = synthetic.AwqCase("awq small", 2, 512, 256, seed=5).make()
    layer = AWQLinear.from_weight(wb, a, bb)
    y = G.bf16_host(layer(G.bf16_dev(xb)))
    p = oawq.pack(formats.bf16_bits_to_float(wb), a)
    want = oawq.linear(formats.bf16_bits_to_float(xb), p["inv_a"], p["q"], p["s"], p["z"],
                       formats.bf16_bits_to_float(bb))
    G.parity("layer", y, want)


def _bits(t):
    """The bf16 output's bit patterns."""
    return t.view(torch.int16).cpu().numpy()


def _problem(xb_dev, k, n, seed, with_bias, use_inv):
    """One AWQ projection of the shared input: its device operands, output and oracle pack."""
    wb, _ = synthetic.weight(k, n, seed, 0.02)
    a = synthetic.awq_scales(k, seed) if use_inv else np.ones(k, np.float32)
    bb = synthetic.bias(n, seed) if with_bias else None
    p = oawq.pack(formats.bf16_bits_to_float(wb), a)
    d = dict(X=xb_dev, inv_awq=G.dev(p["inv_a"]) if use_inv else None, qweight=G.dev(L.awq_pack(p["q"])),
             scales=G.bf16_dev(L.bf16_bits(L.awq_group_pack(p["s"]))),
             zeros=G.bf16_dev(L.bf16_bits(L.awq_group_pack(p["z"]))),
             bias=G.bf16_dev(bb) if with_bias else None, N=n, Y=G.poisoned_bf16(xb_dev.shape[0], n))
    return d, p, bb


@pytest.mark.parametrize("m,k,widths", [
    (2, 3072, (18432, 9216, 18432)),            # a DiT step's modulation projections: one input, mixed widths
    (3, 1024, (64, 320, 128, 64, 256)),         # ragged quad counts, binary search over five problems
    (11, 512, (192, 64)),                       # the 16-row-block kernel
])
def test_awq_grouped_matches_separate_calls_and_oracle(m, k, widths):
    """One grouped launch over several projections of the same input: every output bit-identical to
    its own awq_linear_w4a16 call, and within the parity bar of the oracle."""
    xb, _ = synthetic.activation(m, k, 31 + m)
    X = G.bf16_dev(xb)
    probs = [_problem(X, k, n, 40 + i, with_bias=i % 2 == 0, use_inv=i != 1) for i, n in enumerate(widths)]
    lib.awq_linear_w4a16_grouped([d for d, _, _ in probs], m, k)
    G.check_ok()
    x = formats.bf16_bits_to_float(xb)
    for i, (d, p, bb) in enumerate(probs):
        Ys = G.poisoned_bf16(m, d["N"])
        lib.awq_linear_w4a16(d["X"], d["inv_awq"], d["qweight"], d["scales"], d["zeros"], d["bias"], d["N"], Ys)
        G.check_ok()
        np.testing.assert_array_equal(_bits(d["Y"]), _bits(Ys))
        want = oawq.linear(x, p["inv_a"], p["q"], p["s"], p["z"],
                           formats.bf16_bits_to_float(bb) if bb is not None else None)
        G.parity(f"grouped AWQ {m}x{k}->{d['N']} (problem {i})", G.bf16_host(d["Y"]), want)


def test_awq_grouped_full_step_of_modulations():
    """All 76 modulation projections of a 12B-class DiT step (38 of 3072 -> 18432, 38 of 3072 -> 9216,
    one shared 2-row input) in one launch: sampled problems bit-identical to their own calls."""
    m, k = 2, 3072
    xb, _ = synthetic.activation(m, k, 77)
    X = G.bf16_dev(xb)
    base = [_problem(X, k, n, 90 + j, with_bias=True, use_inv=True) for j, n in enumerate((18432, 9216))]
    probs = []
    for i in range(76):                           # the two packs' weights, each problem its own output
        d, _, _ = base[i % 2]
        probs.append(dict(d, Y=G.poisoned_bf16(m, d["N"])))
    lib.awq_linear_w4a16_grouped(probs, m, k)
    G.check_ok()
    for i in (0, 1, 37, 74, 75):
        d = probs[i]
        Ys = G.poisoned_bf16(m, d["N"])
        lib.awq_linear_w4a16(d["X"], d["inv_awq"], d["qweight"], d["scales"], d["zeros"], d["bias"], d["N"], Ys)
        G.check_ok()
        np.testing.assert_array_equal(_bits(d["Y"]), _bits(Ys))
