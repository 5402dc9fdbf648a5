"""GPU parity at full size on the layer shapes of one denoising step of a
12B-class DiT that the QKV / MLP tests do not already cover:

  single.qkv_mlp  4608 x 3072 -> 21504, GELU on columns 9216.. only
  single.out      4608 x 15360 -> 3072   (K1 at K = 15360)
  dual.img.out    4096 x 3072 -> 3072
  dual.txt        512-row text stream: qkv 3072 -> 9216, out 3072 -> 3072,
                  fc1 3072 -> 12288 (+GELU) then fc2 12288 -> 3072 on fc1's output

(the image-stream qkv / fc1 / fc2 at 4096 rows are the 4608-row shapes of the
QKV and MLP tests with two fewer 256-row tile rows).

Each layer runs in the launch configuration the benchmark uses: K1 on every
row, whose codes and scales must equal the oracle's bit for bit on every row;
K2 on the oracle's own quantized operands (identical on both sides), and the
GPU's own K1 -> K2 chain, both compared with the oracle's layer on sampled
rows.  fc2's input is the oracle's fc1 output rounded to bf16 (its smoothing
and static activation scale are calibrated on it); nothing the GPU computes is
fed to the oracle.
"""
import functools

import numpy as np
import pytest

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import formats, svdquant
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu
TOL = 1e-2
RANK = 32
SEED = 4            # the DiT-step workload's seed


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def _rows(m, count, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(m, size=min(m, count) - 4, replace=False).tolist()) | {0, 1, m - 2, m - 1}
    return np.array(sorted(rows))


@functools.lru_cache(maxsize=None)
def _weight_and_bias(k, n, stream):
    wb, _ = synthetic.weight(k, n, SEED, 0.02, synthetic.count(0.005, k), 8.0, stream=stream)
    return wb, synthetic.bias(n, SEED, stream=stream + 1)


def _layer(name, xb, k, n, stream, epilogue=lib.EPILOGUE_NONE, begin=0, sample=128):
    """Packs the layer with the oracle (calibrated on xb), runs K1 and K2 on the GPU and checks
    them against the oracle.  Returns the oracle's layer output (float64) on every row."""
    m = xb.shape[0]
    x = formats.bf16_bits_to_float(xb)
    wb, bb = _weight_and_bias(k, n, stream)
    p = svdquant.pack(formats.bf16_bits_to_float(wb), np.max(np.abs(x), axis=0).astype(np.float32), RANK)
    d = G.weights_dev(p, RANK)
    bias = formats.bf16_bits_to_float(bb)

    # K1 on every row; codes and scales bit-exact on every row
    bundle, U = G.run_k1(xb, m, k, RANK, d)
    oc, osf, ou = svdquant.quantize_act(x, p["inv_lambda"], p["l1"], p["s_a"], p["s_w"])
    gc, gsf, gu = G.unpack_act(bundle, U, m, k)
    np.testing.assert_array_equal(gc, oc)
    np.testing.assert_array_equal(gsf, osf)
    assert L.bundle_padding_is_zero(G.u8(bundle), m, k, 128)
    G.parity(f"{name} U", L.bf16_bits_to_f64(gu[:, :RANK]), ou, TOL)

    # K2 on the oracle's operands, and the GPU's own chain, against the oracle's layer on sampled rows
    rows = _rows(m, sample, seed=k + n)
    ou16 = formats.bf16_round(ou)
    want = svdquant.w4a4_linear(oc[rows], osf[rows], p["s_a"], p["w_codes"], p["w_sf"], p["s_w"], ou16[rows],
                                p["l2"], bias, epilogue, begin)
    Y, _ = G.run_k2(oc, osf, ou16, d, bb, m, n, k, RANK, epilogue, begin)
    G.parity(f"{name} Y on oracle operands", G.bf16_host(Y)[rows], want, TOL)
    Y2 = G.poisoned_bf16(m, n)
    lib.svdq_linear_w4a4(bundle, U, d["s_a"], d["w_bundle"], d["l2t"], d["s_w"], G.bf16_dev(bb), m, n, k, RANK,
                         epilogue, begin, Y2)
    G.check_ok()
    G.parity(f"{name} Y of the GPU's K1 -> K2 chain", G.bf16_host(Y2)[rows], want, TOL)
    return svdquant.w4a4_linear(oc, osf, p["s_a"], p["w_codes"], p["w_sf"], p["s_w"], ou16, p["l2"], bias,
                                epilogue, begin) if epilogue != lib.EPILOGUE_NONE else None


def _activation(m, k, stream):
    xb, _ = synthetic.activation(m, k, SEED, synthetic.count(0.01, k), 50.0, stream=stream)
    return xb


def test_single_stream_fused_qkv_mlp():
    """single.qkv_mlp: 4608 x 3072 -> 21504, GELU (erf) on the 12288 MLP columns only."""
    _layer("single.qkv_mlp", _activation(4608, 3072, 0), 3072, 21504, stream=4,
           epilogue=lib.EPILOGUE_GELU_ERF, begin=9216)


def test_single_stream_out():
    """single.out: 4608 x 15360 -> 3072 (the attention output and the MLP activation side by side)."""
    _layer("single.out", _activation(4608, 15360, 1), 15360, 3072, stream=6)


def test_image_stream_out():
    """dual.img.out: 4096 x 3072 -> 3072."""
    _layer("dual.img.out", _activation(4096, 3072, 2), 3072, 3072, stream=4)


def test_text_stream_chain():
    """dual.txt at 512 rows: qkv, out, and fc1 (+GELU) -> fc2 on fc1's output."""
    xb = _activation(512, 3072, 3)
    _layer("dual.txt.qkv", xb, 3072, 9216, stream=4, sample=512)
    _layer("dual.txt.out", xb, 3072, 3072, stream=6, sample=512)
    h = _layer("dual.txt.fc1", xb, 3072, 12288, stream=4, epilogue=lib.EPILOGUE_GELU_ERF, sample=512)
    hb = L.bf16_bits(formats.bf16_round(h))
    _layer("dual.txt.fc2", hb, 12288, 3072, stream=6, sample=512)
