"""GPU parity past 32-bit byte offsets.

An activation of 66,048 x 16,384 bf16 is 2.16 GB: rows 65,536 and beyond start past 2^31 bytes of
X, so every offset the kernels form from a row index must be 64-bit.  The layer runs through the C
ABI in both forms, K1 then the GEMM (N = 256, rank 32): the NVFP4 layer and its INT4 variant.
The rows repeat a seeded 2,048-row base (row r is base row r mod 2048), so the oracle needs only
the base; sampled rows on both sides of 2^31 bytes are compared with the oracle's layer on their
base rows (the GPU's own K1 -> GEMM chain against the oracle's quantization and product).
"""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from oracle import formats, int4, svdquant
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu
M, K, N, RANK, BASE = 66048, 16384, 256, 32, 2048
TOL = 1e-2
ROWS = np.array([0, 1, 2047, 2048, 40000, 65535, 65536, 65537, 66000, M - 1])


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


@pytest.fixture(scope="module")
def inputs():
    xb, _ = synthetic.activation(BASE, K, 123, synthetic.count(0.01, K), 50.0)
    wb, _ = synthetic.weight(K, N, 123, 0.02, synthetic.count(0.005, K), 8.0)
    x = formats.bf16_bits_to_float(xb)
    amax = np.max(np.abs(x), axis=0).astype(np.float32)            # the base's maxima are the tiled X's
    X = G.bf16_dev(xb).repeat(M // BASE + 1, 1)[:M].contiguous()    # row r = base row r % BASE
    assert X.numel() * 2 > 2 ** 31 and ROWS[-1] * K * 2 >= 2 ** 31
    return x, formats.bf16_bits_to_float(wb), amax, X, synthetic.bias(N, 124)


def _rows_of(Y):
    return G.bf16_host(Y[torch.as_tensor(ROWS, device=G.DEV)])


def test_nvfp4_chain_past_2gb(inputs):
    x, w, amax, X, bb = inputs
    p = svdquant.pack(w, amax, RANK)
    d = G.weights_dev(p, RANK)
    sz = lib.svdq_act_sizes(M, K)
    bundle = torch.empty(sz["a_bundle"], dtype=torch.uint8, device=G.DEV)
    U = torch.empty(sz["u"], dtype=torch.uint8, device=G.DEV)
    lib.svdq_quantize_act(X, d["inv_lambda"], d["l1t"], RANK, d["s_a"], d["s_w"], bundle, U)
    Y = G.poisoned_bf16(M, N)
    lib.svdq_linear_w4a4(bundle, U, d["s_a"], d["w_bundle"], d["l2t"], d["s_w"], G.bf16_dev(bb), M, N, K, RANK,
                         lib.EPILOGUE_NONE, 0, Y)
    G.check_ok()
    base = ROWS % BASE
    oc, osf, ou = svdquant.quantize_act(x[base], p["inv_lambda"], p["l1"], p["s_a"], p["s_w"])
    want = svdquant.w4a4_linear(oc, osf, p["s_a"], p["w_codes"], p["w_sf"], p["s_w"], formats.bf16_round(ou),
                                p["l2"], formats.bf16_bits_to_float(bb), lib.EPILOGUE_NONE, 0)
    G.parity("NVFP4 chain, rows past 2^31 bytes", _rows_of(Y), want, TOL)


def test_int4_chain_past_2gb(inputs):
    x, w, amax, X, bb = inputs
    p = int4.pack(w, amax, RANK)
    asz = lib.svdq_int4_act_sizes(M, K)
    codes = torch.empty(asz["codes"], dtype=torch.uint8, device=G.DEV)
    scales = torch.empty(asz["scales"], dtype=torch.uint8, device=G.DEV)
    U = torch.empty(lib.svdq_act_sizes(M, K)["u"], dtype=torch.uint8, device=G.DEV)
    lib.svdq_quantize_act_int4(X, G.dev(np.asarray(p["inv_lambda"], np.float32)),
                               G.bf16_dev(L.bf16_bits(p["l1"].T)), RANK, codes, scales, U)
    Y = G.poisoned_bf16(M, N)
    lib.svdq_linear_int4(codes, scales, U, G.dev(L.int4_pack(p["qw"])), G.dev(L.int4_scales_pack(p["sw"], N)),
                         G.dev(L.lowrank_pack(L.bf16_bits(p["l2"].T), 256)), G.bf16_dev(bb), M, N, K, RANK,
                         lib.EPILOGUE_NONE, 0, Y)
    G.check_ok()
    base = ROWS % BASE
    qa, sa, u = int4.quantize_act(x[base], p["inv_lambda"], p["l1"])
    want = int4.int4_linear(qa, sa, p["qw"], p["sw"], formats.bf16_round(u), p["l2"],
                            formats.bf16_bits_to_float(bb), svdquant.EPILOGUE_NONE, 0)
    G.parity("INT4 chain, rows past 2^31 bytes", _rows_of(Y), want, TOL)
