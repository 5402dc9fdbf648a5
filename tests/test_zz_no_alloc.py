"""The allocation-free re-quantizing GEMM (svdq_linear_w4a4_requant_noalloc)
against the entry point that takes a caller workspace.

Callers that cannot allocate device memory (an engine plugin handed only a
layer's tensors, code that must not call cudaMalloc mid-pipeline) use the
variant whose scratch is a fixed array inside the library.  Two calls in a
row, with different shapes, must each give what svdq_linear_w4a4_requant
gives on the same inputs: the next layer's codes and block scales bit for bit,
its low-rank input within the parity tolerance (fp32 sums added in a
different order).  A size beyond the fixed array is refused before anything is
launched.  This file runs last in the suite and passes alone as well.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib, synthetic
from tests import gpu_util as G
from tests import layouts as L

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def _layer(m, k, n, rank, next_rank, seed):
    """fc1's operands (library pack + K1 on the GPU) and the next layer's weights (library pack)."""
    xb, _ = synthetic.activation(m, k, seed, synthetic.count(0.01, k), 50.0)
    wb, _ = synthetic.weight(k, n, seed, 0.02, synthetic.count(0.005, k), 8.0)
    w2, _ = synthetic.weight(n, 64, seed + 1, 0.02)
    amax = np.max(np.abs(synthetic.bf16_bits_to_f32(xb)), axis=0).astype(np.float32)
    p1 = lib.svdq_pack_weights(wb, amax, rank, seed=seed)
    p2 = lib.svdq_pack_weights(w2, np.full(n, 3.0, np.float32), next_rank, seed=seed)
    d1 = {key: G.dev(v) for key, v in p1.items() if key != "l1t"}
    d2 = {key: G.dev(v) for key, v in p2.items() if key != "l1t"}
    d1["l1t"] = G.bf16_dev(p1["l1t"]) if rank else None
    d2["l1t"] = G.bf16_dev(p2["l1t"]) if next_rank else None
    sz = lib.svdq_act_sizes(m, k)
    a = torch.empty(sz["a_bundle"], dtype=torch.uint8, device=G.DEV)
    u = torch.empty(sz["u"], dtype=torch.uint8, device=G.DEV)
    lib.svdq_quantize_act(G.bf16_dev(xb), d1["inv_lambda"], d1["l1t"], rank, d1["s_a"], d1["s_w"], a, u)
    bias = G.bf16_dev(synthetic.bias(n, seed))
    return d1, d2, a, u, bias


def _run(noalloc, m, k, n, rank, next_rank, ops):
    d1, d2, a, u, bias = ops
    nsz = lib.svdq_act_sizes(m, n)
    nb = G.poisoned_u8(nsz["a_bundle"])
    nu = G.poisoned_u8(nsz["u"])
    args = (a, u, d1["s_a"], d1["w_bundle"], d1["l2t"], d1["s_w"], bias, m, n, k, rank, lib.EPILOGUE_GELU_ERF, 0, None,
            d2["inv_lambda"], d2["l1t"], next_rank, d2["s_a"], d2["s_w"], nb, nu if next_rank else None)
    if noalloc:
        lib.svdq_linear_w4a4_requant_noalloc(*args)
    else:
        ws = torch.empty(max(1, lib.svdq_requant_workspace_size(m, next_rank) // 4), dtype=torch.float32,
                         device=G.DEV)
        lib.svdq_linear_w4a4_requant(*args, ws if next_rank else None)
    G.check_ok()
    return G.u8(nb), G.u8(nu)


@pytest.mark.parametrize("calls", [[(4608, 3072, 1024, 32, 32), (300, 512, 384, 16, 64)]])
def test_noalloc_matches_workspace_entry_point_on_two_calls(calls):
    for i, (m, k, n, rank, next_rank) in enumerate(calls):
        ops = _layer(m, k, n, rank, next_rank, seed=20 + i)
        ref_b, ref_u = _run(False, m, k, n, rank, next_rank, ops)
        got_b, got_u = _run(True, m, k, n, rank, next_rank, ops)
        np.testing.assert_array_equal(got_b, ref_b)              # codes and block scales, padding included
        gu = L.lowrank_unpack(got_u, (m + 127) // 128 * 128, 128)
        ru = L.lowrank_unpack(ref_u, (m + 127) // 128 * 128, 128)
        assert (gu[:, next_rank:] == 0).all() and (gu[m:] == 0).all()
        G.parity(f"call {i + 1}: next U, fixed scratch vs workspace", L.bf16_bits_to_f64(gu[:m, :next_rank]),
                 L.bf16_bits_to_f64(ru[:m, :next_rank]), TOL)


def test_noalloc_refuses_sizes_beyond_its_array():
    ops = _layer(8192, 256, 256, 16, 64, seed=30)             # 8192 x 64 > 262144 floats
    with pytest.raises(lib.SvdqError) as e:
        _run(True, 8192, 256, 256, 16, 64, ops)
    assert e.value.status == lib.ERR_SHAPE
    assert "262144" in str(e.value)
