"""The C-ABI library on the CPU: it loads, exports every declared entry point,
and its host-side argument checks and size queries behave (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_w4a4_diffusion_smooth_b200 import lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src, flags=re.M)))


def test_library_loads_and_exports_every_declared_symbol():
    so = lib.load()
    declared = _declared_functions()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(so, name), name
    assert set(lib.EXPORTS) == set(declared)
    assert lib.svdq_version() == 10000


def test_status_strings():
    assert lib.status_name(0) == "SVDQ_OK"
    assert lib.status_name(lib.ERR_TIMEOUT) == "SVDQ_ERR_TIMEOUT"
    assert lib.status_name(99) == "SVDQ_ERR_UNKNOWN"


def test_sizes():
    s = lib.svdq_weight_sizes(3072, 9216, 32)
    assert s["w_bundle"] == 9216 * 1536 + 9216 * 192 * 4   # codes + 4 copies of the scales, 256-row tiles fit exactly
    assert s["l1t"] == 32 * 3072 * 2 and s["l2t"] == 9216 * 64 * 2
    a = lib.svdq_act_sizes(200, 320)
    assert a["a_bundle"] == 2 * 2 * 128 * 144                # rows padded to 256, K to 512
    assert a["u"] == 256 * 128
    with pytest.raises(lib.SvdqError) as e:
        lib.svdq_weight_sizes(100, 256, 16)
    assert e.value.status == lib.ERR_SHAPE
    with pytest.raises(lib.SvdqError) as e:
        lib.svdq_weight_sizes(256, 256, 24)
    assert e.value.status == lib.ERR_SHAPE


def test_device_calls_reject_bad_arguments_before_touching_a_gpu():
    so = lib.load()
    null = ctypes.c_void_p(0)
    rc = so.svdq_quantize_act(null, 64, 256, 256, null, null, 16, null, null, null, null, null)
    assert rc == lib.ERR_INVALID_ARG
    p = ctypes.c_void_p(16)  # never dereferenced: the shape check fails first
    rc = so.svdq_linear_w4a4(p, p, p, p, p, p, None, 64, 256, 100, 16, 0, 0, p, 256, None)
    assert rc == lib.ERR_SHAPE
    assert b"K % 64" in so.svdq_last_error_string()
    rc = so.svdq_linear_w4a4(p, p, p, p, p, p, None, 64, 256, 256, 16, 7, 0, p, 256, None)
    assert rc == lib.ERR_INVALID_ARG
    rc = so.awq_linear_w4a16(p, 17, 256, 256, None, p, p, p, 64, None, 96, p, 96, None)
    assert rc == lib.ERR_SHAPE                                    # N % 64
    rc = so.awq_linear_w4a16(p, 0, 256, 256, None, p, p, p, 64, None, 256, p, 256, None)
    assert rc == lib.ERR_SHAPE                                    # M < 1
    # the re-quantizing GEMM: N is the next layer's K (multiple of 64), next_rank in {0, 16, .., 64}
    rc = so.svdq_linear_w4a4_requant(p, p, p, p, p, p, None, 64, 200, 256, 16, 0, 0, None, 0,
                                     p, p, 16, p, p, p, p, p, None)
    assert rc == lib.ERR_SHAPE
    rc = so.svdq_linear_w4a4_requant(p, p, p, p, p, p, None, 64, 256, 256, 16, 0, 0, None, 0,
                                     p, p, 24, p, p, p, p, p, None)
    assert rc == lib.ERR_SHAPE
    rc = so.svdq_linear_w4a4_requant(p, p, p, p, p, p, None, 64, 256, 256, 16, 0, 0, None, 0,
                                     p, None, 16, p, p, p, p, p, None)
    assert rc == lib.ERR_INVALID_ARG                              # next_l1t missing with next_rank > 0
    assert lib.svdq_requant_workspace_size(4608, 32) == 4608 * 32 * 4
    # the many-row AWQ path: a workspace is required; shapes as the GEMV's
    assert so.awq_linear_w4a16_gemm(p, 100, 256, 256, p, p, p, p, 64, None, 256, p, 256, None, None) == \
        lib.ERR_INVALID_ARG
    assert so.awq_linear_w4a16_gemm(p, 100, 256, 256, p, p, p, p, 64, None, 96, p, 96, p, None) == lib.ERR_SHAPE
    assert lib.awq_gemm_workspace_size(256, 3072, 18432) == 3072 * 18432 * 4 + 256 * 18432 * 4
    # grouped calls: the list, its length and each problem are checked before anything is launched
    assert so.svdq_quantize_act_grouped(None, 1, 16, None) == lib.ERR_INVALID_ARG
    qp = (lib.QuantProblem * 2)()
    for i in range(2):
        qp[i] = lib.QuantProblem(p, 64, 256 if i == 0 else 100, 256, p, p, p, p, p, p)
    assert so.svdq_quantize_act_grouped(qp, lib.MAX_GROUP + 1, 16, None) == lib.ERR_INVALID_ARG
    assert so.svdq_quantize_act_grouped(qp, 2, 16, None) == lib.ERR_SHAPE
    assert b"problem 1" in so.svdq_last_error_string()
    wp = (lib.W4A4Problem * 1)()
    wp[0] = lib.W4A4Problem(p, p, p, p, p, p, None, 64, 256, 100, 0, p, 256)
    assert so.svdq_linear_w4a4_grouped(wp, 0, 16, 0, None) == lib.ERR_INVALID_ARG
    assert so.svdq_linear_w4a4_grouped(wp, 1, 16, 0, None) == lib.ERR_SHAPE
    assert b"problem 0" in so.svdq_last_error_string()
    assert lib.svdq_requant_workspace_size(100, 0) == 0
    rc = so.svdq_act_amax(p, 4, 96, 96, p, p, p, None)
    assert rc == lib.ERR_SHAPE                                    # K % 64
    rc = so.svdq_act_amax(p, 4, 128, 128, p, None, p, None)
    assert rc == lib.ERR_INVALID_ARG                              # no workspace
    assert lib.awq_packed_sizes(3072, 18432) == {"qweight": 3072 * 18432 // 2, "scales": 18432 * 48 * 2,
                                                 "zeros": 18432 * 48 * 2, "inv_awq": 3072 * 4}
    with pytest.raises(lib.SvdqError):
        lib.awq_packed_sizes(3072, 100)
    odd = ctypes.c_void_p(24)
    rc = so.svdq_linear_w4a4(odd, p, p, p, p, p, None, 64, 256, 256, 16, 0, 0, p, 256, None)
    assert rc == lib.ERR_ALIGNMENT
    # the INT4 variant: sizes, then the same argument rules before any device access
    assert lib.svdq_int4_weight_sizes(3072, 9216) == {"codes": 9216 * 1536, "scales": 48 * 9216 * 2}
    assert lib.svdq_int4_act_sizes(200, 320) == {"codes": 256 * 160, "scales": 5 * 256 * 2}
    with pytest.raises(lib.SvdqError) as e:
        lib.svdq_int4_weight_sizes(3072, 200)                     # N % 128
    assert e.value.status == lib.ERR_SHAPE
    assert so.svdq_quantize_act_int4(p, 64, 256, 256, p, None, 16, p, p, p, None) == lib.ERR_INVALID_ARG
    assert so.svdq_quantize_act_int4(p, 64, 200, 256, p, p, 16, p, p, p, None) == lib.ERR_SHAPE
    assert so.svdq_linear_int4(p, p, p, p, p, p, None, 64, 200, 256, 16, 0, 0, p, 256, None) == lib.ERR_SHAPE
    assert so.svdq_linear_int4(p, p, None, p, p, p, None, 64, 256, 256, 16, 0, 0, p, 256, None) == lib.ERR_INVALID_ARG
    assert so.svdq_linear_int4(p, p, p, p, p, p, None, 64, 256, 256, 16, 5, 0, p, 256, None) == lib.ERR_INVALID_ARG
    assert so.svdq_linear_int4(odd, p, p, p, p, p, None, 64, 256, 256, 16, 0, 0, p, 256, None) == lib.ERR_ALIGNMENT


def test_init_without_a_b200_is_an_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(lib.SvdqError) as e:
        lib.svdq_init(0)
    assert e.value.status in (lib.ERR_CUDA, lib.ERR_INVALID_ARG)


def test_pack_argument_checks():
    w = np.zeros((100, 64), np.uint16)
    with pytest.raises(lib.SvdqError):
        lib.svdq_pack_weights(w, np.ones(100, np.float32), 16)
    with pytest.raises(lib.SvdqError):
        lib.awq_pack_weights(np.zeros((64, 48), np.uint16), np.ones(64, np.float32))
    with pytest.raises(lib.SvdqError):
        lib.awq_pack_weights(np.zeros((64, 64), np.uint16), np.zeros(64, np.float32))


def test_empty_inputs_are_rejected_as_shapes():
    """M = 0 (an empty batch) and a zero width are shape errors of every device call and size query,
    reported before anything touches a GPU."""
    so = lib.load()
    p = ctypes.c_void_p(16)  # never dereferenced: the shape check fails first
    assert so.svdq_quantize_act(p, 0, 256, 256, p, p, 16, p, p, p, p, None) == lib.ERR_SHAPE
    assert so.svdq_linear_w4a4(p, p, p, p, p, p, None, 0, 256, 256, 16, 0, 0, p, 256, None) == lib.ERR_SHAPE
    assert so.svdq_linear_w4a4(p, p, p, p, p, p, None, 64, 0, 256, 16, 0, 0, p, 256, None) == lib.ERR_SHAPE
    assert so.svdq_quantize_act_int4(p, 0, 256, 256, p, p, 16, p, p, p, None) == lib.ERR_SHAPE
    assert so.svdq_linear_int4(p, p, p, p, p, p, None, 0, 256, 256, 16, 0, 0, p, 256, None) == lib.ERR_SHAPE
    for call in (lambda: lib.svdq_act_sizes(0, 256), lambda: lib.svdq_int4_act_sizes(0, 256),
                 lambda: lib.svdq_weight_sizes(256, 0, 16), lambda: lib.svdq_int4_weight_sizes(256, 0)):
        with pytest.raises(lib.SvdqError) as e:
            call()
        assert e.value.status == lib.ERR_SHAPE


def test_grouped_awq_rejects_bad_groups_before_touching_a_gpu():
    so = lib.load()
    p = ctypes.c_void_p(16)  # never dereferenced
    arr = (lib.AwqProblem * 2)()
    arr[0] = lib.AwqProblem(p, 256, None, p, p, p, None, 128, p, 128)
    arr[1] = lib.AwqProblem(p, 256, None, p, p, p, None, 96, p, 96)      # N % 64
    assert so.awq_linear_w4a16_grouped(arr, 0, 2, 256, 64, None) == lib.ERR_INVALID_ARG
    assert so.awq_linear_w4a16_grouped(arr, lib.AWQ_MAX_GROUP + 1, 2, 256, 64, None) == lib.ERR_INVALID_ARG
    assert so.awq_linear_w4a16_grouped(arr, 2, 2, 256, 64, None) == lib.ERR_SHAPE
    assert so.awq_linear_w4a16_grouped(arr, 1, 2, 256, 32, None) == lib.ERR_SHAPE   # group 32
    assert so.awq_linear_w4a16_grouped(arr, 1, 0, 256, 64, None) == lib.ERR_SHAPE   # M = 0
