"""ctypes binding of libsvdq_b200.so: the same entry points as include/svdq.h.

Argument marshalling only: every computation happens inside the library (its
CUDA kernels, or its host pack code).  Device arguments are torch CUDA
tensors (torch supplies device memory and streams); host arguments are numpy
arrays.  A missing library raises immediately: there is no fallback path.
"""
import ctypes
import functools
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq_b200.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_SHAPE = 2
ERR_ALIGNMENT = 3
ERR_UNSUPPORTED_DEVICE = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_NOT_INITIALIZED = 7

EPILOGUE_NONE = 0
EPILOGUE_GELU_ERF = 1
EPILOGUE_GELU_TANH = 2
LR_STRIDE = 64
AMAX_WORKSPACE_BYTES = 256
MAX_GROUP = 4

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.POINTER(ctypes.c_size_t)
class QuantProblem(ctypes.Structure):
    """svdq_quant_problem of include/svdq.h."""
    _fields_ = [("X", ctypes.c_void_p), ("M", ctypes.c_int), ("K", ctypes.c_int), ("ldx", ctypes.c_int),
                ("inv_lambda", ctypes.c_void_p), ("l1t", ctypes.c_void_p), ("s_a", ctypes.c_void_p),
                ("s_w", ctypes.c_void_p), ("a_bundle", ctypes.c_void_p), ("U", ctypes.c_void_p)]


class W4A4Problem(ctypes.Structure):
    """svdq_w4a4_problem of include/svdq.h."""
    _fields_ = [("a_bundle", ctypes.c_void_p), ("U", ctypes.c_void_p), ("s_a", ctypes.c_void_p),
                ("w_bundle", ctypes.c_void_p), ("l2t", ctypes.c_void_p), ("s_w", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("M", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int),
                ("gelu_col_begin", ctypes.c_int), ("Y", ctypes.c_void_p), ("ldy", ctypes.c_int)]


class AwqProblem(ctypes.Structure):
    """awq_problem of include/svdq.h."""
    _fields_ = [("X", ctypes.c_void_p), ("ldx", ctypes.c_int), ("inv_awq", ctypes.c_void_p),
                ("qweight", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("N", ctypes.c_int), ("Y", ctypes.c_void_p), ("ldy", ctypes.c_int)]


AWQ_MAX_GROUP = 128

_SIGNATURES = {
    "svdq_version": (_I, []),
    "svdq_last_error_string": (ctypes.c_char_p, []),
    "svdq_status_string": (ctypes.c_char_p, [_I]),
    "svdq_init": (_I, [_I]),
    "svdq_weight_sizes": (_I, [_I, _I, _I, _SZ, _SZ, _SZ, _SZ]),
    "svdq_act_sizes": (_I, [_I, _I, _SZ, _SZ]),
    "svdq_pack_weights": (_I, [_P, _I, _I, _P, _I, _I, ctypes.c_uint64, _P, _P, _P, _P, _P, _P, _P]),
    "svdq_quantize_host": (_I, [_P, _I, _I, ctypes.c_float, _I, _P]),
    "svdq_int4_weight_sizes": (_I, [_I, _I, _SZ, _SZ]),
    "svdq_int4_act_sizes": (_I, [_I, _I, _SZ, _SZ]),
    "svdq_quantize_int4_host": (_I, [_P, _I, _I, _I, _P, _P]),
    "svdq_quantize_act_int4": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P]),
    "svdq_linear_int4": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P]),
    "svdq_quantize_act": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P]),
    "svdq_linear_w4a4": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P]),
    "svdq_quantize_act_grouped": (_I, [ctypes.POINTER(QuantProblem), _I, _I, _P]),
    "svdq_linear_w4a4_grouped": (_I, [ctypes.POINTER(W4A4Problem), _I, _I, _I, _P]),
    "svdq_linear_w4a4_requant": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I,
                                      _P, _P, _I, _P, _P, _P, _P, _P, _P]),
    "svdq_requant_workspace_size": (_I, [_I, _I, _SZ]),
    "svdq_linear_w4a4_requant_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I,
                                              _P, _P, _I, _P, _P, _P, _P, _P]),
    "svdq_act_amax": (_I, [_P, _I, _I, _I, _P, _P, _P, _P]),
    "svdq_calibrate_absmax": (_I, [_P, _I, _I, _I, _P, _P]),
    "svdq_pack_device_workspace_size": (_I, [_I, _I, _I, _SZ]),
    "svdq_pack_weights_device": (_I, [_P, _I, _I, _P, _I, ctypes.c_uint64, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "awq_packed_sizes": (_I, [_I, _I, _I, _SZ, _SZ, _SZ, _SZ]),
    "awq_pack_weights": (_I, [_P, _I, _I, _P, _I, _P, _P, _P, _P]),
    "awq_linear_w4a16": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _P, _I, _P, _I, _P]),
    "awq_linear_w4a16_grouped": (_I, [ctypes.POINTER(AwqProblem), _I, _I, _I, _I, _P]),
    "awq_gemm_workspace_size": (_I, [_I, _I, _I, _SZ]),
    "awq_linear_w4a16_gemm": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _P, _I, _P, _I, _P, _P]),
    "awq_expand_weights": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "awq_linear_w4a16_expanded": (_I, [_P, _I, _I, _I, _P, _I, _P, _I, _P, _P]),
    "svdq_check_status": (_I, [_P]),
    "svdq_debug_wait_timeout": (_I, [ctypes.c_uint64, _P]),
    "svdq_debug_convert": (_I, [_P, _I, _P, _P, _P]),
    "svdq_debug_gelu": (_I, [_P, _I, _I, _P, _P]),
}
EXPORTS = tuple(_SIGNATURES)


class SvdqError(RuntimeError):
    def __init__(self, name, status, text):
        self.status = status
        super().__init__(f"{name}: {status_name(status)}: {text}")


def load():
    """Loads the library once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bit_w4a4_diffusion_smooth_b200.build_lib`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_name(status):
    return load().svdq_status_string(int(status)).decode()


def _check(name, rc):
    if rc != OK:
        raise SvdqError(name, rc, load().svdq_last_error_string().decode())


# ---------------------------------------------------------------- marshalling

def _dptr(t, name, dtype=None, allow_none=False):
    """Device pointer of a CUDA tensor (checked: on a GPU, contiguous rows)."""
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if t.dim() >= 1 and t.stride(-1) != 1:
        raise ValueError(f"{name} must have unit stride in its last dimension")
    return ctypes.c_void_p(t.data_ptr())


def _nbytes(t):
    return t.numel() * t.element_size()


def _need_bytes(t, nbytes, name):
    """Raises unless device buffer `t` holds at least `nbytes` bytes (checked before any call, so a
    short buffer is never handed to a kernel)."""
    if t is not None and _nbytes(t) < nbytes:
        raise ValueError(f"{name} holds {_nbytes(t)} bytes; {nbytes} are needed")


def _need_2d(t, rows, cols, name):
    if t.dim() != 2 or t.shape[0] < rows or t.shape[1] < cols:
        raise ValueError(f"{name} must be 2-D with at least {rows} rows and {cols} columns, got {tuple(t.shape)}")


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _hptr(a, dtype, name):
    if not isinstance(a, np.ndarray) or a.dtype != dtype or not a.flags.c_contiguous:
        raise ValueError(f"{name} must be a C-contiguous numpy array of {np.dtype(dtype).name}")
    return ctypes.c_void_p(a.ctypes.data)


# ---------------------------------------------------------------- entry points

def svdq_version():
    return load().svdq_version()


def svdq_init(device=0):
    _check("svdq_init", load().svdq_init(int(device)))


@functools.lru_cache(maxsize=1024)
def _weight_sizes(K, N, rank):
    s = [ctypes.c_size_t() for _ in range(4)]
    _check("svdq_weight_sizes", load().svdq_weight_sizes(K, N, rank, *[ctypes.byref(x) for x in s]))
    return tuple(x.value for x in s)


@functools.lru_cache(maxsize=1024)
def _act_sizes(M, K):
    s = [ctypes.c_size_t() for _ in range(2)]
    _check("svdq_act_sizes", load().svdq_act_sizes(M, K, *[ctypes.byref(x) for x in s]))
    return tuple(x.value for x in s)


def svdq_weight_sizes(K, N, rank):
    """Byte sizes of a packed layer's buffers (the library's answer, cached per shape: the
    per-call argument checks of the device calls ask it every time)."""
    return dict(zip(("inv_lambda", "l1t", "l2t", "w_bundle"), _weight_sizes(K, N, rank)))


def svdq_act_sizes(M, K):
    """Byte sizes of an activation's bundle and U (cached per shape, like svdq_weight_sizes)."""
    return dict(zip(("a_bundle", "u"), _act_sizes(M, K)))


def svdq_pack_weights(W_bits, act_absmax, rank, num_threads=0, seed=0, want_residual=False):
    """Host pack.  W_bits: uint16 [K, N] bf16 patterns; act_absmax: float32 [K].

    Returns numpy arrays: inv_lambda [K] f32, l1t [rank, K] u16 (bf16), l2t
    (256-row low-rank tiles, u8), w_bundle (256-row NVFP4 bundle, u8), s_w, s_a
    (float32 scalars), and residual [K, N] f32 if asked.
    """
    K, N = W_bits.shape
    sz = svdq_weight_sizes(K, N, rank)
    out = dict(
        inv_lambda=np.zeros(K, np.float32),
        l1t=np.zeros((rank, K), np.uint16),
        l2t=np.zeros(sz["l2t"], np.uint8),
        w_bundle=np.zeros(sz["w_bundle"], np.uint8),
        s_w=np.zeros(1, np.float32),
        s_a=np.zeros(1, np.float32),
    )
    residual = np.zeros((K, N), np.float32) if want_residual else None
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    act_absmax = np.ascontiguousarray(act_absmax, dtype=np.float32)
    rc = load().svdq_pack_weights(
        _hptr(W_bits, np.uint16, "W"), K, N, _hptr(act_absmax, np.float32, "act_absmax"), rank,
        num_threads, seed, _hptr(out["inv_lambda"], np.float32, "inv_lambda"),
        _hptr(out["l1t"], np.uint16, "l1t") if rank else None, _hptr(out["l2t"], np.uint8, "l2t"),
        _hptr(out["w_bundle"], np.uint8, "w_bundle"),
        _hptr(out["s_w"], np.float32, "s_w"), _hptr(out["s_a"], np.float32, "s_a"),
        _hptr(residual, np.float32, "residual") if want_residual else None)
    _check("svdq_pack_weights", rc)
    if want_residual:
        out["residual"] = residual
    return out


def svdq_int4_weight_sizes(K, N):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check("svdq_int4_weight_sizes", load().svdq_int4_weight_sizes(K, N, ctypes.byref(a), ctypes.byref(b)))
    return dict(codes=a.value, scales=b.value)


def svdq_int4_act_sizes(M, K):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check("svdq_int4_act_sizes", load().svdq_int4_act_sizes(M, K, ctypes.byref(a), ctypes.byref(b)))
    return dict(codes=a.value, scales=b.value)


def svdq_quantize_int4_host(T, ld_s=None):
    """INT4 groups of 64 of float32 rows T [rows, K] (host): codes u8 [rows, K/2], scales u16 (bf16)
    [K/64, ld_s]."""
    T = np.ascontiguousarray(T, dtype=np.float32)
    rows, K = T.shape
    ld_s = rows if ld_s is None else ld_s
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((max(K // 64, 1), max(ld_s, 1)), np.uint16)
    _check("svdq_quantize_int4_host", load().svdq_quantize_int4_host(
        _hptr(T, np.float32, "T"), rows, K, ld_s, _hptr(codes, np.uint8, "codes"),
        _hptr(scales, np.uint16, "scales")))
    return codes, scales


def svdq_pack_weights_int4(W_bits, act_absmax, rank, num_threads=0, seed=0):
    """Host pack of the INT4 layer: svdq_pack_weights' smoothing, low-rank branch and residual, the
    residual in INT4 groups along K per output column.  Returns inv_lambda, l1t, l2t (as
    svdq_pack_weights), w_codes u8 [N, K/2], w_scales u16 (bf16) [K/64, N] and the residual."""
    p = svdq_pack_weights(W_bits, act_absmax, rank, num_threads, seed, want_residual=True)
    codes, scales = svdq_quantize_int4_host(np.ascontiguousarray(p["residual"].T))
    return dict(inv_lambda=p["inv_lambda"], l1t=p["l1t"], l2t=p["l2t"], w_codes=codes, w_scales=scales,
                residual=p["residual"])


def svdq_quantize_act_int4(X, inv_lambda, l1t, rank, a_codes, a_scales, U, M=None, K=None, stream=None):
    """Enqueues the INT4 activation kernel.  X: bf16 CUDA [M, ldx]."""
    import torch
    M = X.shape[0] if M is None else M
    K = X.shape[1] if K is None else K
    _need_2d(X, M, K, "X")
    sz = svdq_int4_act_sizes(M, K)
    _need_bytes(a_codes, sz["codes"], "a_codes")
    _need_bytes(a_scales, sz["scales"], "a_scales")
    _need_bytes(U, _act_sizes(M, K)[1], "U")
    _need_bytes(inv_lambda, 4 * K, "inv_lambda")
    if rank:
        _need_bytes(l1t, 2 * rank * K, "l1t")
    _check("svdq_quantize_act_int4", load().svdq_quantize_act_int4(
        _dptr(X, "X", torch.bfloat16), M, K, X.stride(0), _dptr(inv_lambda, "inv_lambda", torch.float32),
        _dptr(l1t, "l1t", allow_none=rank == 0), rank, _dptr(a_codes, "a_codes", torch.uint8),
        _dptr(a_scales, "a_scales"), _dptr(U, "U"), _stream(stream)))


def svdq_linear_int4(a_codes, a_scales, U, w_codes, w_scales, l2t, bias, M, N, K, rank, epilogue, gelu_col_begin, Y,
                     stream=None):
    """Enqueues the INT4 GEMM.  Y: bf16 CUDA [M, ldy]."""
    import torch
    asz, wsz = svdq_int4_act_sizes(M, K), svdq_int4_weight_sizes(K, N)
    _need_bytes(a_codes, asz["codes"], "a_codes")
    _need_bytes(a_scales, asz["scales"], "a_scales")
    _need_bytes(w_codes, wsz["codes"], "w_codes")
    _need_bytes(w_scales, wsz["scales"], "w_scales")
    if rank:
        _need_bytes(U, _act_sizes(M, K)[1], "U")
        _need_bytes(l2t, _weight_sizes(K, N, rank)[2], "l2t")
    _need_bytes(bias, 2 * N, "bias")
    _need_2d(Y, M, N, "Y")
    _check("svdq_linear_int4", load().svdq_linear_int4(
        _dptr(a_codes, "a_codes", torch.uint8), _dptr(a_scales, "a_scales"), _dptr(U, "U", allow_none=rank == 0),
        _dptr(w_codes, "w_codes", torch.uint8), _dptr(w_scales, "w_scales"),
        _dptr(l2t, "l2t", allow_none=rank == 0), _dptr(bias, "bias", allow_none=True), M, N, K, rank, epilogue,
        gelu_col_begin, _dptr(Y, "Y", torch.bfloat16), Y.stride(0), _stream(stream)))


def svdq_quantize_host(T, s_t, tile_rows=128):
    """Host NVFP4 of float32 rows T [rows, K] into a bundle of the given tile height (u8)."""
    T = np.ascontiguousarray(T, dtype=np.float32)
    rows, K = T.shape
    ks = (K + 255) // 256
    tile_bytes = tile_rows * (144 if tile_rows == 128 else 192)
    bundle = np.zeros(((rows + tile_rows - 1) // tile_rows) * ks * tile_bytes, np.uint8)
    _check("svdq_quantize_host", load().svdq_quantize_host(
        _hptr(T, np.float32, "T"), rows, K, ctypes.c_float(float(s_t)), tile_rows,
        _hptr(bundle, np.uint8, "bundle")))
    return bundle


def _quant_problem(X, inv_lambda, l1t, rank, s_a, s_w, a_bundle, U, M=None, K=None):
    """Checks one activation problem's buffers and returns its QuantProblem."""
    import torch
    M = X.shape[0] if M is None else M
    K = X.shape[1] if K is None else K
    _need_2d(X, M, K, "X")
    sz = svdq_act_sizes(M, K)
    _need_bytes(a_bundle, sz["a_bundle"], "a_bundle")
    _need_bytes(U, sz["u"], "U")
    _need_bytes(inv_lambda, 4 * K, "inv_lambda")
    if rank:
        _need_bytes(l1t, 2 * rank * K, "l1t")
    _need_bytes(s_a, 4, "s_a")
    _need_bytes(s_w, 4, "s_w")
    return QuantProblem(_dptr(X, "X", torch.bfloat16), M, K, X.stride(0), _dptr(inv_lambda, "inv_lambda", torch.float32),
                        _dptr(l1t, "l1t", allow_none=rank == 0), _dptr(s_a, "s_a", torch.float32),
                        _dptr(s_w, "s_w", torch.float32), _dptr(a_bundle, "a_bundle", torch.uint8), _dptr(U, "U"))


def svdq_quantize_act(X, inv_lambda, l1t, rank, s_a, s_w, a_bundle, U, M=None, K=None, stream=None):
    """Enqueues the activation kernel.  X: bf16 CUDA [M, ldx] (row stride ldx)."""
    q = _quant_problem(X, inv_lambda, l1t, rank, s_a, s_w, a_bundle, U, M, K)
    _check("svdq_quantize_act", load().svdq_quantize_act(
        q.X, q.M, q.K, q.ldx, q.inv_lambda, q.l1t, rank, q.s_a, q.s_w, q.a_bundle, q.U, _stream(stream)))


def svdq_quantize_act_grouped(problems, rank, stream=None):
    """One launch of the activation kernel over several problems (dicts of svdq_quantize_act's
    keyword arguments X, inv_lambda, l1t, s_a, s_w, a_bundle, U and optionally M, K)."""
    arr = (QuantProblem * len(problems))(*[_quant_problem(rank=rank, **d) for d in problems])
    _check("svdq_quantize_act_grouped", load().svdq_quantize_act_grouped(arr, len(problems), rank, _stream(stream)))


def _w4a4_problem(a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, gelu_col_begin, Y):
    """Checks one GEMM problem's buffers and returns its W4A4Problem."""
    import torch
    asz = svdq_act_sizes(M, K)
    wsz = svdq_weight_sizes(K, N, rank)
    _need_bytes(a_bundle, asz["a_bundle"], "a_bundle")
    _need_bytes(w_bundle, wsz["w_bundle"], "w_bundle")
    if rank:
        _need_bytes(U, asz["u"], "U")
        _need_bytes(l2t, wsz["l2t"], "l2t")
    _need_bytes(bias, 2 * N, "bias")
    _need_bytes(s_a, 4, "s_a")
    _need_bytes(s_w, 4, "s_w")
    _need_2d(Y, M, N, "Y")
    return W4A4Problem(_dptr(a_bundle, "a_bundle", torch.uint8), _dptr(U, "U", allow_none=rank == 0),
                       _dptr(s_a, "s_a", torch.float32), _dptr(w_bundle, "w_bundle", torch.uint8),
                       _dptr(l2t, "l2t", allow_none=rank == 0), _dptr(s_w, "s_w", torch.float32),
                       _dptr(bias, "bias", allow_none=True), M, N, K, gelu_col_begin,
                       _dptr(Y, "Y", torch.bfloat16), Y.stride(0))


def svdq_linear_w4a4(a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, epilogue, gelu_col_begin, Y,
                     stream=None):
    """Enqueues the W4A4 GEMM.  Y: bf16 CUDA [M, ldy]."""
    q = _w4a4_problem(a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, gelu_col_begin, Y)
    _check("svdq_linear_w4a4", load().svdq_linear_w4a4(
        q.a_bundle, q.U, q.s_a, q.w_bundle, q.l2t, q.s_w, q.bias, M, N, K, rank, epilogue, gelu_col_begin, q.Y,
        q.ldy, _stream(stream)))


def svdq_linear_w4a4_grouped(problems, rank, epilogue, stream=None):
    """One launch of the W4A4 GEMM over several problems (dicts of svdq_linear_w4a4's keyword
    arguments a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, gelu_col_begin, Y)."""
    arr = (W4A4Problem * len(problems))(*[_w4a4_problem(rank=rank, **d) for d in problems])
    _check("svdq_linear_w4a4_grouped", load().svdq_linear_w4a4_grouped(arr, len(problems), rank, epilogue,
                                                                       _stream(stream)))


def svdq_act_amax(X, inv_lambda, workspace, s_a, M=None, K=None, stream=None):
    """Enqueues the dynamic activation-scale pass: s_a (f32 CUDA, 1 element) = f32(max |X^|) / 2688."""
    import torch
    M = X.shape[0] if M is None else M
    K = X.shape[1] if K is None else K
    _need_2d(X, M, K, "X")
    _need_bytes(inv_lambda, 4 * K, "inv_lambda")
    _need_bytes(workspace, AMAX_WORKSPACE_BYTES, "workspace")
    _need_bytes(s_a, 4, "s_a")
    _check("svdq_act_amax", load().svdq_act_amax(
        _dptr(X, "X", torch.bfloat16), M, K, X.stride(0), _dptr(inv_lambda, "inv_lambda", torch.float32),
        _dptr(workspace, "workspace"), _dptr(s_a, "s_a", torch.float32), _stream(stream)))


def svdq_calibrate_absmax(X, act_absmax, M=None, K=None, stream=None):
    """act_absmax (f32 CUDA [K]) = max(act_absmax, max over rows of |X|) for a bf16 CUDA X [M, ldx]."""
    import torch
    M = X.shape[0] if M is None else M
    K = X.shape[1] if K is None else K
    _need_2d(X, M, K, "X")
    _need_bytes(act_absmax, 4 * K, "act_absmax")
    _check("svdq_calibrate_absmax", load().svdq_calibrate_absmax(
        _dptr(X, "X", torch.bfloat16), M, K, X.stride(0), _dptr(act_absmax, "act_absmax", torch.float32),
        _stream(stream)))


def svdq_pack_device_workspace_size(K, N, rank):
    n = ctypes.c_size_t()
    _check("svdq_pack_device_workspace_size", load().svdq_pack_device_workspace_size(K, N, rank, ctypes.byref(n)))
    return n.value


def svdq_pack_weights_device(W, act_absmax, rank, seed=0, want_residual=False, stream=None):
    """GPU pack of a bf16 CUDA weight W [K, N] with calibration maxima act_absmax (f32 CUDA [K]).

    Returns CUDA tensors: inv_lambda [K] f32, l1t [rank, K] bf16, l2t (u8 tiles), w_bundle (u8),
    s_w, s_a ([1] f32), and residual [K, N] f32 if asked.
    """
    import torch
    K, N = W.shape
    dev = W.device
    sz = svdq_weight_sizes(K, N, rank)
    out = dict(inv_lambda=torch.empty(K, dtype=torch.float32, device=dev),
               l1t=torch.empty((rank, K), dtype=torch.bfloat16, device=dev),
               l2t=torch.empty(sz["l2t"], dtype=torch.uint8, device=dev),
               w_bundle=torch.empty(sz["w_bundle"], dtype=torch.uint8, device=dev),
               s_w=torch.empty(1, dtype=torch.float32, device=dev), s_a=torch.empty(1, dtype=torch.float32, device=dev))
    residual = torch.empty((K, N), dtype=torch.float32, device=dev) if want_residual else None
    ws = torch.empty(svdq_pack_device_workspace_size(K, N, rank), dtype=torch.uint8, device=dev)
    _need_2d(W, K, N, "W")
    _need_bytes(act_absmax, 4 * K, "act_absmax")
    _check("svdq_pack_weights_device", load().svdq_pack_weights_device(
        _dptr(W, "W", torch.bfloat16), K, N, _dptr(act_absmax, "act_absmax", torch.float32), rank, seed,
        _dptr(out["inv_lambda"], "inv_lambda"), _dptr(out["l1t"], "l1t") if rank else None,
        _dptr(out["l2t"], "l2t"), _dptr(out["w_bundle"], "w_bundle"), _dptr(out["s_w"], "s_w"),
        _dptr(out["s_a"], "s_a"), _dptr(residual, "residual", allow_none=True), _dptr(ws, "workspace"),
        _stream(stream)))
    if want_residual:
        out["residual"] = residual
    return out


def awq_packed_sizes(K, N, group=64):
    s = [ctypes.c_size_t() for _ in range(4)]
    _check("awq_packed_sizes", load().awq_packed_sizes(K, N, group, *[ctypes.byref(x) for x in s]))
    return dict(zip(("qweight", "scales", "zeros", "inv_awq"), (x.value for x in s)))


def svdq_requant_workspace_size(M, next_rank):
    n = ctypes.c_size_t()
    _check("svdq_requant_workspace_size", load().svdq_requant_workspace_size(M, next_rank, ctypes.byref(n)))
    return n.value


def svdq_linear_w4a4_requant(a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, epilogue, gelu_col_begin,
                             Y, next_inv_lambda, next_l1t, next_rank, next_s_a, next_s_w, next_a_bundle, next_U,
                             workspace, stream=None):
    """Enqueues the W4A4 GEMM that re-quantizes its output for the next SVDQ layer (K_next = N).
    Y: bf16 CUDA [M, ldy] or None (no bf16 output)."""
    import torch
    asz = svdq_act_sizes(M, K)
    wsz = svdq_weight_sizes(K, N, rank)
    nsz = svdq_act_sizes(M, N)
    _need_bytes(a_bundle, asz["a_bundle"], "a_bundle")
    _need_bytes(w_bundle, wsz["w_bundle"], "w_bundle")
    if rank:
        _need_bytes(U, asz["u"], "U")
        _need_bytes(l2t, wsz["l2t"], "l2t")
    _need_bytes(bias, 2 * N, "bias")
    _need_bytes(s_a, 4, "s_a")
    _need_bytes(s_w, 4, "s_w")
    if Y is not None:
        _need_2d(Y, M, N, "Y")
    _need_bytes(next_inv_lambda, 4 * N, "next_inv_lambda")
    _need_bytes(next_s_a, 4, "next_s_a")
    _need_bytes(next_s_w, 4, "next_s_w")
    _need_bytes(next_a_bundle, nsz["a_bundle"], "next_a_bundle")
    if next_rank:
        _need_bytes(next_l1t, 2 * next_rank * N, "next_l1t")
        _need_bytes(next_U, nsz["u"], "next_U")
        _need_bytes(workspace, svdq_requant_workspace_size(M, next_rank), "workspace")
    _check("svdq_linear_w4a4_requant", load().svdq_linear_w4a4_requant(
        _dptr(a_bundle, "a_bundle", torch.uint8), _dptr(U, "U", allow_none=rank == 0),
        _dptr(s_a, "s_a", torch.float32), _dptr(w_bundle, "w_bundle", torch.uint8),
        _dptr(l2t, "l2t", allow_none=rank == 0), _dptr(s_w, "s_w", torch.float32),
        _dptr(bias, "bias", allow_none=True), M, N, K, rank, epilogue, gelu_col_begin,
        _dptr(Y, "Y", torch.bfloat16, allow_none=True), Y.stride(0) if Y is not None else N,
        _dptr(next_inv_lambda, "next_inv_lambda", torch.float32),
        _dptr(next_l1t, "next_l1t", allow_none=next_rank == 0), next_rank,
        _dptr(next_s_a, "next_s_a", torch.float32), _dptr(next_s_w, "next_s_w", torch.float32),
        _dptr(next_a_bundle, "next_a_bundle", torch.uint8), _dptr(next_U, "next_U", allow_none=next_rank == 0),
        _dptr(workspace, "workspace", torch.float32, allow_none=next_rank == 0), _stream(stream)))


def svdq_linear_w4a4_requant_noalloc(a_bundle, U, s_a, w_bundle, l2t, s_w, bias, M, N, K, rank, epilogue,
                                     gelu_col_begin, Y, next_inv_lambda, next_l1t, next_rank, next_s_a, next_s_w,
                                     next_a_bundle, next_U, stream=None):
    """svdq_linear_w4a4_requant for callers that cannot allocate: the partial sums use the library's
    fixed device array (M * next_rank <= 262144), so no workspace is passed."""
    import torch
    asz = svdq_act_sizes(M, K)
    wsz = svdq_weight_sizes(K, N, rank)
    nsz = svdq_act_sizes(M, N)
    _need_bytes(a_bundle, asz["a_bundle"], "a_bundle")
    _need_bytes(w_bundle, wsz["w_bundle"], "w_bundle")
    if rank:
        _need_bytes(U, asz["u"], "U")
        _need_bytes(l2t, wsz["l2t"], "l2t")
    _need_bytes(bias, 2 * N, "bias")
    if Y is not None:
        _need_2d(Y, M, N, "Y")
    _need_bytes(next_inv_lambda, 4 * N, "next_inv_lambda")
    _need_bytes(next_a_bundle, nsz["a_bundle"], "next_a_bundle")
    if next_rank:
        _need_bytes(next_l1t, 2 * next_rank * N, "next_l1t")
        _need_bytes(next_U, nsz["u"], "next_U")
    _check("svdq_linear_w4a4_requant_noalloc", load().svdq_linear_w4a4_requant_noalloc(
        _dptr(a_bundle, "a_bundle", torch.uint8), _dptr(U, "U", allow_none=rank == 0),
        _dptr(s_a, "s_a", torch.float32), _dptr(w_bundle, "w_bundle", torch.uint8),
        _dptr(l2t, "l2t", allow_none=rank == 0), _dptr(s_w, "s_w", torch.float32),
        _dptr(bias, "bias", allow_none=True), M, N, K, rank, epilogue, gelu_col_begin,
        _dptr(Y, "Y", torch.bfloat16, allow_none=True), Y.stride(0) if Y is not None else N,
        _dptr(next_inv_lambda, "next_inv_lambda", torch.float32),
        _dptr(next_l1t, "next_l1t", allow_none=next_rank == 0), next_rank,
        _dptr(next_s_a, "next_s_a", torch.float32), _dptr(next_s_w, "next_s_w", torch.float32),
        _dptr(next_a_bundle, "next_a_bundle", torch.uint8), _dptr(next_U, "next_U", allow_none=next_rank == 0),
        _stream(stream)))


def awq_pack_weights(W_bits, awq_scale, group=64):
    """Host AWQ pack: returns qweight (u32, fragment order), scales, zeros (u16 [N/64, K/g, 64]), inv_awq."""
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    awq_scale = np.ascontiguousarray(awq_scale, dtype=np.float32)
    K, N = W_bits.shape
    gshape = (N // 64, K // group, 64) if N % 64 == 0 and K % group == 0 else (N, max(K // group, 1))
    out = dict(qweight=np.zeros(N * K // 8, np.uint32), scales=np.zeros(gshape, np.uint16),
               zeros=np.zeros(gshape, np.uint16), inv_awq=np.zeros(K, np.float32))
    _check("awq_pack_weights", load().awq_pack_weights(
        _hptr(W_bits, np.uint16, "W"), K, N, _hptr(awq_scale, np.float32, "awq_scale"), group,
        _hptr(out["qweight"], np.uint32, "qweight"), _hptr(out["scales"], np.uint16, "scales"),
        _hptr(out["zeros"], np.uint16, "zeros"), _hptr(out["inv_awq"], np.float32, "inv_awq")))
    return out


def awq_linear_w4a16(X, inv_awq, qweight, scales, zeros, bias, N, Y, group=64, M=None, K=None, stream=None):
    """Enqueues the W4A16 GEMV.  X: bf16 CUDA [M, ldx]; Y: bf16 CUDA [M, ldy]."""
    import torch
    M = X.shape[0] if M is None else M
    K = X.shape[1] if K is None else K
    _need_2d(X, M, K, "X")
    _need_2d(Y, M, N, "Y")
    _need_bytes(qweight, N * K // 2, "qweight")
    _need_bytes(scales, 2 * N * (K // group), "scales")
    _need_bytes(zeros, 2 * N * (K // group), "zeros")
    _need_bytes(inv_awq, 4 * K, "inv_awq")
    _need_bytes(bias, 2 * N, "bias")
    _check("awq_linear_w4a16", load().awq_linear_w4a16(
        _dptr(X, "X", torch.bfloat16), M, K, X.stride(0), _dptr(inv_awq, "inv_awq", allow_none=True),
        _dptr(qweight, "qweight"), _dptr(scales, "scales"), _dptr(zeros, "zeros"), group,
        _dptr(bias, "bias", allow_none=True), N, _dptr(Y, "Y", torch.bfloat16), Y.stride(0),
        _stream(stream)))



def awq_linear_w4a16_grouped(problems, M, K, group=64, stream=None):
    """One launch of the W4A16 GEMV over several projections of the same M and K (dicts of
    awq_linear_w4a16's arguments X, inv_awq, qweight, scales, zeros, bias, N, Y); outputs are
    bit-identical to separate calls."""
    import torch
    if not 1 <= len(problems) <= AWQ_MAX_GROUP:
        raise ValueError(f"a grouped AWQ launch takes 1..{AWQ_MAX_GROUP} problems, got {len(problems)}")
    arr = (AwqProblem * len(problems))()
    for i, d in enumerate(problems):
        X, Y, N = d["X"], d["Y"], d["N"]
        _need_2d(X, M, K, "X")
        _need_2d(Y, M, N, "Y")
        _need_bytes(d["qweight"], N * K // 2, "qweight")
        _need_bytes(d["scales"], 2 * N * (K // group), "scales")
        _need_bytes(d["zeros"], 2 * N * (K // group), "zeros")
        _need_bytes(d.get("inv_awq"), 4 * K, "inv_awq")
        _need_bytes(d.get("bias"), 2 * N, "bias")
        arr[i] = AwqProblem(_dptr(X, "X", torch.bfloat16), X.stride(0), _dptr(d.get("inv_awq"), "inv_awq", allow_none=True),
                            _dptr(d["qweight"], "qweight"), _dptr(d["scales"], "scales"), _dptr(d["zeros"], "zeros"),
                            _dptr(d.get("bias"), "bias", allow_none=True), N, _dptr(Y, "Y", torch.bfloat16),
                            Y.stride(0))
    _check("awq_linear_w4a16_grouped", load().awq_linear_w4a16_grouped(arr, len(problems), M, K, group,
                                                                       _stream(stream)))

def awq_gemm_workspace_size(M, K, N):
    n = ctypes.c_size_t()
    _check("awq_gemm_workspace_size", load().awq_gemm_workspace_size(M, K, N, ctypes.byref(n)))
    return n.value


def awq_linear_w4a16_gemm(X, inv_awq, qweight, scales, zeros, bias, N, Y, workspace, group=64, M=None, K=None,
                          stream=None):
    """Enqueues the many-row W4A16 path (weights expanded into `workspace`, then one bf16 GEMM)."""
    import torch
    M = X.shape[0] if M is None else M
    K = X.shape[1] if K is None else K
    _need_2d(X, M, K, "X")
    _need_2d(Y, M, N, "Y")
    _need_bytes(qweight, N * K // 2, "qweight")
    _need_bytes(scales, 2 * N * (K // group), "scales")
    _need_bytes(zeros, 2 * N * (K // group), "zeros")
    _need_bytes(inv_awq, 4 * K, "inv_awq")
    _need_bytes(bias, 2 * N, "bias")
    _need_bytes(workspace, awq_gemm_workspace_size(M, K, N), "workspace")
    _check("awq_linear_w4a16_gemm", load().awq_linear_w4a16_gemm(
        _dptr(X, "X", torch.bfloat16), M, K, X.stride(0), _dptr(inv_awq, "inv_awq"),
        _dptr(qweight, "qweight"), _dptr(scales, "scales"), _dptr(zeros, "zeros"), group,
        _dptr(bias, "bias", allow_none=True), N, _dptr(Y, "Y", torch.bfloat16), Y.stride(0),
        _dptr(workspace, "workspace"), _stream(stream)))


def awq_expand_weights(inv_awq, qweight, scales, zeros, K, N, workspace, group=64, stream=None):
    """Writes the layer's expanded weights into the first 4 K N bytes of `workspace`."""
    _need_bytes(qweight, N * K // 2, "qweight")
    _need_bytes(scales, 2 * N * (K // group), "scales")
    _need_bytes(zeros, 2 * N * (K // group), "zeros")
    _need_bytes(inv_awq, 4 * K, "inv_awq")
    _need_bytes(workspace, 4 * K * N, "workspace")
    _check("awq_expand_weights", load().awq_expand_weights(
        _dptr(inv_awq, "inv_awq"), _dptr(qweight, "qweight"), _dptr(scales, "scales"), _dptr(zeros, "zeros"),
        K, N, group, _dptr(workspace, "workspace"), _stream(stream)))


def awq_linear_w4a16_expanded(X, bias, N, Y, workspace, M=None, K=None, stream=None):
    """The GEMM half of the many-row path, on the expansion already in `workspace`."""
    import torch
    M = X.shape[0] if M is None else M
    K = X.shape[1] if K is None else K
    _need_2d(X, M, K, "X")
    _need_2d(Y, M, N, "Y")
    _need_bytes(bias, 2 * N, "bias")
    _need_bytes(workspace, awq_gemm_workspace_size(M, K, N), "workspace")
    _check("awq_linear_w4a16_expanded", load().awq_linear_w4a16_expanded(
        _dptr(X, "X", torch.bfloat16), M, K, X.stride(0), _dptr(bias, "bias", allow_none=True), N,
        _dptr(Y, "Y", torch.bfloat16), Y.stride(0), _dptr(workspace, "workspace"), _stream(stream)))


def svdq_check_status(stream=None):
    """Synchronizes `stream`, returns the status code and clears it (no raise)."""
    return load().svdq_check_status(_stream(stream))


def svdq_debug_wait_timeout(limit_ns, stream=None):
    _check("svdq_debug_wait_timeout", load().svdq_debug_wait_timeout(int(limit_ns), _stream(stream)))


def svdq_debug_convert(x, e2m1_out, e4m3_out, stream=None):
    import torch
    _check("svdq_debug_convert", load().svdq_debug_convert(
        _dptr(x, "x", torch.float32), x.numel(), _dptr(e2m1_out, "e2m1_out", torch.uint8),
        _dptr(e4m3_out, "e4m3_out", torch.uint8), _stream(stream)))


def svdq_debug_gelu(x, kind, out, stream=None):
    """out = GELU(x) through the epilogue's device function (x, out: float32 CUDA)."""
    import torch
    _check("svdq_debug_gelu", load().svdq_debug_gelu(
        _dptr(x, "x", torch.float32), x.numel(), int(kind), _dptr(out, "out", torch.float32), _stream(stream)))
