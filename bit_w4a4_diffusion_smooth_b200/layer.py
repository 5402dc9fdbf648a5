"""User-facing layers on top of the C ABI: SVDQLinear (W4A4 + low-rank branch)
and AWQLinear (W4A16).  They hold the packed weights on the GPU and reuse
activation buffers per row count; all arithmetic runs in the library.
"""
import numpy as np
import torch

from . import lib


def _dev(a, device, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(device)


class SVDQLinear:
    """Y = (X^ L1) L2 + Q(X^) Q(R) + b  (one SVDQuant linear layer).

    Build with `from_weight` (offline host pack of a bf16 weight [K, N] and
    calibration maxima) or `from_packed` (a dict from lib.svdq_pack_weights).
    """

    def __init__(self, packed, K, N, rank, bias_bits=None, epilogue=lib.EPILOGUE_NONE, gelu_col_begin=0,
                 device="cuda"):
        self.K, self.N, self.rank = K, N, rank
        self.epilogue, self.gelu_col_begin = epilogue, gelu_col_begin
        self.device = torch.device(device)
        lib.svdq_init(self.device.index or 0)
        self.inv_lambda = _dev(packed["inv_lambda"], device)
        self.l1t = _dev(packed["l1t"], device, torch.bfloat16) if rank else None
        self.l2t = _dev(packed["l2t"], device)
        self.w_bundle = _dev(packed["w_bundle"], device)
        self.s_w = _dev(np.asarray(packed["s_w"], np.float32).reshape(1), device)
        self.s_a = _dev(np.asarray(packed["s_a"], np.float32).reshape(1), device)
        self.bias = _dev(bias_bits, device, torch.bfloat16) if bias_bits is not None else None
        self._bufs = {}

    @classmethod
    def from_weight(cls, W_bits, act_absmax, rank, bias_bits=None, epilogue=lib.EPILOGUE_NONE,
                    gelu_col_begin=0, device="cuda", seed=0):
        K, N = W_bits.shape
        packed = lib.svdq_pack_weights(W_bits, act_absmax, rank, seed=seed)
        return cls(packed, K, N, rank, bias_bits, epilogue, gelu_col_begin, device)

    def buffers(self, M):
        """Activation-side buffers for M rows (allocated once per M)."""
        if M not in self._bufs:
            sz = lib.svdq_act_sizes(M, self.K)
            self._bufs[M] = dict(
                a_bundle=torch.empty(sz["a_bundle"], dtype=torch.uint8, device=self.device),
                U=torch.empty(sz["u"], dtype=torch.uint8, device=self.device))
        return self._bufs[M]

    def quantize(self, X, stream=None):
        b = self.buffers(X.shape[0])
        lib.svdq_quantize_act(X, self.inv_lambda, self.l1t, self.rank, self.s_a, self.s_w,
                              b["a_bundle"], b["U"], stream=stream)
        return b

    def gemm(self, b, M, Y, stream=None):
        lib.svdq_linear_w4a4(b["a_bundle"], b["U"], self.s_a, self.w_bundle, self.l2t, self.s_w, self.bias,
                             M, self.N, self.K, self.rank, self.epilogue, self.gelu_col_begin, Y, stream=stream)
        return Y

    def __call__(self, X, Y=None, stream=None):
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.N), dtype=torch.bfloat16, device=self.device)
        return self.gemm(self.quantize(X, stream), M, Y, stream)


class AWQLinear:
    """Y = (X diag(inv_awq)) deq(W_a) + b with 4-bit group-64 weights (any M; blocks of 16 rows)."""

    def __init__(self, packed, K, N, bias_bits=None, device="cuda"):
        self.K, self.N = K, N
        self.device = torch.device(device)
        lib.svdq_init(self.device.index or 0)
        self.qweight = _dev(packed["qweight"], device)
        self.scales = _dev(packed["scales"], device, torch.bfloat16)
        self.zeros = _dev(packed["zeros"], device, torch.bfloat16)
        self.inv_awq = _dev(packed["inv_awq"], device)
        self.bias = _dev(bias_bits, device, torch.bfloat16) if bias_bits is not None else None

    @classmethod
    def from_weight(cls, W_bits, awq_scale, bias_bits=None, device="cuda"):
        K, N = W_bits.shape
        return cls(lib.awq_pack_weights(W_bits, awq_scale), K, N, bias_bits, device)

    def __call__(self, X, Y=None, stream=None):
        if Y is None:
            Y = torch.empty((X.shape[0], self.N), dtype=torch.bfloat16, device=self.device)
        lib.awq_linear_w4a16(X, self.inv_awq, self.qweight, self.scales, self.zeros, self.bias, self.N, Y,
                             stream=stream)
        return Y
