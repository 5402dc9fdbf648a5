"""User-facing layers on top of the C ABI: SVDQLinear (W4A4 + low-rank branch),
SVDQLinearInt4 (its INT4 variant) and AWQLinear (W4A16).  They hold the packed weights on the GPU and reuse
activation buffers per row count; all arithmetic runs in the library.

A layer instance keeps one set of activation buffers per row count, shared by
all its calls: use an instance from one stream at a time (two calls with the
same row count that overlap on different streams would race on them).
"""
import numpy as np
import torch

from . import lib


def _resolve(device):
    """torch.device with an explicit index ('cuda' means the caller's current device)."""
    d = torch.device(device)
    if d.type != "cuda":
        raise ValueError(f"the layers run on a CUDA device, got {d}")
    return d if d.index is not None else torch.device("cuda", torch.cuda.current_device())


def _init_on(device):
    """svdq_init for `device` (it validates the GPU and makes it current), then restores the
    caller's current device."""
    prev = torch.cuda.current_device()
    try:
        lib.svdq_init(device.index)
    finally:
        torch.cuda.set_device(prev)


def _dev(a, device, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(device)


def _check_input(X, K, device, name):
    if X.dim() != 2 or X.shape[1] != K:
        raise ValueError(f"{name}: X must be [M, {K}], got {tuple(X.shape)}")
    if X.dtype != torch.bfloat16 or X.device != device:
        raise ValueError(f"{name}: X must be bf16 on {device}, got {X.dtype} on {X.device}")


def _raw_stream(stream, device):
    """The CUDA stream handle a call enqueues on: `stream`, else the caller's current stream."""
    if stream is not None:
        return stream.cuda_stream
    get = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    return get(device.index) if get is not None else torch.cuda.current_stream(device).cuda_stream


class _Plans:
    """Marshalled C-ABI arguments of a layer's calls, per set of buffers.

    The key holds every property the checked path validates (pointers, shapes, strides and
    dtypes of X and Y, and the stream), so a hit repeats a call that already passed the
    checks with the same buffers; the library then finds its tensor maps cached as well.
    Bounded: the table is cleared when it fills."""

    LIMIT = 64

    def __init__(self):
        self._t = {}

    @staticmethod
    def key(X, Y, s):
        return (X.data_ptr(), X.shape[0], X.shape[1], X.stride(0), X.stride(1), X.dtype,
                Y.data_ptr(), Y.shape[0], Y.shape[1], Y.stride(0), Y.stride(1), Y.dtype, s)

    def get(self, k):
        return self._t.get(k)

    def put(self, k, plan):
        if len(self._t) >= self.LIMIT:
            self._t.clear()
        self._t[k] = plan


def _check_output(Y, M, N, device, name):
    if tuple(Y.shape) != (M, N) or Y.dtype != torch.bfloat16 or Y.device != device:
        raise ValueError(f"{name}: Y must be bf16 [{M}, {N}] on {device}, got {Y.dtype} {tuple(Y.shape)} "
                         f"on {Y.device}")


class SVDQLinear:
    """Y = (X^ L1) L2 + Q(X^) Q(R) + b  (one SVDQuant linear layer).

    Build with `from_weight` (offline host pack of a bf16 weight [K, N] and
    calibration maxima) or with the constructor from a dict returned by
    lib.svdq_pack_weights.
    """

    def __init__(self, packed, K, N, rank, bias_bits=None, epilogue=lib.EPILOGUE_NONE, gelu_col_begin=0,
                 device="cuda"):
        self.K, self.N, self.rank = K, N, rank
        self.epilogue, self.gelu_col_begin = epilogue, gelu_col_begin
        self.device = _resolve(device)
        _init_on(self.device)
        device = self.device
        self.inv_lambda = _dev(packed["inv_lambda"], device)
        self.l1t = _dev(packed["l1t"], device, torch.bfloat16) if rank else None
        self.l2t = _dev(packed["l2t"], device)
        self.w_bundle = _dev(packed["w_bundle"], device)
        self.s_w = _dev(np.asarray(packed["s_w"], np.float32).reshape(1), device)
        self.s_a = _dev(np.asarray(packed["s_a"], np.float32).reshape(1), device)
        self.bias = _dev(bias_bits, device, torch.bfloat16) if bias_bits is not None else None
        if self.bias is not None and self.bias.numel() != N:
            raise ValueError(f"SVDQLinear: bias must have {N} elements")
        self._bufs = {}
        self._plans = _Plans()

    @classmethod
    def from_weight(cls, W_bits, act_absmax, rank, bias_bits=None, epilogue=lib.EPILOGUE_NONE,
                    gelu_col_begin=0, device="cuda", seed=0):
        K, N = W_bits.shape
        packed = lib.svdq_pack_weights(W_bits, act_absmax, rank, seed=seed)
        return cls(packed, K, N, rank, bias_bits, epilogue, gelu_col_begin, device)

    def buffers(self, M):
        """Activation-side buffers for M rows (allocated once per M, shared by every call)."""
        if M not in self._bufs:
            sz = lib.svdq_act_sizes(M, self.K)
            self._bufs[M] = dict(
                a_bundle=torch.empty(sz["a_bundle"], dtype=torch.uint8, device=self.device),
                U=torch.empty(sz["u"], dtype=torch.uint8, device=self.device))
        return self._bufs[M]

    def quantize(self, X, stream=None):
        _check_input(X, self.K, self.device, "SVDQLinear")
        b = self.buffers(X.shape[0])
        lib.svdq_quantize_act(X, self.inv_lambda, self.l1t, self.rank, self.s_a, self.s_w,
                              b["a_bundle"], b["U"], stream=stream)
        return b

    def gemm(self, b, M, Y, stream=None):
        _check_output(Y, M, self.N, self.device, "SVDQLinear")
        lib.svdq_linear_w4a4(b["a_bundle"], b["U"], self.s_a, self.w_bundle, self.l2t, self.s_w, self.bias,
                             M, self.N, self.K, self.rank, self.epilogue, self.gelu_col_begin, Y, stream=stream)
        return Y

    def __call__(self, X, Y=None, stream=None):
        _check_input(X, self.K, self.device, "SVDQLinear")
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.N), dtype=torch.bfloat16, device=self.device)
        s = _raw_stream(stream, self.device)
        key = _Plans.key(X, Y, s)
        plan = self._plans.get(key)
        if plan is None:
            # first call with these buffers: the checked wrappers, then the marshalled arguments
            self.gemm(self.quantize(X, stream), M, Y, stream)
            b = self.buffers(M)
            p = lambda t: None if t is None else t.data_ptr()
            q = (p(X), M, self.K, X.stride(0), p(self.inv_lambda), p(self.l1t), self.rank, p(self.s_a),
                 p(self.s_w), p(b["a_bundle"]), p(b["U"]), s)
            g = (p(b["a_bundle"]), p(b["U"]), p(self.s_a), p(self.w_bundle), p(self.l2t), p(self.s_w), p(self.bias),
                 M, self.N, self.K, self.rank, self.epilogue, self.gelu_col_begin, p(Y), Y.stride(0), s)
            self._plans.put(key, (q, g))
            return Y
        L = lib.load()
        lib._check("svdq_quantize_act", L.svdq_quantize_act(*plan[0]))
        lib._check("svdq_linear_w4a4", L.svdq_linear_w4a4(*plan[1]))
        return Y


class SVDQLinearInt4:
    """The INT4 W4A4 variant of SVDQLinear: the same smoothing and low-rank branch, the 4-bit
    branch in INT4 groups of 64 along K with bf16 scales (svdq_quantize_act_int4 +
    svdq_linear_int4).

    Build with `from_weight` (host pack) or from a dict returned by lib.svdq_pack_weights_int4.
    N must be a multiple of 128 (a multiple of 256 runs on the tensor cores).
    """

    def __init__(self, packed, K, N, rank, bias_bits=None, epilogue=lib.EPILOGUE_NONE, gelu_col_begin=0,
                 device="cuda"):
        self.K, self.N, self.rank = K, N, rank
        self.epilogue, self.gelu_col_begin = epilogue, gelu_col_begin
        self.device = _resolve(device)
        _init_on(self.device)
        device = self.device
        self.inv_lambda = _dev(packed["inv_lambda"], device)
        self.l1t = _dev(packed["l1t"], device, torch.bfloat16) if rank else None
        self.l2t = _dev(packed["l2t"], device)
        self.w_codes = _dev(packed["w_codes"], device)
        self.w_scales = _dev(packed["w_scales"], device)
        self.bias = _dev(bias_bits, device, torch.bfloat16) if bias_bits is not None else None
        if self.bias is not None and self.bias.numel() != N:
            raise ValueError(f"SVDQLinearInt4: bias must have {N} elements")
        self._bufs = {}

    @classmethod
    def from_weight(cls, W_bits, act_absmax, rank, bias_bits=None, epilogue=lib.EPILOGUE_NONE,
                    gelu_col_begin=0, device="cuda", seed=0):
        K, N = W_bits.shape
        packed = lib.svdq_pack_weights_int4(W_bits, act_absmax, rank, seed=seed)
        return cls(packed, K, N, rank, bias_bits, epilogue, gelu_col_begin, device)

    def buffers(self, M):
        """Activation-side buffers for M rows (allocated once per M, shared by every call)."""
        if M not in self._bufs:
            sz = lib.svdq_int4_act_sizes(M, self.K)
            self._bufs[M] = dict(
                codes=torch.empty(sz["codes"], dtype=torch.uint8, device=self.device),
                scales=torch.empty(sz["scales"], dtype=torch.uint8, device=self.device),
                U=torch.empty(lib.svdq_act_sizes(M, self.K)["u"], dtype=torch.uint8, device=self.device))
        return self._bufs[M]

    def __call__(self, X, Y=None, stream=None):
        _check_input(X, self.K, self.device, "SVDQLinearInt4")
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.N), dtype=torch.bfloat16, device=self.device)
        _check_output(Y, M, self.N, self.device, "SVDQLinearInt4")
        b = self.buffers(M)
        lib.svdq_quantize_act_int4(X, self.inv_lambda, self.l1t, self.rank, b["codes"], b["scales"], b["U"],
                                   stream=stream)
        lib.svdq_linear_int4(b["codes"], b["scales"], b["U"], self.w_codes, self.w_scales, self.l2t, self.bias, M,
                             self.N, self.K, self.rank, self.epilogue, self.gelu_col_begin, Y, stream=stream)
        return Y


class SplitProjection:
    """A fused projection's packed checkpoint mapped onto split modules.

    The pages note that a checkpoint whose query, key and value projections
    are fused into one grouped operation does not map by itself onto a model
    that keeps them as separate modules: the mapping needs the tensor order
    and a small runtime adapter.  This is that adapter for an SVDQLinear
    packed over the concatenation [W_0 | W_1 | ...] of the parts along N
    (in that order): every part keeps the fused layer's smoothing, L1, s_a
    and s_w, and takes its own columns of the residual codes and scales, of
    L2^T and of the bias - views of the fused layer's device buffers, no
    copy.  One call quantizes X once (the parts share the activation side)
    and runs the parts' GEMMs as one grouped launch; part i's output equals
    columns [n_i, n_i + size_i) of the fused layer's output bit for bit.
    Part sizes must be multiples of 256 (the weight bundle's tile rows).
    """

    def __init__(self, fused, sizes, names=None):
        if sum(sizes) != fused.N or any(sz <= 0 or sz % 256 for sz in sizes):
            raise ValueError(f"SplitProjection: part sizes {sizes} must be positive multiples of 256 adding up to "
                             f"N = {fused.N}")
        if len(sizes) > lib.MAX_GROUP:
            raise ValueError(f"SplitProjection: at most {lib.MAX_GROUP} parts")
        self.fused = fused
        self.names = list(names) if names is not None else [str(i) for i in range(len(sizes))]
        tile_bytes = lib.svdq_weight_sizes(fused.K, 256, fused.rank)["w_bundle"]   # one 256-row tile row, all K
        self.parts = []
        n0 = 0
        for sz in sizes:
            n1 = n0 + sz
            begin = min(max(fused.gelu_col_begin - n0, 0), sz)
            self.parts.append(dict(n0=n0, N=sz, gelu_col_begin=begin,
                                   w_bundle=fused.w_bundle[n0 // 256 * tile_bytes:n1 // 256 * tile_bytes],
                                   l2t=fused.l2t[n0 * 2 * lib.LR_STRIDE:n1 * 2 * lib.LR_STRIDE],
                                   bias=fused.bias[n0:n1] if fused.bias is not None else None))
            n0 = n1

    def __call__(self, X, out=None, stream=None):
        """X: bf16 CUDA [M, K] -> {name: Y_i bf16 [M, size_i]} (or into the tensors of `out`)."""
        f = self.fused
        M = X.shape[0]
        b = f.quantize(X, stream)
        ys = {}
        probs = []
        for name, p in zip(self.names, self.parts):
            Y = out[name] if out is not None else torch.empty((M, p["N"]), dtype=torch.bfloat16, device=f.device)
            _check_output(Y, M, p["N"], f.device, "SplitProjection")
            ys[name] = Y
            probs.append(dict(a_bundle=b["a_bundle"], U=b["U"], s_a=f.s_a, w_bundle=p["w_bundle"], l2t=p["l2t"],
                              s_w=f.s_w, bias=p["bias"], M=M, N=p["N"], K=f.K, gelu_col_begin=p["gelu_col_begin"],
                              Y=Y))
        lib.svdq_linear_w4a4_grouped(probs, f.rank, f.epilogue, stream=stream)
        return ys


class AWQLinear:
    """Y = (X diag(inv_awq)) deq(W_a) + b with 4-bit group-64 weights, any M.

    Up to `gemm_rows` rows run on the GEMV (one pass over the packed weights per
    block of 16 rows); more rows run the GEMM path on weights expanded once into
    a workspace the layer keeps (allocated on first use, grown with M).
    """

    gemm_rows = 48

    def __init__(self, packed, K, N, bias_bits=None, device="cuda"):
        self.K, self.N = K, N
        self.device = _resolve(device)
        _init_on(self.device)
        device = self.device
        self.qweight = _dev(packed["qweight"], device)
        self.scales = _dev(packed["scales"], device, torch.bfloat16)
        self.zeros = _dev(packed["zeros"], device, torch.bfloat16)
        self.inv_awq = _dev(packed["inv_awq"], device)
        self.bias = _dev(bias_bits, device, torch.bfloat16) if bias_bits is not None else None
        if self.bias is not None and self.bias.numel() != N:
            raise ValueError(f"AWQLinear: bias must have {N} elements")

    @classmethod
    def from_weight(cls, W_bits, awq_scale, bias_bits=None, device="cuda"):
        K, N = W_bits.shape
        return cls(lib.awq_pack_weights(W_bits, awq_scale), K, N, bias_bits, device)

    def __call__(self, X, Y=None, stream=None):
        _check_input(X, self.K, self.device, "AWQLinear")
        if Y is None:
            Y = torch.empty((X.shape[0], self.N), dtype=torch.bfloat16, device=self.device)
        _check_output(Y, X.shape[0], self.N, self.device, "AWQLinear")
        if X.shape[0] > self.gemm_rows:
            need = lib.awq_gemm_workspace_size(X.shape[0], self.K, self.N)
            if getattr(self, "_workspace", None) is None or self._workspace.numel() < need:
                # (re)allocated: the expanded weights are written once into its head and reused
                self._workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
                lib.awq_expand_weights(self.inv_awq, self.qweight, self.scales, self.zeros, self.K, self.N,
                                       self._workspace, stream=stream)
            lib.awq_linear_w4a16_expanded(X, self.bias, self.N, Y, self._workspace, stream=stream)
        else:
            lib.awq_linear_w4a16(X, self.inv_awq, self.qweight, self.scales, self.zeros, self.bias, self.N, Y,
                                 stream=stream)
        return Y
