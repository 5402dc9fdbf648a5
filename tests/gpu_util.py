"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
reading results back, and the normalised error of the parity bar."""
import numpy as np
import torch

from bit_w4a4_diffusion_smooth_b200 import lib
from tests import layouts as L

DEV = torch.device("cuda:0")
POISON = 0xA5


def init():
    lib.svdq_init(0)
    torch.cuda.set_device(0)


def bf16_dev(bits, rows=None):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(DEV)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def bf16_host(t):
    """bf16 CUDA tensor -> float64 numpy (exact)."""
    return t.float().cpu().numpy().astype(np.float64)


def u8(t):
    return t.cpu().numpy()


def poisoned_u8(*shape):
    return torch.full(shape, POISON, dtype=torch.uint8, device=DEV)


def poisoned_bf16(*shape):
    return torch.full(shape, float("nan"), dtype=torch.bfloat16, device=DEV)


def row_rms_error(got, want):
    """max_i max_j |got - want| / rms_j(want[i, :]) (rows with rms 0 use 1)."""
    rms = np.sqrt(np.mean(want ** 2, axis=1))
    rms = np.where(rms == 0, 1.0, rms)
    return float(np.max(np.abs(got - want) / rms[:, None]))


def bf16_ulp(v):
    """Spacing of bf16 numbers just above |v|'s power of two (2^-133 at 0)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(np.maximum(e, -126) - 7), 2.0 ** -133)


def excess_error(got, want):
    """The parity measure for bf16 outputs: max over a row of
    max(0, |got - want| - ulp(got) / 2) divided by the RMS of the oracle's row.

    A kernel that returns bf16 cannot be closer to the exact value than half a
    bf16 spacing of its own result; this measures what the kernel's arithmetic
    adds beyond that rounding of its output (a lower bound of
    |pre-rounding result - want|).
    """
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    rms = np.sqrt(np.mean(want ** 2, axis=1))
    rms = np.where(rms == 0, 1.0, rms)
    d = np.maximum(0.0, np.abs(got - want) - 0.5 * bf16_ulp(got))
    return float(np.max(d / rms[:, None]))


def check_ok():
    rc = lib.svdq_check_status()
    assert rc == lib.OK, lib.status_name(rc)


def weights_dev(p, rank):
    """An oracle SVDQ pack (oracle.svdquant.pack) in the library's device layout."""
    k = p["inv_lambda"].shape[0]
    n = p["w_codes"].shape[0]
    l2t = np.zeros((n, lib.LR_STRIDE), np.uint16)
    l2t[:, :rank] = L.bf16_bits(p["l2"].T)
    return dict(
        inv_lambda=dev(p["inv_lambda"]),
        l1t=bf16_dev(L.bf16_bits(p["l1"].T)) if rank else None,
        l2t=bf16_dev(l2t),
        w_codes=dev(L.pack_codes(p["w_codes"])),
        w_scales=dev(L.tile_scales(p["w_sf"], n, k)),
        s_w=dev(np.array([p["s_w"]], np.float32)),
        s_a=dev(np.array([p["s_a"]], np.float32)),
    )


def run_k1(xb, m, k, rank, d, ldx=None):
    """K1 on a bf16 bit array; poisoned outputs so unwritten bytes show."""
    X = bf16_dev(xb)
    if ldx is not None and ldx != k:  # strided rows
        Xp = torch.zeros((m, ldx), dtype=torch.bfloat16, device=DEV)
        Xp[:, :k] = X
        X = Xp[:, :k]
    sz = lib.svdq_act_sizes(m, k)
    codes = poisoned_u8(m, k // 2)
    scales = poisoned_u8(sz["scales"])
    U = poisoned_bf16(m, lib.LR_STRIDE)
    lib.svdq_quantize_act(X, d["inv_lambda"], d["l1t"], rank, d["s_a"], d["s_w"], codes, scales, U, M=m, K=k)
    check_ok()
    return codes, scales, U


def run_k2(oc, osf, ou, d, bias_bits, m, n, k, rank, epilogue, begin, ldy=None):
    """K2 on the oracle's activation operands (codes, scales, bf16-valued U/alpha)."""
    U = np.zeros((m, lib.LR_STRIDE), np.uint16)
    U[:, :rank] = L.bf16_bits(ou)
    ldy = n if ldy is None else ldy
    Yfull = poisoned_bf16(m, ldy)
    Y = Yfull[:, :n]
    lib.svdq_linear_w4a4(dev(L.pack_codes(oc)), dev(L.tile_scales(osf, m, k)), bf16_dev(U), d["s_a"],
                         d["w_codes"], d["w_scales"], d["l2t"], d["s_w"],
                         bf16_dev(bias_bits) if bias_bits is not None else None,
                         m, n, k, rank, epilogue, begin, Y)
    check_ok()
    return Y, Yfull
