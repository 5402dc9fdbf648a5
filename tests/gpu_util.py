"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
reading results back, and the normalised error of the parity bar."""
import os

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


# Every parity comparison of the session: both measures, for the report printed at the end of the
# run (tests/conftest.py) and written as JSON to $PARITY_REPORT when that is set.
PARITY = []


def parity(label, got, want, tol=1e-2):
    """Asserts the parity bar (excess_error <= tol) and records it together with the raw
    row_rms_error, so a reader sees whether the raw bar holds as well."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    ex, raw = excess_error(got, want), row_rms_error(got, want)
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    PARITY.append({"test": test, "case": label, "excess": ex, "raw": raw, "tol": tol,
                   "raw_within_tol": raw <= tol})
    print(f"parity {test} {label}: excess {ex:.3e}  raw {raw:.3e}  (tol {tol:g})")
    assert ex <= tol, f"{label}: excess error {ex:.3e} > {tol:g} (raw {raw:.3e})"
    return ex, raw


def check_ok():
    rc = lib.svdq_check_status()
    assert rc == lib.OK, lib.status_name(rc)


def weights_dev(p, rank):
    """An oracle SVDQ pack (oracle.svdquant.pack) in the library's device layout."""
    k = p["inv_lambda"].shape[0]
    n = p["w_codes"].shape[0]
    return dict(
        inv_lambda=dev(p["inv_lambda"]),
        l1t=bf16_dev(L.bf16_bits(p["l1"].T)) if rank else None,
        l2t=dev(L.lowrank_pack(L.bf16_bits(p["l2"].T), 256)),
        w_bundle=dev(L.bundle_pack(p["w_codes"], p["w_sf"], n, k, 256)),
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
    bundle = poisoned_u8(sz["a_bundle"])
    U = poisoned_u8(sz["u"])
    lib.svdq_quantize_act(X, d["inv_lambda"], d["l1t"], rank, d["s_a"], d["s_w"], bundle, U, M=m, K=k)
    check_ok()
    return bundle, U


def run_k2(oc, osf, ou, d, bias_bits, m, n, k, rank, epilogue, begin, ldy=None):
    """K2 on the oracle's activation operands (codes, scales, bf16-valued U/alpha)."""
    U = L.lowrank_pack(L.bf16_bits(ou), 128)
    ldy = n if ldy is None else ldy
    Yfull = poisoned_bf16(m, ldy)
    Y = Yfull[:, :n]
    lib.svdq_linear_w4a4(dev(L.bundle_pack(oc, osf, m, k, 128)), dev(U), d["s_a"], d["w_bundle"], d["l2t"],
                         d["s_w"], bf16_dev(bias_bits) if bias_bits is not None else None,
                         m, n, k, rank, epilogue, begin, Y)
    check_ok()
    return Y, Yfull


def unpack_act(bundle, U, m, k):
    """GPU activation outputs -> (codes [m, k], scales [m, k/16], U bf16 bits [m, 64])."""
    codes, sf = L.bundle_unpack(u8(bundle), m, k, 128)
    return codes, sf, L.lowrank_unpack(u8(U), m, 128)
