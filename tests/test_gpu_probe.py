"""The hardware conversions the kernels rely on, and the bounded-wait path.

The kernels produce e2m1 codes and e4m3 block scales with cvt...satfinite;
these tests check those instructions against the format definitions of the
oracle (bit-exact, negative zero included), and check that a wait nothing
completes runs out and is reported, with the context still usable.
"""
import numpy as np
import pytest
import torch

from bit_w4a4_diffusion_smooth_b200 import lib
from oracle import formats
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _init():
    G.init()


def _sweep_e2m1():
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    pts = set()
    for g in grid:
        pts.update(np.nextafter(np.float32(g), [np.float32(-1), np.float32(100)]).tolist() + [g])
    for lo, hi in zip(grid[:-1], grid[1:]):
        m = np.float32((lo + hi) / 2)
        pts.update([m, np.nextafter(m, np.float32(-1)), np.nextafter(m, np.float32(100))])
    pts.update([7.0, 100.0, 1e30, 1e-30, 0.0, 0.1])
    rng = np.random.default_rng(0)
    pts.update(rng.uniform(0, 8, 4000).astype(np.float32).tolist())
    xs = np.array(sorted(pts), dtype=np.float32)
    xs = np.concatenate([xs, -xs, np.array([-0.0, 0.0], np.float32)])
    if xs.size % 2:
        xs = np.append(xs, np.float32(1.0))
    return xs


def test_e2m1_conversion_matches_definition():
    xs = _sweep_e2m1()
    e2 = torch.empty(xs.size // 2, dtype=torch.uint8, device=G.DEV)
    e4 = torch.empty(xs.size, dtype=torch.uint8, device=G.DEV)
    lib.svdq_debug_convert(G.dev(xs), e2, e4)
    got = G.u8(e2)
    codes = formats.e2m1_encode(xs)
    want = (codes[1::2] << 4) | codes[0::2]
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(xs[2 * i], xs[2 * i + 1], hex(got[i]), hex(want[i])) for i in bad[:8]]


def test_e4m3_conversion_matches_definition():
    vals = formats.ue4m3_decode(np.arange(127))
    pts = set(vals.astype(np.float32).tolist())
    for lo, hi in zip(vals[:-1], vals[1:]):
        m = np.float32((lo + hi) / 2)
        pts.update([m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9))])
    pts.update([449.0, 464.0, 479.0, 480.0, 1e6, 2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11])
    rng = np.random.default_rng(1)
    pts.update(np.exp2(rng.uniform(-12, 10, 6000)).astype(np.float32).tolist())
    xs = np.array(sorted(pts), dtype=np.float32)
    if xs.size % 2:
        xs = np.append(xs, np.float32(1.0))
    e2 = torch.empty(xs.size // 2, dtype=torch.uint8, device=G.DEV)
    e4 = torch.empty(xs.size, dtype=torch.uint8, device=G.DEV)
    lib.svdq_debug_convert(G.dev(xs), e2, e4)
    got = G.u8(e4)
    want = formats.ue4m3_encode(xs)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(xs[i], hex(got[i]), hex(want[i])) for i in bad[:8]]


def test_bounded_wait_reports_timeout_and_context_survives():
    assert lib.svdq_check_status() == lib.OK
    lib.svdq_debug_wait_timeout(20_000_000)  # 20 ms; nothing ever completes the barrier
    assert lib.svdq_check_status() == lib.ERR_TIMEOUT
    assert lib.svdq_check_status() == lib.OK  # cleared
    x = torch.arange(10, device=G.DEV).sum().item()
    assert x == 45


def test_init_rejects_missing_device():
    with pytest.raises(lib.SvdqError) as e:
        lib.svdq_init(torch.cuda.device_count() + 3)
    assert e.value.status == lib.ERR_INVALID_ARG


def _gelu_probe(x, kind):
    xs = torch.from_numpy(x).to(G.DEV)
    out = torch.empty_like(xs)
    lib.svdq_debug_gelu(xs, kind, out)
    G.check_ok()
    return out.cpu().numpy().astype(np.float64)


def test_gelu_erf_matches_definition():
    """The epilogue's erf-form GELU (erf by Abramowitz & Stegun 7.1.26, |error| <= 1.5e-7, through
    fast exp / division) against 0.5 x (1 + erf(x / sqrt 2)) in float64: absolute error within
    1e-6 |x| + 1e-30 over [-12, 12], far below the bf16 rounding of the output it feeds."""
    from scipy.special import erf
    rng = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-12, 12, 200001), rng.normal(0, 3, 100000),
                        [0.0, -0.0, 1e-30, -1e-30, 1e-6, -1e-6, 30.0, -30.0]]).astype(np.float32)
    got = _gelu_probe(x, lib.EPILOGUE_GELU_ERF)
    xd = x.astype(np.float64)
    want = 0.5 * xd * (1.0 + erf(xd / np.sqrt(2.0)))
    err = np.abs(got - want)
    assert np.all(err <= 1e-6 * np.abs(xd) + 1e-30), float(np.max(err / (np.abs(xd) + 1e-30)))
    assert got[x == 30.0][0] == 30.0 and got[x == -30.0][0] == 0.0
    # GELU of a negative input is negative: the sign survives down to the smallest results (it
    # decides the sign of a zero e2m1 code when the output is re-quantized), and results the
    # format can hold are not flushed to zero
    neg = x < 0
    assert np.signbit(got[neg]).all()
    assert (got[(x < -1.0) & (x > -12.0)] < 0).all()


def test_gelu_tanh_matches_definition():
    rng = np.random.default_rng(4)
    x = np.concatenate([np.linspace(-12, 12, 100001), rng.normal(0, 3, 50000)]).astype(np.float32)
    got = _gelu_probe(x, lib.EPILOGUE_GELU_TANH)
    xd = x.astype(np.float64)
    want = 0.5 * xd * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (xd + 0.044715 * xd ** 3)))
    assert np.all(np.abs(got - want) <= 2e-6 * np.abs(xd) + 1e-30)
