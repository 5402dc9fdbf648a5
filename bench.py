"""Throughput of the SVDQuant W4A4 linear (+ AWQ W4A16 projection) on B200.

One step = the whole hot path over one batch of synthetic input, on the layer
shapes of one block of a 12B-class DiT at 1024x1024 (4096 image + 512 text
tokens, rank 32):
  qkv   K1 + K2    X [4608 x 3072] -> [4608 x 9216]
  fc1   K1 + K2    X [4608 x 3072] -> H [4608 x 12288], GELU (erf) epilogue
  fc2   K1 + K2    H [4608 x 12288] -> [4608 x 3072]   (fc1's output re-quantized)
  adaLN K3         [2 x 3072] -> [2 x 18432]           (AWQ W4A16, group 64)
K1 = activation quantize + low-rank down-projection, K2 = tcgen05 NVFP4 GEMM +
low-rank up-projection + epilogue, K3 = W4A16 GEMV.

value = algorithmic FLOPs of the step / step time (TFLOP/s, all ranks).
Weights, inputs, intermediates and outputs rotate over buffer sets that
together exceed twice the L2 cache, so no step reads what the previous one
left in L2.  Multi-GPU runs are independent replicas (the layer needs no
exchange between GPUs): weak scaling.

After the timed region every kernel of the step is timed alone, back to back
over the rotating sets, so that the per-kernel figures carry no event between
two different kernels; the roofline object reports the fc1 GEMM
(4608 x 3072 x 12288 with GELU), the largest kernel of the step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload layers|dit-step]

--workload dit-step times every projection linear of one denoising step of a
12B-class DiT (228 W4A4 layers + 76 AWQ projections) as one CUDA graph.
"""
import argparse
import hashlib
import json
import platform
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

RANK = 32
TOKENS, HIDDEN, MLP = 4608, 3072, 12288
# name -> (M, K, N, GELU epilogue); fc2 reads fc1's output
LAYERS = {"qkv": (TOKENS, HIDDEN, 3 * HIDDEN, False),
          "fc1": (TOKENS, HIDDEN, MLP, True),
          "fc2": (TOKENS, MLP, HIDDEN, False)}
AM, AK, AN = 2, HIDDEN, 6 * HIDDEN
MIN_SETS = 6                   # rotating buffer sets: 6 x 32 MB (the AWQ weights) > 1.5 x L2
WORKLOAD = ("one 12B-class DiT block's SVDQ W4A4 linears at 4608 tokens, rank 32 (NVFP4, group 16): "
            "QKV 3072->9216, MLP fc1 3072->12288 +GELU then fc2 12288->3072 on fc1's output; "
            "+ AWQ W4A16 adaLN projection 2x3072->18432 (INT4, group 64)")
METRIC = "SVDQ W4A4 linear TFLOPS and % of B200 dense-FP4 peak; W4A16 GB/s vs HBM"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0            # nominal dense FP4 / dense bf16 ratio (9 / 2.25 PFLOP/s)
FP4_NOMINAL_TFLOPS = 9000.0    # NVIDIA's dense FP4 figure for B200


def gemm_flops(m, k, n, r=RANK):
    """FP4 main branch + the low-rank up-projection done inside K2."""
    return 2 * m * k * n + 2 * m * r * n


def layer_flops(m, k, n, r=RANK):
    """The whole SVDQ layer: K2's work + K1's low-rank down-projection."""
    return gemm_flops(m, k, n, r) + 2 * m * k * r


AWQ_FLOPS = 2 * AM * AK * AN
STEP_FLOPS = sum(layer_flops(m, k, n) for m, k, n, _ in LAYERS.values()) + AWQ_FLOPS


def k1_bytes(m, k, r=RANK):
    """Algorithmic bytes of K1: X, L1T, inv_lambda in; codes, scales, U out."""
    return m * k * 2 + k * r * 2 + k * 4 + m * k // 2 + m * k // 16 + m * r * 2


def k2_bytes(m, k, n, r=RANK):
    return (m * k // 2 + m * k // 16 + m * r * 2 + n * k // 2 + n * k // 16 + n * r * 2 + n * 2 + m * n * 2)


K3_BYTES = (AN * AK // 2 + 2 * AN * (AK // 64) * 2      # qweight, scales + zeros
            + AM * AK * 2 + AK * 4 + AN * 2 + AM * AN * 2)

# DRAM traffic of one fc1-shaped K2 launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
# ncu capture summarised in profiles/, and the hash of the GEMM sources it was taken on: when the
# source has changed since, the counters no longer describe the kernel and `traffic` is null.
K2_TRAFFIC = {"bytes": 130053632, "source_sha16": "d448269f86494399"}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return PEAKS_FALLBACK, "fallback"


K2_SOURCES = ("gemm_w4a4_kernel.cuh", "device_common.cuh", "svdq_internal.h")


def source_sha16(names=K2_SOURCES):
    """Hash of the sources a kernel is compiled from (the GEMM's by default)."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "bit_w4a4_diffusion_smooth_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


# ------------------------------------------------------------------ replicas
# The layer needs no exchange between GPUs, so N GPUs run N independent
# replicas of the step.  The process group carries only the barriers around
# the timed region and the max-over-ranks reduction of the timings.
def init_replicas(world, backend, device=None, timeout_s=120):
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        kw = {"device_id": device} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)


def max_over_ranks(values, world, device="cpu"):
    """Element-wise max over ranks of this rank's timings (every rank gets it)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_tflops(flops_per_replica_step, world, ms_per_step):
    """Whole-job throughput: the work of all replicas over the slowest rank's step time."""
    return flops_per_replica_step * world / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU is under the bench's load."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu):
        self.gpu = gpu
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        # nvidia-smi needs a moment before its first sample: start timing only once it samples
        t_end = time.time() + 5.0
        while time.time() < t_end:
            self.out.flush()
            try:
                if os.path.getsize(self.out.name) > 0:
                    break
            except OSError:
                break
            time.sleep(0.05)
        time.sleep(0.1)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        smax = max(float(r[2]) for r in rows)
        loaded = [float(r[1]) for r in rows if float(r[3]) > 250.0] or sm
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded)}


# ------------------------------------------------------------------ our arm
def _bf(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _t(arr):
    import torch
    return torch.from_numpy(np.ascontiguousarray(arr))


class Workload:
    """Packed weights (host pack of the library), inputs and buffers of the step, on one device,
    as `sets` rotating copies."""

    def __init__(self, device):
        import torch

        from bit_w4a4_diffusion_smooth_b200 import lib, synthetic

        self.device = device
        lib.svdq_init(device.index)
        cases = {"qkv": synthetic.QKV, "fc1": synthetic.MLP_FC1, "fc2": synthetic.MLP_FC2}
        self.host_w = {}
        self.x_bits = {}
        self.w_bits = {}
        for name in ("qkv", "fc1"):
            c = cases[name]
            xb, wb, bb = c.make()
            amax = np.max(np.abs(synthetic.bf16_bits_to_f32(xb)), axis=0).astype(np.float32)
            self.x_bits[name] = xb
            self.w_bits[name] = (wb, amax, bb)
            self.host_w[name] = (lib.svdq_pack_weights(wb, amax, RANK, seed=c.seed), bb)
        # fc2: calibrated on fc1's output for this input (one untimed fc1 pass on the device)
        c2 = cases["fc2"]
        wb2, _ = synthetic.weight(c2.k, c2.n, c2.seed, 0.02, c2.w_outlier_rows, c2.w_factor)
        bb2 = synthetic.bias(c2.n, c2.seed + 100)
        one = self._layer_dev("fc1")
        xs = _bf(self.x_bits["fc1"]).to(device)
        sz = lib.svdq_act_sizes(TOKENS, HIDDEN)
        ab = torch.empty(sz["a_bundle"], dtype=torch.uint8, device=device)
        u = torch.empty(sz["u"], dtype=torch.uint8, device=device)
        h = torch.empty((TOKENS, MLP), dtype=torch.bfloat16, device=device)
        lib.svdq_quantize_act(xs, one["inv_lambda"], one["l1t"], RANK, one["s_a"], one["s_w"], ab, u)
        lib.svdq_linear_w4a4(ab, u, one["s_a"], one["w_bundle"], one["l2t"], one["s_w"], one["bias"],
                             TOKENS, MLP, HIDDEN, RANK, lib.EPILOGUE_GELU_ERF, 0, h)
        amax2 = h.float().abs().amax(dim=0).cpu().numpy().astype(np.float32)
        self.host_w["fc2"] = (lib.svdq_pack_weights(wb2, amax2, RANK, seed=c2.seed), bb2)
        del one, xs, ab, u, h
        a = synthetic.AWQ
        axb, awb, abb, asc = a.make()
        self.awq_x_bits = axb
        self.host_awq = (lib.awq_pack_weights(awb, asc), abb)
        self.sets = []

    def _layer_dev(self, name):
        p, bb = self.host_w[name]
        d = self.device
        return dict(inv_lambda=_t(p["inv_lambda"]).to(d), l1t=_bf(p["l1t"]).to(d), l2t=_t(p["l2t"]).to(d),
                    w_bundle=_t(p["w_bundle"]).to(d), s_w=_t(p["s_w"]).to(d), s_a=_t(p["s_a"]).to(d),
                    bias=_bf(bb).to(d))

    def add_set(self):
        import torch

        from bit_w4a4_diffusion_smooth_b200 import lib
        d = self.device
        s = {}
        for name, (m, k, n, _) in LAYERS.items():
            L = self._layer_dev(name)
            sz = lib.svdq_act_sizes(m, k)
            L["a_bundle"] = torch.empty(sz["a_bundle"], dtype=torch.uint8, device=d)
            L["U"] = torch.empty(sz["u"], dtype=torch.uint8, device=d)
            L["Y"] = torch.empty((m, n), dtype=torch.bfloat16, device=d)
            s[name] = L
        s["qkv"]["X"] = _bf(self.x_bits["qkv"]).to(d)
        s["fc1"]["X"] = _bf(self.x_bits["fc1"]).to(d)
        s["fc2"]["X"] = s["fc1"]["Y"]                    # unfused path: fc2's K1 reads fc1's output
        s["requant_ws"] = torch.empty(lib.svdq_requant_workspace_size(TOKENS, RANK) // 4, dtype=torch.float32,
                                      device=d)
        apk, abb = self.host_awq
        s["awq"] = dict(X=_bf(self.awq_x_bits).to(d), qweight=_t(apk["qweight"]).to(d),
                        scales=_bf(apk["scales"]).to(d), zeros=_bf(apk["zeros"]).to(d),
                        inv_awq=_t(apk["inv_awq"]).to(d), bias=_bf(abb).to(d),
                        Y=torch.empty((AM, AN), dtype=torch.bfloat16, device=d))
        self.sets.append(s)
        seen, total = set(), 0
        for part in s.values():
            for v in (part.values() if isinstance(part, dict) else [part]):
                if v.data_ptr() not in seen:
                    seen.add(v.data_ptr())
                    total += v.numel() * v.element_size()
        return total


def k1(L, name):
    from bit_w4a4_diffusion_smooth_b200 import lib
    m, k, n, _ = LAYERS[name]
    lib.svdq_quantize_act(L["X"], L["inv_lambda"], L["l1t"], RANK, L["s_a"], L["s_w"], L["a_bundle"], L["U"],
                          M=m, K=k)


def k2(L, name):
    from bit_w4a4_diffusion_smooth_b200 import lib
    m, k, n, gelu = LAYERS[name]
    lib.svdq_linear_w4a4(L["a_bundle"], L["U"], L["s_a"], L["w_bundle"], L["l2t"], L["s_w"], L["bias"], m, n, k,
                         RANK, lib.EPILOGUE_GELU_ERF if gelu else lib.EPILOGUE_NONE, 0, L["Y"])


def k2_requant(s):
    """fc1's GEMM writing fc2's input operands (codes, scales, U) instead of its bf16 output."""
    from bit_w4a4_diffusion_smooth_b200 import lib
    m, k, n, gelu = LAYERS["fc1"]
    L, nx = s["fc1"], s["fc2"]
    lib.svdq_linear_w4a4_requant(L["a_bundle"], L["U"], L["s_a"], L["w_bundle"], L["l2t"], L["s_w"], L["bias"], m, n,
                                 k, RANK, lib.EPILOGUE_GELU_ERF if gelu else lib.EPILOGUE_NONE, 0, None,
                                 nx["inv_lambda"], nx["l1t"], RANK, nx["s_a"], nx["s_w"], nx["a_bundle"], nx["U"],
                                 s["requant_ws"])


def k3(A):
    from bit_w4a4_diffusion_smooth_b200 import lib
    lib.awq_linear_w4a16(A["X"], A["inv_awq"], A["qweight"], A["scales"], A["zeros"], A["bias"], AN, A["Y"])


# The step's kernels in order: (label, function of one buffer set).  The MLP pair runs either
# fused - fc1's GEMM re-quantizes its GELU output for fc2 in its epilogue, so fc2 needs no K1 pass
# and the 4608 x 12288 bf16 activation between the two layers never travels through memory - or
# unfused (fc1's plain GEMM writes the bf16 activation, fc2's K1 reads it back); the other form is
# timed alone for comparison.
def step_kernels(mlp):
    head = [("K1 qkv", lambda s: k1(s["qkv"], "qkv")), ("K2 qkv", lambda s: k2(s["qkv"], "qkv")),
            ("K1 fc1", lambda s: k1(s["fc1"], "fc1"))]
    tail = [("K2 fc2", lambda s: k2(s["fc2"], "fc2")), ("K3 adaLN", lambda s: k3(s["awq"]))]
    if mlp == "fused":
        return head + FUSED_MLP + tail
    return head + UNFUSED_MLP + tail


FUSED_MLP = [("K2 fc1 -> fc2 operands", k2_requant)]
UNFUSED_MLP = [("K2 fc1 (plain, bf16 out)", lambda s: k2(s["fc1"], "fc1")),
               ("K1 fc2 (on fc1's bf16 out)", lambda s: k1(s["fc2"], "fc2"))]
MLP_DEFAULT = "unfused"   # measured faster on B200 (the fused epilogue is the longer path)
STEP_KERNELS = step_kernels(MLP_DEFAULT)


def launches_per_step(mlp):
    """My kernels per step; the re-quantizing call launches the GEMM and a small finalize kernel."""
    return len(step_kernels(mlp)) + (1 if mlp == "fused" else 0)


LAUNCHES_PER_STEP = launches_per_step(MLP_DEFAULT)


def step(sets, i, kernels=None):
    s = sets[i % len(sets)]
    for _, fn in (kernels or STEP_KERNELS):
        fn(s)


def requant_flops():
    """fc1's GEMM plus, in its epilogue, fc2's low-rank down-projection (2 M N r)."""
    m, k, n, _ = LAYERS["fc1"]
    return gemm_flops(m, k, n) + 2 * m * n * RANK


def kernel_table(pk):
    """label -> (algorithmic amount per launch, unit, bound, peak)."""
    fp4_peak = pk["bf16_tflops"] * FP4_OVER_BF16
    t = {}
    for name, (m, k, n, _) in LAYERS.items():
        t[f"K1 {name}"] = (k1_bytes(m, k), "GB/s", "hbm", pk["hbm_gbs"])
        t[f"K2 {name}"] = (gemm_flops(m, k, n), "TFLOP/s", "tensor", fp4_peak)
    t["K2 fc1 -> fc2 operands"] = (requant_flops(), "TFLOP/s", "tensor", fp4_peak)
    t["K2 fc1 (plain, bf16 out)"] = t["K2 fc1"]
    t["K1 fc2 (on fc1's bf16 out)"] = t["K1 fc2"]
    t["K3 adaLN"] = (K3_BYTES, "GB/s", "hbm", pk["hbm_gbs"])
    return t


class L2Flush:
    """Reads a buffer of twice the L2 size, so that the next kernel finds none of its data in L2.  A read
    leaves the cache clean: a flush by writing would leave ~L2-size of dirty lines for the timed kernel
    to write back."""

    def __init__(self, device):
        import torch
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        self.buf = torch.zeros(2 * l2 // 4, dtype=torch.int32, device=device)
        self.out = torch.zeros((), dtype=torch.int64, device=device)

    def __call__(self):
        import torch
        torch.sum(self.buf, dim=0, dtype=torch.int64, out=self.out)


def time_back_to_back(fn, sets, reps, barrier):
    """Mean device time (ms) per launch of `fn` launched `reps` times back to back over the rotating
    sets, with one event before the first launch and one after the last."""
    import torch
    for i in range(2):
        fn(sets[i % len(sets)])
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(reps):
        fn(sets[i % len(sets)])
    b.record()
    barrier()
    return a.elapsed_time(b) / reps


def time_cold(fn, sets, reps, flush):
    """Mean device time (ms) of one launch of `fn` with L2 flushed before it: each launch sits alone
    between two events on the stream, after a read of twice the L2 size."""
    import torch
    for i in range(2):
        fn(sets[i % len(sets)])
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i in range(reps):
        flush()
        ev[i][0].record()
        fn(sets[i % len(sets)])
        ev[i][1].record()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / reps


def awq_many_rows(W, device, m=256, reps=10):
    """The adaLN projection on a batch of m rows: K3's blocks of 16 rows against the GEMM path on weights
    expanded once (mean device time of `reps` back-to-back launches each, after warm-up)."""
    import torch
    from bit_w4a4_diffusion_smooth_b200 import lib
    A = W.sets[0]["awq"]
    gen = torch.Generator(device=device)
    gen.manual_seed(7)
    X = torch.randn(m, AK, device=device, generator=gen).to(torch.bfloat16)
    Y = torch.empty(m, AN, dtype=torch.bfloat16, device=device)
    ws = torch.empty(lib.awq_gemm_workspace_size(m, AK, AN), dtype=torch.uint8, device=device)
    lib.awq_expand_weights(A["inv_awq"], A["qweight"], A["scales"], A["zeros"], AK, AN, ws)
    out = {}
    for name, fn in (("gemv_blocks_of_16_us", lambda: lib.awq_linear_w4a16(X, A["inv_awq"], A["qweight"], A["scales"],
                                                                           A["zeros"], A["bias"], AN, Y)),
                     ("gemm_on_expanded_us", lambda: lib.awq_linear_w4a16_expanded(X, A["bias"], AN, Y, ws))):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out[name] = round(e0.elapsed_time(e1) / reps * 1e3, 2)
    out["what"] = f"{m}x{AK}->{AN} AWQ W4A16, {reps} launches back to back (the many-row path of the adaLN projection)"
    return out


def int4_variant(W, device, pk, reps=20):
    """The INT4 W4A4 variant on the MLP fc1 layer (4608 x 3072 -> 12288, erf GELU, rank 32): its
    activation kernel and its GEMM, each launched back to back over rotating copies of every buffer
    (six: each launch's data evicted from L2 by the others), beside the NVFP4 kernels of the step."""
    import torch
    from bit_w4a4_diffusion_smooth_b200 import lib
    m, k, n, _ = LAYERS["fc1"]
    wb, amax, bb = W.w_bits["fc1"]
    pack = lib.svdq_pack_weights_int4(wb, amax, RANK, seed=11)
    asz = lib.svdq_int4_act_sizes(m, k)
    sets = []
    for s in W.sets[:MIN_SETS]:
        sets.append(dict(X=s["fc1"]["X"], inv=_t(pack["inv_lambda"]).to(device), l1t=_bf(pack["l1t"]).to(device),
                         l2t=_t(pack["l2t"]).to(device), wc=_t(pack["w_codes"]).to(device),
                         ws=_t(pack["w_scales"]).to(device), bias=s["fc1"]["bias"],
                         ac=torch.empty(asz["codes"], dtype=torch.uint8, device=device),
                         asc=torch.empty(asz["scales"], dtype=torch.uint8, device=device),
                         U=torch.empty(lib.svdq_act_sizes(m, k)["u"], dtype=torch.uint8, device=device),
                         Y=s["fc1"]["Y"]))

    def k1(d):
        lib.svdq_quantize_act_int4(d["X"], d["inv"], d["l1t"], RANK, d["ac"], d["asc"], d["U"], M=m, K=k)

    def k2(d):
        lib.svdq_linear_int4(d["ac"], d["asc"], d["U"], d["wc"], d["ws"], d["l2t"], d["bias"], m, n, k, RANK,
                             lib.EPILOGUE_GELU_ERF, 0, d["Y"])

    def sync():
        torch.cuda.synchronize()
    k1_ms = time_back_to_back(k1, sets, reps, sync)
    k2_ms = time_back_to_back(k2, sets, reps, sync)
    rc = lib.svdq_check_status()
    if rc != lib.OK:
        raise RuntimeError(f"device status after the INT4 pass: {lib.status_name(rc)}")
    f16_peak = pk["bf16_tflops"]           # the GEMM's tensor-core arithmetic is fp16 x fp16 -> fp32
    k1_gbs = k1_bytes(m, k) / (k1_ms * 1e-3) / 1e9
    k2_tops = gemm_flops(m, k, n) / (k2_ms * 1e-3) / 1e12
    return {"K1 int4 fc1": {"us": round(k1_ms * 1e3, 2), "GB/s": round(k1_gbs, 1),
                            "frac": round(k1_gbs / pk["hbm_gbs"], 4)},
            "K2 int4 fc1 +GELU": {"us": round(k2_ms * 1e3, 2), "TFLOP/s": round(k2_tops, 1),
                                  "frac_of_fp16_tensor_peak": round(k2_tops / f16_peak, 4)},
            "fp16_tensor_peak_tflops": round(f16_peak, 1),
            "what": "INT4 W4A4 (groups of 64, bf16 scales) on the fc1 layer: back-to-back launches over 6 rotating "
                    "buffer sets; B200 has no 4-bit integer MMA, so the GEMM turns the codes into exact fp16 "
                    "operands q*s in shared memory and runs tcgen05 kind::f16 (fp32 accumulation), against the "
                    "16-bit tensor peak"}


def host_path_point(device, m=512, k=3072, n=9216, reps=100):
    """Host cost of a layer call: a 512-row text-stream projection (m x k -> n, rank 32) through
    SVDQLinear's repeated calls (the marshalled arguments of its first call with these buffers),
    launched from the host back to back, against the same calls replayed from a CUDA graph.
    Random-valid packed bytes (speed only)."""
    import time

    import torch

    from bit_w4a4_diffusion_smooth_b200 import lib
    from bit_w4a4_diffusion_smooth_b200.layer import SVDQLinear
    rng = np.random.default_rng(5)
    ws = lib.svdq_weight_sizes(k, n, RANK)
    packed = dict(inv_lambda=np.ones(k, np.float32), l1t=np.zeros((RANK, k), np.uint16),
                  l2t=rng.integers(0, 256, ws["l2t"], dtype=np.uint8) & 0x3F,
                  w_bundle=rng.integers(0, 256, ws["w_bundle"], dtype=np.uint8) & 0x77, s_w=1e-3, s_a=1.0)
    layer = SVDQLinear(packed, k, n, RANK, device=device)
    X = (torch.randn(m, k, device=device) * 0.5).to(torch.bfloat16)
    Y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
    for _ in range(5):
        layer(X, Y)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        layer(X, Y)
    e1.record()
    torch.cuda.synchronize()
    launched = e0.elapsed_time(e1) / reps * 1e3
    t = time.perf_counter()
    for _ in range(reps):
        layer(X, Y)
    host = (time.perf_counter() - t) / reps * 1e6
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(10):
            layer(X, Y)
    graph.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps // 10):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    replayed = e0.elapsed_time(e1) / reps * 1e3
    del graph
    return {"layer": f"SVDQLinear {m}x{k}->{n} r{RANK}, repeated calls on the same buffers",
            "host_launched_us": round(launched, 2), "graph_us": round(replayed, 2),
            "host_us_per_call": round(host, 2),
            "what": "GPU time per call (K1 + K2) of 100 calls launched from the host back to back, against the "
                    "same calls replayed from a CUDA graph; host_us_per_call is the host's own time per call"}


def copy_floor(device, nbytes, reps=24):
    """A library copy of `nbytes` (torch, device to device) with L2 flushed before it, timed like the
    kernels: the HBM rate a plain stream of this size reaches on this GPU, as (GB/s counting read +
    write, us per copy)."""
    import torch
    n = nbytes // 2
    src = torch.empty(n, dtype=torch.bfloat16, device=device).fill_(1.0)
    dst = torch.empty(n, dtype=torch.bfloat16, device=device)
    flush = L2Flush(device)
    ms = time_cold(lambda b: b[1].copy_(b[0]), [(src, dst)], reps, flush)
    del src, dst, flush
    return 2 * nbytes / (ms * 1e-3) / 1e9, ms * 1e3


def fp4_library_point(device, m, k, n, reps=20):
    """torch._scaled_mm (cuBLASLt) on NVFP4 operands of the same shape as a library reference
    point: e2m1 A [m, k] and B [n, k], ue4m3 block scales of 16 in the blocked layout.  Returns
    (TFLOP/s of the 2mkn product, us) or an error string when the call is not supported here."""
    import torch
    try:
        fp4 = torch.float4_e2m1fn_x2
        sets = []
        for i in range(2):
            a = (torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device=device) & 0x77).view(fp4)
            b = (torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=device) & 0x77).view(fp4)
            rm, rn, rk = (m + 127) // 128 * 128, (n + 127) // 128 * 128, (k // 16 + 3) // 4 * 4
            sa = torch.full((rm * rk,), 0x38, dtype=torch.uint8, device=device).view(torch.float8_e4m3fn)
            sb = torch.full((rn * rk,), 0x38, dtype=torch.uint8, device=device).view(torch.float8_e4m3fn)
            sets.append((a, b, sa, sb))

        def run(s):
            return torch._scaled_mm(s[0], s[1].t(), s[2], s[3], out_dtype=torch.bfloat16)

        y = run(sets[0])
        torch.cuda.synchronize()
        if tuple(y.shape) != (m, n):
            return f"unexpected output shape {tuple(y.shape)}"
        flush = L2Flush(device)
        ms = time_cold(run, sets, reps, flush)
        return 2 * m * k * n / (ms * 1e-3) / 1e12, ms * 1e3
    except Exception as e:  # noqa: BLE001 - a reference point only: record why it is missing
        return f"{type(e).__name__}: {str(e).splitlines()[0][:200]}"


def run_ours(args):
    import torch
    import torch.distributed as dist

    from bit_w4a4_diffusion_smooth_b200 import lib

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_replicas(world, "nccl", device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    W = Workload(device)
    set_bytes = W.add_set()
    # enough sets that a kernel run back to back over them (the smallest one touches ~32 MB of a
    # set) finds its data evicted from L2 each time, as it does inside the step
    while len(W.sets) < MIN_SETS or len(W.sets) * set_bytes < 2 * l2:
        W.add_set()
    sets = W.sets

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    kernels = step_kernels(args.mlp)
    other = UNFUSED_MLP if args.mlp == "fused" else FUSED_MLP
    for i in range(args.warmup):
        step(sets, i, kernels)
    rc = lib.svdq_check_status()
    if rc != lib.OK:
        raise RuntimeError(f"device status after warm-up: {lib.status_name(rc)}")

    # ---- device-timed region: exactly K steps between two events on the launching stream
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        step(sets, i, kernels)
    t1.record()
    barrier()
    ms = t0.elapsed_time(t1)
    # ---- the same steps again with an event after every kernel: each kernel's mean duration inside
    # the running step, on the launching stream.  An event between two kernels costs their launch
    # overlap, so this pass is slower than the region above; it gives the per-kernel split and the
    # roofline, not the headline.  The first steps after the barrier are left out (the queue is
    # still filling).
    skip, nb = 3, max(1, min(args.steps, 100))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(kernels) + 1)] for _ in range(skip + nb)]
    barrier()
    for i in range(skip + nb):
        s = sets[i % len(sets)]
        evs[i][0].record()
        for j, (_, fn) in enumerate(kernels):
            fn(s)
            evs[i][j + 1].record()
    barrier()
    live = {label: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(skip, skip + nb)) / nb
            for j, (label, _) in enumerate(kernels)}
    # ---- each kernel back to back: its launches over the rotating sets between two events and none
    # in between, so consecutive launches keep their overlap as in the step; these per-kernel times
    # add up to about the step time
    b2b = {label: time_back_to_back(fn, sets, max(8, min(args.steps, 50)), barrier) for label, fn in kernels}
    # ---- each kernel alone after an L2 flush; the clock sampler keeps running under this load
    flush = L2Flush(device)
    per = {label: time_cold(fn, sets, args.kernel_reps, flush) for label, fn in kernels}
    extra = {label: time_cold(fn, sets, args.kernel_reps, flush) for label, fn in other}
    del flush
    clk = clocks.stop()
    rc = lib.svdq_check_status()
    if rc != lib.OK:
        raise RuntimeError(f"device status after timing: {lib.status_name(rc)}")

    # ---- end to end through the public API, host buffers in and out.  Every step copies its
    # inputs in from pinned host memory and its outputs back out; the uploads, the kernels and
    # the downloads of consecutive steps run on three streams (the two DMA directions and the
    # compute stream), ordered by events, over the rotating device buffer sets.
    host_in = {"qkv": _bf(W.x_bits["qkv"]).pin_memory(), "fc1": _bf(W.x_bits["fc1"]).pin_memory(),
               "awq": _bf(W.awq_x_bits).pin_memory()}
    outs = (("qkv", (TOKENS, 3 * HIDDEN)), ("fc2", (TOKENS, HIDDEN)), ("awq", (AM, AN)))
    host_out = [{k: torch.empty(shape, dtype=torch.bfloat16, pin_memory=True) for k, shape in outs}
                for _ in range(2)]
    e_steps = max(3, min(args.steps, 20))
    main_s = torch.cuda.current_stream(device)
    in_s, out_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(e_steps)]
    ev_done = [torch.cuda.Event() for _ in range(e_steps)]
    ev_out = [torch.cuda.Event() for _ in range(e_steps)]
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(main_s)
    in_s.wait_event(e0)
    out_s.wait_event(e0)
    for i in range(e_steps):
        s = sets[i % len(sets)]
        with torch.cuda.stream(in_s):
            if i >= len(sets):
                in_s.wait_event(ev_done[i - len(sets)])    # the set's previous inputs have been consumed
            for k, v in host_in.items():
                s[k]["X"].copy_(v, non_blocking=True)
            ev_in[i].record(in_s)
        main_s.wait_event(ev_in[i])
        if i >= len(sets):
            main_s.wait_event(ev_out[i - len(sets)])       # the set's previous outputs have been read out
        step(sets, i, kernels)
        ev_done[i].record(main_s)
        with torch.cuda.stream(out_s):
            out_s.wait_event(ev_done[i])
            for k, _ in outs:
                host_out[i % 2][k].copy_(s[k]["Y"], non_blocking=True)
            ev_out[i].record(out_s)
    main_s.wait_event(ev_out[e_steps - 1])
    e1.record(main_s)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    h2d = sum(v.numel() * 2 for v in host_in.values())
    d2h = sum(v.numel() * 2 for v in host_out[0].values())

    # ---- reference points on this GPU: a library copy of the activation's size, and cuBLASLt's
    # NVFP4 GEMM on the fc1 shape
    floor_gbs, floor_us = copy_floor(device, TOKENS * HIDDEN * 2)
    awq_batch = awq_many_rows(W, device)
    pk_local, _ = peaks()
    int4_pass = int4_variant(W, device, pk_local)
    host_path = host_path_point(device)
    fp4_lib = fp4_library_point(device, *LAYERS["fc1"][:3]) if not args.no_library_points else "skipped"

    # ---- max over ranks
    labels = [label for label, _ in kernels]
    xlabels = [label for label, _ in other]
    vals = max_over_ranks([ms, e2e_ms] + [per[x] for x in labels] + [extra[x] for x in xlabels]
                          + [live[x] for x in labels] + [b2b[x] for x in labels], world, device)
    ms, e2e_ms = vals[0], vals[1]
    nl, nx = len(labels), len(xlabels)
    per = dict(zip(labels, vals[2:2 + nl]))
    extra = dict(zip(xlabels, vals[2 + nl:2 + nl + nx]))
    live = dict(zip(labels, vals[2 + nl + nx:2 + 2 * nl + nx]))
    b2b = dict(zip(labels, vals[2 + 2 * nl + nx:]))
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    pk, how = peaks()
    fp4_peak = pk["bf16_tflops"] * FP4_OVER_BF16
    ms_step = ms / args.steps
    table = kernel_table(pk)
    def entry(label, ms_, cold_ms=None, b2b_ms=None):
        amount, unit, bound, peak = table[label]

        def rate(t_ms):
            return amount / (t_ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
        e = {"us": round(ms_ * 1e3, 2), unit: round(rate(ms_), 1), "frac": round(rate(ms_) / peak, 4)}
        if b2b_ms is not None:
            e.update({"b2b_us": round(b2b_ms * 1e3, 2), "b2b_frac": round(rate(b2b_ms) / peak, 4)})
        if cold_ms is not None:
            e.update({"cold_us": round(cold_ms * 1e3, 2), "cold_frac": round(rate(cold_ms) / peak, 4)})
        return e

    ktab = {label: entry(label, live[label], per[label], b2b[label]) for label in labels}
    ktab["sum_us"] = round(sum(live.values()) * 1e3, 2)
    ktab["b2b_sum_us"] = round(sum(b2b.values()) * 1e3, 2)
    ktab["timing"] = (f"us/frac: mean over {nb} steps of the step's own launches, an event after every kernel "
                      "on the launching stream (those events cost the launch overlap, so sum_us exceeds "
                      "ms_per_step); b2b_us/b2b_frac: the kernel's own launches back to back over the rotating "
                      f"sets ({len(sets)}, each launch's data evicted from L2 by the others), between two events "
                      f"and none in between; cold_us/cold_frac: each kernel alone, mean of {args.kernel_reps} "
                      "launches, each after an L2 flush (a read of twice the L2 size) and between its own two "
                      "events")
    ktab[f"{'unfused' if args.mlp == 'fused' else 'fused'}_mlp_for_comparison"] = dict(
        {label: entry(label, extra[label]) for label in xlabels}, timing="alone after an L2 flush, like cold_us")
    m, k, n, _ = LAYERS["fc1"]
    if args.mlp == "fused":
        k2_label, k2_flops = "K2 fc1 -> fc2 operands", requant_flops()
    else:
        k2_label, k2_flops = "K2 fc1 (plain, bf16 out)", gemm_flops(m, k, n)
    k2_us = live[k2_label] * 1e3
    k2_tflops = k2_flops / (k2_us * 1e-6) / 1e12
    traffic = K2_TRAFFIC["bytes"] if K2_TRAFFIC["source_sha16"] == source_sha16() else None
    line = {
        "metric": METRIC,
        "value": round(aggregate_tflops(STEP_FLOPS, world, ms_step), 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3-scaled, fp32 accumulate); bf16 low-rank; int4 x bf16",
        "data": "synthetic (seeded; outlier channels/rows as in the workload)",
        "config": {"workload": WORKLOAD, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2; {len(sets)} rotating sets of weights, inputs and outputs, "
                         f"{len(sets) * set_bytes / 1e6:.0f} MB > 2x L2",
                   "flops_per_step": STEP_FLOPS, "launches_per_step": launches_per_step(args.mlp),
                   "mlp": ("fused: fc1's GEMM writes fc2's NVFP4 operands and U (no bf16 activation, no K1 for fc2)"
                           if args.mlp == "fused" else "unfused: fc1 writes its bf16 output, fc2's K1 reads it")},
        "roofline": {"bound": "tensor",
                     "kernel": ("svdq_linear_w4a4_requant, fc1 4608x3072x12288 +GELU re-quantized for fc2"
                                if args.mlp == "fused" else "svdq_linear_w4a4, fc1 4608x3072x12288 +GELU"),
                     "achieved": round(k2_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(k2_tflops / fp4_peak, 4), "traffic": traffic,
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_source": f"{how} bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/bf16)",
                     "frac_of_nominal_9pf": round(k2_tflops / FP4_NOMINAL_TFLOPS, 4),
                     "duration": "mean in-step duration of the launch (the kernels table's us)",
                     "algorithmic": ("2MKN (FP4) + 2MrN (low-rank up-projection) + 2MNr (fc2's low-rank "
                                     "down-projection in the epilogue) per launch" if args.mlp == "fused" else
                                     "2MKN (FP4) + 2MrN (low-rank up-projection) per launch")},
        "kernels": ktab,
        "awq_many_rows": awq_batch,
        "int4_w4a4": int4_pass,
        "host_path": host_path,
        "reference_points": {
            "hbm_copy_same_bytes": {"GB/s": round(floor_gbs, 1), "us": round(floor_us, 2),
                                    "what": f"torch copy of {TOKENS}x{HIDDEN} bf16, timed like the kernels "
                                            "(L2 flushed first; read + write)"},
            "cublaslt_nvfp4_fc1_shape": (
                {"TFLOP/s": round(fp4_lib[0], 1), "us": round(fp4_lib[1], 2),
                 "what": "torch._scaled_mm, NVFP4 A/B, block-16 e4m3 scales, bf16 out, no low-rank branch; timed "
                        "like the kernels (L2 flushed first)"}
                if isinstance(fp4_lib, tuple) else {"unavailable": fp4_lib}),
            "hbm_peak_gbs": pk["hbm_gbs"], "peak_source": how},
        "e2e": {"value": round(aggregate_tflops(STEP_FLOPS, world, e2e_ms), 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step(args.mlp) * args.steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(rows=16, reps=1)
    print(json.dumps(line))


# ------------------------------------------------------------------ oracle timing
class OracleWorkload:
    """The oracle's own packs of the step's layers (untimed) and its bounded samples (timed)."""

    def __init__(self):
        from bit_w4a4_diffusion_smooth_b200 import synthetic
        from oracle import awq as oawq
        from oracle import formats, svdquant

        self.f = formats
        self.sq = svdquant
        self.oawq = oawq
        self.x = {}
        self.p = {}
        self.b = {}
        for name, c in (("qkv", synthetic.QKV), ("fc1", synthetic.MLP_FC1)):
            xb, wb, bb = c.make()
            x = formats.bf16_bits_to_float(xb)
            self.x[name] = x
            self.p[name] = svdquant.pack(formats.bf16_bits_to_float(wb),
                                         np.max(np.abs(x), axis=0).astype(np.float32), RANK)
            self.b[name] = formats.bf16_bits_to_float(bb)
        c2 = synthetic.MLP_FC2
        wb2, _ = synthetic.weight(c2.k, c2.n, c2.seed, 0.02, c2.w_outlier_rows, c2.w_factor)
        self.b["fc2"] = formats.bf16_bits_to_float(synthetic.bias(c2.n, c2.seed + 100))
        # fc2's calibration: the oracle's own fc1 output on a sample of rows
        h = formats.bf16_round(svdquant.forward(self.x["fc1"][::36], self.p["fc1"], self.b["fc1"],
                                                svdquant.EPILOGUE_GELU_ERF))
        self.p["fc2"] = svdquant.pack(formats.bf16_bits_to_float(wb2),
                                      np.max(np.abs(h), axis=0).astype(np.float32), RANK)
        a = synthetic.AWQ
        axb, awb, abb, asc = a.make()
        ap = oawq.pack(formats.bf16_bits_to_float(awb), asc)
        self.awq = (formats.bf16_bits_to_float(axb), ap["inv_a"], ap["q"], ap["s"], ap["z"],
                    formats.bf16_bits_to_float(abb))

    def sample(self, rows):
        """`rows` rows of every SVDQ layer (fc2 on the oracle's fc1 output of those rows) and the
        whole AWQ projection; returns (FLOPs it stands for, seconds)."""
        sq, f = self.sq, self.f
        t = time.perf_counter()
        sq.forward(self.x["qkv"][:rows], self.p["qkv"], self.b["qkv"])
        h = sq.forward(self.x["fc1"][:rows], self.p["fc1"], self.b["fc1"], sq.EPILOGUE_GELU_ERF)
        sq.forward(f.bf16_round(h), self.p["fc2"], self.b["fc2"])
        self.oawq.linear(*self.awq)
        dt = time.perf_counter() - t
        flops = rows / TOKENS * sum(layer_flops(m, k, n) for m, k, n, _ in LAYERS.values()) + AWQ_FLOPS
        return flops, dt


def _cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(rows=16, reps=1):
    ow = OracleWorkload()
    flops = secs = 0.0
    for _ in range(reps):
        f, s = ow.sample(rows)
        flops += f
        secs += s
    # the same sample with numpy's BLAS held to one thread
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):
            f1, s1 = ow.sample(rows)
        one = round(f1 / s1 / 1e12, 6)
    except Exception:
        one = None
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "one_thread_value": one, "cpu_model": _cpu_model(),
            "sample": f"{rows} of {TOKENS} rows of each SVDQ layer (QKV, fc1, fc2 on fc1's output: quantize + "
                      f"two-branch float64 GEMM) + the full 2x3072->18432 AWQ projection, {reps} repetition(s); "
                      "the oracle's packs are untimed"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    ow = OracleWorkload()
    rows = 8
    for _ in range(args.warmup):
        ow.sample(rows)
    flops = secs = 0.0
    for _ in range(args.steps):
        f, s = ow.sample(rows)
        flops += f
        secs += s
    v = round(flops / secs / 1e12, 6)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (CPU oracle)",
        "data": "synthetic", "config": {"workload": WORKLOAD, "parallelism": "single host process"},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                         "sample": f"{rows} of {TOKENS} rows of each SVDQ layer + the full AWQ projection per "
                                   "step"},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------------------------ one DiT denoising step
DIT_METRIC = "DiT step: every projection linear (SVDQ W4A4 + AWQ W4A16), FLOP-weighted TFLOPS"


def dit_step_plan():
    """Layers of one step in execution order: (kind, name, m, k, n, gelu_col_begin or None)."""
    from bit_w4a4_diffusion_smooth_b200 import synthetic
    d = synthetic.DitStep()
    by_name = {name: (m, k, n, gelu, gbeg) for name, m, k, n, gelu, gbeg, _ in d.layers}
    plan = []
    for _ in range(d.dual_blocks):
        for stream in ("img", "txt"):
            plan.append(("awq", f"dual.{stream}.adaln", 2, d.hidden, 6 * d.hidden, None))
        for name in ("qkv", "out", "fc1", "fc2"):   # each projection on both streams (fc2 after fc1)
            for stream in ("img", "txt"):
                m, k, n, gelu, gbeg = by_name[f"dual.{stream}.{name}"]
                plan.append(("w4a4", f"dual.{stream}.{name}", m, k, n, gbeg if gelu else None))
    for _ in range(d.single_blocks):
        plan.append(("awq", "single.adaln", 2, d.hidden, 3 * d.hidden, None))
        for name in ("single.qkv_mlp", "single.out"):
            m, k, n, gelu, gbeg = by_name[name]
            plan.append(("w4a4", name, m, k, n, gbeg if gelu else None))
    return d, plan


def run_dit_step(args):
    """Every projection linear of one denoising step of a 12B-class DiT (19 dual-stream and 38
    single-stream blocks: 228 SVDQ W4A4 layers, each K1 + K2, and 76 AWQ W4A16 projections),
    on distinct random-valid packed weights, replayed as one CUDA graph.  fc2 reads fc1's
    output; the other layers read synthetic activations from rotating pools."""
    import torch

    from bit_w4a4_diffusion_smooth_b200 import lib

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_replicas(world, "nccl", device)
    lib.svdq_init(device.index)
    d, plan = dit_step_plan()
    r = d.rank
    gen = torch.Generator(device=device)
    gen.manual_seed(d.seed)

    def rand_bundle(nbytes):
        # valid NVFP4 bytes: e2m1 codes 0..7 in both nibbles, e4m3 scales <= 240 (no NaN)
        return torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device=device, generator=gen) & 0x77

    def rand_bf16(*shape, std=1.0):
        return (torch.randn(*shape, device=device, generator=gen) * std).to(torch.bfloat16)

    one_t = torch.ones(1, device=device)
    s_w = torch.full((1,), 1e-3, device=device)
    pools, act, layers = {}, {}, []
    cond = {}     # the modulation projections all read the step's conditioning vector
    for kind, name, m, k, n, gbeg in plan:
        if kind == "awq":
            g_n = k // 64
            if (m, k) not in cond:
                cond[(m, k)] = rand_bf16(m, k)
            layers.append(dict(kind=kind, m=m, k=k, n=n,
                               X=cond[(m, k)], inv=torch.ones(k, device=device),
                               qw=torch.randint(0, 2 ** 31, (k // 8 * n,), dtype=torch.int32, device=device,
                                                generator=gen),
                               sc=(torch.rand(g_n * n, device=device, generator=gen) * 1e-3).to(torch.bfloat16),
                               z=torch.randint(0, 16, (g_n * n,), device=device, generator=gen).to(torch.bfloat16),
                               b=rand_bf16(n, std=0.01), Y=torch.empty(m, n, dtype=torch.bfloat16, device=device)))
            continue
        ws = lib.svdq_weight_sizes(k, n, r)
        if (m, k) not in act:
            sz = lib.svdq_act_sizes(m, k)
            act[(m, k)] = (torch.empty(sz["a_bundle"], dtype=torch.uint8, device=device),
                           torch.empty(sz["u"], dtype=torch.uint8, device=device))
        if (m, k) not in pools:  # 6 rotating inputs per shape: more than L2 holds for the big ones
            pools[(m, k)] = [rand_bf16(m, k) for _ in range(6)]
        layers.append(dict(kind=kind, name=name, m=m, k=k, n=n, gbeg=gbeg,
                           inv=torch.ones(k, device=device), l1t=rand_bf16(r, k, std=0.02),
                           l2t=rand_bundle(ws["l2t"]) & 0x3F, w=rand_bundle(ws["w_bundle"]),
                           b=rand_bf16(n, std=0.01), Y=torch.empty(m, n, dtype=torch.bfloat16, device=device)))
    use = {}
    prev_fc1 = {}
    for L in layers:  # inputs: fc2 takes its stream's fc1 output, the rest a pool buffer
        if L["kind"] != "w4a4":
            continue
        if L["name"].endswith(".fc2"):
            L["X"] = prev_fc1[L["name"].rsplit(".", 1)[0]]
        else:
            key = (L["m"], L["k"])
            i = use.get(key, 0)
            use[key] = i + 1
            L["X"] = pools[key][i % 6]
        if L["name"].endswith(".fc1"):
            prev_fc1[L["name"].rsplit(".", 1)[0]] = L["Y"]

    # launch units: with --group-streams on, the image and text instances of a dual-stream block's
    # projection run as one grouped K1 and one grouped K2 launch (adjacent in the plan); with
    # --group-awq on, every modulation projection of the step (they depend only on the conditioning
    # vector) runs in one grouped AWQ launch at the start of the step
    units = []
    awq_layers = [L for L in layers if L["kind"] == "awq"]
    if args.group_awq == "on" and awq_layers:
        units.append(awq_layers)
    for L in layers:
        if args.group_awq == "on" and L["kind"] == "awq":
            continue
        prev = units[-1] if units else None
        if (args.group_streams == "on" and L["kind"] == "w4a4" and L["name"].startswith("dual.txt.") and prev
                and prev[0]["kind"] == "w4a4" and prev[0]["name"] == L["name"].replace(".txt.", ".img.")):
            prev.append(L)
        else:
            units.append([L])

    def run_unit(unit):
        L = unit[0]
        if L["kind"] == "awq" and len(unit) > 1:
            lib.awq_linear_w4a16_grouped([dict(X=u["X"], inv_awq=u["inv"], qweight=u["qw"], scales=u["sc"],
                                               zeros=u["z"], bias=u["b"], N=u["n"], Y=u["Y"]) for u in unit],
                                         L["m"], L["k"])
            return
        if L["kind"] == "awq":
            lib.awq_linear_w4a16(L["X"], L["inv"], L["qw"], L["sc"], L["z"], L["b"], L["n"], L["Y"])
            return
        epi = lib.EPILOGUE_GELU_ERF if L["gbeg"] is not None else lib.EPILOGUE_NONE
        if len(unit) == 1:
            ab, U = act[(L["m"], L["k"])]
            lib.svdq_quantize_act(L["X"], L["inv"], L["l1t"], r, one_t, s_w, ab, U)
            lib.svdq_linear_w4a4(ab, U, one_t, L["w"], L["l2t"], s_w, L["b"], L["m"], L["n"], L["k"], r, epi,
                                 L["gbeg"] or 0, L["Y"])
            return
        lib.svdq_quantize_act_grouped(
            [dict(X=u["X"], inv_lambda=u["inv"], l1t=u["l1t"], s_a=one_t, s_w=s_w, a_bundle=act[(u["m"], u["k"])][0],
                  U=act[(u["m"], u["k"])][1]) for u in unit], r)
        lib.svdq_linear_w4a4_grouped(
            [dict(a_bundle=act[(u["m"], u["k"])][0], U=act[(u["m"], u["k"])][1], s_a=one_t, w_bundle=u["w"],
                  l2t=u["l2t"], s_w=s_w, bias=u["b"], M=u["m"], N=u["n"], K=u["k"], gelu_col_begin=u["gbeg"] or 0,
                  Y=u["Y"]) for u in unit], r, epi)

    def step():
        for unit in units:
            run_unit(unit)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc = lib.svdq_check_status()
    if rc != lib.OK:
        raise RuntimeError(f"device status after warm-up: {lib.status_name(rc)}")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph.replay()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        graph.replay()
    t1.record()
    barrier()
    clk = clocks.stop()
    rc = lib.svdq_check_status()
    if rc != lib.OK:
        raise RuntimeError(f"device status after timing: {lib.status_name(rc)}")
    (ms,) = max_over_ranks([t0.elapsed_time(t1) / args.steps], world, device)
    del graph

    # per layer type: one instance's K1 + K2 (or K3) replayed back to back, times the count
    per_type = {}
    for L in layers:
        key = (L["kind"], L.get("name", "adaln"), L["m"], L["k"], L["n"])
        per_type.setdefault(key, [L, 0])[1] += 1
    breakdown = []
    for (kind, name, m, k, n), (L, cnt) in per_type.items():
        def one(L=L):
            if L["kind"] == "awq":
                lib.awq_linear_w4a16(L["X"], L["inv"], L["qw"], L["sc"], L["z"], L["b"], L["n"], L["Y"])
                return
            ab, U = act[(L["m"], L["k"])]
            lib.svdq_quantize_act(L["X"], L["inv"], L["l1t"], r, one_t, s_w, ab, U)
            epi = lib.EPILOGUE_GELU_ERF if L["gbeg"] is not None else lib.EPILOGUE_NONE
            lib.svdq_linear_w4a4(ab, U, one_t, L["w"], L["l2t"], s_w, L["b"], L["m"], L["n"], L["k"], r, epi,
                                 L["gbeg"] or 0, L["Y"])
        for _ in range(3):
            one()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            one()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / 10 * 1e3
        fl = 2 * m * k * n + (2 * m * r * (k + n) if kind == "w4a4" else 0)
        breakdown.append({"layer": name if kind == "w4a4" else f"{name} (AWQ)", "m": m, "k": k, "n": n,
                          "count": cnt, "us_each": round(us, 2), "TFLOP/s": round(fl / (us * 1e-6) / 1e12, 1),
                          "ms_per_step": round(us * cnt / 1e3, 3)})
    if args.group_awq == "on" and awq_layers:  # the grouped modulation launch alone
        for _ in range(3):
            run_unit(awq_layers)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            run_unit(awq_layers)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / 10 * 1e3
        wbytes = sum(L["n"] * L["k"] // 2 + 2 * 2 * L["n"] * (L["k"] // 64) for L in awq_layers)
        breakdown.append({"layer": f"all {len(awq_layers)} modulation projections (AWQ, one grouped launch)",
                          "us_each": round(us, 2), "count": 1, "ms_per_step": round(us / 1e3, 3),
                          "weight_GB/s": round(wbytes / (us * 1e-6) / 1e9, 1)})
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    w4a4 = sum(2 * L["m"] * L["k"] * L["n"] for L in layers if L["kind"] == "w4a4")
    lowrank = sum(2 * L["m"] * r * (L["k"] + L["n"]) for L in layers if L["kind"] == "w4a4")
    awq = sum(2 * L["m"] * L["k"] * L["n"] for L in layers if L["kind"] == "awq")
    flops = w4a4 + lowrank + awq
    n_w4a4 = sum(1 for L in layers if L["kind"] == "w4a4")
    n_awq = len(layers) - n_w4a4
    print(json.dumps({
        "metric": DIT_METRIC, "value": round(aggregate_tflops(flops, world, ms), 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3-scaled, fp32 accumulate); bf16 low-rank; int4 x bf16",
        "data": "synthetic (random-valid packed weights per layer; seeded activations)",
        "config": {"workload": "all projection linears of one denoising step of a 12B-class DiT: 19 dual-stream "
                               "blocks (img 4096 / txt 512 tokens: QKV 3072->9216, out 3072->3072, "
                               "fc1 3072->12288 +GELU, fc2 12288->3072) + 38 single-stream blocks (4608 tokens: "
                               "3072->21504 with GELU on the last 12288 columns, 15360->3072), rank 32; "
                               "adaLN AWQ 2x3072->18432 (x38) and 2x3072->9216 (x38)",
                   "parallelism": f"replicas x{world}", "graph": "one CUDA graph per step",
                   "group_streams": (f"{args.group_streams}: a dual-stream block's image and text instances of "
                                     "each projection run as one grouped K1 and one grouped K2 launch"
                                     if args.group_streams == "on" else "off: every layer its own launches"),
                   "group_awq": ("on: the step's modulation projections (one shared conditioning vector) run as "
                                 "one grouped AWQ launch" if args.group_awq == "on" else
                                 "off: every modulation projection its own launch"),
                   "layers": {"w4a4": n_w4a4, "awq": n_awq}, "flops_per_step": flops},
        "breakdown": breakdown,
        "gpu_launches": args.steps * sum(1 if u[0]["kind"] == "awq" else 2 for u in units),
        "clocks": clk,
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 300 for the layer step; 200 for --workload dit-step; 10 for "
                         "--impl reference)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-library-points", action="store_true",
                    help="skip the cuBLASLt NVFP4 reference point")
    ap.add_argument("--kernel-reps", type=int, default=20,
                    help="back-to-back launches per kernel for the per-kernel times")
    ap.add_argument("--mlp", choices=("fused", "unfused"), default=MLP_DEFAULT,
                    help="MLP pair: fc1's GEMM re-quantizing for fc2 (fused) or fc1 bf16 out + fc2 K1 (unfused)")
    ap.add_argument("--workload", choices=("layers", "dit-step"), default="layers",
                    help="layers: QKV + MLP pair + AWQ projection (default); dit-step: one whole DiT step")
    ap.add_argument("--group-streams", choices=("on", "off"), default="on",
                    help="dit-step: image and text instances of a dual-stream projection as one grouped launch")
    ap.add_argument("--group-awq", choices=("on", "off"), default="on",
                    help="dit-step: the step's modulation projections (one shared input) as one grouped AWQ launch")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = {"reference": 10}.get(args.impl, 300 if args.workload == "layers" else 200)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "dit-step":
        run_dit_step(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
