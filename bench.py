"""Throughput of the SVDQuant W4A4 linear (+ AWQ W4A16 projection) on B200.

One step = the whole hot path over one batch of synthetic input:
  K1  activation quantize + low-rank down-projection   X [4608 x 3072] bf16
  K2  tcgen05 NVFP4 GEMM + low-rank up-projection      -> Y [4608 x 9216] bf16
  K3  AWQ W4A16 projection                             [2 x 3072] -> [2 x 18432]
(the attention-QKV-shaped layer of a 12B-class DiT at 1024x1024: 4096 image +
512 text tokens, rank 32; and its adaLN modulation projection).

value = algorithmic FLOPs of the step / step time (TFLOP/s, all ranks).
Inputs rotate over buffer sets that together exceed twice the L2 cache, so no
step reads what the previous one left in L2.  Multi-GPU runs are independent
replicas (the layer needs no exchange between GPUs): weak scaling.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload qkv|dit-step]

--workload dit-step times every projection linear of one denoising step of a
12B-class DiT (228 W4A4 layers + 76 AWQ projections) as one CUDA graph.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, K, N, RANK = 4608, 3072, 9216, 32
AM, AK, AN = 2, 3072, 18432
WORKLOAD = ("attention-QKV SVDQ W4A4 linear 4608x3072->9216 rank 32 (NVFP4, group 16) "
            "+ AWQ W4A16 adaLN projection 2x3072->18432 (INT4, group 64)")
METRIC = "SVDQ W4A4 linear TFLOPS and % of B200 dense-FP4 peak; W4A16 GB/s vs HBM"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / dense bf16 ratio (9 / 2.25 PFLOP/s)

W4A4_FLOPS = 2 * M * K * N                # 4-bit main branch
LOWRANK_FLOPS = 2 * M * K * RANK + 2 * M * RANK * N
AWQ_FLOPS = 2 * AM * AK * AN
STEP_FLOPS = W4A4_FLOPS + LOWRANK_FLOPS + AWQ_FLOPS
# Algorithmic bytes per launch (each byte the kernel must move once).
K1_BYTES = (M * K * 2 + K * RANK * 2 + K * 4            # X, L1T, inv_lambda
            + M * K // 2 + M * K // 16 + M * RANK * 2)  # codes, scales, U
K2_BYTES = (M * K // 2 + M * K // 16 + M * RANK * 2     # activation codes, scales, U
            + N * K // 2 + N * K // 16 + N * RANK * 2   # weight codes, scales, L2T
            + N * 2 + M * N * 2)                        # bias, Y
K3_BYTES = (AN * AK // 2 + 2 * AN * (AK // 64) * 2    # qweight, scales + zeros
            + AM * AK * 2 + AK * 4 + AN * 2 + AM * AN * 2)
# DRAM bytes of one K2 launch (dram__bytes_read.sum + dram__bytes_write.sum) from the ncu capture
# summarised in profiles/gemm_w4a4_qkv_4608x3072x9216.md; None until that capture matches the
# current K2 again.
K2_TRAFFIC_BYTES = 33_172_992 + 46_266_880
# Steps of the timed region that carry per-kernel CUDA events (1 in EV_EVERY).
EV_EVERY = 16


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return PEAKS_FALLBACK, "fallback"


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
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
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
def setup(device, sets):
    import torch

    from bit_w4a4_diffusion_smooth_b200 import lib, synthetic

    lib.svdq_init(device.index)
    c = synthetic.QKV
    xb, wb, bb = c.make()
    x = synthetic.bf16_bits_to_f32(xb)
    amax = np.max(np.abs(x), axis=0).astype(np.float32)
    packed = lib.svdq_pack_weights(wb, amax, RANK, seed=c.seed)
    a = synthetic.AWQ
    axb, awb, abb, asc = a.make()
    apk = lib.awq_pack_weights(awb, asc)

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

    def t(arr):
        return torch.from_numpy(np.ascontiguousarray(arr))

    host = dict(X=bf(xb).pin_memory(), AX=bf(axb).pin_memory())
    sz = lib.svdq_act_sizes(M, K)
    S = []
    for _ in range(sets):
        S.append(dict(
            X=bf(xb).to(device), inv_lambda=t(packed["inv_lambda"]).to(device), l1t=bf(packed["l1t"]).to(device),
            l2t=t(packed["l2t"]).to(device), w_bundle=t(packed["w_bundle"]).to(device),
            s_w=t(packed["s_w"]).to(device), s_a=t(packed["s_a"]).to(device), bias=bf(bb).to(device),
            a_bundle=torch.empty(sz["a_bundle"], dtype=torch.uint8, device=device),
            U=torch.empty(sz["u"], dtype=torch.uint8, device=device),
            Y=torch.empty((M, N), dtype=torch.bfloat16, device=device),
            AX=bf(axb).to(device), qweight=t(apk["qweight"]).to(device), ascales=bf(apk["scales"]).to(device),
            azeros=bf(apk["zeros"]).to(device), inv_awq=t(apk["inv_awq"]).to(device), abias=bf(abb).to(device),
            AY=torch.empty((AM, AN), dtype=torch.bfloat16, device=device)))
    set_bytes = sum(v.numel() * v.element_size() for v in S[0].values())
    return S, host, set_bytes


def step(S, i, ev=None):
    from bit_w4a4_diffusion_smooth_b200 import lib
    s = S[i % len(S)]
    if ev is not None:
        ev[0].record()
    lib.svdq_quantize_act(s["X"], s["inv_lambda"], s["l1t"], RANK, s["s_a"], s["s_w"], s["a_bundle"], s["U"])
    if ev is not None:
        ev[1].record()
    lib.svdq_linear_w4a4(s["a_bundle"], s["U"], s["s_a"], s["w_bundle"], s["l2t"], s["s_w"], s["bias"],
                         M, N, K, RANK, 0, 0, s["Y"])
    if ev is not None:
        ev[2].record()
    lib.awq_linear_w4a16(s["AX"], s["inv_awq"], s["qweight"], s["ascales"], s["azeros"], s["abias"], AN, s["AY"])
    if ev is not None:
        ev[3].record()


def run_ours(args):
    import torch
    import torch.distributed as dist

    from bit_w4a4_diffusion_smooth_b200 import lib

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_replicas(world, "nccl", device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    sets = 4
    S, host, set_bytes = setup(device, sets)
    while sets * set_bytes < 2 * l2:
        sets += 1
        S, host, set_bytes = setup(device, sets)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(args.warmup):
        step(S, i)
    rc = lib.svdq_check_status()
    if rc != lib.OK:
        raise RuntimeError(f"device status after warm-up: {lib.status_name(rc)}")

    # ---- device-timed region: K steps; per-kernel events on every EV_EVERY-th step only, since an
    # event between two kernels keeps the next one from launching early (dependent launches)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(0, args.steps, EV_EVERY)]
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        step(S, i, evs[i // EV_EVERY] if i % EV_EVERY == 0 else None)
    t1.record()
    barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    k1 = sum(e[0].elapsed_time(e[1]) for e in evs) / len(evs)
    k2 = sum(e[1].elapsed_time(e[2]) for e in evs) / len(evs)
    k3 = sum(e[2].elapsed_time(e[3]) for e in evs) / len(evs)
    rc = lib.svdq_check_status()
    if rc != lib.OK:
        raise RuntimeError(f"device status after timing: {lib.status_name(rc)}")

    # ---- end to end through the public API, host buffers in and out.  Every step copies its
    # inputs in from pinned host memory and its outputs back out; the uploads, the kernels and
    # the downloads of consecutive steps run on three streams (the two DMA directions and the
    # compute stream), ordered by events, over the rotating device buffer sets.
    yh = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    ayh = [torch.empty((AM, AN), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
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
        s = S[i % len(S)]
        with torch.cuda.stream(in_s):
            if i >= len(S):
                in_s.wait_event(ev_done[i - len(S)])    # the set's previous inputs have been consumed
            s["X"].copy_(host["X"], non_blocking=True)
            s["AX"].copy_(host["AX"], non_blocking=True)
            ev_in[i].record(in_s)
        main_s.wait_event(ev_in[i])
        if i >= len(S):
            main_s.wait_event(ev_out[i - len(S)])       # the set's previous outputs have been read out
        step(S, i)
        ev_done[i].record(main_s)
        with torch.cuda.stream(out_s):
            out_s.wait_event(ev_done[i])
            yh[i % 2].copy_(s["Y"], non_blocking=True)
            ayh[i % 2].copy_(s["AY"], non_blocking=True)
            ev_out[i].record(out_s)
    main_s.wait_event(ev_out[e_steps - 1])
    e1.record(main_s)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e_steps

    # ---- max over ranks
    ms, k1, k2, k3, e2e_ms = max_over_ranks([ms, k1, k2, k3, e2e_ms], world, device)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    pk, how = peaks()
    fp4_peak = pk["bf16_tflops"] * FP4_OVER_BF16
    ms_step = ms / args.steps
    k2_tflops = (W4A4_FLOPS + 2 * M * RANK * N) / (k2 * 1e-3) / 1e12
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
                   "l2": f"{len(S)} rotating input/output sets, {len(S) * set_bytes / 1e6:.0f} MB > 2x L2",
                   "flops_per_step": STEP_FLOPS},
        "roofline": {"bound": "tensor", "kernel": "svdq_linear_w4a4 (K2)",
                     "achieved": round(k2_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(k2_tflops / fp4_peak, 4), "traffic": K2_TRAFFIC_BYTES,
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_source": f"{how} bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/bf16)"},
        "kernels": {
            "K1_quantize_act": {"us": round(k1 * 1e3, 2), "GB/s": round(K1_BYTES / (k1 * 1e-3) / 1e9, 1),
                                "frac_hbm": round(K1_BYTES / (k1 * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
            "K2_linear_w4a4": {"us": round(k2 * 1e3, 2), "TFLOP/s": round(k2_tflops, 1),
                               "frac_fp4": round(k2_tflops / fp4_peak, 4)},
            "K3_awq_w4a16": {"us": round(k3 * 1e3, 2), "GB/s": round(K3_BYTES / (k3 * 1e-3) / 1e9, 1),
                             "frac_hbm": round(K3_BYTES / (k3 * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
            "hbm_peak_gbs": pk["hbm_gbs"], "peak_source": how,
            "events_on": f"{len(evs)} of {args.steps} timed steps (per-kernel CUDA events)",
        },
        "e2e": {"value": round(aggregate_tflops(STEP_FLOPS, world, e2e_ms), 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2 + AM * AK * 2, "d2h_bytes_per_step": M * N * 2 + AM * AN * 2},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(rows=64, reps=2)
    print(json.dumps(line))


# ------------------------------------------------------------------ oracle timing
def oracle_sample(rows, x, packed, bb, awq_case):
    """One bounded sample of the step on the CPU oracle; returns (flops, seconds)."""
    from oracle import awq as oawq
    from oracle import formats, svdquant

    def bf(bits):
        return formats.bf16_bits_to_float(np.asarray(bits, np.uint16))

    l1, l2, w_codes, w_sf = packed["l1"], packed["l2"], packed["w_codes"], packed["w_sf"]
    axb, ainv, aq, as_, az, abias = awq_case
    t = time.perf_counter()
    codes, sf, u = svdquant.quantize_act(x[:rows], packed["inv_lambda"], l1, packed["s_a"], packed["s_w"])
    svdquant.w4a4_linear(codes, sf, packed["s_a"], w_codes, w_sf, packed["s_w"], u, l2, bf(bb))
    oawq.linear(axb, ainv, aq, as_, az, abias)
    dt = time.perf_counter() - t
    flops = rows / M * (W4A4_FLOPS + LOWRANK_FLOPS) + AWQ_FLOPS
    return flops, dt


def _oracle_inputs():
    from bit_w4a4_diffusion_smooth_b200 import synthetic
    from oracle import awq as oawq
    from oracle import formats, svdquant

    c = synthetic.QKV
    xb, wb, bb = c.make()
    x = formats.bf16_bits_to_float(xb)
    # the oracle's own pack; its cost is not part of the timed sample
    packed = svdquant.pack(formats.bf16_bits_to_float(wb), np.max(np.abs(x), axis=0).astype(np.float32), RANK)
    a = synthetic.AWQ
    axb, awb, abb, asc = a.make()
    ap = oawq.pack(formats.bf16_bits_to_float(awb), asc)
    awq_case = (formats.bf16_bits_to_float(axb), ap["inv_a"], ap["q"], ap["s"], ap["z"], formats.bf16_bits_to_float(abb))
    return x, packed, bb, awq_case


def _cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(rows=64, reps=2):
    x, packed, bb, awq_case = _oracle_inputs()
    flops = secs = 0.0
    for _ in range(reps):
        f, s = oracle_sample(rows, x, packed, bb, awq_case)
        flops += f
        secs += s
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": f"{rows} of {M} rows of the QKV layer (quantize + two-branch float64 GEMM) + the full "
                      f"2x3072->18432 AWQ projection, {reps} repetitions"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    x, packed, bb, awq_case = _oracle_inputs()
    rows = 32
    for _ in range(args.warmup):
        oracle_sample(rows, x, packed, bb, awq_case)
    flops = secs = 0.0
    for _ in range(args.steps):
        f, s = oracle_sample(rows, x, packed, bb, awq_case)
        flops += f
        secs += s
    v = round(flops / secs / 1e12, 6)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (CPU oracle)",
        "data": "synthetic", "config": {"workload": WORKLOAD, "parallelism": "single host process"},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                         "sample": f"{rows} of {M} rows of the QKV layer + the full AWQ projection per step"},
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
        for stream in ("img", "txt"):
            for name in ("qkv", "out", "fc1", "fc2"):
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
    for kind, name, m, k, n, gbeg in plan:
        if kind == "awq":
            g_n = k // 64
            layers.append(dict(kind=kind, m=m, k=k, n=n,
                               X=rand_bf16(m, k), inv=torch.ones(k, device=device),
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

    def step():
        for L in layers:
            if L["kind"] == "awq":
                lib.awq_linear_w4a16(L["X"], L["inv"], L["qw"], L["sc"], L["z"], L["b"], L["n"], L["Y"])
                continue
            ab, U = act[(L["m"], L["k"])]
            lib.svdq_quantize_act(L["X"], L["inv"], L["l1t"], r, one_t, s_w, ab, U)
            epi = lib.EPILOGUE_GELU_ERF if L["gbeg"] is not None else lib.EPILOGUE_NONE
            lib.svdq_linear_w4a4(ab, U, one_t, L["w"], L["l2t"], s_w, L["b"], L["m"], L["n"], L["k"], r, epi,
                                 L["gbeg"] or 0, L["Y"])

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
                   "layers": {"w4a4": n_w4a4, "awq": n_awq}, "flops_per_step": flops},
        "breakdown": breakdown,
        "gpu_launches": args.steps * (2 * n_w4a4 + n_awq),
        "clocks": clk,
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 3000 for the layer step, about 0.4 s timed, so that the clock "
                         "sampler sees the timed region; 200 for --workload dit-step and --impl reference)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=("qkv", "dit-step"), default="qkv",
                    help="qkv: the QKV layer + AWQ projection (default); dit-step: one whole DiT step")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 3000 if (args.impl == "ours" and args.workload == "qkv") else 200
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
