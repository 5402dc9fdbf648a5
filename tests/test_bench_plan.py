"""Host-side checks of the benchmark's workloads (no GPU): the DiT-step layer plan matches the
12B-class DiT layer list (228 SVDQ W4A4 layers, 76 AWQ projections, 5.949e13 W4A4 FLOP)."""
import collections
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_dit_step_plan_counts_and_flops():
    d, plan = bench.dit_step_plan()
    kinds = collections.Counter(p[0] for p in plan)
    assert kinds == {"w4a4": 228, "awq": 76}
    assert sum(2 * m * k * n for kind, _, m, k, n, _ in plan if kind == "w4a4") == d.w4a4_flops() == 59489592016896
    shapes = collections.Counter((name, m, k, n, g) for kind, name, m, k, n, g in plan)
    assert shapes[("single.qkv_mlp", 4608, 3072, 21504, 9216)] == 38      # GELU on the MLP columns only
    assert shapes[("dual.img.fc1", 4096, 3072, 12288, 0)] == 19
    assert shapes[("dual.txt.fc2", 512, 12288, 3072, None)] == 19
    assert shapes[("dual.img.adaln", 2, 3072, 18432, None)] == 19
    assert shapes[("single.adaln", 2, 3072, 9216, None)] == 38


def test_dit_step_plan_orders_fc1_before_its_fc2():
    _, plan = bench.dit_step_plan()
    names = [p[1] for p in plan]
    for stream in ("img", "txt"):
        fc1 = [i for i, n in enumerate(names) if n == f"dual.{stream}.fc1"]
        fc2 = [i for i, n in enumerate(names) if n == f"dual.{stream}.fc2"]
        assert len(fc1) == len(fc2) == 19
        assert all(a < b for a, b in zip(fc1, fc2))


def test_qkv_step_flops():
    assert bench.STEP_FLOPS == 2 * 4608 * 3072 * 9216 + 2 * 4608 * 32 * (3072 + 9216) + 2 * 2 * 3072 * 18432
