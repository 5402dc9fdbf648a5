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


def test_layer_step_flops_and_kernels():
    """The default step: QKV, MLP fc1 (+GELU) and fc2 on fc1's output, each K1 + K2, then K3."""
    def layer(m, k, n, r=32):
        return 2 * m * k * n + 2 * m * r * (k + n)
    want = layer(4608, 3072, 9216) + layer(4608, 3072, 12288) + layer(4608, 12288, 3072) + 2 * 2 * 3072 * 18432
    assert bench.STEP_FLOPS == want
    labels = [label for label, _ in bench.step_kernels("fused")]
    assert labels == ["K1 qkv", "K2 qkv", "K1 fc1", "K2 fc1 -> fc2 operands", "K2 fc2", "K3 adaLN"]
    labels = [label for label, _ in bench.step_kernels("unfused")]
    assert labels == ["K1 qkv", "K2 qkv", "K1 fc1", "K2 fc1 (plain, bf16 out)", "K1 fc2 (on fc1's bf16 out)",
                      "K2 fc2", "K3 adaLN"]
    assert bench.LAYERS["fc1"] == (4608, 3072, 12288, True)
    assert bench.launches_per_step("fused") == 7           # the re-quantizing call also runs its finalize kernel
    assert bench.launches_per_step("unfused") == 7
    assert bench.requant_flops() == 2 * 4608 * 3072 * 12288 + 2 * 4608 * 32 * 12288 * 2


def test_kernel_table_units():
    t = bench.kernel_table({"hbm_gbs": 6000.0, "bf16_tflops": 1500.0})
    assert t["K2 fc1"] == (2 * 4608 * 3072 * 12288 + 2 * 4608 * 32 * 12288, "TFLOP/s", "tensor", 6000.0)
    assert t["K1 qkv"][0] == 4608 * 3072 * 2 + 3072 * 32 * 2 + 3072 * 4 + 4608 * 3072 // 2 + 4608 * 3072 // 16 \
        + 4608 * 32 * 2
    assert t["K3 adaLN"][1:] == ("GB/s", "hbm", 6000.0)
