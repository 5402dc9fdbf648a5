import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


def pytest_terminal_summary(terminalreporter):
    """Both measures of every GPU parity comparison of the session (excess and raw row-RMS error)."""
    mod = sys.modules.get("tests.gpu_util")
    rows = getattr(mod, "PARITY", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.section("parity: excess / raw row-RMS error")
    for r in rows:
        flag = "" if r["raw_within_tol"] else "   (raw above tol: only the excess bar holds)"
        tr.write_line(f"{r['excess']:.3e}  {r['raw']:.3e}  {r['test']} {r['case']}{flag}")
    out = os.environ.get("PARITY_REPORT")
    if out:
        import json
        with open(out, "w") as f:
            json.dump(rows, f, indent=1)
