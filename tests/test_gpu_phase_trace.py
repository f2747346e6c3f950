"""The tracing build of the library (per-phase timestamps of the step
kernel): it builds, runs steps exactly like the product build (in its own
process, so this process keeps the product library), and every CTA's
phases come in order."""
import os
import re
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_phase_trace_runs_in_order():
    res = subprocess.run([sys.executable, "-m", "sparse_long_context_mse_b200.phase_trace",
                          "gqa32x8_L16384_B16"], cwd=ROOT, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    last = res.stdout.strip().split("step ")[-1]
    med = {int(m.group(1)): float(m.group(2))
           for m in re.finditer(r"^\s+(\d+) .*?med\s+([-\d.]+)", last, re.M)}
    assert med[0] == 0.0 or med[0] < 1.0
    order = [0, 1, 2, 3, 4, 5, 8, 9, 10, 11, 12, 14, 15, 16, 17, 18]
    meds = [med[i] for i in order if i in med]
    assert len(meds) >= 12 and meds == sorted(meds)
