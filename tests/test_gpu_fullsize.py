"""Full-size parity, every element, one child process per case.

Each case of ``tests/fullsize_cases.py`` runs in a fresh Python process: a sticky CUDA
fault (which poisons the rest of a process's CUDA context) fails that case alone, and the
other cases still run. The child's report (element counts, LoRA ulp statistics, the largest
error relative to its bound) is printed with ``pytest -s`` and kept in the failure message.
"""
import json
import os
import subprocess
import sys

import pytest

from tests.fullsize_cases import CASES

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("case", list(CASES))
def test_full_size_every_element(case):
    r = subprocess.run([sys.executable, "-m", "tests.fullsize_cases", case], cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-4000:]
    assert r.returncode == 0, f"{case} failed (exit {r.returncode}):\n{tail}"
    reports = [ln[len("REPORT "):] for ln in r.stdout.splitlines() if ln.startswith("REPORT ")]
    assert reports, tail
    print(json.dumps(json.loads(reports[-1])))
