"""Concurrent calls from several host threads on their own streams, in a fresh process (see
tests/concurrency_case.py): each result must equal the same call made alone, bit for bit."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_entry_point_at_once_from_threads_and_streams():
    r = subprocess.run([sys.executable, "-m", "tests.concurrency_case"], cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    tail = (r.stdout + r.stderr)[-4000:]
    assert r.returncode == 0, f"exit {r.returncode}:\n{tail}"
    assert "CONCURRENCY ok" in r.stdout, tail
