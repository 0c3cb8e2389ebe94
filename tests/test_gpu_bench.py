"""bench.py's profiling mode on the GPU: `--forwards N` runs the launches the
committed profiler commands capture (N forwards of a workload in the
benchmark's launch configuration) and nothing else."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def test_bench_forwards_mode_runs_the_layer():
    """Two forwards of the small layer through this library: exit 0 with the
    device error word clear (the mode checks it) and one status line."""
    r = subprocess.run([sys.executable, "bench.py", "--workload", "tiny", "--forwards", "2"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().splitlines()[-1] == "tiny: 2 forwards"
