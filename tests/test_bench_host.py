"""Host-side arithmetic of bench.py that needs no GPU: the algorithmic bytes
of the launches around the GEMM and their GB/s, checked against sums worked by
hand for the decode layer (T=128, H=7168, E=32, top-8, FP8 x) and the BF16
variant of the same shape."""
import os

import pytest

from workloads.synth import WORKLOADS

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_side_kernel_bytes_decode():
    b = _load_bench().side_kernel_bytes(WORKLOADS["decode"])
    # route: 1024 ids in (4 KiB); perm + inv out (8 KiB); 32 counts + 33 offsets.
    assert b["route_alone"] == 4096 + 8192 + 65 * 4
    # gather: 128 token rows read + 1024 slot rows written, 7168 B + 56 scale
    # bytes each; 1024 perm entries read.
    assert b["gather_alone"] == 1152 * 7224 + 4096
    assert b["route_gather"] == b["route_alone"] + b["gather_alone"]
    # combine: 1024 bf16 y rows + weights + inv in, 128 bf16 rows out.
    assert b["combine"] == 1024 * 14336 + 8192 + 128 * 14336


def test_side_kernel_bytes_bf16_has_no_scales():
    wl = WORKLOADS["bf16"]
    b = _load_bench().side_kernel_bytes(wl)
    assert b["gather_alone"] == (wl.T + wl.S) * wl.H * 2 + wl.S * 4


def test_kernels_gbs_uses_mean_time_and_skips_missing():
    bench = _load_bench()
    wl = WORKLOADS["decode"]
    split = {"combine": [0.01, 0.03], "fc1_fc2": [0.2], "route_alone": []}
    g = bench.kernels_gbs(wl, split)
    assert set(g) == {"combine"}
    assert g["combine"] == pytest.approx(bench.side_kernel_bytes(wl)["combine"] / 0.02e-3 / 1e9,
                                         abs=0.05)


def test_reference_arm_line_on_the_small_config():
    """The oracle arm runs on the host alone and prints one line with the
    contract's keys and the workload-defining config keys of the other arm."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "1"], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    wl = WORKLOADS["tiny"]
    want = _load_bench().workload_config(wl, line["config"]["active_experts"])
    assert {k: line["config"][k] for k in want} == want
    assert 1 <= line["config"]["active_experts"] <= wl.E
    assert line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_gpus_without_a_launcher_respawns_under_torchrun(monkeypatch):
    """`bench.py --gpus N` with no WORLD_SIZE in the environment starts N ranks
    of the same command under torch.distributed.run (one process per GPU, the
    rendezvous on 127.0.0.1) and exits with its status."""
    import sys
    bench = _load_bench()
    calls = []
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: calls.append(cmd) or 0)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "7"])
    with pytest.raises(SystemExit) as ei:
        bench.main()
    assert ei.value.code == 0
    (cmd,) = calls
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "7"]


def test_gpus_disagreeing_with_world_size_is_refused(monkeypatch):
    import sys
    bench = _load_bench()
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4"])
    with pytest.raises(SystemExit) as ei:
        bench.main()
    assert "WORLD_SIZE=2" in str(ei.value.code)


def test_forwards_mode_dispatches_without_timing(monkeypatch):
    """--forwards N runs only the profiler's launches (run_forwards) on the
    workload and tokens given, never the timed benchmark or the oracle arm."""
    import sys
    bench = _load_bench()
    seen = []
    monkeypatch.setattr(bench, "run_forwards", lambda args, wl: seen.append((args.forwards, wl.name)))
    monkeypatch.setattr(bench, "run_b200", lambda args: pytest.fail("timed run started"))
    monkeypatch.setattr(bench, "run_reference", lambda args, wl: pytest.fail("oracle arm started"))
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "mxfp4", "--tokens", "128",
                                      "--forwards", "4"])
    bench.main()
    assert seen == [(4, bench.workload("mxfp4", 128).name)]
