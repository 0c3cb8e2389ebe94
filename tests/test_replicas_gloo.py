"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks (replicas, no data
exchange) agree on the slowest rank's time, the whole-job throughput counts every
rank's tokens, the reference arm runs on rank 0 only, and the whole line is
assembled from per-rank measurements (stubbed layer timings) the same way on
every rank."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        bench = _load_bench()
        # Rank r measured (10 + r) ms for its steps and (20 - r) ms end to end.
        got = bench.max_over_ranks([10.0 + rank, 20.0 - rank], world, "cpu")
        value = bench.replica_throughput(128, world, got[0], 5)
        # The reference arm: every rank but 0 returns without work or output.
        out = io.StringIO()
        if rank != 0:
            with redirect_stdout(out):
                r = bench.run_reference(None, None)
            ref_silent = r is None and out.getvalue() == ""
        else:
            ref_silent = True
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, got, value, ref_silent, None))
    except Exception as e:   # report to the parent instead of hanging it
        q.put((rank, None, None, None, repr(e)))


def test_two_replica_ranks_take_the_slowest_time_and_count_all_tokens():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, got, value, ref_silent, err = q.get(timeout=120)
        assert err is None, f"rank {rank}: {err}"
        res[rank] = (got, value, ref_silent)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        got, value, ref_silent = res[rank]
        assert got == [11.0, 20.0]                      # max over ranks, element-wise
        assert value == pytest.approx(128 * 2 / (11.0e-3 / 5))
        assert ref_silent


def _stub_measurements(bench, rank):
    """What measure_rank returns on a GPU, with made-up times: rank r is slower
    by r ms per step on the headline and by 2r ms on each per-config entry."""
    from workloads.synth import WORKLOADS
    wl = WORKLOADS["mxfp4"].with_tokens(32768)
    steps = 4
    split = {"route_gather": [0.5] * steps, "fc1_fc2": [14.0 + rank] * steps,
             "combine": [0.4] * steps, "route_alone": [0.2] * steps}
    main = {"wl": wl, "step_ms": [15.0 + rank] * steps, "eager_ms": [15.5] * steps,
            "split": split, "e2e_ms": [20.0 - rank] * steps, "h2d": 1000, "d2h": 2000,
            "clocks": {"sm_mhz": 1500.0, "reasons": []}, "active": 48, "alg_bytes": 10 ** 9,
            "w_bytes": 9 * 10 ** 8, "pairs": False, "tiled": False, "chunked": True, "swap": 2,
            "launches": 5}
    per = []
    for name, tokens in (("decode", None), ("mxfp4", 128)):
        w = WORKLOADS[name] if tokens is None else WORKLOADS[name].with_tokens(tokens)
        per.append({"wl": w, "step_ms": [0.25 + 2 * rank] * 3,
                    "split": {"route_gather": [0.02] * 3, "fc1_fc2": [0.2] * 3,
                              "combine": [0.01] * 3},
                    "active": 28, "alg_bytes": 10 ** 9, "w_bytes": 10 ** 9, "pairs": False,
                    "clocks": {"sm_mhz": 1600.0, "reasons": ["sw_power_cap"]}})
    return main, per


def _line_rank(rank, world, port, q):
    import datetime
    import types

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        bench = _load_bench()
        main, per = _stub_measurements(bench, rank)
        args = types.SimpleNamespace(warmup=3)
        line = bench.assemble_line(args, world, "cpu", main, per, None)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, line, None))
    except Exception as e:   # report to the parent instead of hanging it
        import traceback
        q.put((rank, None, traceback.format_exc()))


def test_two_replica_ranks_assemble_the_same_line():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_line_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    lines = {}
    for _ in range(world):
        rank, line, err = q.get(timeout=120)
        assert err is None, f"rank {rank}: {err}"
        lines[rank] = line
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert lines[0] == lines[1]                     # every rank computes the same line
    line = lines[0]
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    # slowest rank: 16 ms per step; both ranks' tokens count
    assert line["ms_per_step"] == pytest.approx(16.0)
    assert line["value"] == pytest.approx(2 * 32768 / 16e-3, rel=1e-6)
    assert line["e2e"]["value"] == pytest.approx(2 * 32768 / 20e-3, rel=1e-6)
    assert line["roofline"]["bound"] == "tensor"
    flops = 6.0 * 32768 * 6 * 7168 * 3072
    assert line["roofline"]["achieved"] == pytest.approx(flops / 15e-3 / 1e12, abs=0.1)
    dec, fp4 = line["per_config"]
    assert dec["workload"] == "decode" and fp4["workload"] == "mxfp4@T=128"
    assert dec["ms_per_step"] == pytest.approx(2.25)     # max over ranks: 0.25 + 2
    assert dec["tokens_per_s"] == pytest.approx(2 * 128 / 2.25e-3, rel=1e-6)
    assert dec["roofline"]["bound"] == "hbm"
    assert line["gpu_launches"] == 5 * 4
    assert line["kernels_ms"]["fc1_fc2"] == pytest.approx(15.0)   # the slower rank's split
