"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks (replicas, no data
exchange) agree on the slowest rank's time, the whole-job throughput counts every
rank's tokens, and the reference arm runs on rank 0 only."""
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
