"""Throughput benchmark of the fused MoE expert layer on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl {b200,reference}]

One step = one whole layer (route, gather, FC1 + SwiGLU + FP8 requant, FC2,
combine) over one batch of seeded synthetic inputs already resident in HBM.
The headline workload is the largest configuration that fits one GPU: the
FP8-activation x MXFP4-weight layer at T=32768 (H=7168, I=3072, E=48, top-6);
`per_config` adds a shorter record (tokens/s, step time, fused-GEMM time and
its roofline fraction) of every configuration: decode, prefill, OAI, the BF16
variant and MXFP4 at 128, 1024, 8192 and 32768 tokens.  With N > 1 (launched
by torch.distributed.run, or started by `--gpus N` itself) every
rank runs its own replica of the layer on its own GPU: the path has no exchange
step, so there is no collective on the data path (weak scaling); the elapsed
device time is the maximum over ranks.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream; L2 is flushed (a 256 MiB buffer is overwritten)
before every timed step, outside the events.  `e2e` times K steps through the
C ABI's host-buffer entry point (moe_forward_hostio_batches: every step's
pinned host inputs copied in and its output copied back, overlapped with the
neighbouring steps' layers, all inside the events; the weights are larger
than L2).

`--impl reference` times the float64 CPU oracle on the host cores instead (a
bounded sample of the workload's tokens per step) and prints the same line.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and achieved TFLOPS or HBM GB/s vs roofline, 1×B200"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _dist():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix=f"moe_clocks_gpu{gpu_index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "window": "continuous steps of the same layer around the timed steps, the "
                          "eager steps and the per-kernel split"}


KERNEL_SOURCES = ("moe_expert_ffn_permute_b200/csrc/gemm.cu",
                  "moe_expert_ffn_permute_b200/csrc/gemm2.cu",
                  "moe_expert_ffn_permute_b200/csrc/sm100.cuh",
                  "moe_expert_ffn_permute_b200/csrc/sm100_pair.cuh",
                  "moe_expert_ffn_permute_b200/csrc/internal.h")


def _strip_comments(src):
    """C++ source without comments and blank lines (string literals in these
    kernel sources hold no comment markers)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash():
    """Hash of the GEMM kernel sources' code (comments and blank lines do not
    count), which the recorded DRAM traffic is valid for."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload):
    """DRAM bytes per launch of the GEMM kernel from the committed ncu summary
    (profiles/gemm_traffic.json), or None when the kernel sources changed since
    the counters were taken or no capture exists for this workload."""
    try:
        with open(os.path.join(ROOT, "profiles", "gemm_traffic.json")) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


def algorithmic_bytes(wl, d):
    """Bytes the layer must move at minimum: the weights and scales of the
    experts that receive tokens, x and its scales, the routing, the output."""
    import torch
    counts = torch.bincount(d["topk_idx"].reshape(-1).long(), minlength=wl.E)[:wl.E]
    active = int((counts > 0).sum())
    def nbytes(t):
        return 0 if t is None else t.numel() * t.element_size()
    per_expert_w = sum(nbytes(d[k][0]) if d[k] is not None else 0
                       for k in ("w1", "w1_scales", "w2", "w2_scales"))
    act_bytes = (nbytes(d["x"]) + nbytes(d["x_scales"]) + d["topk_idx"].numel() * 4 +
                 d["topk_w"].numel() * 4 + wl.T * wl.H * 2)
    return active * per_expert_w + act_bytes, active * per_expert_w, active


def workload_config(wl, active):
    """The keys of the line's ``config`` that define the workload; both arms
    (this library's and the oracle's) report them."""
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k,
            "w_dtype": wl.w_dtype, "routing": wl.routing, "act": wl.act,
            "active_experts": active}


def side_kernel_bytes(wl):
    """Algorithmic bytes of the launches around the GEMM, per launch.
    route: topk_idx in; perm, inv, counts and offsets out.  gather: x and its
    1x128 scales read once, one row (and its scales) written per slot, perm
    read.  combine: y, topk_w and inv read per slot; out written."""
    S = wl.S
    xe = 2 if wl.w_dtype == "bf16" else 1
    sf = 0 if wl.w_dtype == "bf16" else wl.H // 128
    route = S * 4 + 2 * S * 4 + (2 * wl.E + 1) * 4
    gather = (wl.T + S) * (wl.H * xe + sf) + S * 4
    combine = S * wl.H * 2 + 2 * S * 4 + wl.T * wl.H * 2
    return {"route_gather": route + gather, "route_alone": route, "gather_alone": gather,
            "combine": combine}


def kernels_gbs(wl, split):
    """GB/s of the launches around the GEMM from their mean split times (ms)."""
    return {k: round(b / (statistics.mean(split[k]) * 1e-3) / 1e9, 1)
            for k, b in side_kernel_bytes(wl).items() if split.get(k)}


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank times (each rank gets the result): a
    replica job is as fast as its slowest rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def replica_throughput(tokens_per_rank, world, total_ms, steps):
    """Whole-job tokens/s of `world` independent replicas (weak scaling), each
    processing tokens_per_rank per step, timed by the slowest rank."""
    return tokens_per_rank * world / (total_ms * 1e-3 / steps)


# The line's headline workload: the largest configuration that fits one GPU
# (the FP8-activation x MXFP4-weight layer at 32768 tokens); the per-config
# record covers every configuration of the layer.
HEADLINE = ("mxfp4", 32768)
PER_CONFIG = (("decode", None), ("prefill", None), ("oai", None), ("bf16", None),
              ("mxfp4", 128), ("mxfp4", 1024), ("mxfp4", 8192), ("mxfp4", 32768))
PER_CONFIG_STEPS = 10


def workload(name, tokens=None):
    from workloads.synth import WORKLOADS
    wl = WORKLOADS[name]
    return wl.with_tokens(tokens) if tokens else wl


def roofline(wl, alg_bytes, w_bytes, active, gemm_ms, pairs=False):
    """Roofline of the dominant kernel (the fused FC1+FC2 GEMM launch) from its
    mean split time: HBM-bound workloads count the active experts' weight and
    scale bytes per launch against the measured copy bandwidth, tensor-bound
    ones count 6*S*H*I FLOP against the measured sustained bf16 GEMM rate (x2
    for FP8 and FP8 x FP4 operands: the GEMM time comes from continuous steps,
    the sustained power-capped state)."""
    hbm, bf16_burst, bf16_sus, peak_src = _peaks()
    flops = 6.0 * wl.S * wl.H * wl.I
    tc_mult = 1.0 if wl.w_dtype == "bf16" else 2.0
    hbm_bound = alg_bytes / (hbm * 1e9) > flops / (tc_mult * bf16_sus * 1e12)
    if hbm_bound:
        roof = {"bound": "hbm", "achieved": round(w_bytes / (gemm_ms * 1e-3) / 1e9, 1),
                "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": round(flops / (gemm_ms * 1e-3) / 1e12, 1),
                "peak": round(tc_mult * bf16_sus, 1), "unit": "TFLOP/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    if not hbm_bound:
        # For a kernel whose clock stayed near its maximum (no power capping
        # in the samples) the burst figure is the closer denominator.
        roof["frac_of_burst_peak"] = round(roof["achieved"] / (tc_mult * bf16_burst), 4)
    roof["traffic"] = measured_traffic(wl.name)
    roof["kernel"] = (("moe_gemm_pair_kernel (CTA pairs, 2-SM MMA; with its weight-scale "
                       "expansion launch)" if pairs else "moe_gemm_kernel") +
                      ": FC1 + SwiGLU + " + ("bf16 activation" if wl.w_dtype == "bf16"
                                              else "FP8 requant") +
                      " and FC2 in one persistent launch")
    roof["per_launch"] = (f"{w_bytes} B of expert weights+scales ({active} active experts)"
                          if hbm_bound else f"{flops:.4g} FLOP (6*S*H*I)")
    roof["peak_source"] = f"{peak_src}" + (" copy bandwidth" if roof["unit"] == "GB/s" else
                                           " bf16 sustained" if tc_mult == 1.0 else
                                           " bf16 sustained x2 (FP8 = 2x bf16 nominal)")
    return roof


class LayerBench:
    """One workload on this rank's GPU: seeded inputs, weights in the layout the
    library streams fastest (FP8/BF16 tiles, MXFP4 scale chunks; prepacked once,
    as at model load), the layer, and a CUDA graph of moe_forward."""

    def __init__(self, wl, args, dev, keep_row_major=False):
        import torch

        import moe_expert_ffn_permute_b200 as moe
        from workloads.synth import make_inputs
        self.moe, self.wl, self.args, self.dev = moe, wl, args, dev
        d = make_inputs(wl, device=dev)
        self.tiled = not args.row_major_weights      # FP8/BF16 tiles; MXFP4 code tiles
        self.chunked = wl.w_dtype == "e2m1" and not args.row_major_weights
        self.lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                                alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, device=dev,
                                tiled_weights=self.tiled,
                                cta_pairs=args.cta_pairs if self.tiled else None,
                                swap_ab=args.swap_ab, chunked_scales=self.chunked)
        self.pairs = moe.moe_plan_cta_pairs_active(self.lay.plan)
        self.alg_bytes, self.w_bytes, self.active = algorithmic_bytes(wl, d)
        self.d_row_major = dict(d) if keep_row_major else None   # the oracle's layout
        if self.tiled:
            d["w1"], d["w2"] = self.lay.prepack(d["w1"], d["w2"])
        if self.chunked:
            d["w1_scales"], d["w2_scales"] = self.lay.prepack_scales(d["w1_scales"],
                                                                     d["w2_scales"])
        torch.cuda.synchronize()
        self.d = d
        self.out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
        self.stream = torch.cuda.current_stream()
        self.graph = None

    def fwd(self):
        """moe_forward on the current stream (inside graph capture: the capture
        stream, so that the graph records the launches)."""
        import torch
        d = self.d
        self.moe.moe_forward(self.lay.plan, d["x"], d["x_scales"], d["topk_idx"], d["topk_w"],
                             d["w1"], d["w1_scales"], d["w2"], d["w2_scales"], self.out,
                             self.lay.workspace, torch.cuda.current_stream())

    def steps(self, unfused=False):
        """The launch sequence of moe_forward one call per step (route+gather,
        FC1+FC2, combine), or with routing, gather and the two GEMMs as separate
        launches (informational)."""
        moe, d, lay, st = self.moe, self.d, self.lay, self.stream
        if not unfused:
            return [("route_gather", lambda: moe.moe_route_gather(lay.plan, d["topk_idx"], d["x"],
                                                                  d["x_scales"], lay.workspace, st)),
                    ("fc1_fc2", lambda: moe.moe_fc1_fc2(lay.plan, d["w1"], d["w1_scales"], d["w2"],
                                                        d["w2_scales"], lay.workspace, st)),
                    ("combine", lambda: moe.moe_combine(lay.plan, d["topk_w"], self.out,
                                                        lay.workspace, st))]
        return [("route_alone", lambda: moe.moe_route(lay.plan, d["topk_idx"], lay.workspace, st)),
                ("gather_alone", lambda: moe.moe_gather(lay.plan, d["x"], d["x_scales"],
                                                        lay.workspace, st)),
                ("fc1_alone", lambda: moe.moe_fc1(lay.plan, d["w1"], d["w1_scales"],
                                                  lay.workspace, st)),
                ("fc2_alone", lambda: moe.moe_fc2(lay.plan, d["w2"], d["w2_scales"],
                                                  lay.workspace, st))]

    def prepare(self, warmup):
        import torch
        for _ in range(warmup):
            self.fwd()
        torch.cuda.synchronize()
        if self.lay.check() != 0:
            raise RuntimeError(f"device error during warm-up of {self.wl.name}")
        # The timed step replays a CUDA graph of moe_forward (the same kernels
        # with the same arguments; the routing kernel resets the GEMM
        # scheduler's counters inside the graph, so every replay starts clean).
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.fwd()
        torch.cuda.synchronize()
        # The replay must run the layer: a graph that captured nothing would
        # time an empty replay.  One replay into a poisoned output proves it.
        self.out.fill_(float("nan"))
        self.graph.replay()
        torch.cuda.synchronize()
        if bool(torch.isnan(self.out).any()):
            raise RuntimeError(f"graph replay of {self.wl.name} did not recompute the output")

    def soak(self, seconds):
        import torch
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            for _ in range(20):
                self.graph.replay()
            torch.cuda.synchronize()

    def timed(self, fn, steps, flush):
        """Per-step device times (ms): CUDA events on the launching stream, L2
        flushed before every step outside the events."""
        import torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(self.stream)
            fn()
            ev[i][1].record(self.stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def split(self, steps, flush, unfused=False):
        """Per-launch device times (ms) of the launch sequence, one event per
        launch boundary on the launching stream."""
        import torch
        seqs = [self.steps()] + ([self.steps(unfused=True)] if unfused else [])
        out = {name: [] for seq in seqs for name, _ in seq}
        for seq in seqs:
            for i in range(steps):
                flush.fill_(i & 0xFF)
                evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(seq) + 1)]
                evs[0].record(self.stream)
                for j, (_, fn) in enumerate(seq):
                    fn()
                    evs[j + 1].record(self.stream)
                torch.cuda.synchronize()
                for j, (name, _) in enumerate(seq):
                    out[name].append(evs[j].elapsed_time(evs[j + 1]))
        return out

    def e2e(self, steps, warmup, flush):
        """Device time (ms per step) through the host-buffer entry point: every
        step's inputs copied in from pinned host memory and its output copied
        back, all inside the events (moe_forward_hostio_batches: the copies of
        one step overlap the layer of the neighbouring steps)."""
        import torch
        moe, d, lay = self.moe, self.d, self.lay
        host = {k: (None if d[k] is None else d[k].cpu().pin_memory())
                for k in ("x", "x_scales", "topk_idx", "topk_w")}
        out_h = torch.empty(self.wl.T, self.wl.H, dtype=torch.bfloat16).pin_memory()

        def call(n):
            moe.moe_forward_hostio_batches(
                lay.plan, [host["x"]] * n,
                None if host["x_scales"] is None else [host["x_scales"]] * n,
                [host["topk_idx"]] * n, [host["topk_w"]] * n, d["w1"], d["w1_scales"], d["w2"],
                d["w2_scales"], [out_h] * n, lay.workspace, self.stream)
        call(max(warmup, 1))
        torch.cuda.synchronize()
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        call(steps)
        b.record(self.stream)
        torch.cuda.synchronize()
        total = a.elapsed_time(b)
        h2d = int(sum(v.numel() * v.element_size() for v in host.values() if v is not None))
        return [total / steps] * steps, h2d, int(out_h.numel() * 2)

    def release(self):
        import torch
        self.graph = None
        self.lay = None
        self.d = None
        self.out = None
        torch.cuda.empty_cache()


def measure_rank(args, dev):
    """This rank's measurements: the headline workload (timed steps, eager
    steps, per-launch split, e2e, clocks) and a shorter record of every
    configuration.  Returns plain numbers so that the line can be assembled
    from any number of ranks (``assemble_line``)."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rank, world, local = _dist()
    wl = workload(args.workload, args.tokens)
    lb = LayerBench(wl, args, dev, keep_row_major=(rank == 0 and not args.no_cpu_baseline))
    lb.prepare(args.warmup)
    clocks = Clocks(local)
    clocks.start()
    # The clock sampler needs ~100 ms per sample, longer than K steps take, so
    # the timed steps sit between continuous (untimed) steps of the same layer.
    lb.soak(0.6)
    step_ms = lb.timed(lb.graph.replay, args.steps, flush)
    lb.soak(0.3)
    eager_ms = lb.timed(lb.fwd, args.steps, flush)
    lb.soak(0.3)
    split = lb.split(args.steps, flush, unfused=True)
    lb.soak(0.3)
    clk = clocks.stop()
    e2e_ms, h2d, d2h = lb.e2e(args.steps, args.warmup, flush)
    if lb.lay.check() != 0:
        raise RuntimeError("device error during timing")
    main = {"wl": wl, "step_ms": step_ms, "eager_ms": eager_ms, "split": split,
            "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h, "clocks": clk, "active": lb.active,
            "alg_bytes": lb.alg_bytes, "w_bytes": lb.w_bytes, "pairs": lb.pairs,
            "tiled": lb.tiled, "chunked": lb.chunked,
            "swap": lb.moe.moe_plan_swap_ab_active(lb.lay.plan),
            "wide": lb.moe.moe_plan_wide_tiles_active(lb.lay.plan),
            "launches": lb.moe.moe_forward_launch_count(lb.lay.plan)}
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, lb.d_row_major, args)
    lb.release()
    per = []
    if not args.no_per_config:
        for name, tokens in PER_CONFIG:
            w = workload(name, tokens)
            b = LayerBench(w, args, dev)
            b.prepare(min(args.warmup, 3))
            c = Clocks(local)
            c.start()
            b.soak(0.3)
            ms = b.timed(b.graph.replay, PER_CONFIG_STEPS, flush)
            sp = b.split(PER_CONFIG_STEPS, flush)
            b.soak(0.1)
            cc = c.stop()
            if b.lay.check() != 0:
                raise RuntimeError(f"device error during timing of {w.name}")
            per.append({"wl": w, "step_ms": ms, "split": sp, "active": b.active,
                        "alg_bytes": b.alg_bytes, "w_bytes": b.w_bytes, "pairs": b.pairs,
                        "clocks": cc, "wide": b.moe.moe_plan_wide_tiles_active(b.lay.plan)})
            b.release()
    return main, per, cpu


def assemble_line(args, world, device, main, per, cpu):
    """The contract's JSON line from this rank's measurements: every time is
    first replaced by its maximum over ranks (one all-reduce, the same on every
    rank), so a replica job is as fast as its slowest rank and `value` counts
    the tokens of all ranks (weak scaling)."""
    wl = main["wl"]
    steps = len(main["step_ms"])
    # Every time on the line, as (key, local value); one all-reduce of them all.
    keys = [("total", sum(main["step_ms"])), ("e2e", sum(main["e2e_ms"])),
            ("eager", sum(main["eager_ms"]))]
    keys += [(("split", k), statistics.mean(v)) for k, v in main["split"].items() if v]
    for i, p in enumerate(per):
        keys.append((("per", i, "total"), sum(p["step_ms"])))
        keys += [(("per", i, k), statistics.mean(v)) for k, v in p["split"].items() if v]
    red = dict(zip([k for k, _ in keys], max_over_ranks([v for _, v in keys], world, device)))
    total_ms, e2e_total, eager_total = red["total"], red["e2e"], red["eager"]
    split_ms = {k[1]: v for k, v in red.items() if isinstance(k, tuple) and k[0] == "split"}
    gemm_ms = split_ms["fc1_fc2"]
    ms_per_step = total_ms / steps
    flops = 6.0 * wl.S * wl.H * wl.I
    res = {
        "metric": METRIC, "value": round(replica_throughput(wl.T, world, total_ms, steps), 1),
        "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"e4m3": "fp8_e4m3", "e2m1": "fp8_e4m3xe2m1",
                                       "bf16": "bf16"}[wl.w_dtype],
        "data": "synthetic (seeded; random-init weights)",
        "config": {**workload_config(wl, main["active"]),
                   "l2": "flushed (256 MiB write) before each step",
                   "weights": ("tiled codes and chunked scales (moe_prepack_weights and "
                               "moe_prepack_weight_scales, once)" if main["chunked"] else
                               "tiled (moe_prepack_weights, once)" if main["tiled"] else
                               "row-major"),
                   "gemm_tiles": {0: "token rows", 1: "token-major (swap AB)",
                                  2: "token-major for tiles of <= 96 tokens, else token rows"}[
                       main["swap"]] + ("; wide token-major tiles over two m-tiles (up to 240 "
                                        "tokens)" if main.get("wide") else ""),
                   "parallelism": f"replicas x{world}"},
        "achieved": {"tflops": round(flops / (ms_per_step * 1e-3) / 1e12, 2),
                     "hbm_gbs": round(main["alg_bytes"] / (ms_per_step * 1e-3) / 1e9, 1),
                     "alg_bytes": main["alg_bytes"], "flops": flops},
        "kernels_ms": {k: round(v, 4) for k, v in split_ms.items()},
        "kernels_gbs": kernels_gbs(wl, {k: [v] for k, v in split_ms.items()}),
        "eager_ms_per_step": round(eager_total / steps, 4),
        "timing": "CUDA-graph replay of moe_forward, events on the launching stream",
        "roofline": roofline(wl, main["alg_bytes"], main["w_bytes"], main["active"], gemm_ms,
                             main["pairs"]),
        "e2e": {"value": round(replica_throughput(wl.T, world, e2e_total, steps), 1),
                "unit": "tokens/s", "h2d_bytes_per_step": main["h2d"],
                "d2h_bytes_per_step": main["d2h"]},
        "gpu_launches": main["launches"] * steps,
        "clocks": main["clocks"],
    }
    per_out = []
    for i, p in enumerate(per):
        w = p["wl"]
        t_ms, g_ms = red[("per", i, "total")], red[("per", i, "fc1_fc2")]
        n = len(p["step_ms"])
        roof = roofline(w, p["alg_bytes"], p["w_bytes"], p["active"], g_ms, p["pairs"])
        per_out.append({
            "workload": w.name, "T": w.T, "w_dtype": w.w_dtype, "active_experts": p["active"],
            "tokens_per_s": round(replica_throughput(w.T, world, t_ms, n), 1),
            "ms_per_step": round(t_ms / n, 4), "fc1_fc2_ms": round(g_ms, 4),
            "route_gather_ms": round(red[("per", i, "route_gather")], 4),
            "combine_ms": round(red[("per", i, "combine")], 4),
            "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac")},
            "sm_mhz": p["clocks"].get("sm_mhz"), "reasons": p["clocks"].get("reasons"),
            "wide_tiles": bool(p.get("wide")), "steps": n})
    if per_out:
        res["per_config"] = per_out
    if cpu is not None:
        res["cpu_baseline"] = cpu
    return res


def run_b200(args):
    import datetime

    import torch
    import torch.distributed as dist

    from moe_expert_ffn_permute_b200.build import build

    rank, world, local = _dist()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    import moe_expert_ffn_permute_b200 as moe
    moe.lib()
    dev = torch.device("cuda", local)
    main, per, cpu = measure_rank(args, dev)
    if world > 1:
        dist.barrier()
    res = assemble_line(args, world, dev, main, per, cpu)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))


def run_forwards(args, wl):
    """N forwards of one workload in the benchmark's launch configuration
    (prepared weights, automatic tiles) and nothing else: the launches a
    profiler captures, without the benchmark's timing around them."""
    import torch

    from moe_expert_ffn_permute_b200.build import build

    build()
    dev = torch.device("cuda", 0)
    lb = LayerBench(wl, args, dev)
    for _ in range(args.forwards):
        lb.fwd()
    torch.cuda.synchronize()
    if lb.lay.check() != 0:
        sys.exit(f"bench.py: device error word set after {args.forwards} forwards of {wl.name}")
    print(f"{wl.name}: {args.forwards} forwards")
    lb.release()


def _oracle_sample(wl, dn, tokens):
    from oracle import layer as L
    sub = dict(dn)
    for key in ("x", "x_scales", "topk_idx", "topk_w"):
        if dn[key] is not None:
            sub[key] = dn[key][tokens]
    if wl.w_dtype == "bf16":
        return L.layer_bf16(sub["x"], sub["topk_idx"], sub["topk_w"], dn["w1"], dn["w2"],
                            alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit)
    return L.layer(sub["x"], sub["x_scales"], sub["topk_idx"], sub["topk_w"], dn["w1"],
                   dn["w1_scales"], dn["w2"], dn["w2_scales"], w_dtype=wl.w_dtype,
                   alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit)


def _cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
        return int(n)
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl, d, args, ntok=None):
    """The float64 oracle, as it stands, on a bounded sample of the workload's
    tokens (the oracle's cost is dominated by dequantising the touched experts'
    weights, so a few tokens already take seconds)."""
    from workloads.synth import to_numpy
    dn = to_numpy(d)
    ntok = ntok or args.cpu_tokens
    t0 = time.perf_counter()
    _oracle_sample(wl, dn, list(range(ntok)))
    dt = time.perf_counter() - t0
    return {"value": round(ntok / dt, 4), "unit": "tokens/s", "cores": _cores(),
            "kind": "oracle", "sample": f"first {ntok} of {wl.T} tokens of {wl.name}, "
                                        f"float64 NumPy, {dt:.1f} s"}


def run_reference(args, wl):
    rank, world, _ = _dist()
    if rank != 0:
        return
    import torch
    from workloads.synth import make_inputs, to_numpy
    d = make_inputs(wl, device="cuda" if torch.cuda.is_available() else "cpu")
    dn = to_numpy(d)
    ntok = args.ref_tokens
    for i in range(args.warmup):
        _oracle_sample(wl, dn, [i % wl.T])
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        _oracle_sample(wl, dn, [(j + i * ntok) % wl.T for j in range(ntok)])
        times.append(time.perf_counter() - t0)
    total = sum(times)
    val = ntok * args.steps / total
    res = {"metric": METRIC, "value": round(val, 4), "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(1e3 * total / args.steps, 2), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "impl": "reference",
           "config": {**workload_config(wl, algorithmic_bytes(wl, d)[2]),
                      "parallelism": "float64 oracle on the host cores (rank 0)"},
           "cpu_baseline": {"value": round(val, 4), "unit": "tokens/s", "cores": _cores(),
                            "kind": "oracle",
                            "sample": f"{ntok} token(s) of {wl.name} per step"},
           "e2e": {"value": round(val, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res))


def _respawn_under_torchrun(n):
    """`--gpus N` without a launcher: start N ranks of this same command under
    torch.distributed.run (one process per GPU) and return its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE[0])
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (the mxfp4 sweep); default: the headline's 32768 tokens "
                         "for the mxfp4 workload")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=2,
                    help="tokens of the oracle sample beside the GPU line (cpu_baseline)")
    ap.add_argument("--ref-tokens", type=int, default=1,
                    help="tokens per step of the oracle arm (--impl reference)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-configuration record (headline workload only)")
    ap.add_argument("--cta-pairs", type=int, default=0, choices=[0, 1, 2],
                    help="GEMM on CTA pairs: 0 automatic, 1 never, 2 always (tiled FP8 only)")
    ap.add_argument("--swap-ab", type=int, default=0, choices=[0, 1, 2],
                    help="token-major GEMM tiles: 0 tile by tile (automatic), 1 never, 2 always")
    ap.add_argument("--row-major-weights", action="store_true",
                    help="weights as given (row-major, 2-D TMA; MXFP4 scales unchunked) "
                         "instead of prepacked")
    ap.add_argument("--forwards", type=int, default=0,
                    help="only run this many forwards of the workload on one GPU, untimed "
                         "(the launches a profiler captures), and print no JSON line")
    args = ap.parse_args()
    if args.tokens is None and args.workload == HEADLINE[0]:
        args.tokens = HEADLINE[1]
    world_env = os.environ.get("WORLD_SIZE")
    if args.gpus > 1 and world_env is None:
        sys.exit(_respawn_under_torchrun(args.gpus))
    if world_env is not None and int(world_env) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world_env}: launch one rank "
                 f"per GPU (torch.distributed.run --nproc-per-node {args.gpus})")
    wl = workload(args.workload, args.tokens)
    if args.forwards > 0:
        run_forwards(args, wl)
    elif args.impl == "reference":
        run_reference(args, wl)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
