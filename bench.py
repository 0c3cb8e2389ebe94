"""Throughput benchmark of the fused MoE expert layer on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl {b200,reference}]

One step = one whole layer (route, gather, FC1 + SwiGLU + FP8 requant, FC2,
combine) over one batch of seeded synthetic inputs already resident in HBM.
The default workload is the decode-size layer (T=128, H=7168, I=2048, E=32,
top-8, skewed routing).  With N > 1 (launched by torch.distributed.run) every
rank runs its own replica of the layer on its own GPU: the path has no exchange
step, so there is no collective on the data path (weak scaling); the elapsed
device time is the maximum over ranks.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream; L2 is flushed (a 256 MiB buffer is overwritten)
before every timed step, outside the events.  `e2e` times the same layer
through the C ABI's host-buffer entry point (pinned host inputs copied in,
output copied back, all inside the events).

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


def run_b200(args, wl):
    import torch
    import torch.distributed as dist

    import moe_expert_ffn_permute_b200 as moe
    from moe_expert_ffn_permute_b200.build import build
    from workloads.synth import make_inputs

    rank, world, local = _dist()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    torch.cuda.set_device(local)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    lib = moe.lib()
    dev = torch.device("cuda", local)
    d = make_inputs(wl, device=dev)
    # FP8 weights are rearranged once into the tensor-core tile layout (as at
    # model load); the timed steps read them in that layout.
    tiled = wl.w_dtype in ("e4m3", "bf16") and not args.row_major_weights
    chunked = wl.w_dtype == "e2m1" and not args.row_major_weights
    lay = moe.MoELayer(wl.T, wl.H, wl.I, wl.E, wl.k, w_dtype=wl.w_dtype, act=wl.act,
                       alpha=wl.alpha, up_bias=wl.up_bias, limit=wl.limit, device=dev,
                       tiled_weights=tiled, cta_pairs=args.cta_pairs if tiled else None,
                       swap_ab=args.swap_ab, chunked_scales=chunked)
    pairs = moe.moe_plan_cta_pairs_active(lay.plan)
    d_row_major = dict(d)          # the oracle reads the original layout
    if tiled:
        d["w1"], d["w2"] = lay.prepack(d["w1"], d["w2"])
        torch.cuda.synchronize()
    if chunked:
        d["w1_scales"], d["w2_scales"] = lay.prepack_scales(d["w1_scales"], d["w2_scales"])
        torch.cuda.synchronize()
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    args_dev = (d["x"], d["x_scales"], d["topk_idx"], d["topk_w"], d["w1"], d["w1_scales"],
                d["w2"], d["w2_scales"])

    def fwd(st=None):
        moe.moe_forward(lay.plan, *args_dev, out, lay.workspace,
                        st if st is not None else torch.cuda.current_stream())

    steps = [("route_gather", lambda: moe.moe_route_gather(lay.plan, d["topk_idx"], d["x"],
                                                           d["x_scales"], lay.workspace,
                                                           stream)),
             ("fc1_fc2", lambda: moe.moe_fc1_fc2(lay.plan, d["w1"], d["w1_scales"], d["w2"],
                                                 d["w2_scales"], lay.workspace, stream)),
             ("combine", lambda: moe.moe_combine(lay.plan, d["topk_w"], out, lay.workspace,
                                                 stream))]
    # Routing and gather as separate launches, and the two GEMMs as separate
    # launches (informational; moe_forward fuses each pair).
    extra = [("route_alone", lambda: moe.moe_route(lay.plan, d["topk_idx"], lay.workspace,
                                                   stream)),
             ("gather_alone", lambda: moe.moe_gather(lay.plan, d["x"], d["x_scales"],
                                                     lay.workspace, stream)),
             ("fc1_alone", lambda: moe.moe_fc1(lay.plan, d["w1"], d["w1_scales"],
                                               lay.workspace, stream)),
             ("fc2_alone", lambda: moe.moe_fc2(lay.plan, d["w2"], d["w2_scales"],
                                               lay.workspace, stream))]

    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    if lay.check() != 0:
        raise RuntimeError("device error during warm-up")

    # The timed step replays a CUDA graph of moe_forward (the same kernels with
    # the same arguments; the routing kernel resets the GEMM scheduler's
    # counters inside the graph, so every replay starts from a clean state).
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fwd()
    torch.cuda.synchronize()

    def step():
        graph.replay()

    # ---- timed: whole layer, device-resident inputs.  The clock sampler needs
    # ~100 ms per sample, longer than K steps of this layer take, so the timed
    # steps sit inside a window of continuous (untimed) steps of the same layer
    # that starts and ends 0.6 s around them; all samples are taken under load.
    clocks = Clocks(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()

    def soak(seconds):
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            for _ in range(20):
                step()
            torch.cuda.synchronize()

    def timed(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    soak(0.6)
    step_ms = timed(step)
    # ---- per-kernel split (the launch sequence of moe_forward, one event per
    # step boundary, on the launching stream), then the unfused launches.
    split = {name: [] for name, _ in steps + extra}

    def split_timing():
        for seq in (steps, extra):
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(seq) + 1)]
                evs[0].record(stream)
                for j, (_, fn) in enumerate(seq):
                    fn()
                    evs[j + 1].record(stream)
                torch.cuda.synchronize()
                for j, (name, _) in enumerate(seq):
                    split[name].append(evs[j].elapsed_time(evs[j + 1]))

    # Everything on the line is measured in the same sustained state: the
    # eager calls and the per-kernel split also sit between continuous steps.
    soak(0.3)
    eager_ms = timed(fwd)
    soak(0.3)
    split_timing()
    soak(0.3)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    total_ms = sum(step_ms)

    # ---- e2e through the host-buffer entry point
    host = {k: (None if d[k] is None else d[k].cpu().pin_memory())
            for k in ("x", "x_scales", "topk_idx", "topk_w")}
    out_h = torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory()
    for _ in range(args.warmup):
        moe.moe_forward_hostio(lay.plan, host["x"], host["x_scales"], host["topk_idx"],
                               host["topk_w"], d["w1"], d["w1_scales"], d["w2"], d["w2_scales"],
                               out_h, lay.workspace, stream)
    torch.cuda.synchronize()
    e2e_ms = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        moe.moe_forward_hostio(lay.plan, host["x"], host["x_scales"], host["topk_idx"],
                               host["topk_w"], d["w1"], d["w1_scales"], d["w2"], d["w2_scales"],
                               out_h, lay.workspace, stream)
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    if lay.check() != 0:
        raise RuntimeError("device error during timing")

    # ---- max over ranks
    total_ms, e2e_total = max_over_ranks([total_ms, sum(e2e_ms)], world, dev)

    alg_bytes, w_bytes, active = algorithmic_bytes(wl, d)
    hbm, bf16, bf16_sus, peak_src = _peaks()
    flops = 6.0 * wl.S * wl.H * wl.I
    gemm_ms = statistics.mean(split["fc1_fc2"])
    # Tensor peak of the GEMM's own input type: the measured bf16 figure for
    # BF16 weights, twice it for FP8 (and E4M3 x E2M1) operands.  The GEMM time
    # comes from the split taken between continuous steps, so the sustained
    # (power-capped) bf16 measurement is the matching denominator.
    tc_mult = 1.0 if wl.w_dtype == "bf16" else 2.0
    hbm_bound = alg_bytes / (hbm * 1e9) > flops / (tc_mult * bf16_sus * 1e12)
    if hbm_bound:
        roof = {"bound": "hbm", "achieved": round(w_bytes / (gemm_ms * 1e-3) / 1e9, 1),
                "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": round(flops / (gemm_ms * 1e-3) / 1e12, 1),
                "peak": round(tc_mult * bf16_sus, 1), "unit": "TFLOP/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
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

    ms_per_step = total_ms / args.steps
    res = {
        "metric": METRIC, "value": round(replica_throughput(wl.T, world, total_ms, args.steps), 1),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"e4m3": "fp8_e4m3", "e2m1": "fp8_e4m3xe2m1",
                                       "bf16": "bf16"}[wl.w_dtype],
        "data": "synthetic (seeded; random-init weights)",
        "config": {**workload_config(wl, active), "l2": "flushed (256 MiB write) before each step",
                   "weights": ("tiled (moe_prepack_weights, once)" if tiled else
                               "row-major codes, chunked scales (moe_prepack_weight_scales, once)"
                               if chunked else "row-major"),
                   "gemm_tiles": {0: "token rows", 1: "token-major (swap AB)",
                                  2: "token-major for tiles of <= 96 tokens, else token rows"}[
                       moe.moe_plan_swap_ab_active(lay.plan)],
                   "parallelism": f"replicas x{world}"},
        "achieved": {"tflops": round(flops / (ms_per_step * 1e-3) / 1e12, 2),
                     "hbm_gbs": round(alg_bytes / (ms_per_step * 1e-3) / 1e9, 1),
                     "alg_bytes": alg_bytes, "flops": flops},
        "kernels_ms": {k: round(statistics.mean(v), 4) for k, v in split.items()},
        "kernels_gbs": kernels_gbs(wl, split),
        "eager_ms_per_step": round(sum(eager_ms) / args.steps, 4),
        "timing": "CUDA-graph replay of moe_forward, events on the launching stream",
        "roofline": roof,
        "e2e": {"value": round(replica_throughput(wl.T, world, e2e_total, args.steps), 1),
                "unit": "tokens/s",
                "h2d_bytes_per_step": int(sum(v.numel() * v.element_size() for v in host.values()
                                              if v is not None)),
                "d2h_bytes_per_step": int(out_h.numel() * 2)},
        "gpu_launches": moe.moe_forward_launch_count(lay.plan) * args.steps,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, d_row_major, args)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))


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
    ntok = args.cpu_tokens
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode")
    ap.add_argument("--tokens", type=int, default=None, help="override T (mxfp4 sweep)")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cta-pairs", type=int, default=0, choices=[0, 1, 2],
                    help="GEMM on CTA pairs: 0 automatic, 1 never, 2 always (tiled FP8 only)")
    ap.add_argument("--swap-ab", type=int, default=0, choices=[0, 1, 2],
                    help="token-major GEMM tiles: 0 tile by tile (automatic), 1 never, 2 always")
    ap.add_argument("--row-major-weights", action="store_true",
                    help="weights as given (row-major, 2-D TMA; MXFP4 scales unchunked) "
                         "instead of prepacked")
    args = ap.parse_args()
    from workloads.synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.with_tokens(args.tokens)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_b200(args, wl)


if __name__ == "__main__":
    main()
