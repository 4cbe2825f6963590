#!/usr/bin/env python
"""Benchmark of the DCNv4 hot path on B200.

One step = DCNv4 forward + DCNv4 backward + MSDCN forward over one batch of
the InternImage-stage workload (N64 56x56 C128 G8, bf16; MSDCN inputs of the
same shape), inputs resident in HBM. Each op is captured once in a CUDA graph
and replayed; L2 is flushed (256 MB write) before every timed step; CUDA
events on the launching stream time each op. The reported value is effective
bandwidth: the operator's ideal bytes (input and output once, 27 offset/weight
values per pixel and group; DCNv4 digest "GPU效率的理论分析") per second of device
time, summed over all ranks (weak scaling: every rank runs a full batch).
Outside the timed step, `next_rows` times MSDCN backward and the offset/weight
producer (depthwise 3x3 + merged linear) on the same shape, graph-replayed
with the same L2 flush; they are reported, not counted in the value.
`configs` times every workload of the table below the same way (median of
graph replays, L2 flushed before each): forward, backward (fp32 accumulation
of grad_input across CTAs, the default, and the 16-bit cross-CTA variant
acc16), MSDCN forward and backward, and the forward with the offset/weight
sub-network fused in (dcn4_fused_forward, next to the producer + forward
chain it replaces), each with ideal bytes, GB/s, the fraction of the HBM
peak and the fraction of samples outside the image.
The CPU-baseline leg, which runs the oracle, also checks one image of every
(config, op) against it (scaled max error and an elementwise error with an
rms floor). `e2e` runs the step through the public calls from pinned host
memory, every step's input copies and result reads inside the timed region,
with the transfers of neighbouring steps overlapped (two device buffer sets,
input / compute / output streams); the one-after-another figure is kept
beside it (`sequential_value`).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DCNv4 fwd/bwd GB/s and Gsample·ch/s at 1 B200; % of HBM roofline"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 256 << 20

# (label, workload, ops) timed outside the step; "bwd" is the default
# backward (fp32 accumulation across CTAs), "bwd_acc16" the 16-bit cross-CTA
# accumulation, "msbwd" the MSDCN backward (default math), "fused" the
# forward with the offset/weight sub-network in front (one call)
CONFIG_TABLE = [
    ("c1", "tiny_f32", ["fwd", "bwd"]),
    ("c2", "internimage_bf16", ["fwd", "bwd", "bwd_acc16", "msfwd", "msbwd", "fused"]),
    ("c2", "internimage_f32", ["fwd", "bwd"]),
    ("c3a", "ldm64_f16", ["fwd", "bwd", "bwd_acc16"]),
    ("c3b", "ldm32_f16", ["fwd", "bwd", "bwd_acc16"]),
    ("c4", "flowdcn_msdcn_bf16", ["msfwd", "msbwd"]),
    ("c5", "highres_bf16", ["fwd", "bwd", "bwd_acc16", "fused"]),
]


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="internimage_bf16")
    p.add_argument("--no-cpu-baseline", action="store_true")
    # time the step alone: skip the next_rows and configs diagnostics and the
    # end-to-end leg (used by the profiler's launch list)
    p.add_argument("--step-only", action="store_true")
    return p.parse_args(argv)


# ---------------------------------------------------------------- accounting
def ideal_bytes(wl, Ho, Wo):
    """Ideal traffic of each op in bytes (inputs read once, outputs written once)."""
    eb = 4 if wl.dtype == "f32" else 2
    nin = wl.N * wl.H * wl.W * wl.C
    nout = wl.N * Ho * Wo * wl.C
    now = wl.N * Ho * Wo * wl.G * wl.K * 3
    return {
        "dcn4_forward": (nin + nout + now) * eb,
        "dcn4_backward": (nin + nout + now + nin + now) * eb,
        "msdcn_forward": (nin + nout + now + wl.N * Ho * Wo * wl.G) * eb,
    }


def samples_ch(wl, Ho, Wo):
    """Bilinear samples x channels of one forward (K per output element)."""
    return wl.K * wl.N * Ho * Wo * wl.C


def msdcn_variant(wl):
    return wl.replace(kind="msdcn", offset_dist=("normal", 1.0))


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    """Hash of the kernel sources' code: comments removed and whitespace
    collapsed, so that a documentation edit does not invalidate recorded
    measurements while any change to the code does."""
    import re
    csrc = os.path.join(ROOT, "deformable_convolution_dcn4_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            code = f.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        code = " ".join(code.split())
        h.update(name.encode() + code.encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    e = rec.get(f"{kernel}@{workload}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------- distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value, device="cpu"):
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(step_bytes_per_rank, step_ms_max, world):
    """Whole-job throughput in GB/s: every rank processes its own full batch
    (step_bytes_per_rank), the job takes the slowest rank's time."""
    return world * step_bytes_per_rank / (step_ms_max * 1e-3) / 1e9


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle
def oracle_step_sample(wl, n_images):
    """The oracle's fwd + bwd + MSDCN fwd on the first n_images of the
    workload; returns (seconds, ideal bytes processed)."""
    import oracle
    from deformable_convolution_dcn4_b200.workloads import make_inputs
    orc = oracle.default()
    sub = wl.replace(N=n_images)
    p = orc.problem(sub.N, sub.H, sub.W, sub.C, sub.G, sub.kh, sub.kw, sub.stride, sub.pad,
                    sub.dilation, sub.offset_scale)
    Ho, Wo = orc.out_hw(p)
    d = make_inputs(sub, (Ho, Wo), with_grad=True)
    ms = make_inputs(msdcn_variant(sub), (Ho, Wo))
    arr = {k: v.float().numpy() for k, v in d.items()}
    marr = {k: v.float().numpy() for k, v in ms.items()}
    t0 = time.perf_counter()
    orc.forward(p, arr["input"], arr["offset_weight"])
    orc.backward(p, arr["input"], arr["offset_weight"], arr["grad_out"])
    orc.msdcn_forward(p, marr["input"], marr["dir_weight"], marr["scale_raw"], marr["s0"],
                      sub.smax)
    dt = time.perf_counter() - t0
    return dt, sum(ideal_bytes(sub, Ho, Wo).values())


def cpu_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    if n and n.isdigit():
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s=10.0):
    """Times the oracle on a bounded sample: whole images, the count growing
    until one run takes a sizeable part of budget_s (at most the whole batch),
    then repeated until about budget_s of oracle time has been spent."""
    n, total_t, total_b, runs = 1, 0.0, 0.0, 0
    while True:
        dt, b = oracle_step_sample(wl, n)
        total_t, total_b, runs = total_t + dt, total_b + b, runs + 1
        if total_t >= budget_s or runs >= 64:
            break
        if n < wl.N:
            n = min(wl.N, max(n + 1, int(n * budget_s / max(dt, 1e-3) * 0.25)))
    # once more on one thread (one image)
    import oracle
    orc = oracle.default()
    orc.set_threads(1)
    try:
        dt1, b1 = oracle_step_sample(wl, 1)
    finally:
        orc.set_threads(cpu_threads())
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": cpu_threads(),
            "kind": "oracle",
            "sample": f"{runs} oracle runs of fwd+bwd+MSDCN fwd, the last on {n} of {wl.N} "
                      f"images of {wl.name}, {total_t:.1f} s of oracle time",
            "single_thread": {"value": round(b1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"1 image of {wl.name}, {dt1:.2f} s"}}


# ---------------------------------------------------------------- our arm
def describe(wl, Ho, Wo):
    return {"workload": f"{wl.name}: N{wl.N} {wl.H}x{wl.W} C{wl.C} G{wl.G} (D{wl.D}) "
                        f"{wl.kh}x{wl.kw} s{wl.stride[0]} p{wl.pad[0]} d{wl.dilation[0]} "
                        f"{wl.dtype}; offsets {wl.offset_dist[0]}({wl.offset_dist[1]}) px, "
                        f"m ~ N(0,{wl.weight_sigma}); MSDCN inputs of the same shape "
                        f"(dir ~ N(0,1), raw ~ N(0,1), s0 = 1,1,2,2,.., Smax {wl.smax})",
            "ops_per_step": ["dcn4_forward", "dcn4_backward", "msdcn_forward"],
            "N": wl.N, "H": wl.H, "W": wl.W, "C": wl.C, "G": wl.G, "Ho": Ho, "Wo": Wo,
            "l2": "flushed before every timed step (256 MB write)",
            "parallelism": "batch replicas, one process per GPU"}


def run_ours(args):
    import torch

    import deformable_convolution_dcn4_b200 as dcn
    from deformable_convolution_dcn4_b200.workloads import WORKLOADS, make_inputs

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    dcn.load()

    wl = WORKLOADS[args.workload]
    desc = dcn.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, 0, (wl.kh, wl.kw), wl.stride, wl.pad,
                         wl.dilation, wl.offset_scale)
    Ho, Wo = dcn.dcn4_out_shape(desc)
    host = make_inputs(wl, (Ho, Wo), with_grad=True)
    mhost = make_inputs(msdcn_variant(wl), (Ho, Wo))
    d = {k: v.to(dev) for k, v in host.items()}
    m = {k: (v if k == "s0" else v.to(dev)) for k, v in mhost.items()}
    kw = dict(group=wl.G, kernel_size=(wl.kh, wl.kw), stride=wl.stride, pad=wl.pad,
              dilation=wl.dilation, offset_scale=wl.offset_scale)
    out = torch.empty((wl.N, Ho, Wo, wl.C), dtype=d["input"].dtype, device=dev)
    ms_out = torch.empty_like(out)
    gin = torch.empty_like(d["input"])
    gow = torch.empty_like(d["offset_weight"])
    dsc = dcn.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, d["input"].dtype, (wl.kh, wl.kw),
                        wl.stride, wl.pad, wl.dilation, wl.offset_scale)
    ws = torch.empty(max(dcn.dcn4_backward_workspace_size(dsc), 16), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    ops = {
        "dcn4_forward": lambda: dcn.dcn4_forward(d["input"], d["offset_weight"], out=out, **kw),
        "dcn4_backward": lambda: dcn.dcn4_backward(d["input"], d["offset_weight"], d["grad_out"],
                                                   workspace=ws, grad_input=gin,
                                                   grad_offset_weight=gow, **kw),
        "msdcn_forward": lambda: dcn.msdcn_forward(m["input"], m["dir_weight"], m["scale_raw"],
                                                   m["s0"], wl.smax, out=ms_out, **kw),
    }
    for f in ops.values():  # first calls set kernel attributes outside any capture
        f()
    torch.cuda.synchronize()
    graphs = {}
    launches = {}  # library kernels recorded into each op's graph
    for name, f in ops.items():
        g = torch.cuda.CUDAGraph()
        before = dcn.dcn4_kernel_launches()
        with torch.cuda.graph(g):
            f()
        launches[name] = dcn.dcn4_kernel_launches() - before
        graphs[name] = g
    torch.cuda.synchronize()
    names = list(ops)
    stream = torch.cuda.current_stream(dev)

    def timed_step():
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        ev[0].record(stream)
        for i, n in enumerate(names):
            graphs[n].replay()
            ev[i + 1].record(stream)
        return ev

    for _ in range(args.warmup):
        timed_step()
    torch.cuda.synchronize()
    barrier(dev)
    torch.cuda.synchronize()
    per_op = {n: 0.0 for n in names}
    with ClockSampler(local) as clocks:
        evs = [timed_step() for _ in range(args.steps)]
        torch.cuda.synchronize()
    samples = {n: [] for n in names}
    for ev in evs:
        for i, n in enumerate(names):
            dt = ev[i].elapsed_time(ev[i + 1])
            per_op[n] += dt
            samples[n].append(dt)
    step_ms_local = sum(per_op.values()) / args.steps
    barrier(dev)
    torch.cuda.synchronize()
    step_ms = max_over_ranks(step_ms_local, dev)
    ib = ideal_bytes(wl, Ho, Wo)
    step_bytes = sum(ib.values())
    value = weak_scaling_value(step_bytes, step_ms, world)
    op_ms = {n: per_op[n] / args.steps for n in names}
    # diagnostics outside the timed region: the same ops without the L2
    # flush (inputs partly L2-resident), median of a few replays each
    warm = {n: [] for n in names}
    for _ in range(max(3, min(args.steps, 10))):
        for n in names:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graphs[n].replay()
            b.record(stream)
            torch.cuda.synchronize()
            warm[n].append(a.elapsed_time(b))
    peak, peak_kind = hbm_peak()
    breakdown = {}
    for n in names:
        gbs = ib[n] / (op_ms[n] * 1e-3) / 1e9
        breakdown[n] = {"ms": round(op_ms[n], 5), "median_ms": round(statistics.median(samples[n]), 5),
                        "warm_l2_median_ms": round(statistics.median(warm[n]), 5),
                        "ideal_bytes": ib[n], "GB/s": round(gbs, 1),
                        f"frac_of_{peak_kind}_hbm": round(gbs / peak, 4)}
    breakdown["dcn4_forward"]["Gsample_ch_per_s"] = round(
        samples_ch(wl, Ho, Wo) / (op_ms["dcn4_forward"] * 1e-3) / 1e9, 1)
    breakdown["msdcn_forward"]["Gsample_ch_per_s"] = round(
        samples_ch(wl, Ho, Wo) / (op_ms["msdcn_forward"] * 1e-3) / 1e9, 1)
    dom = max(names, key=lambda n: op_ms[n])
    dom_gbs = ib[dom] / (op_ms[dom] * 1e-3) / 1e9
    traffic = recorded_traffic(dom, wl.name)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(dom_gbs, 1), "peak": peak,
                "unit": "GB/s", "frac": round(dom_gbs / peak, 4), "traffic": traffic,
                "peak_source": f"{peak_kind} copy bandwidth",
                "bytes_per_launch": ib[dom]}

    # next rows beyond the step (MSDCN backward; the offset/weight producer),
    # timed the same way outside the timed region, reported on their own
    extra, configs, samples, e2e = None, None, [], None
    if not args.step_only:
        extra = next_rows(dcn, wl, Ho, Wo, d, m, kw, ws, flush, stream, peak, peak_kind)

        # every workload of the table, each op timed on its own (outside the step)
        configs, samples = time_configs(dcn, flush, stream, peak, peak_kind)

        # end to end: pinned host buffers, H2D copies + the three calls + D2H reads,
        # one after another and pipelined over steps
        e2e = run_e2e(args, dcn, host, mhost, ops, d, m, out, ms_out, gin, gow, dev, stream,
                      step_bytes, world)
        e2e_pipe = run_e2e_pipelined(args, dcn, wl, kw, host, mhost, dev, step_bytes, world)
        e2e["sequential_value"] = e2e["value"]
        e2e["sequential_ms_per_step"] = e2e["ms_per_step"]
        for k in ("value", "ms_per_step", "steps", "path"):
            e2e[k] = e2e_pipe[k]

    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic (seeded; shapes and distributions of an "
                                       "InternImage stage)",
            "config": describe(wl, Ho, Wo), "roofline": roofline, "ops": breakdown,
            "gpu_launches": args.steps * sum(launches.values()),
            "launches_per_step": launches, "e2e": e2e, "next_rows": extra,
            "configs": configs, "clocks": clocks.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.step_only:
        line["cpu_baseline"] = cpu_baseline(wl)
        for key, per_op in oracle_config_checks(samples).items():
            for op, errs in per_op.items():
                configs[key]["ops"][op].update(errs)
    barrier(dev)
    for g in graphs.values():
        del g
    graphs.clear()
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


def graph_median_ms(fn, flush, stream, reps=10):
    """Median device time of one graph replay of fn, L2 flushed before each."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    ts = []
    for _ in range(reps + 3):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    del g
    return statistics.median(ts[3:])


def next_rows(dcn, wl, Ho, Wo, d, m, kw, ws, flush, stream, peak, peak_kind):
    """MSDCN backward and the offset/weight producer (depthwise 3x3 + merged
    linear) on the step's shape: median ms, ideal bytes, GB/s."""
    import torch
    from deformable_convolution_dcn4_b200.workloads import make_producer_inputs
    eb = 4 if wl.dtype == "f32" else 2
    nin = wl.N * wl.H * wl.W * wl.C
    nout = wl.N * Ho * Wo * wl.C
    now = wl.N * Ho * Wo * wl.G * wl.K * 3
    graw = wl.N * Ho * Wo * wl.G
    gin = torch.empty_like(m["input"])
    gdw = torch.empty_like(m["dir_weight"])
    gsr = torch.empty_like(m["scale_raw"])
    go = d["grad_out"]
    res = {}
    ms = graph_median_ms(lambda: dcn.msdcn_backward(
        m["input"], m["dir_weight"], m["scale_raw"], m["s0"], wl.smax, go, workspace=ws,
        grad_input=gin, grad_dir_weight=gdw, grad_scale_raw=gsr, **kw), flush, stream)
    ib = (nin + now + graw + nout + nin + now + graw) * eb
    res["msdcn_backward"] = {"median_ms": round(ms, 5), "ideal_bytes": ib,
                             "GB/s": round(ib / (ms * 1e-3) / 1e9, 1),
                             f"frac_of_{peak_kind}_hbm": round(ib / (ms * 1e-3) / 1e9 / peak, 4)}
    if wl.H * wl.W == Ho * Wo:
        p = make_producer_inputs(wl.N, wl.H, wl.W, wl.C, wl.G, wl.K, wl.dtype, seed=wl.seed,
                                 device=d["input"].device)
        pout = torch.empty_like(d["offset_weight"])
        J = wl.G * wl.K * 3
        ms = graph_median_ms(lambda: dcn.dcn4_offset_producer(
            p["x"], p["dw_weight"], p["dw_bias"], p["lin_weight"], p["lin_bias"], out=pout,
            **kw), flush, stream)
        ib = (nin + now + 10 * wl.C + J * wl.C + J) * eb
        flops = 2.0 * nin * J + 18.0 * nin
        res["dcn4_offset_producer"] = {
            "median_ms": round(ms, 5), "ideal_bytes": ib, "GB/s": round(ib / (ms * 1e-3) / 1e9, 1),
            f"frac_of_{peak_kind}_hbm": round(ib / (ms * 1e-3) / 1e9 / peak, 4),
            "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1)}
    return res


def op_ideal_bytes(wl, Ho, Wo, op):
    """Ideal bytes of one op: every tensor it reads or writes once (DCNv4
    digest "GPU效率的理论分析" for the forward; the backward reads input,
    grad_out and offset_weight and writes grad_input and grad_offset_weight;
    MSDCN adds the raw scales, read and, in the backward, their gradient)."""
    eb = 4 if wl.dtype == "f32" else 2
    nin = wl.N * wl.H * wl.W * wl.C
    nout = wl.N * Ho * Wo * wl.C
    now = wl.N * Ho * Wo * wl.G * wl.K * 3
    nraw = wl.N * Ho * Wo * wl.G
    J = wl.G * wl.K * 3
    elems = {"fwd": nin + nout + now, "bwd": 2 * nin + nout + 2 * now,
             "bwd_acc16": 2 * nin + nout + 2 * now, "msfwd": nin + nout + now + nraw,
             "msbwd": 2 * nin + nout + 2 * now + 2 * nraw,
             # input and x read once, output written once, the sub-network's
             # weights; the records stay on chip
             "fused": 2 * nin + nout + 10 * wl.C + J * wl.C + J}[op]
    return elems * eb


def oob_fraction(wl, d, Ho, Wo, msdcn):
    """Fraction of bilinear samples whose position lies outside (-1, W) x
    (-1, H), i.e. that contribute nothing (a statistic of the synthetic
    inputs, printed next to the timings)."""
    import torch
    ow = (d["dir_weight"] if msdcn else d["offset_weight"]).float()
    dx, dy = ow[..., 0], ow[..., 1]
    if msdcn:
        raw = d["scale_raw"].float()
        s0 = d["s0"].to(raw.device).view(1, 1, 1, -1)
        s = torch.clamp(s0 * torch.nn.functional.softplus(raw), max=wl.smax).unsqueeze(-1)
        dx, dy = s * dx, s * dy
    dev = ow.device
    i = torch.arange(wl.kh, device=dev).repeat_interleave(wl.kw).view(1, 1, 1, 1, -1)
    j = torch.arange(wl.kw, device=dev).repeat(wl.kh).view(1, 1, 1, 1, -1)
    ho = torch.arange(Ho, device=dev).view(1, -1, 1, 1, 1)
    wo = torch.arange(Wo, device=dev).view(1, 1, -1, 1, 1)
    x = (wo * wl.stride[1] - wl.pad[1] + j * wl.dilation[1]).float() + dx * wl.offset_scale
    y = (ho * wl.stride[0] - wl.pad[0] + i * wl.dilation[0]).float() + dy * wl.offset_scale
    inside = (x > -1) & (x < wl.W) & (y > -1) & (y < wl.H)
    return round(1.0 - inside.float().mean().item(), 4)


def time_configs(dcn, flush, stream, peak, peak_kind):
    """Times every (config, op) of CONFIG_TABLE; returns (table, samples) where
    samples keep one image's inputs and GPU outputs (host, fp32) per op for the
    oracle check of the CPU-baseline leg."""
    import torch
    from deformable_convolution_dcn4_b200.workloads import WORKLOADS, make_fused_inputs, make_inputs
    table, samples = {}, []
    dev = flush.device
    for label, wname, ops in CONFIG_TABLE:
        wl = WORKLOADS[wname]
        desc = dcn.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, 0, (wl.kh, wl.kw), wl.stride, wl.pad,
                             wl.dilation, wl.offset_scale)
        Ho, Wo = dcn.dcn4_out_shape(desc)
        kw = dict(group=wl.G, kernel_size=(wl.kh, wl.kw), stride=wl.stride, pad=wl.pad,
                  dilation=wl.dilation, offset_scale=wl.offset_scale)
        entry = {"label": label, "shape": f"N{wl.N} {wl.H}x{wl.W} C{wl.C} G{wl.G} (D{wl.D}) "
                                          f"{wl.dtype}", "ops": {}}
        needs_dcn = any(not o.startswith("ms") and o != "fused" for o in ops)
        needs_ms = any(o.startswith("ms") for o in ops)
        dh = make_inputs(wl, (Ho, Wo), with_grad=True) if needs_dcn and wl.kind != "msdcn" else None
        mwl = wl if wl.kind == "msdcn" else msdcn_variant(wl)
        mh = make_inputs(mwl, (Ho, Wo), with_grad=True) if needs_ms else None
        d = {k: v.to(dev) for k, v in dh.items()} if dh else None
        m = {k: (v if k == "s0" else v.to(dev)) for k, v in mh.items()} if mh else None
        f = None
        if "fused" in ops:
            f = make_fused_inputs(wl.N, wl.H, wl.W, wl.C, wl.G, wl.dtype, seed=wl.seed,
                                  device=dev)
            # the records the call uses (written out once, untimed): the oob
            # statistic and the oracle check of the aggregation read them
            f["offset_weight"] = torch.empty((wl.N, Ho, Wo, wl.G, wl.K, 3), dtype=f["x"].dtype,
                                             device=dev)
            dcn.dcn4_fused_forward(f["input"], f["x"], f["dw_weight"], f["dw_bias"],
                                   f["lin_weight"], f["lin_bias"],
                                   offset_weight_out=f["offset_weight"], **kw)
        ws = torch.empty(max(wl.N * wl.H * wl.W * wl.C * 4, 16), dtype=torch.uint8, device=dev)
        n_s = wl.N - 1  # the image the oracle checks
        for op in ops:
            src = m if op.startswith("ms") else f if op == "fused" else d
            x = src["input"]
            chain_ms = kernel_ms = None
            if op == "fwd":
                outs = [torch.empty((wl.N, Ho, Wo, wl.C), dtype=x.dtype, device=dev)]
                fn = lambda: dcn.dcn4_forward(d["input"], d["offset_weight"], out=outs[0], **kw)
            elif op in ("bwd", "bwd_acc16"):
                outs = [torch.empty_like(x), torch.empty_like(d["offset_weight"])]
                math = "acc16" if op == "bwd_acc16" else "default"
                fn = lambda: dcn.dcn4_backward(d["input"], d["offset_weight"], d["grad_out"],
                                               workspace=ws, grad_input=outs[0],
                                               grad_offset_weight=outs[1], math=math, **kw)
            elif op == "msfwd":
                outs = [torch.empty((wl.N, Ho, Wo, wl.C), dtype=x.dtype, device=dev)]
                fn = lambda: dcn.msdcn_forward(m["input"], m["dir_weight"], m["scale_raw"],
                                               m["s0"], mwl.smax, out=outs[0], **kw)
            elif op == "fused":
                outs = [torch.empty((wl.N, Ho, Wo, wl.C), dtype=x.dtype, device=dev)]
                # scratch for the records and the forward's escapes, used
                # where the call takes the two-kernel chain (faster than the
                # fused kernel there)
                fdesc = dcn.make_desc(wl.N, wl.H, wl.W, wl.C, wl.G, f["x"].dtype)
                fws = torch.empty(max(16, dcn.dcn4_fused_forward_workspace_size(fdesc)),
                                  dtype=torch.uint8, device=dev)
                fn = lambda: dcn.dcn4_fused_forward(f["input"], f["x"], f["dw_weight"],
                                                    f["dw_bias"], f["lin_weight"],
                                                    f["lin_bias"], out=outs[0], workspace=fws,
                                                    **kw)
                kout = torch.empty_like(outs[0])
                kernel_ms = graph_median_ms(
                    lambda: dcn.dcn4_fused_forward(f["input"], f["x"], f["dw_weight"],
                                                   f["dw_bias"], f["lin_weight"], f["lin_bias"],
                                                   out=kout, algo="halo", **kw), flush, stream)
                # the two-kernel chain it replaces, same inputs, same flush
                rec_buf = torch.empty_like(f["offset_weight"])
                chain_out = torch.empty_like(outs[0])

                def chain():
                    dcn.dcn4_offset_producer(f["x"], f["dw_weight"], f["dw_bias"],
                                             f["lin_weight"], f["lin_bias"], out=rec_buf, **kw)
                    dcn.dcn4_forward(f["input"], rec_buf, out=chain_out, **kw)
                chain_ms = graph_median_ms(chain, flush, stream)
            else:  # msbwd
                outs = [torch.empty_like(x), torch.empty_like(m["dir_weight"]),
                        torch.empty_like(m["scale_raw"])]
                fn = lambda: dcn.msdcn_backward(m["input"], m["dir_weight"], m["scale_raw"],
                                                m["s0"], mwl.smax, m["grad_out"], workspace=ws,
                                                grad_input=outs[0], grad_dir_weight=outs[1],
                                                grad_scale_raw=outs[2], **kw)
            n0 = dcn.dcn4_kernel_launches()
            fn()
            launches = dcn.dcn4_kernel_launches() - n0
            ms = graph_median_ms(fn, flush, stream)
            ib = op_ideal_bytes(wl, Ho, Wo, op)
            gbs = ib / (ms * 1e-3) / 1e9
            rec = {"median_ms": round(ms, 5), "ideal_bytes": ib, "GB/s": round(gbs, 1),
                   f"frac_of_{peak_kind}_hbm": round(gbs / peak, 4), "launches": launches,
                   "oob_fraction": oob_fraction(mwl if op.startswith("ms") else wl, src, Ho, Wo,
                                                op.startswith("ms"))}
            if op in ("fwd", "msfwd", "fused"):
                rec["Gsample_ch_per_s"] = round(samples_ch(wl, Ho, Wo) / (ms * 1e-3) / 1e9, 1)
            if chain_ms is not None:
                rec["path"] = "fused kernel" if launches == 1 else "producer + forward"
                rec["fused_kernel_ms"] = round(kernel_ms, 5)
                rec["producer_plus_forward_ms"] = round(chain_ms, 5)
                rec["speedup_vs_chain"] = round(chain_ms / ms, 3)
            entry["ops"][op] = rec
            torch.cuda.synchronize()
            samples.append({"key": f"{label}_{wname}", "op": op,
                            "wl": (mwl if op.startswith("ms") else wl).replace(N=1),
                            "inputs": {k: sample_of(op, k, v, n_s) for k, v in src.items()},
                            "outputs": [t[n_s:n_s + 1].float().cpu() for t in outs]})
        table[f"{label}_{wname}"] = entry
        del d, m, f, ws, dh, mh
        torch.cuda.empty_cache()
    return table, samples


def sample_of(op, k, v, n):
    """Image n of an input tensor (host, fp32) for the oracle check; s0 and
    the fused call's sub-network weights as they are."""
    if k == "s0":
        return v
    if op == "fused" and v.dim() < 4:
        return v.float().cpu()
    return v[n:n + 1].float().cpu()


def oracle_config_checks(samples):
    """Part of the CPU-baseline leg: the oracle on the one sampled image of
    every (config, op), compared with the GPU result. Returns
    {key: {op: {max_scaled_err, max_rel_err_rms_floor}}} over all outputs."""
    import numpy as np

    import oracle
    orc = oracle.default()
    res = {}
    for smp in samples:
        wl, op, a = smp["wl"], smp["op"], {k: (v if k == "s0" else v.numpy())
                                            for k, v in smp["inputs"].items()}
        prob = orc.problem(1, wl.H, wl.W, wl.C, wl.G, wl.kh, wl.kw, wl.stride, wl.pad,
                           wl.dilation, wl.offset_scale)
        if op == "fwd":
            refs = [orc.forward(prob, a["input"], a["offset_weight"])]
        elif op in ("bwd", "bwd_acc16"):
            refs = list(orc.backward(prob, a["input"], a["offset_weight"], a["grad_out"]))
        elif op == "msfwd":
            refs = [orc.msdcn_forward(prob, a["input"], a["dir_weight"], a["scale_raw"],
                                      a["s0"].numpy(), wl.smax)]
        elif op == "fused":
            # the aggregation on the records the call used; those records
            # against the oracle's producer
            refs = [orc.forward(prob, a["input"], a["offset_weight"])]
            rec_ref = orc.offset_producer(prob, a["x"], a["dw_weight"], a["dw_bias"],
                                          a["lin_weight"], a["lin_bias"])
            rd = np.abs(a["offset_weight"].reshape(rec_ref.shape) - rec_ref)
            res.setdefault(smp["key"], {}).setdefault(op, {})["records_max_scaled_err"] = \
                float(f"{rd.max() / np.abs(rec_ref).max():.3e}")
        else:
            refs = list(orc.msdcn_backward(prob, a["input"], a["dir_weight"], a["scale_raw"],
                                           a["s0"].numpy(), wl.smax, a["grad_out"]))
        scaled, elem = 0.0, 0.0
        for got, ref in zip(smp["outputs"], refs):
            got = got.numpy().astype(np.float64)
            ref = np.asarray(ref, np.float64)
            diff = np.abs(got - ref)
            scale = np.abs(ref).max()
            rms = float(np.sqrt(np.mean(ref * ref)))
            scaled = max(scaled, float(diff.max() / scale) if scale > 0 else float(diff.max()))
            elem = max(elem, float((diff / (np.abs(ref) + rms)).max()) if rms > 0 else 0.0)
        res.setdefault(smp["key"], {}).setdefault(op, {}).update(
            {"max_scaled_err": float(f"{scaled:.3e}"),
             "max_rel_err_rms_floor": float(f"{elem:.3e}")})
    return res


def run_e2e_pipelined(args, dcn, wl, kw, host, mhost, dev, step_bytes, world):
    """The end-to-end step with transfers overlapped across steps: two sets
    of device buffers, three streams (host -> device copies, the three calls,
    device -> host reads). Step i's input copies wait until step i-2's calls
    have read that buffer set, its calls wait for its input copies and for
    step i-2's reads of the outputs, its reads wait for its calls; so step
    i+1's inputs cross PCIe while step i computes and its results come back.
    Every step still copies all its inputs in and all its results out."""
    import torch
    pin = {k: v.pin_memory() for k, v in host.items()}
    mpin = {k: (v if k == "s0" else v.pin_memory()) for k, v in mhost.items()}
    sets = []
    for _ in range(2):
        d = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in pin.items()}
        m = {k: (v if k == "s0" else torch.empty(v.shape, dtype=v.dtype, device=dev))
             for k, v in mpin.items()}
        out = torch.empty_like(d["input"])
        ms_out = torch.empty_like(m["input"])
        gin = torch.empty_like(d["input"])
        gow = torch.empty_like(d["offset_weight"])
        ws = torch.empty(max(d["input"].numel() * 4, 16), dtype=torch.uint8, device=dev)
        outs = [out, gin, gow, ms_out]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        sets.append((d, m, outs, hout, ws))
    h2d = sum(v.numel() * v.element_size() for v in pin.values()) + \
        sum(v.numel() * v.element_size() for k, v in mpin.items() if k != "s0")
    d2h = sum(t.numel() * t.element_size() for t in sets[0][2])
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ran = [torch.cuda.Event() for _ in range(2)]      # the set's calls are done
    read = [torch.cuda.Event() for _ in range(2)]     # the set's outputs are read back
    loaded = [torch.cuda.Event() for _ in range(2)]   # the set's inputs are in

    def step(i):
        b = i & 1
        d, m, outs, hout, ws = sets[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ran[b])
            for k, v in pin.items():
                d[k].copy_(v, non_blocking=True)
            for k, v in mpin.items():
                if k != "s0":
                    m[k].copy_(v, non_blocking=True)
            loaded[b].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(loaded[b])
            s_run.wait_event(read[b])
            dcn.dcn4_forward(d["input"], d["offset_weight"], out=outs[0], **kw)
            dcn.dcn4_backward(d["input"], d["offset_weight"], d["grad_out"], workspace=ws,
                              grad_input=outs[1], grad_offset_weight=outs[2], **kw)
            dcn.msdcn_forward(m["input"], m["dir_weight"], m["scale_raw"], m["s0"], wl.smax,
                              out=outs[3], **kw)
            ran[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ran[b])
            for t, h in zip(outs, hout):
                h.copy_(t, non_blocking=True)
            read[b].record(s_out)

    for b in range(2):  # events start out completed
        ran[b].record(s_run)
        read[b].record(s_out)
    for i in range(max(1, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    barrier(dev)
    steps = max(1, min(args.steps, 10))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    s_run.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(steps):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    t1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    return {"value": round(weak_scaling_value(step_bytes, ms, world), 2), "unit": "GB/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps,
            "path": "Python binding -> C ABI, pinned host buffers, cudaMemcpyAsync both ways "
                    "inside the timed region, transfers of neighbouring steps overlapped (two "
                    "device buffer sets, input / compute / output streams)"}


def run_e2e(args, dcn, host, mhost, ops, d, m, out, ms_out, gin, gow, dev, stream, step_bytes,
            world):
    import torch
    pin = {k: v.pin_memory() for k, v in host.items()}
    mpin = {k: (v if k == "s0" else v.pin_memory()) for k, v in mhost.items()}
    outs = [out, gin, gow, ms_out]
    hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    h2d = sum(v.numel() * v.element_size() for v in pin.values()) + \
        sum(v.numel() * v.element_size() for k, v in mpin.items() if k != "s0")
    d2h = sum(t.numel() * t.element_size() for t in outs)

    def step():
        for k, v in pin.items():
            d[k].copy_(v, non_blocking=True)
        for k, v in mpin.items():
            if k != "s0":
                m[k].copy_(v, non_blocking=True)
        for f in ops.values():
            f()
        for t, h in zip(outs, hout):
            h.copy_(t, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(dev)
    steps = max(1, min(args.steps, 10))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    return {"value": round(weak_scaling_value(step_bytes, ms, world), 2), "unit": "GB/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps, "path": "Python binding -> C ABI, pinned host buffers, "
                                    "cudaMemcpyAsync both ways inside the timed region"}


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    from deformable_convolution_dcn4_b200.workloads import WORKLOADS
    rank, world, _ = dist_env()
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    n_img = wl.N  # the whole batch: a fraction of a second per step on 16 host cores
    for _ in range(args.warmup):
        oracle_step_sample(wl, n_img)
    times, nbytes = [], 0.0
    for _ in range(args.steps):
        dt, b = oracle_step_sample(wl, n_img)
        times.append(dt)
        nbytes = b
    step_s = sum(times) / len(times)
    value = nbytes / step_s / 1e9
    sample = (f"fwd+bwd+MSDCN fwd of the CPU oracle on {n_img} of {wl.N} images of {wl.name} "
              f"per step")
    import oracle
    orc = oracle.default()
    Ho, Wo = orc.out_hw(orc.problem(wl.N, wl.H, wl.W, wl.C, wl.G, wl.kh, wl.kw, wl.stride,
                                    wl.pad, wl.dilation, wl.offset_scale))
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": describe(wl, Ho, Wo),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
