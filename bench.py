#!/usr/bin/env python
"""Throughput of the bucketed gradient-quantization step on B200.

One step = one pass of the whole hot path over one batch: for each of W simulated workers,
error feedback (v = g + r), per-bucket level fit, Philox stochastic rounding, dense bit packing
into the worker's message, residual update, and the decode + average of the W dequantized
gradients (gq_fused_step, messages written).

Default workload: 1e9-element fp32 gradient per worker (1000 blocks of 1e6 elements, block
sigma log-uniform in [1e-5, 1e-2]), W = 8 workers on one GPU, ORQ-5, d = 512, error feedback
on: 71 GB resident in HBM, far larger than L2.  Metric: gradient worker-elements per second.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gq|reference]

--impl reference times the CPU oracle (plain C, all host cores) on bounded samples of the same
workload.  With N > 1 (torchrun) every rank runs an independent replica on its GPU: the path
has no exchange between GPUs.

Other one-line modes (one GPU):
  --unfused   gq_encode per worker and gq_decode_accumulate, each against its own bytes
  --sweep     bucket sizes 128 .. 32768: throughput and normalised quantization variance
  --entropy   base-s packing of the W messages (gq_entropy_pack / gq_entropy_unpack)
  --elias     Elias-gamma coding of the W messages (gq_elias_pack / gq_elias_unpack), for an
              odd-level QSGD-family scheme such as --scheme qsgd_l2 --levels 3
  --exchange  the data-parallel exchange (exchange.Exchange): one worker per rank under
              torchrun, gq_encode + NCCL all-gather of the packed messages + gq_decode_accumulate
  --scheme terngrad_layer --workload resnet50
              TernGrad with one scale per parameter tensor (two passes: the tensors' maxima,
              then the rounding)
"""
import argparse
import concurrent.futures as cf
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gradient elems/s (encode+pack+decode+sum), ORQ-5 d=512; % of HBM peak"


def metric_name(args):
    """The headline metric's name for the default configuration (ORQ-5, d = 512); the same
    metric for another scheme, level count or bucket size names that configuration."""
    if (args.scheme, args.levels, args.bucket) == ("orq", 5, 512):
        return METRIC
    return "gradient elems/s (encode+pack+decode+sum), %s-%d d=%d; %% of HBM peak" % (
        args.scheme, args.levels, args.bucket)
UNIT = "elem/s"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0  # B200 HBM3e specification, shown beside the measured-peak fraction


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gq", choices=["gq", "reference"])
    ap.add_argument("--workload", default="blocks1b")
    ap.add_argument("--scheme", default="orq")
    ap.add_argument("--levels", type=int, default=5)
    ap.add_argument("--bucket", type=int, default=512)
    ap.add_argument("--clip", type=float, default=0.0)
    ap.add_argument("--elements", type=int, default=0, help="truncate the workload (profiling runs)")
    ap.add_argument("--no-msgs", action="store_true", help="do not write the messages")
    ap.add_argument("--base-s", action="store_true",
                    help="base-s messages (s = 3, 5, 9 levels) written by the encode and read by the decode")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--unfused", action="store_true",
                    help="the unfused path: gq_encode per worker, then gq_decode_accumulate; per-kernel "
                         "rooflines, one JSON line")
    ap.add_argument("--sweep", action="store_true",
                    help="bucket-size sweep (1e8 elements, W = 8, no error feedback): throughput and "
                         "normalised quantization variance per bucket size, one JSON line")
    ap.add_argument("--entropy", action="store_true",
                    help="base-s packing: gq_entropy_pack then gq_entropy_unpack of the W messages of one "
                         "step; per-kernel rooflines and the compression ratios, one JSON line")
    ap.add_argument("--exchange", action="store_true",
                    help="the quantized all-gather exchange, one worker per rank (W = the number of ranks): "
                         "per-phase times (encode, all-gather, decode), one JSON line from rank 0")
    ap.add_argument("--elias", action="store_true",
                    help="Elias-gamma coding: gq_elias_pack then gq_elias_unpack of the W messages of one "
                         "step (an odd-level QSGD-family scheme, e.g. --scheme qsgd_l2 --levels 3); "
                         "per-call rooflines and the bits per element, one JSON line")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------------
# bookkeeping shared by both arms
# ---------------------------------------------------------------------------------------------
def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def table_len(scheme_id, levels):
    """Floats per level table: the scale for the QSGD family (QSGD, TernGrad, QSGD-nearest,
    QSGD-l2), two levels for BinGrad-b / BinGrad-pb / SignSGD, s levels for ORQ."""
    return 1 if scheme_id in (0, 1, 5, 7) else (2 if scheme_id in (2, 3, 6) else levels)


# base-s groups: s -> (g codes, B bits)
BASE_S_GROUPS = {3: (5, 8), 5: (3, 7), 9: (5, 16)}


def message_bytes_per_elem(scheme_id, levels, d, base_s=False):
    """A message's bytes per element: the codes (b/8, or a bucket's base-s words over d) and the
    level table's share."""
    L = table_len(scheme_id, levels)
    if base_s:
        g, B = BASE_S_GROUPS[levels]
        return 4.0 * ((-(-d // g) * B + 31) // 32) / d + 4.0 * L / d
    return (levels - 1).bit_length() / 8.0 + 4.0 * L / d


def bytes_per_worker_elem(scheme_id, levels, d, W, ef, msgs, base_s=False):
    """Algorithmic HBM bytes per worker-element of the fused step: read g (and r), write r',
    the message and the worker's share of the average."""
    b = 4.0 + (8.0 if ef else 0.0) + 4.0 / W
    if msgs:
        b += message_bytes_per_elem(scheme_id, levels, d, base_s)
    return b


def max_over_ranks(x, device):
    """The largest of the ranks' values (every rank gets it): the job's time is its slowest rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, workers, n, steps, elapsed_ms):
    """Whole-job throughput: worker-elements processed by all ranks / the slowest rank's time."""
    return world * workers * n * steps / (elapsed_ms / 1000.0)


# The sources the fused warp-per-bucket kernel (d <= 512) is compiled and launched from: its
# code, its instantiation, its launch configuration and the plan it reads.  A stored traffic
# figure stands only while these are byte-identical to what was captured.
FUSED_KERNEL_SOURCES = ("gq_api.cu", "gq_device.cuh", "gq_internal.h", "gq_round.cuh", "gq_warp.cu",
                        "gq_warp.cuh", "gq_warp_orq.cu")


def source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gradient_quantization_communication_b200", "csrc")
    for fn in FUSED_KERNEL_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel_key):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_key)
    except Exception:
        return None
    if rec and rec.get("source_hash") == source_hash():
        return rec
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region (one GPU)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = bus_id
        self.proc = None
        self.out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus_id:
            cmd += ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [ln.split(", ") for ln in self.out.read().splitlines() if ln.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for nm, val in zip(names, r[5:9]):
                if val.strip() == "Active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def pci_bus_id(dev):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        return None


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------------------------
def oracle_sample_rate(wl, args, gs_host, nbuckets, threads):
    """Worker-elements per second of the oracle's fused step over the first nbuckets buckets of
    every worker (host arrays gs_host), split over `threads` host threads."""
    import numpy as np

    import oracle as O
    d = args.bucket
    n = nbuckets * d
    sid = O.SCHEMES[args.scheme]
    cfg = O.Config(sid, args.levels, d, wl.workers, int(wl.error_feedback), args.clip, wl.rounding_seed, n)
    gs = [np.ascontiguousarray(g[:n]) for g in gs_host]
    rs = [np.zeros(n, np.float32) for _ in gs] if wl.error_feedback else None
    bounds = [(nbuckets * i // threads, nbuckets * (i + 1) // threads) for i in range(threads)]
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda b: O.fused_step(cfg, 0, gs, rs, not args.no_msgs, b[0], b[1]), bounds))
    dt = time.perf_counter() - t0
    return wl.workers * n / dt, dt


def host_sample(wl_name, workers, nelem):
    import torch

    from gradient_quantization_communication_b200 import synth
    return [synth.gradient(wl_name, w, 0, n=nelem).numpy() for w in range(workers)]


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def calibrated_buckets(wl, args, gs_host, threads, seconds):
    probe = 8 * threads
    rate, dt = oracle_sample_rate(wl, args, gs_host, probe, threads)
    per_bucket = dt / probe
    return max(threads, int(seconds / per_bucket)), rate


# ---------------------------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gradient_quantization_communication_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    threads = cpu_threads()
    max_buckets = 64 * threads * 8
    gs_host = host_sample(args.workload, wl.workers, max_buckets * args.bucket)
    # size each step to about half a second of work on all host cores
    nbk, _ = calibrated_buckets(wl, args, gs_host, threads, 0.5)
    nbk = min(nbk, max_buckets)
    for _ in range(args.warmup):
        oracle_sample_rate(wl, args, gs_host, nbk, threads)
    times = []
    for _ in range(args.steps):
        _, dt = oracle_sample_rate(wl, args, gs_host, nbk, threads)
        times.append(dt)
    total = sum(times)
    value = wl.workers * nbk * args.bucket * args.steps / total
    sample = "first %d buckets (d=%d) of each of the %d workers per step" % (nbk, args.bucket, wl.workers)
    line = {
        "impl": "reference", "metric": metric_name(args), "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args, wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(args, wl):
    return {"workload": "%s: %d fp32 elements x W=%d workers, %s-%d, d=%d, error feedback %s%s" % (
        args.workload, wl.n, wl.workers, args.scheme, args.levels, args.bucket,
        "on" if wl.error_feedback else "off", (", clip %.1f sigma" % args.clip) if args.clip else ""),
        "elements": wl.n, "workers": wl.workers, "scheme": args.scheme, "levels": args.levels,
        "bucket": args.bucket, "messages_written": not args.no_msgs,
        "message_format": "base-s" if getattr(args, "base_s", False) else "dense",
        "l2": ("inputs larger than L2 (working set %.1f GB, L2 126 MB): no flush needed" % (wl.n * wl.workers * 12 / 1e9)
               if wl.n * wl.workers * 12 > 4 * 126e6 else "working set within a few L2 sizes: timings include L2 reuse"),
        "gradients": "drawn once in HBM before timing; the residual evolves every step"}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------
def fused_roofline(args, d, W, n, ef, write_msgs, bpe, achieved, peak, peak_kind):
    """The roofline object of the fused kernel's line (None above d = 512, where the step is two
    kernels).  The stored DRAM traffic is per launch of the captured configuration: it stands for
    this run only when the workload, error feedback, message writes and clip match, scaled by the
    elements processed."""
    if achieved is None:
        return None
    kernel_key = "fused_%s%d_d%d_w%d%s" % (args.scheme, args.levels, d, W, "_bases" if getattr(args, "base_s", False) else "")
    traffic = traffic_record(kernel_key)
    if traffic and (traffic.get("workload"), traffic.get("error_feedback"), traffic.get("messages_written"),
                    traffic.get("clip")) != (args.workload, bool(ef), bool(write_msgs), float(args.clip)):
        traffic = None
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "traffic": traffic["bytes_per_launch"] * n / traffic["elements"] if traffic else None,
            "algorithmic_bytes_per_launch": bpe * W * n, "kernel": kernel_key}


def default_line(args, wl, value, world, W, n, ms_per_step, bpe, peak, roofline, cpu, e2e, gpu_launches, clocks):
    """The default run's JSON line (rank 0)."""
    gbs = bpe * W * n / (ms_per_step / 1000.0) / 1e9  # one rank's bytes over the step time
    return {
        "metric": metric_name(args), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": workload_config(args, wl),
        "hbm_gbs_achieved": round(gbs, 1),
        "pct_hbm_peak": round(100.0 * gbs / peak, 2),
        "pct_hbm_spec": round(100.0 * gbs / SPEC_HBM_GBS, 2),
        "elem_per_s_per_worker": value / (W * world),
        "bytes_per_worker_elem": bpe,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": gpu_launches, "clocks": clocks,
    }


def run_gq(args):
    import torch
    import torch.distributed as dist

    import gradient_quantization_communication_b200.gq as G
    from gradient_quantization_communication_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = synth.WORKLOADS[args.workload]
    if args.elements:
        wl = dataclasses.replace(wl, n=min(wl.n, args.elements))
    W, n, d, ef = wl.workers, wl.n, args.bucket, wl.error_feedback
    sid = G.SCHEMES[args.scheme]
    cfg = G.gq_config(sid, args.levels, d, W, ef, args.clip, wl.rounding_seed, n)
    plan = G.Plan(cfg, fmt=G.GQ_FORMAT_BASE_S if args.base_s else G.GQ_FORMAT_DENSE)
    stream = torch.cuda.current_stream()
    g = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    for w in range(W):
        synth.gradient(args.workload, w, 0, n=n, out=g[w])
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if ef else None
    write_msgs = not args.no_msgs
    msgs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)] if write_msgs else None
    avg = torch.empty(n, dtype=torch.float32, device=dev)
    # d <= 512: the fused kernel over the full buckets, plus one launch for a ragged last bucket;
    # d > 512: one fused launch of the large-bucket kernel
    launches_per_step = ((1 if n >= d else 0) + (1 if n % d else 0)) if d <= 512 else 1

    def step(t):
        G.gq_fused_step(plan.handle, t, g, r, msgs, avg, stream)

    for t in range(args.warmup):
        step(t)
    torch.cuda.synchronize()
    if G.gq_plan_status(plan.handle, stream) != G.GQ_OK:
        raise RuntimeError("non-finite input in the benchmark workload")

    sampler = ClockSampler(pci_bus_id(dev)) if rank == 0 else None
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        ev[k][0].record(stream)
        step(args.warmup + k)
        ev[k][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    elapsed_ms = t_start.elapsed_time(t_end)
    per_launch_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    if world > 1:
        elapsed_ms = max_over_ranks(elapsed_ms, dev)
    ms_per_step = elapsed_ms / args.steps
    value = job_value(world, W, n, args.steps, elapsed_ms)

    bpe = bytes_per_worker_elem(sid, args.levels, d, W, ef, write_msgs, args.base_s)
    peak, peak_kind = measured_hbm_peak()
    achieved = bpe * W * n / (per_launch_ms / 1000.0) / 1e9 if d <= 512 else None
    roofline = fused_roofline(args, d, W, n, ef, write_msgs, bpe, achieved, peak, peak_kind)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, G, plan, W, n, g, r, msgs, avg, dev, stream, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(args, wl, g)

    plan.close()
    if rank == 0:
        line = default_line(args, wl, value, world, W, n, ms_per_step, bpe, peak, roofline, cpu, e2e,
                            launches_per_step * args.steps, clocks)
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def all_ranks_min(x, device):
    """The smallest of the ranks' values (every rank gets it); the value itself when alone."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return t.item()


def e2e_host_mode(W, n, avail, local_world):
    """Pinned host buffers the e2e leg can afford: 2 = one per worker plus the average,
    1 = one gradient buffer copied into every worker's device gradient plus the average (the same
    bytes cross PCIe every step), 0 = none.  The local ranks share the host's memory."""
    if avail is None:
        return 2
    budget = avail / (1.5 * max(1, local_world))
    if 4 * (W + 1) * n <= budget:
        return 2
    if 8 * n <= budget:
        return 1
    return 0


def run_e2e(args, G, plan, W, n, g, r, msgs, avg, dev, stream, world):
    """The same step through the C ABI with the gradients in pinned host memory: every step
    copies the W gradients host -> device, runs gq_fused_step and reads the average back, the
    steps pipelined when the device holds a second set of gradients and averages.  All ranks take
    the same decisions (and so the same collective calls) whatever their memory."""
    import torch
    try:
        with open("/proc/meminfo") as f:
            avail = 1024 * int(next(ln for ln in f if ln.startswith("MemAvailable")).split()[1])
    except Exception:
        avail = None
    local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
    mode = int(all_ranks_min(e2e_host_mode(W, n, avail, local_world), dev))
    if mode == 0:
        return {"value": None, "unit": UNIT, "error": "host memory: %s GB available for %d local ranks"
                % ("?" if avail is None else avail >> 30, local_world)}
    host_g, host_avg = [], None
    try:
        host_g = [torch.empty(n, dtype=torch.float32, pin_memory=True) for _ in range(W if mode == 2 else 1)]
        host_avg = torch.empty(n, dtype=torch.float32, pin_memory=True)
        ok = 1
    except Exception:
        ok = 0
    if all_ranks_min(ok, dev) < 1:
        del host_g, host_avg
        return {"value": None, "unit": UNIT, "error": "pinned host allocation failed on some rank"}
    for i, hg in enumerate(host_g):
        hg.copy_(g[i])
    # Pipelined across steps when a second set of device gradients and a second average fit: step
    # t's copy in (its own stream) fills the set step t - 1 is not reading, overlapping that
    # step's kernel, and step t - 1's average goes out on a third stream while step t's inputs
    # come in (PCIe carries both directions at once).  Every step still copies all of its inputs
    # in and its average out inside the timed region.
    try:
        g2 = [torch.empty_like(x) for x in g]
        avg2 = torch.empty_like(avg)
        ok = 1
    except Exception:
        g2, avg2, ok = None, None, 0
    pipelined = all_ranks_min(ok, dev) >= 1
    if not pipelined:
        g2, avg2 = None, None
        torch.cuda.empty_cache()
    gsets, avgs = ([g, g2], [avg, avg2]) if pipelined else ([g], [avg])
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    nb = len(gsets)
    read_done = [torch.cuda.Event() for _ in range(nb)]  # the kernel that read gradient set k
    out_done = [torch.cuda.Event() for _ in range(nb)]   # the copy out of average k
    for k in range(nb):
        read_done[k].record(stream)
        out_done[k].record(stream)

    def step(t):
        k = t % nb
        s_in.wait_event(read_done[k])
        with torch.cuda.stream(s_in):
            for w in range(W):
                gsets[k][w].copy_(host_g[w if mode == 2 else 0], non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_event(out_done[k])
        G.gq_fused_step(plan.handle, 1000 + t, gsets[k], r, msgs, avgs[k], stream)
        read_done[k].record(stream)
        s_out.wait_event(read_done[k])
        with torch.cuda.stream(s_out):
            host_avg.copy_(avgs[k], non_blocking=True)
        out_done[k].record(s_out)

    step(0)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for t in range(args.e2e_steps):
        step(1 + t)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    if world > 1:
        ms = max_over_ranks(ms, dev)
    del g2, avg2
    del host_g, host_avg
    return {"value": world * W * n * args.e2e_steps / (ms / 1000.0), "unit": UNIT,
            "h2d_bytes_per_step": 4 * W * n, "d2h_bytes_per_step": 4 * n, "steps": args.e2e_steps,
            "host_gradients": "one pinned buffer per worker" if mode == 2 else
            "one pinned buffer copied into every worker's gradient (host memory shared by %d ranks)" % local_world,
            "pipelined": ("copies in, kernel and copy out of consecutive steps overlap (two device gradient sets)"
                          if pipelined else "one device gradient set: copy in, kernel, copy out in sequence")}


def run_cpu_baseline(args, wl, g):
    """The oracle on all host cores, on the first buckets of every worker: a probe of 8 buckets
    per thread calibrates the rate, then a sample sized to about args.cpu_seconds of CPU work
    (at most 2 GB of host copies) is timed once."""
    threads = cpu_threads()
    d = args.bucket
    probe = min(8 * threads, wl.n // d)
    gs_probe = [x[:probe * d].cpu().numpy() for x in g]
    _, dt = oracle_sample_rate(wl, args, gs_probe, probe, threads)
    nbk = int(args.cpu_seconds / (dt / probe))
    nbk = max(probe, min(nbk, wl.n // d, (2 << 30) // (4 * d * wl.workers)))
    gs_host = [x[:nbk * d].cpu().numpy() for x in g]
    rate, dt = oracle_sample_rate(wl, args, gs_host, nbk, threads)
    # the same oracle on one thread, over the probe's buckets
    rate1, dt1 = oracle_sample_rate(wl, args, gs_probe, probe, 1)
    return {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "seconds": round(dt, 2),
            "sample": "first %d buckets (d=%d) of each of the %d workers, one step" % (nbk, d, wl.workers),
            "single_thread": {"value": rate1, "seconds": round(dt1, 2),
                              "sample": "first %d buckets of each worker" % probe}}


def run_unfused(args):
    """The step as its separate calls: gq_encode for each worker (fit, round, pack, residual; the
    message written to HBM), then gq_decode_accumulate over the W messages.  Each launch is
    timed with events on the launching stream; the line gives the step's throughput and, per
    kernel kind, the algorithmic bytes per launch over the mean launch time."""
    import torch

    import gradient_quantization_communication_b200.gq as G
    from gradient_quantization_communication_b200 import synth

    wl = synth.WORKLOADS[args.workload]
    if args.elements:
        wl = dataclasses.replace(wl, n=min(wl.n, args.elements))
    W, n, d, ef = wl.workers, wl.n, args.bucket, wl.error_feedback
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    sid = G.SCHEMES[args.scheme]
    cfg = G.gq_config(sid, args.levels, d, W, ef, args.clip, wl.rounding_seed, n)
    plan = G.Plan(cfg, fmt=G.GQ_FORMAT_BASE_S if args.base_s else G.GQ_FORMAT_DENSE)
    stream = torch.cuda.current_stream()
    g = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    for w in range(W):
        synth.gradient(args.workload, w, 0, n=n, out=g[w])
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if ef else None
    msgs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]
    avg = torch.empty(n, dtype=torch.float32, device=dev)

    def step(t, evs=None):
        for w in range(W):
            if evs is not None:
                evs[w][0].record(stream)
            G.gq_encode(plan.handle, w, t, g[w], r[w] if ef else None, msgs[w], stream)
            if evs is not None:
                evs[w][1].record(stream)
        if evs is not None:
            evs[W][0].record(stream)
        G.gq_decode_accumulate(plan.handle, msgs, avg, stream)
        if evs is not None:
            evs[W][1].record(stream)

    for t in range(args.warmup):
        step(t)
    torch.cuda.synchronize()
    if G.gq_plan_status(plan.handle, stream) != G.GQ_OK:
        raise RuntimeError("non-finite input in the benchmark workload")
    sampler = ClockSampler(pci_bus_id(dev))
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(W + 1)]
           for _ in range(args.steps)]
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(args.warmup + k, evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1) / args.steps
    enc_ms = statistics.mean(a.elapsed_time(b) for e in evs for a, b in e[:W])
    dec_ms = statistics.mean(e[W][0].elapsed_time(e[W][1]) for e in evs)
    plan.close()
    msg_b = message_bytes_per_elem(sid, args.levels, d, args.base_s)
    enc_b = 4.0 + (8.0 if ef else 0.0) + msg_b          # per element of one worker
    dec_b = W * msg_b + 4.0                             # per element of the average
    peak, peak_kind = measured_hbm_peak()

    def roof(bytes_per_launch, launch_ms):
        a = bytes_per_launch / (launch_ms / 1000.0) / 1e9
        return {"bound": "hbm", "achieved": round(a, 1), "peak": peak, "unit": "GB/s", "frac": round(a / peak, 4),
                "peak_kind": peak_kind, "algorithmic_bytes_per_launch": bytes_per_launch, "ms_per_launch": launch_ms}

    print(json.dumps({
        "metric": "unfused step: gq_encode x W + gq_decode_accumulate, worker-elements/s", "value": W * n / (ms / 1000.0),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "f32", "data": "synthetic", "config": workload_config(args, wl),
        "encode": roof(enc_b * n, enc_ms), "decode": roof(dec_b * n, dec_ms),
        "bytes": {"encode_per_worker_elem": enc_b, "decode_per_elem": dec_b},
        "gpu_launches": (W + 1) * args.steps, "clocks": clocks}))
    return 0


def run_layer(args):
    """TernGrad with one scale per parameter tensor (--scheme terngrad_layer) on a workload with
    tensor structure (resnet18 / resnet50: their parameter tensors; blocks1b: its 1e6-element
    blocks).  The fused step is two launches: the per-tensor maxima of |g + r| (a pass over g and
    r), then the rounding, residual, message and average (a second pass).  Both passes belong to
    the method: an element's scale depends on its whole tensor, which is far larger than the
    chip's memory for most tensors, so the algorithmic bytes count g and r twice."""
    import torch

    import gradient_quantization_communication_b200.gq as G
    from gradient_quantization_communication_b200 import synth

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
    if args.elements:
        wl = dataclasses.replace(wl, n=min(wl.n, args.elements))
    W, n, d, ef = wl.workers, wl.n, args.bucket, wl.error_feedback
    off = synth.tensor_offsets(args.workload, n)
    nseg = len(off) - 1
    cfg = G.gq_config(G.SCHEMES["terngrad_layer"], 3, d, W, ef, 0.0, wl.rounding_seed, n)
    plan = G.Plan(cfg, segments=off)
    stream = torch.cuda.current_stream()
    g = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    for w in range(W):
        synth.gradient(args.workload, w, 0, n=n, out=g[w])
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if ef else None
    msgs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]
    avg = torch.empty(n, dtype=torch.float32, device=dev)
    for t in range(args.warmup):
        G.gq_fused_step(plan.handle, t, g, r, msgs, avg, stream)
    torch.cuda.synchronize()
    if G.gq_plan_status(plan.handle, stream) != G.GQ_OK:
        raise RuntimeError("non-finite input in the benchmark workload")
    sampler = ClockSampler(pci_bus_id(dev))
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        G.gq_fused_step(plan.handle, args.warmup + k, g, r, msgs, avg, stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1) / args.steps
    msg_bytes = plan.msg_bytes
    plan.close()
    rw = 8.0 if ef else 4.0  # g (and r) per element and pass
    bpe = 2.0 * rw + (4.0 if ef else 0.0) + msg_bytes / n + 4.0 / W
    peak, peak_kind = measured_hbm_peak()
    achieved = bpe * W * n / (ms / 1000.0) / 1e9
    config = workload_config(args, wl)
    config.update({"scheme": "terngrad_layer", "levels": 3, "tensors": nseg,
                   "workload": "%s: %d fp32 elements in %d tensors x W=%d workers, terngrad_layer (one scale per "
                               "tensor), error feedback %s" % (args.workload, n, nseg, W, "on" if ef else "off")})
    print(json.dumps({
        "metric": "TernGrad with one scale per tensor, fused step, worker-elements/s", "value": W * n / (ms / 1000.0),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "f32", "data": "synthetic", "config": config,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind, "traffic": None,
                     "algorithmic_bytes_per_worker_elem": bpe,
                     "note": "both passes over g and r counted: the per-tensor scale needs the whole tensor first"},
        "gpu_launches": 2 * args.steps, "clocks": clocks}))
    return 0


# Measured peer copy between two B200s of this machine over NVLink, one direction (900 nominal).
PEER_LINK_GBS = 770.0


def run_exchange(args):
    """The data-parallel exchange of exchange.Exchange, one worker per rank: rank w quantizes its
    own gradient (worker index w) with gq_encode, the W packed messages are all-gathered over NCCL
    and every rank decodes and averages them with gq_decode_accumulate.  Each phase is timed with
    events on the launching stream (the all-gather's completion is ordered onto it); the step
    time is the slowest rank's.  Per-worker elements: the workload's n; W = the number of ranks.
    With one rank the all-gather is a copy on the GPU and no byte crosses a link."""
    import datetime

    import torch
    import torch.distributed as dist

    import gradient_quantization_communication_b200.gq as G
    from gradient_quantization_communication_b200 import synth
    from gradient_quantization_communication_b200.exchange import Exchange

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(_free_port()))
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wl = synth.WORKLOADS[args.workload]
    if args.elements:
        wl = dataclasses.replace(wl, n=min(wl.n, args.elements))
    n, d, ef, W = wl.n, args.bucket, wl.error_feedback, world
    sid = G.SCHEMES[args.scheme]
    cfg = G.gq_config(sid, args.levels, d, W, ef, args.clip, wl.rounding_seed, n)
    ex = Exchange(cfg, device=dev)
    g = torch.empty(n, dtype=torch.float32, device=dev)
    synth.gradient(args.workload, rank, 0, n=n, out=g)
    r = torch.zeros(n, dtype=torch.float32, device=dev) if ef else None
    avg = torch.empty(n, dtype=torch.float32, device=dev)
    for t in range(args.warmup):
        ex.step(t, g, r, avg)
    torch.cuda.synchronize()
    if G.gq_plan_status(ex.plan.handle) != G.GQ_OK:
        raise RuntimeError("non-finite input in the benchmark workload")
    sampler = ClockSampler(pci_bus_id(dev)) if rank == 0 else None
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for k in range(args.steps):
        ex.step(args.warmup + k, g, r, avg, events=evs[k])
    t1.record()
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop() if sampler else None
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), dev)
    phase = [max_over_ranks(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs), dev) for i in range(3)]
    msg_bytes = ex.msg_bytes
    ex.close()
    dist.destroy_process_group()
    if rank != 0:
        return 0
    ms = elapsed_ms / args.steps
    msg_b = message_bytes_per_elem(sid, args.levels, d)
    enc_b = 4.0 + (8.0 if ef else 0.0) + msg_b  # per element of this rank's worker
    dec_b = W * msg_b + 4.0                     # per element of the average
    peak, peak_kind = measured_hbm_peak()

    def roof(bytes_per_call, call_ms):
        a = bytes_per_call / (call_ms / 1000.0) / 1e9
        return {"bound": "hbm", "achieved": round(a, 1), "peak": peak, "unit": "GB/s", "frac": round(a / peak, 4),
                "peak_kind": peak_kind, "algorithmic_bytes_per_call": bytes_per_call, "ms_per_call": call_ms}

    recv = (W - 1) * msg_bytes  # bytes that reach each rank over the links
    link = {"bound": "nvlink", "ms_per_call": phase[1], "bytes_received_per_rank": recv,
            "achieved": round(recv / (phase[1] / 1000.0) / 1e9, 1) if recv else None, "peak": PEER_LINK_GBS,
            "unit": "GB/s", "frac": round(recv / (phase[1] / 1000.0) / 1e9 / PEER_LINK_GBS, 4) if recv else None,
            "peak_kind": "measured peer copy, one direction"}
    config = workload_config(args, wl)
    config.update({"workload": "%s: %d fp32 elements per worker x W=%d workers (one per rank), %s-%d, d=%d, "
                               "error feedback %s" % (args.workload, n, W, args.scheme, args.levels, d,
                                                      "on" if ef else "off"),
                   "workers": W, "elements_per_worker": n,
                   "parallelism": "one worker per rank, all-gather of the packed messages"})
    tail = 1 if n % d else 0
    print(json.dumps({
        "metric": "quantized exchange step (encode + all-gather + decode), worker-elements/s",
        "value": W * n / (ms / 1000.0), "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config,
        "encode": roof(enc_b * n, phase[0]), "allgather": link, "decode": roof(dec_b * n, phase[2]),
        "bytes": {"encode_per_elem": enc_b, "decode_per_elem": dec_b, "message": msg_bytes},
        "gpu_launches": ((1 if n >= d else 0) + tail + 1) * args.steps, "clocks": clocks}))
    return 0


def _free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def run_entropy(args):
    """Base-s packing of the W messages of one fused step: a timed step is gq_entropy_pack of
    every worker's message followed by gq_entropy_unpack of every base-s message (each launch
    timed with events on the launching stream).  After timing, the unpacked messages must equal
    the dense ones byte for byte."""
    import torch

    import gradient_quantization_communication_b200.gq as G
    from gradient_quantization_communication_b200 import synth

    wl = synth.WORKLOADS[args.workload]
    if args.elements:
        wl = dataclasses.replace(wl, n=min(wl.n, args.elements))
    W, n, d, ef = wl.workers, wl.n, args.bucket, wl.error_feedback
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    sid = G.SCHEMES[args.scheme]
    cfg = G.gq_config(sid, args.levels, d, W, ef, args.clip, wl.rounding_seed, n)
    stream = torch.cuda.current_stream()
    plan = G.Plan(cfg)
    msgs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]
    g = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    for w in range(W):
        synth.gradient(args.workload, w, 0, n=n, out=g[w])
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if ef else None
    avg = torch.empty(n, dtype=torch.float32, device=dev)
    G.gq_fused_step(plan.handle, 0, g, r, msgs, avg, stream)
    if G.gq_plan_status(plan.handle, stream) != G.GQ_OK:
        raise RuntimeError("non-finite input in the benchmark workload")
    plan.close()
    del g, r, avg
    torch.cuda.empty_cache()
    ebytes, _, _ = G.gq_entropy_layout(cfg)
    emsgs = [torch.empty(ebytes, dtype=torch.uint8, device=dev) for _ in range(W)]
    backs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]

    def step(evs=None):
        for w in range(W):
            if evs is not None:
                evs[w][0].record(stream)
            G.gq_entropy_pack(cfg, msgs[w], emsgs[w], stream)
            if evs is not None:
                evs[w][1].record(stream)
        for w in range(W):
            if evs is not None:
                evs[W + w][0].record(stream)
            G.gq_entropy_unpack(cfg, emsgs[w], backs[w], stream)
            if evs is not None:
                evs[W + w][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(pci_bus_id(dev))
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2 * W)]
           for _ in range(args.steps)]
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    for w in range(W):
        if not torch.equal(backs[w], msgs[w]):
            raise RuntimeError("base-s round trip differs for worker %d" % w)
    ms = t0.elapsed_time(t1) / args.steps
    pack_ms = statistics.mean(a.elapsed_time(b) for e in evs for a, b in e[:W])
    unpack_ms = statistics.mean(a.elapsed_time(b) for e in evs for a, b in e[W:])
    # algorithmic bytes per launch: the dense message read and the base-s message written (or
    # the reverse), codes and level tables, without the padding
    bits = (args.levels - 1).bit_length()
    L = table_len(sid, args.levels)
    nb = (n + d - 1) // d
    gsz, B = {3: (5, 8), 5: (3, 7), 9: (5, 16)}[args.levels]
    ew = (-(-d // gsz) * B + 31) // 32
    dense_b = nb * (d * bits // 8 + 4 * L)
    base_b = nb * (4 * ew + 4 * L)
    peak, peak_kind = measured_hbm_peak()

    def roof(bytes_per_launch, launch_ms):
        a = bytes_per_launch / (launch_ms / 1000.0) / 1e9
        return {"bound": "hbm", "achieved": round(a, 1), "peak": peak, "unit": "GB/s", "frac": round(a / peak, 4),
                "peak_kind": peak_kind, "algorithmic_bytes_per_launch": dense_b + base_b, "ms_per_launch": launch_ms}

    print(json.dumps({
        "metric": "base-s pack + unpack of the W messages, worker-elements/s", "value": W * n / (ms / 1000.0),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "u32", "data": "synthetic", "config": workload_config(args, wl),
        "pack": roof(dense_b + base_b, pack_ms), "unpack": roof(dense_b + base_b, unpack_ms),
        "compression": {"dense_bits_per_elem": 8.0 * dense_b / n, "base_s_bits_per_elem": 8.0 * base_b / n,
                        "ratio_vs_fp32_dense": round(32.0 * n / (8.0 * dense_b), 3),
                        "ratio_vs_fp32_base_s": round(32.0 * n / (8.0 * base_b), 3),
                        "ratio_vs_fp32_base_s_codes_only": round(32.0 * d / (32.0 * ew), 3)},
        "round_trip": "exact", "gpu_launches": 2 * W * args.steps, "clocks": clocks}))
    return 0


def run_elias(args):
    """Elias-gamma coding of the W messages of one fused step: a timed step is gq_elias_pack of
    every worker's message (five launches) followed by gq_elias_unpack of every Elias message
    (one launch), each call timed with events on the launching stream.  After timing, every
    unpacked message must equal its dense message byte for byte."""
    import numpy as np
    import torch

    import gradient_quantization_communication_b200.gq as G
    from gradient_quantization_communication_b200 import synth

    wl = synth.WORKLOADS[args.workload]
    if args.elements:
        wl = dataclasses.replace(wl, n=min(wl.n, args.elements))
    W, n, d, ef = wl.workers, wl.n, args.bucket, wl.error_feedback
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    sid = G.SCHEMES[args.scheme]
    cfg = G.gq_config(sid, args.levels, d, W, ef, args.clip, wl.rounding_seed, n)
    stream = torch.cuda.current_stream()
    plan = G.Plan(cfg)
    msgs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]
    g = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    for w in range(W):
        synth.gradient(args.workload, w, 0, n=n, out=g[w])
    r = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(W)] if ef else None
    avg = torch.empty(n, dtype=torch.float32, device=dev)
    G.gq_fused_step(plan.handle, 0, g, r, msgs, avg, stream)
    if G.gq_plan_status(plan.handle, stream) != G.GQ_OK:
        raise RuntimeError("non-finite input in the benchmark workload")
    plan.close()
    del g, r, avg
    torch.cuda.empty_cache()
    cap, _, _, _ = G.gq_elias_layout(cfg)
    emsgs = [torch.empty(cap, dtype=torch.uint8, device=dev) for _ in range(W)]
    backs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]

    def step(evs=None):
        for w in range(W):
            if evs is not None:
                evs[w][0].record(stream)
            G.gq_elias_pack(cfg, msgs[w], emsgs[w], stream)
            if evs is not None:
                evs[w][1].record(stream)
        for w in range(W):
            if evs is not None:
                evs[W + w][0].record(stream)
            G.gq_elias_unpack(cfg, emsgs[w], backs[w], stream)
            if evs is not None:
                evs[W + w][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(pci_bus_id(dev))
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2 * W)]
           for _ in range(args.steps)]
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    for w in range(W):
        if not torch.equal(backs[w], msgs[w]):
            raise RuntimeError("Elias round trip differs for worker %d" % w)
    ms = t0.elapsed_time(t1) / args.steps
    pack_ms = statistics.mean(a.elapsed_time(b) for e in evs for a, b in e[:W])
    unpack_ms = statistics.mean(a.elapsed_time(b) for e in evs for a, b in e[W:])
    T = [int(e[:8].cpu().numpy().view(np.uint64)[0]) for e in emsgs]
    used = [G.gq_elias_used_bytes(cfg, t) for t in T]
    bits = (args.levels - 1).bit_length()
    L = table_len(sid, args.levels)
    nb = (n + d - 1) // d
    dense_b = nb * (d * bits // 8 + 4 * L)
    elias_b = statistics.mean(used)
    # algorithmic bytes of one call: the dense message read and the Elias message written (or
    # the reverse); pack also reads and writes the per-bucket counts once more for the scan
    algo = dense_b + elias_b
    peak, peak_kind = measured_hbm_peak()

    def roof(bytes_per_call, call_ms):
        a = bytes_per_call / (call_ms / 1000.0) / 1e9
        return {"bound": "hbm", "achieved": round(a, 1), "peak": peak, "unit": "GB/s", "frac": round(a / peak, 4),
                "peak_kind": peak_kind, "algorithmic_bytes_per_call": bytes_per_call, "ms_per_call": call_ms}

    print(json.dumps({
        "metric": "Elias-gamma pack + unpack of the W messages, worker-elements/s", "value": W * n / (ms / 1000.0),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "u32", "data": "synthetic", "config": workload_config(args, wl),
        "pack": roof(algo, pack_ms), "unpack": roof(algo, unpack_ms),
        "compression": {"dense_bits_per_elem": 8.0 * dense_b / n, "stream_bits_per_elem": statistics.mean(T) / n,
                        "elias_bits_per_elem": 8.0 * elias_b / n,
                        "ratio_vs_fp32_dense": round(32.0 * n / (8.0 * dense_b), 3),
                        "ratio_vs_fp32_elias": round(32.0 * n / (8.0 * elias_b), 3)},
        "round_trip": "exact", "gpu_launches": 6 * W * args.steps, "clocks": clocks}))
    return 0


def run_sweep(args):
    """Fused-step throughput and normalised quantization variance sum (b-u)(u-a) / sum u^2 for
    every bucket size of the sweep workload, for ORQ-5 and QSGD-5."""
    import torch

    import gradient_quantization_communication_b200.gq as G
    from gradient_quantization_communication_b200 import synth

    wl = synth.WORKLOADS["mixture100m"]
    n = min(wl.n, args.elements) if args.elements else wl.n
    W = wl.workers
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    g = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(W)]
    for w in range(W):
        synth.gradient("mixture100m", w, 0, n=n, out=g[w])
    avg = torch.empty(n, dtype=torch.float32, device=dev)
    out = torch.zeros(3, dtype=torch.float64, device=dev)
    peak, _ = measured_hbm_peak()
    rows = []
    for scheme, levels, _clip in wl.schemes:
        for d in wl.buckets_sweep:
            cfg = G.gq_config(scheme, levels, d, W, False, 0.0, wl.rounding_seed, n)
            with G.Plan(cfg) as plan:
                msgs = [torch.empty(plan.msg_bytes, dtype=torch.uint8, device=dev) for _ in range(W)]
                for t in range(args.warmup):
                    G.gq_fused_step(plan.handle, t, g, None, msgs, avg)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                a.record()
                for t in range(args.steps):
                    G.gq_fused_step(plan.handle, args.warmup + t, g, None, msgs, avg)
                b.record()
                torch.cuda.synchronize()
                ms = a.elapsed_time(b) / args.steps
                e = uu = 0.0
                for w in range(W):
                    G.gq_quant_error(plan.handle, w, 0, g[w], None, out)
                    o = out.cpu().tolist()
                    e += o[0]
                    uu += o[1]
                sid = G.SCHEMES[scheme]
                bpe = bytes_per_worker_elem(sid, levels, d, W, False, True)
                rows.append({"scheme": "%s-%d" % (scheme, levels), "bucket": d, "ms_per_step": round(ms, 4),
                             "elem_per_s": W * n / (ms / 1000.0), "bytes_per_worker_elem": round(bpe, 4),
                             "pct_hbm_peak": round(100.0 * bpe * W * n / (ms / 1000.0) / 1e9 / peak, 2),
                             "normalised_variance": e / uu})
                del msgs
    print(json.dumps({"metric": "bucket-size sweep: throughput and normalised quantization variance",
                      "workload": "mixture100m: %d fp32 elements x W=%d, error feedback off" % (n, W),
                      "steps": args.steps, "warmup": args.warmup, "data": "synthetic", "sweep": rows}))
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.unfused:
        return run_unfused(args)
    if args.entropy:
        return run_entropy(args)
    if args.elias:
        return run_elias(args)
    if args.exchange:
        return run_exchange(args)
    if args.scheme == "terngrad_layer":
        return run_layer(args)
    return run_gq(args)


if __name__ == "__main__":
    sys.exit(main())
