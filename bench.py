"""Benchmark of the sink-aware GQA attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl {flint,reference}]

One step is one attention-layer forward (flint_attn_fwd: key preparation +
attention kernel) over one batch of seeded synthetic input already resident
in HBM.  The default workload is the full-attention layer at S=4096 (32 query
heads, 4 KV heads, head dim 128, no RoPE, FP32 sinks), the configuration the
headline metric (attention TFLOP/s, ms per layer) is quoted on.  Inputs are
smaller than L2, so L2 is flushed (a 256 MiB write) before every timed step.

With --gpus N > 1 (launched by torch.distributed.run) every rank runs its own
replica on its own GPU (weak scaling, no data-path collective); NCCL is only
used for the barriers and the max-over-ranks of the timings.

--workload bwd_<name> times the gradient (flint_attn_bwd) on workload <name>
instead; decode_* workloads time one decode step.

--impl reference times the FP64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "sink-attn fwd TFLOP/s (BF16) and % of B200 tensor peak; ms/layer at S=4096"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "full_s4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# sources of the attention kernel; a recorded ncu traffic figure is used only
# while they are unchanged
KERNEL_SOURCES = [os.path.join(os.path.dirname(os.path.abspath(__file__)), "full_gqa_learned_b200",
                               "csrc", f) for f in ("flint_attn.cu", "flint_common.cuh", "sm100.cuh")]


def recorded_traffic(workload, profiles_dir=None):
    """DRAM bytes (read + write) per attention-kernel launch from the committed
    ncu summary of `workload`, or None when there is none or the kernel's
    sources changed since it was taken."""
    if profiles_dir is None:
        profiles_dir = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles")
    for name in ("attn_fwd_kernel", "attn_fwd_qprep_kernel"):
        path = os.path.join(profiles_dir, "%s_%s_ncu.md" % (name, workload))
        if os.path.exists(path):
            break
    else:
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            key, sep, val = line.partition(":")
            if sep:
                vals[key.strip()] = val.strip()
    if "traffic_bytes_per_launch" not in vals or "kernel_source_sha256" not in vals:
        return None
    if kernel_code_sha256() != vals["kernel_source_sha256"]:
        return None
    return float(vals["traffic_bytes_per_launch"])


def strip_comments(text):
    """C/C++ source without // and /* */ comments (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "".join(out)


def kernel_code_sha256():
    """SHA-256 of the attention kernel's sources with comments removed and
    whitespace collapsed: a recorded profile stays valid across comment and
    layout edits, not code edits."""
    h = hashlib.sha256()
    for src in KERNEL_SOURCES:
        with open(src, encoding="utf-8") as f:
            # whitespace runs collapsed: a removed comment leaves no trace
            h.update(" ".join(strip_comments(f.read()).split()).encode("utf-8"))
    return h.hexdigest()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def row_flops(w, rows):
    """Window-aware FLOPs of the given query rows: 4*128*32 per visible key,
    a valid query i of a segment starting at s seeing min(i-s+1, window) keys."""
    import oracle
    doc = oracle.doc_ids(w.T, w.cu_seqlens, w.pad_mask)
    start = np.zeros(w.T, np.int64)
    for t in range(1, w.T):
        start[t] = start[t - 1] if doc[t] == doc[t - 1] else t
    rows = np.asarray(rows)
    n = rows - start[rows] + 1
    if w.window > 0:
        n = np.minimum(n, w.window)
    n = np.where(doc[rows] >= 0, n, 0)
    return 4.0 * 128 * 32 * float(n.sum())


def max_over_ranks(values, device=None):
    """Element-wise maximum of per-rank timings (ms) across all ranks of the
    default process group (any backend); identity on a single process."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_tflops(flops_per_rank_step, steps, world, max_total_ms):
    """Throughput of the whole job: every rank processes its own replica, so
    the units done are world x steps x flops per step, over the slowest
    rank's time."""
    return world * flops_per_rank_step * steps / (max_total_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
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
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- flint arm

def soak(args, work, sync):
    """About args.soak seconds of untimed load while the clock sampler runs,
    so that it records the clocks of the part under this workload (a timed
    region of a few milliseconds ends before nvidia-smi's first sample)."""
    if args.profile:
        return
    time.sleep(0.3)
    t_end = time.time() + args.soak
    while time.time() < t_end:
        for _ in range(20):
            work()
        sync()


def run_flint(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import full_gqa_learned_b200 as fa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = W.make(args.workload)
    T = w.T

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16)
    host = dict(q=bf(w.q), k=bf(w.k), v=bf(w.v), q_norm_w=torch.from_numpy(w.q_norm_w),
                k_norm_w=torch.from_numpy(w.k_norm_w),
                sinks=torch.from_numpy(np.ascontiguousarray(w.sinks, np.float32)))
    if w.pos_ids is not None:
        host["pos_ids"] = torch.from_numpy(w.pos_ids)
    if w.cu_seqlens is not None:
        host["cu_seqlens"] = torch.from_numpy(w.cu_seqlens)
    if w.pad_mask is not None:
        host["pad_mask"] = torch.from_numpy(w.pad_mask)
    d = {k: v.to(dev) for k, v in host.items()}
    nseg = (len(w.cu_seqlens) - 1) if w.cu_seqlens is not None else (
        w.pad_mask.shape[0] if w.pad_mask is not None else 1)
    out = torch.empty((T, 4096), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((32, T), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.workspace_bytes(T, nseg), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kw = dict(pos_ids=d.get("pos_ids"), cu_seqlens=d.get("cu_seqlens"),
              pad_mask=d.get("pad_mask"), window=w.window, use_rope=w.use_rope,
              rope_theta=w.rope_theta, eps=w.eps, out=out, lse=lse, workspace=ws,
              stream=stream)

    def step(ev=None):
        if ev is None:
            fa.attn_fwd(d["q"], d["k"], d["v"], d["q_norm_w"], d["k_norm_w"], d["sinks"], **kw)
            return
        ev[0].record(stream)
        fa.attn_fwd(d["q"], d["k"], d["v"], d["q_norm_w"], d["k_norm_w"], d["sinks"],
                    stage="prepare", **kw)
        ev[1].record(stream)
        fa.attn_fwd(d["q"], d["k"], d["v"], d["q_norm_w"], d["k_norm_w"], d["sinks"],
                    stage="attend", **kw)
        ev[2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up, then a ~1 s soak so the clock sampler sees the part under load
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    st = fa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status %s" % fa.STATUS.get(st, st))
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    if not args.profile:
        time.sleep(0.3)
    t_end = time.time() + (0.0 if args.profile else args.soak)
    while time.time() < t_end:
        for _ in range(20):
            step()
        torch.cuda.synchronize(dev)

    # timed region: exactly K steps of the one-call public path, L2 flushed
    # before each
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    st = fa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status %s" % fa.STATUS.get(st, st))
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = sum(step_ms)

    # the two kernels apart (stage by stage, same inputs and flushes): the
    # attention kernel's duration for its roofline, the preparation kernel's
    # for the breakdown
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step(evs[i])
    torch.cuda.synchronize(dev)
    prep_ms = [e[0].elapsed_time(e[1]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    attn_avg = sum(attn_ms) / len(attn_ms)

    if args.profile:
        return dict(w=w, total_ms=total_ms, attn_avg=attn_avg, prep_avg=sum(prep_ms) / len(prep_ms),
                    e2e_ms=float("nan"), h2d=0, d2h=0, clocks=clocks, launches=2 * args.steps,
                    gpu=torch.cuda.get_device_name(dev))

    # end-to-end through the public API from pinned host buffers
    pinned = {k: v.pin_memory() for k, v in host.items()}
    out_h = torch.empty((T, 4096), dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty((32, T), dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_h.numel() * 2 + lse_h.numel() * 4
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        dd = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
        o, l = fa.attn_fwd(dd["q"], dd["k"], dd["v"], dd["q_norm_w"], dd["k_norm_w"],
                           dd["sinks"], pos_ids=dd.get("pos_ids"), cu_seqlens=dd.get("cu_seqlens"),
                           pad_mask=dd.get("pad_mask"), window=w.window, use_rope=w.use_rope,
                           rope_theta=w.rope_theta, eps=w.eps, workspace=ws)
        out_h.copy_(o, non_blocking=True)
        lse_h.copy_(l, non_blocking=True)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = 0.0
    for _ in range(e2e_steps):
        flush.fill_(3)
        e0.record(stream)
        dd = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
        o, l = fa.attn_fwd(dd["q"], dd["k"], dd["v"], dd["q_norm_w"], dd["k_norm_w"],
                           dd["sinks"], pos_ids=dd.get("pos_ids"), cu_seqlens=dd.get("cu_seqlens"),
                           pad_mask=dd.get("pad_mask"), window=w.window, use_rope=w.use_rope,
                           rope_theta=w.rope_theta, eps=w.eps, workspace=ws)
        out_h.copy_(o, non_blocking=True)
        lse_h.copy_(l, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms += e0.elapsed_time(e1)
    e2e_ms /= e2e_steps

    # max over ranks
    total_ms, attn_avg, e2e_ms = max_over_ranks([total_ms, attn_avg, e2e_ms], device=dev)
    return dict(w=w, total_ms=total_ms, attn_avg=attn_avg, prep_avg=sum(prep_ms) / len(prep_ms),
                e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, clocks=clocks, launches=2 * args.steps,
                gpu=torch.cuda.get_device_name(dev))


def time_config(name, dev, steps=20, warmup=5):
    """Layer, attention-kernel and preparation-kernel times (ms, CUDA events,
    L2 flushed before every step) of one named workload: the per-config
    record of the default run.  Inputs are the workload's seeded tensors,
    already resident in HBM."""
    import torch
    import full_gqa_learned_b200 as fa
    w = W.make(name)

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(dev)
    d = dict(q=bf(w.q), k=bf(w.k), v=bf(w.v), q_norm_w=torch.from_numpy(w.q_norm_w).to(dev),
             k_norm_w=torch.from_numpy(w.k_norm_w).to(dev),
             sinks=torch.from_numpy(np.ascontiguousarray(w.sinks, np.float32)).to(dev))
    opt = {n: torch.from_numpy(getattr(w, n)).to(dev) for n in ("pos_ids", "cu_seqlens", "pad_mask")
           if getattr(w, n) is not None}
    nseg = (len(w.cu_seqlens) - 1) if w.cu_seqlens is not None else (
        w.pad_mask.shape[0] if w.pad_mask is not None else 1)
    out = torch.empty((w.T, 4096), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((32, w.T), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.workspace_bytes(w.T, nseg), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kw = dict(window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps, out=out,
              lse=lse, workspace=ws, stream=stream, **opt)

    def call(stage="both"):
        fa.attn_fwd(d["q"], d["k"], d["v"], d["q_norm_w"], d["k_norm_w"], d["sinks"], stage=stage, **kw)
    for _ in range(warmup):
        flush.fill_(1)
        call()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
        flush.fill_((i + 7) & 0xFF)
        ev[i][2].record(stream)
        call("prepare")
        ev[i][3].record(stream)
        call("attend")
        ev[i][4].record(stream)
    torch.cuda.synchronize(dev)
    st = fa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status %s on %s" % (fa.STATUS.get(st, st), name))
    layer = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    prep = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    attn = statistics.mean(e[3].elapsed_time(e[4]) for e in ev)
    del d, opt, out, lse, ws, flush
    torch.cuda.empty_cache()
    return w, layer, attn, prep


def configs_record(dev, peak, main=None):
    """Per-config record of every named workload (the driver's default run
    carries it): layer and kernel times, TFLOP/s and fractions of the peak."""
    rec = {}
    for name in W.CONFIGS:
        if main is not None and name == main["name"]:
            w_flops, layer, attn, prep = main["flops"], main["layer"], main["attn"], main["prep"]
        else:
            w, layer, attn, prep = time_config(name, dev)
            w_flops = w.flops()
        rec[name] = dict(layer_ms=round(layer, 5), attn_kernel_ms=round(attn, 5),
                         prep_kernel_ms=round(prep, 5),
                         layer_tflops=round(w_flops / (layer * 1e-3) / 1e12, 2),
                         attn_tflops=round(w_flops / (attn * 1e-3) / 1e12, 2),
                         layer_frac=round(w_flops / (layer * 1e-3) / 1e12 / peak, 4),
                         attn_frac=round(w_flops / (attn * 1e-3) / 1e12 / peak, 4),
                         flops=w_flops)
    return rec


def cpu_baseline(w, budget_s, nthreads=0):
    """The oracle, as it stands, on a bounded sample of query rows."""
    import oracle
    rng = np.random.default_rng(12345)
    n = 32
    rows = np.sort(rng.choice(w.T, n, replace=False))
    t0 = time.time()
    oracle.attn_fwd_workload(w, rows=rows, nthreads=nthreads)
    dt = time.time() - t0
    # grow the sample to roughly the time budget
    if dt < budget_s / 4:
        n = int(min(w.T, n * max(1.0, budget_s / max(dt, 1e-3) * 0.8)))
        rows = np.sort(rng.choice(w.T, n, replace=False))
        t0 = time.time()
        oracle.attn_fwd_workload(w, rows=rows, nthreads=nthreads)
        dt = time.time() - t0
    fl = row_flops(w, rows)
    cores = nthreads if nthreads > 0 else os.cpu_count()
    return dict(value=fl / dt / 1e12, unit=UNIT, cores=cores, kind="oracle",
                sample="%d of %d query rows x 32 heads of %s (seeded), %.1f s" %
                (len(rows), w.T, w.name, dt))


DECODE_METRIC = "decode step: algorithmic HBM bytes per second (window keys and values once)"


def run_decode(args, rank, world, local_rank):
    """One decode step per timed step (flint_attn_decode), L2 flushed before
    each; the step rewrites the same cache slot with the same values, so
    repeating it is idempotent."""
    import torch
    import full_gqa_learned_b200 as fa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    d = W.make_decode_named(args.workload)

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(dev)
    t = dict(q=bf(d.q), k=bf(d.k), v=bf(d.v), k_cache=bf(d.k_cache), v_cache=bf(d.v_cache),
             cache_len=torch.from_numpy(d.cache_len).to(dev), q_norm_w=torch.from_numpy(d.q_norm_w).to(dev),
             k_norm_w=torch.from_numpy(d.k_norm_w).to(dev),
             sinks=torch.from_numpy(np.ascontiguousarray(d.sinks, np.float32)).to(dev))
    out = torch.empty((d.B, 4096), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((32, d.B), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.decode_workspace_bytes(d.B, d.cap, d.window), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.attn_decode(t["q"], t["k"], t["v"], t["q_norm_w"], t["k_norm_w"], t["sinks"], t["k_cache"],
                       t["v_cache"], t["cache_len"], window=d.window, use_rope=d.use_rope,
                       rope_theta=d.rope_theta, eps=d.eps, out=out, lse=lse, workspace=ws, stream=stream)
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    st = fa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status %s" % fa.STATUS.get(st, st))
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    soak(args, lambda: (flush.fill_(1), step()), lambda: torch.cuda.synchronize(dev))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    (total_ms,) = max_over_ranks([total_ms], device=dev)
    return d, total_ms, clocks


def decode_cpu_baseline(d, budget_s):
    """The decode oracle, as it stands, on the first sequences of the step
    (about budget_s seconds of single-threaded numpy): algorithmic bytes of
    those sequences per second."""
    import oracle.decode as OD
    t0 = time.time()
    n = 0
    for b in range(d.B):
        OD.decode_step(d.q[b:b + 1], d.k[b:b + 1], d.v[b:b + 1], d.k_cache[b:b + 1], d.v_cache[b:b + 1],
                       d.cache_len[b:b + 1], d.q_norm_w, d.k_norm_w, d.sinks, window=d.window,
                       use_rope=d.use_rope)
        n = b + 1
        if time.time() - t0 > budget_s:
            break
    dt = time.time() - t0
    frac = n / d.B
    return dict(value=d.algorithmic_bytes() * frac / dt / 1e9, unit="GB/s", cores=1, kind="oracle",
                sample="%d of %d sequences of %s, %.1f s" % (n, d.B, d.name, dt))


def decode_line(args, world, d, total_ms, clocks):
    peaks, src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    nbytes = d.algorithmic_bytes()
    step_ms = total_ms / args.steps
    gbs = nbytes / (step_ms * 1e-3) / 1e9
    return dict(
        metric=DECODE_METRIC, value=round(gbs * world, 3), unit="GB/s", n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=round(step_ms, 5), higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="f32", data="synthetic (seeded N(0,1) BF16 q/k/v and caches)",
        config=dict(workload=d.name, B=d.B, cap=d.cap, window=d.window, use_rope=bool(d.use_rope),
                    keys=int(d.keys_per_sequence().sum()), l2="flushed before every timed step (256 MiB write)",
                    per_rank="independent replica"),
        roofline=dict(bound="hbm", achieved=round(gbs, 3), peak=peak, unit="GB/s", frac=round(gbs / peak, 4),
                      traffic=None, kernel="flint::decode_tc_kernel (whole step: reset kernel, tile kernel, CUDA-core kernel returning at once)",
                      peak_source="%s hbm_gbs" % src, bytes_per_step=nbytes),
        gpu_launches=3 * args.steps, clocks=clocks)


# ---------------------------------------------------------------- backward leg

BWD_PREFIX = "bwd_"
BWD_METRIC = ("sink-attn backward TFLOP/s (window-aware algorithmic FLOPs: 2.5x the forward's, "
              "five contractions per pair and head)")


def bwd_flops(w):
    return 2.5 * w.flops()


def run_bwd(args, rank, world, local_rank):
    """One flint_attn_bwd call per timed step on the forward's out and lse of
    the named workload and a seeded N(0,1) BF16 upstream gradient; L2
    flushed before each step."""
    import torch
    import full_gqa_learned_b200 as fa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = W.make(args.workload[len(BWD_PREFIX):])
    T = w.T

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16)
    host = dict(q=bf(w.q), k=bf(w.k), v=bf(w.v), q_norm_w=torch.from_numpy(w.q_norm_w),
                k_norm_w=torch.from_numpy(w.k_norm_w),
                sinks=torch.from_numpy(np.ascontiguousarray(w.sinks, np.float32)))
    for name in ("pos_ids", "cu_seqlens", "pad_mask"):
        if getattr(w, name) is not None:
            host[name] = torch.from_numpy(getattr(w, name))
    rng = np.random.default_rng(w.seed + 1000)
    host["dout"] = bf(W.bf16_bits(rng.standard_normal((T, 4096), dtype=np.float32)))
    d = {k: v.to(dev) for k, v in host.items()}
    kw = dict(pos_ids=d.get("pos_ids"), cu_seqlens=d.get("cu_seqlens"), pad_mask=d.get("pad_mask"),
              window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    out, lse = fa.attn_fwd(d["q"], d["k"], d["v"], d["q_norm_w"], d["k_norm_w"], d["sinks"], **kw)
    host["out"], host["lse"] = out.cpu(), lse.cpu()
    d["out"], d["lse"] = out, lse
    shapes = {"dq": (T, 32, 128), "dk": (T, 4, 128), "dv": (T, 4, 128), "dq_norm_w": (128,),
              "dk_norm_w": (128,), "dsinks": (32,)}
    grads = {n: torch.empty(sh, dtype=torch.float32, device=dev) for n, sh in shapes.items()}
    ws = torch.empty(fa.bwd_workspace_bytes(T), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call(dd, g):
        fa.attn_bwd(dd["q"], dd["k"], dd["v"], dd["q_norm_w"], dd["k_norm_w"], dd["sinks"], dd["out"],
                    dd["lse"], dd["dout"], pos_ids=dd.get("pos_ids"), cu_seqlens=dd.get("cu_seqlens"),
                    pad_mask=dd.get("pad_mask"), window=w.window, use_rope=w.use_rope,
                    rope_theta=w.rope_theta, eps=w.eps, grads=g, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        flush.fill_(1)
        call(d, grads)
    st = fa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status %s" % fa.STATUS.get(st, st))
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    soak(args, lambda: (flush.fill_(1), call(d, grads)), lambda: torch.cuda.synchronize(dev))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        call(d, grads)
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = sum(e[0].elapsed_time(e[1]) for e in evs)

    e2e_ms, h2d, d2h = float("nan"), 0, 0
    if not args.profile:
        # end to end: inputs from pinned host memory, gradients back to it
        pinned = {k: v.pin_memory() for k, v in host.items()}
        g_h = {n: torch.empty(sh, dtype=torch.float32).pin_memory() for n, sh in shapes.items()}
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())
        d2h = sum(v.numel() * 4 for v in g_h.values())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        e2e_ms = 0.0
        for _ in range(n_e2e):
            flush.fill_(3)
            e0.record(stream)
            dd = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
            call(dd, grads)
            for n in g_h:
                g_h[n].copy_(grads[n], non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            e2e_ms += e0.elapsed_time(e1)
        e2e_ms /= n_e2e
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device=dev)
    return dict(w=w, total_ms=total_ms, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, clocks=clocks,
                gpu=torch.cuda.get_device_name(dev))


def bwd_cpu_baseline(w, budget_s):
    """The backward oracle, as it stands, on a prefix of the workload's
    tokens (a prefix of a causal layer is a self-contained problem), grown
    until a run takes about budget_s seconds: algorithmic FLOPs per second."""
    from threadpoolctl import threadpool_limits
    from oracle import backward as OB
    with threadpool_limits(limits=1):          # one BLAS thread: `cores` below is exact
        return _bwd_cpu_sample(w, budget_s, OB, np.random.default_rng(1))


def _bwd_cpu_sample(w, budget_s, OB, rng):
    n, dt = 32, 0.0
    while True:
        sub = W.make_small(n, seed=w.seed, window=w.window, use_rope=w.use_rope)
        sub.q, sub.k, sub.v = w.q[:n], w.k[:n], w.v[:n]
        sub.q_norm_w, sub.k_norm_w, sub.sinks = w.q_norm_w, w.k_norm_w, w.sinks
        dO = rng.standard_normal((n, 32, 128))
        t0 = time.time()
        OB.attn_bwd_workload(sub, dO)
        dt = time.time() - t0
        if dt > budget_s / 4 or 2 * n > w.T:
            break
        n *= 2
    return dict(value=bwd_flops(sub) / dt / 1e12, unit=UNIT, cores=1, kind="oracle",
                sample="first %d tokens of %s (one document), %.2f s" % (n, w.name, dt))


def bwd_line(args, world, r):
    w = r["w"]
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    flops = bwd_flops(w)
    step_ms = r["total_ms"] / args.steps
    tf = flops / (step_ms * 1e-3) / 1e12
    return dict(
        metric=BWD_METRIC, value=round(tf * world, 4), unit=UNIT, n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=round(step_ms, 5), higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="bf16",
        data="synthetic (the forward workload's seeded inputs; N(0,1) BF16 upstream gradient)",
        config=dict(workload=args.workload, T=w.T, window=w.window, use_rope=bool(w.use_rope),
                    l2="flushed before every timed step (256 MiB write)", per_rank="independent replica",
                    seed=w.seed, gpu=r["gpu"]),
        roofline=dict(bound="tensor", achieved=round(tf, 4), peak=peak, unit=UNIT,
                      frac=round(tf / peak, 4), traffic=None,
                      kernel="flint bwd call (segments, prep, tcgen05 dq and dk/dv, adjoint, finish kernels)",
                      peak_source="%s bf16_tflops (burst)" % src, flops_per_launch=flops,
                      note="algorithmic FLOPs (5 products per pair); the tensor cores run 7"),
        e2e=dict(value=round(flops / (r["e2e_ms"] * 1e-3) / 1e12 * world, 4), unit=UNIT,
                 h2d_bytes_per_step=r["h2d"], d2h_bytes_per_step=r["d2h"], ms_per_step=round(r["e2e_ms"], 4)),
        gpu_launches=6 * args.steps, clocks=r["clocks"])


# ---------------------------------------------------------------- whole-layer leg

LAYER_METRIC = ("attention layer TFLOP/s (q/k/v projection GEMM + sink attention + o_proj GEMM, "
                "BF16, window-aware attention FLOPs)")


def run_layer(args, rank, world, local_rank):
    """One flint_attn_layer_fwd call per timed step (hidden states to the
    layer's output), L2 flushed before each; then the two projection GEMMs
    apart for their own roofline."""
    import torch
    import full_gqa_learned_b200 as fa
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lw = W.make_layer_named(args.workload)
    w = lw.attn

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16)
    host = dict(x=bf(lw.x), w_qkv=bf(lw.w_qkv), w_o=bf(lw.w_o), q_norm_w=torch.from_numpy(w.q_norm_w),
                k_norm_w=torch.from_numpy(w.k_norm_w),
                sinks=torch.from_numpy(np.ascontiguousarray(w.sinks, np.float32)))
    for n in ("pos_ids", "cu_seqlens", "pad_mask"):
        if getattr(w, n) is not None:
            host[n] = torch.from_numpy(getattr(w, n))
    d = {k: v.to(dev) for k, v in host.items()}
    kw = dict(pos_ids=d.get("pos_ids"), cu_seqlens=d.get("cu_seqlens"), pad_mask=d.get("pad_mask"),
              window=w.window, use_rope=w.use_rope, rope_theta=w.rope_theta, eps=w.eps)
    out = fa.attn_layer_fwd(d["x"], d["w_qkv"], d["w_o"], d["q_norm_w"], d["k_norm_w"], d["sinks"], **kw)
    ws = fa.attn_layer_fwd.last_workspace
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.attn_layer_fwd(d["x"], d["w_qkv"], d["w_o"], d["q_norm_w"], d["k_norm_w"], d["sinks"],
                          out=out, workspace=ws, stream=stream, **kw)
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    st = fa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status %s" % fa.STATUS.get(st, st))
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    soak(args, lambda: (flush.fill_(1), step()), lambda: torch.cuda.synchronize(dev))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    st = fa.device_status(ws)
    if st != 0:
        raise RuntimeError("device status %s" % fa.STATUS.get(st, st))
    # the projection GEMMs apart (same inputs, L2 flushed before each)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        fa.qkv_proj(d["x"], d["w_qkv"], q=out["q"], k=out["k"], v=out["v"], stream=stream)
        ev[i][1].record(stream)
        flush.fill_((i + 3) & 0xFF)
        ev[i][2].record(stream)
        fa.o_proj(out["attn_out"], d["w_o"], y=out["y"], stream=stream)
        ev[i][3].record(stream)
    torch.cuda.synchronize(dev)
    qkv_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    o_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)

    e2e_ms, h2d, d2h = float("nan"), 0, 0
    if not args.profile:
        pinned = {k: v.pin_memory() for k, v in host.items()}
        y_h = torch.empty(tuple(out["y"].shape), dtype=torch.bfloat16).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())
        d2h = y_h.numel() * 2
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        e2e_ms = 0.0
        for _ in range(n_e2e):
            flush.fill_(3)
            e0.record(stream)
            dd = {k: v.to(dev, non_blocking=True) for k, v in pinned.items()}
            fa.attn_layer_fwd(dd["x"], dd["w_qkv"], dd["w_o"], dd["q_norm_w"], dd["k_norm_w"], dd["sinks"],
                              pos_ids=dd.get("pos_ids"), cu_seqlens=dd.get("cu_seqlens"),
                              pad_mask=dd.get("pad_mask"), window=w.window, use_rope=w.use_rope,
                              rope_theta=w.rope_theta, eps=w.eps, out=out, workspace=ws, stream=stream)
            y_h.copy_(out["y"], non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            e2e_ms += e0.elapsed_time(e1)
        e2e_ms /= n_e2e
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device=dev)
    return dict(lw=lw, total_ms=total_ms, qkv_ms=qkv_ms, o_ms=o_ms, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h,
                clocks=clocks, gpu=torch.cuda.get_device_name(dev))


def layer_cpu_baseline(lw, budget_s):
    """The layer oracle (FP64 projections, attention oracle, o_proj), as it
    stands, on a prefix of the workload's tokens (a prefix of a causal single
    sequence is a self-contained problem), grown until a run takes about
    budget_s seconds: algorithmic FLOPs per second."""
    from oracle import projection as OP
    n, dt = 16, 0.0
    while True:
        sub = W.make_layer(n, seed=0, hidden=lw.hidden, window=lw.attn.window, use_rope=lw.attn.use_rope)
        a = lw.attn
        t0 = time.time()
        OP.attn_layer(lw.x[:n], lw.w_qkv[:4096], lw.w_qkv[4096:4608], lw.w_qkv[4608:], lw.w_o, a.q_norm_w,
                      a.k_norm_w, a.sinks, window=a.window, use_rope=a.use_rope, rope_theta=a.rope_theta,
                      eps=a.eps)
        dt = time.time() - t0
        if dt > budget_s / 4 or 2 * n > lw.T:
            break
        n *= 2
    return dict(value=sub.flops() / dt / 1e12, unit=UNIT, cores=os.cpu_count(), kind="oracle",
                sample="first %d tokens of %s (one sequence), %.2f s" % (n, lw.name, dt))


def layer_line(args, world, r):
    lw = r["lw"]
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    flops = lw.flops()
    step_ms = r["total_ms"] / args.steps
    tf = flops / (step_ms * 1e-3) / 1e12
    qkv_flops = 2.0 * lw.T * lw.hidden * 5120
    o_flops = 2.0 * lw.T * 4096 * lw.hidden
    qkv_tf = qkv_flops / (r["qkv_ms"] * 1e-3) / 1e12
    return dict(
        metric=LAYER_METRIC, value=round(tf * world, 3), unit=UNIT, n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=round(step_ms, 5), higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="bf16",
        data="synthetic (seeded N(0,1) BF16 hidden states, N(0,1/fan_in) BF16 weights, 1+N(0,0.1) norm "
             "weights, N(0,1) sinks)",
        config=dict(workload=lw.name, T=lw.T, hidden=lw.hidden, window=lw.attn.window,
                    use_rope=bool(lw.attn.use_rope), l2="flushed before every timed step (256 MiB write)",
                    per_rank="independent replica", gpu=r["gpu"]),
        roofline=dict(bound="tensor", achieved=round(qkv_tf, 3), peak=peak, unit=UNIT,
                      frac=round(qkv_tf / peak, 4), traffic=None, kernel="flint::gemm_kernel (q/k/v projection)",
                      peak_source="%s bf16_tflops (burst)" % src, flops_per_launch=qkv_flops,
                      kernel_ms=round(r["qkv_ms"], 5), o_proj_ms=round(r["o_ms"], 5),
                      o_proj_tflops=round(o_flops / (r["o_ms"] * 1e-3) / 1e12, 3),
                      layer_frac=round(tf / peak, 4)),
        e2e=dict(value=round(flops / (r["e2e_ms"] * 1e-3) / 1e12 * world, 3), unit=UNIT,
                 h2d_bytes_per_step=r["h2d"], d2h_bytes_per_step=r["d2h"], ms_per_step=round(r["e2e_ms"], 4)),
        gpu_launches=4 * args.steps, clocks=r["clocks"])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(W.CONFIGS) + sorted(W.PROFILE_CONFIGS) + sorted(W.DECODE_CONFIGS)
                    + sorted(W.LAYER_CONFIGS)
                    + sorted(BWD_PREFIX + n for n in W.CONFIGS))
    ap.add_argument("--impl", default="flint", choices=["flint", "reference"])
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed load before timing")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-config record of the other named workloads")
    ap.add_argument("--profile", action="store_true",
                    help="warm-up and timed steps only (for ncu captures): no soak, e2e or CPU leg")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu DRAM bytes per attention launch (default: the committed ncu "
                         "summary of the workload, if the kernel is unchanged since)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        if args.workload in W.DECODE_CONFIGS:
            d = W.make_decode_named(args.workload)
            vals, cb = [], None
            for i in range(args.warmup + args.steps):
                cb = decode_cpu_baseline(d, budget_s=min(args.cpu_budget, 60.0 / max(1, args.steps + args.warmup)))
                if i >= args.warmup:
                    vals.append(cb["value"])
            value = statistics.median(vals)
            cb["value"] = value
            print(json.dumps(dict(impl="reference", metric=DECODE_METRIC, value=value, unit="GB/s",
                                  n_gpus=args.gpus, steps=args.steps, warmup=args.warmup, ms_per_step=None,
                                  higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                                  data="synthetic", config=dict(workload=d.name, B=d.B, cap=d.cap,
                                                                window=d.window, use_rope=d.use_rope),
                                  cpu_baseline=cb,
                                  e2e=dict(value=value, unit="GB/s", h2d_bytes_per_step=0,
                                           d2h_bytes_per_step=0))))
            return 0
        if args.workload in W.LAYER_CONFIGS:
            lw = W.make_layer_named(args.workload)
            vals, cb = [], None
            for i in range(args.warmup + args.steps):
                cb = layer_cpu_baseline(lw, budget_s=min(args.cpu_budget, 60.0 / max(1, args.steps + args.warmup)))
                if i >= args.warmup:
                    vals.append(cb["value"])
            value = statistics.median(vals)
            cb["value"] = value
            print(json.dumps(dict(impl="reference", metric=LAYER_METRIC, value=value, unit=UNIT,
                                  n_gpus=args.gpus, steps=args.steps, warmup=args.warmup, ms_per_step=None,
                                  higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                                  data="synthetic", config=dict(workload=lw.name, T=lw.T, hidden=lw.hidden,
                                                                window=lw.attn.window,
                                                                use_rope=lw.attn.use_rope),
                                  cpu_baseline=cb,
                                  e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0,
                                           d2h_bytes_per_step=0))))
            return 0
        if args.workload.startswith(BWD_PREFIX):
            w = W.make(args.workload[len(BWD_PREFIX):])
            vals, cb = [], None
            for i in range(args.warmup + args.steps):
                cb = bwd_cpu_baseline(w, budget_s=min(args.cpu_budget, 60.0 / max(1, args.steps + args.warmup)))
                if i >= args.warmup:
                    vals.append(cb["value"])
            value = statistics.median(vals)
            cb["value"] = value
            print(json.dumps(dict(impl="reference", metric=BWD_METRIC, value=value, unit=UNIT,
                                  n_gpus=args.gpus, steps=args.steps, warmup=args.warmup, ms_per_step=None,
                                  higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                                  data="synthetic", config=dict(workload=args.workload, T=w.T,
                                                                window=w.window, use_rope=w.use_rope),
                                  cpu_baseline=cb,
                                  e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0,
                                           d2h_bytes_per_step=0))))
            return 0
        w = W.make(args.workload)
        times, cb = [], None
        for i in range(args.warmup + args.steps):
            r = cpu_baseline(w, budget_s=min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup)))
            if i >= args.warmup:
                times.append(r["value"])
            cb = r
        value = statistics.median(times)
        cb["value"] = value
        line = dict(impl="reference", metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus,
                    steps=args.steps, warmup=args.warmup, ms_per_step=None,
                    higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                    data="synthetic", config=dict(workload=w.name, T=w.T, window=w.window,
                                                  use_rope=w.use_rope),
                    cpu_baseline=cb,
                    e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if args.workload in W.DECODE_CONFIGS:
        d, total_ms, clocks = run_decode(args, rank, world, local_rank)
        line = decode_line(args, world, d, total_ms, clocks)
        if rank == 0 and world == 1 and not args.profile:
            line["cpu_baseline"] = decode_cpu_baseline(d, budget_s=args.cpu_budget)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line))
        return 0
    if args.workload in W.LAYER_CONFIGS:
        r = run_layer(args, rank, world, local_rank)
        line = layer_line(args, world, r)
        if rank == 0 and world == 1 and not args.profile:
            line["cpu_baseline"] = layer_cpu_baseline(r["lw"], budget_s=args.cpu_budget)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line))
        return 0
    if args.workload.startswith(BWD_PREFIX):
        r = run_bwd(args, rank, world, local_rank)
        line = bwd_line(args, world, r)
        if rank == 0 and world == 1 and not args.profile:
            line["cpu_baseline"] = bwd_cpu_baseline(r["w"], budget_s=args.cpu_budget)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line))
        return 0
    r = run_flint(args, rank, world, local_rank)
    w = r["w"]
    peaks, src = load_peaks()
    flops = w.flops()
    value = whole_job_tflops(flops, args.steps, world, r["total_ms"])
    attn_tflops = flops / (r["attn_avg"] * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    line = dict(
        metric=METRIC, value=round(value, 3), unit=UNIT, n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=round(r["total_ms"] / args.steps, 5),
        higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
        data="synthetic (seeded N(0,1) BF16 q/k/v, 1+N(0,0.1) norm weights, N(0,1) sinks)",
        config=dict(workload=w.name, T=w.T, window=w.window, use_rope=bool(w.use_rope),
                    q_heads=32, kv_heads=4, head_dim=128, qk_operands="fp16 (post-norm)",
                    pv_operands="bf16", l2="flushed before every timed step (256 MiB write)",
                    per_rank="independent replica", seed=w.seed, gpu=r["gpu"]),
        roofline=dict(bound="tensor", achieved=round(attn_tflops, 3), peak=peak, unit=UNIT,
                      frac=round(attn_tflops / peak, 4), kernel_frac=round(attn_tflops / peak, 4),
                      layer_frac=round(value / world / peak, 4),
                      traffic=args.traffic if args.traffic is not None else recorded_traffic(w.name),
                      kernel=("flint::attn_fwd_qprep_kernel" if w.window > 0 else "flint::attn_fwd_kernel"),
                      peak_source="%s bf16_tflops (burst)" % src,
                      flops_per_launch=flops,
                      kernel_ms=round(r["attn_avg"], 5), prep_kernel_ms=round(r["prep_avg"], 5)),
        e2e=dict(value=round(whole_job_tflops(flops, 1, world, r["e2e_ms"]), 3), unit=UNIT,
                 h2d_bytes_per_step=r["h2d"], d2h_bytes_per_step=r["d2h"],
                 ms_per_step=round(r["e2e_ms"], 4)),
        gpu_launches=r["launches"], clocks=r["clocks"],
        pct_of_tensor_peak=round(100.0 * value / world / peak, 2),
    )
    if rank == 0 and world == 1 and not args.profile:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    if world == 1 and not args.profile and not args.no_configs:
        main = dict(name=w.name, flops=flops, layer=r["total_ms"] / args.steps, attn=r["attn_avg"],
                    prep=r["prep_avg"])
        line["configs"] = configs_record(torch.device("cuda", local_rank), peak, main)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
