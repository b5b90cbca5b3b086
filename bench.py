#!/usr/bin/env python
"""Benchmark of libssd, the Mamba-2 SSD layer, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...     (one process per GPU)

Prints ONE JSON line (rank 0).  The headline is prefill throughput of the 2.7B-shaped
SSD layer (batch 1, L = 4096, 80 heads x 64 channels, d_state 128, chunk 256, bf16 x/B/C,
fp32 dt/A/D/state/y): one step = one ssd_prefill of that layer (chunk state, state
passing and chunk scan, each starting its set-up under the tail of the one before).  The batched cached-decode workload (batch 256 x 80 heads, fp32 state
671 MB, 1024 steps) is reported under "decode" in the same line.

Timing: CUDA events on the launching stream; W untimed warm-up steps; K timed steps
bracketed by a barrier and a device synchronise on both sides; the max over ranks.  The
prefill inputs fit in L2, so a 256 MiB buffer is written before every timed prefill step
(outside that step's events).  Per-kernel durations (the roofline figures) come from a
second pass of K steps with an event between kernels, which runs them serially.  The
decode state (671 MB) is larger than L2.
Multi-GPU: every rank runs its own independent sequence (weak scaling), no collective
on the data path.

`--impl reference` times the fp64 CPU oracle on this machine's cores instead (rank 0
only), on a bounded sample of the same workload per step.
"""
import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

PREFILL_WORKLOAD = "mamba2_2.7b_prefill"
DECODE_WORKLOAD = "mamba2_2.7b_decode_b256"
METRIC = "SSD prefill tokens/s (TFLOP/s) and decode steps/s with HBM GB/s vs peak"
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20   # B200 L2
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x FMA x max clock


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init_dist(world, backend, device=None):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = {}
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def barrier(world, device=None):
    import torch.distributed as dist
    if world > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, world: int, device) -> float:
    import torch
    import torch.distributed as dist
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Every rank draws its own independent sequence."""
    return base_seed + 1000 * rank


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (read-only) while
    the timed regions run."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        self._active = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    self.h = h
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            if self._active.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    try:
                        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    except AttributeError:
                        r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                    self.samples.append(mhz)
                    for bit, name in self.REASONS.items():
                        if r & bit and bit != 0x1:
                            self.reasons.add(name)
                except Exception:
                    pass
            time.sleep(self.period)

    def start(self):
        if self.ok and self._thread is None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def active(self, on: bool):
        (self._active.set if on else self._active.clear)()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def source_digest(files):
    """Digest of the code in `files` with comments and whitespace removed, so that a change
    to a comment does not void counters taken from unchanged kernels."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary (profiles/<kernel>.<workload>.txt),
    or None if there is none or the kernel's sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}.{workload}.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.split("=", 1)
            kv[k.strip()] = v.strip()
    try:
        files = kv["sources"].split()
        if source_digest(files) != kv["sources_sha256"]:
            return None
        return float(kv["traffic_bytes_per_launch"])
    except (KeyError, OSError, ValueError):
        return None


# ------------------------------------------------------------------------ work models

def prefill_work(w, Q=None):
    """Algorithmic FLOPs and minimum bytes of one prefill of workload w."""
    Q = Q or w.chunk
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    tok = b * L
    el = 2 if w.dtype == "bf16" else 4
    flops_dense = tok * H * (2 * Q * P + 4 * N * P) + tok * G * 2 * Q * N
    flops_causal = tok * H * ((Q + 1) * P + 4 * N * P) + tok * G * (Q + 1) * N
    min_bytes = (tok * H * P * el + 2 * tok * G * N * el + tok * H * 4 + 2 * H * 4
                 + tok * H * P * 4 + b * H * P * N * 4)
    return flops_dense, flops_causal, min_bytes


def kernel_work(name, w, Q):
    """(bound, pipeline bytes per launch, DRAM-minimum bytes per launch, flops per launch) of
    one prefill kernel.

    Pipeline bytes are what the kernel moves given the pipeline's intermediates: the chunk
    states S (fp32, written by chunk_state, read by state passing), the state entering each
    chunk (bf16, written by state passing, read by chunk_scan) and the decay table.  Those
    intermediates normally stay in L2, so pipeline bytes are not an HBM figure.  The
    DRAM-minimum bytes count only what must cross DRAM: the kernel's own inputs read once
    and its outputs written once (for state passing, the final state)."""
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    tok, nc = b * L, -(-w.seqlen // Q)
    el = 2 if w.dtype == "bf16" else 4
    x_b, bc_b, dt_b, y_b = tok * H * P * el, tok * G * N * el, tok * H * 4, tok * H * P * 4
    states = b * nc * H * P * N
    final_b = b * H * P * N * 4
    tab_b = b * H * nc * (4 + 2 * Q) * 4   # decay table rows (tensor-core path)
    flops_state = tok * H * 2 * N * P
    flops_scan = tok * H * (2 * Q * P + 2 * N * P) + tok * G * 2 * Q * N
    if name.startswith("dA_cumsum"):
        return "hbm", dt_b + b * H * nc * Q * 4, dt_b, 0
    if name == "state_passing":
        return "hbm", 2 * states * 4 + final_b, final_b, 0
    if name.startswith("state_passing"):
        return "hbm", states * 4 + states * 2 + final_b + b * H * nc * 4, final_b, 0
    if name == "chunk_state_tc":
        return "tensor", x_b + bc_b + dt_b + tab_b + states * 4 + b * H * nc * 4, x_b + bc_b + dt_b, flops_state
    if name == "chunk_scan_tc":
        return "tensor", x_b + 2 * bc_b + tab_b + states * 2 + y_b, x_b + 2 * bc_b + y_b, flops_scan
    if name.startswith("chunk_state"):
        return "flops", flops_state, x_b + bc_b + dt_b, flops_state
    if name.startswith("chunk_scan"):
        return "flops", flops_scan, x_b + 2 * bc_b + y_b, flops_scan
    return "hbm", 0, 0, 0


TRAFFIC_NOTE = ("DRAM bytes read + written per launch, from the committed ncu summary of this kernel "
                "(ncu --cache-control none on a launch inside back-to-back prefills, so the L2 is as the "
                "pipeline leaves it; null once its sources changed)")


def roofline_entry(name, w, Q, avg_ms, peaks, traffic):
    """Roofline of one prefill kernel from its average event-timed launch.

    The tensor-core kernels lead with their tensor-pipe work: dense-tile FLOPs per launch
    over the launch time, against the measured bf16 peak.  Beside it, the DRAM-minimum
    bytes over the same time against the measured HBM copy bandwidth, and the pipeline
    bytes (including L2-resident intermediates) under their own name."""
    kind, pipe, dram_min, flops = kernel_work(name, w, Q)
    secs = avg_ms / 1e3
    hbm = {"bytes": dram_min, "GB/s": dram_min / secs / 1e9, "frac": dram_min / secs / 1e9 / peaks["hbm_gbs"],
           "peak": peaks["hbm_gbs"], "what": "DRAM-minimum bytes: the kernel's inputs read once, outputs written once"}
    pipeline = {"bytes": pipe, "GB/s": pipe / secs / 1e9,
                "what": "pipeline bytes, including intermediates that stay in L2; not an HBM figure"}
    if kind == "tensor":
        achieved = flops / secs / 1e12
        return {"kernel": name, "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                "traffic_what": TRAFFIC_NOTE, "flops_per_launch": flops,
                "peak_source": f"{peaks['source']} bf16_tflops (burst)", "hbm_min": hbm, "pipeline": pipeline}
    if kind == "hbm":
        # state passing: its chunk states come from L2, so only its pipeline bytes mean much
        achieved = pipe / secs / 1e9
        return {"kernel": name, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "traffic_what": TRAFFIC_NOTE,
                "achieved_what": "pipeline bytes over time (reads its inputs from L2: an L2-bound kernel "
                                 "measured against the HBM figure)",
                "peak_source": f"{peaks['source']} hbm_gbs", "hbm_min": hbm}
    achieved = pipe / secs / 1e12
    if name.endswith("_simt"):  # fp32 FMA on CUDA cores
        return {"kernel": name, "bound": "alu", "achieved": achieved, "peak": FP32_SIMT_PEAK_TFLOPS,
                "unit": "TFLOP/s", "frac": achieved / FP32_SIMT_PEAK_TFLOPS, "traffic": traffic,
                "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1.965 GHz"}
    return {"kernel": name, "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
            "peak_source": f"{peaks['source']} bf16_tflops (burst)"}


# ------------------------------------------------------------------------ CPU oracle legs

def oracle_prefill_rate(w, seed, min_seconds=10.0, max_seconds=30.0, heads=None):
    """Oracle tokens/s of the whole layer, timed over repeated runs of a sample (all heads by
    default).  Returns (tokens_per_s, description, threads, seconds)."""
    import oracle
    from selective_state_space_10_b200 import inputs
    si = inputs.workload_sequence(w, seed=seed)
    H = w.nheads if heads is None else heads
    f64 = lambda a: np.ascontiguousarray(a, dtype=np.float64)
    args = (f64(si.x[:, :, :H]), f64(si.dt[:, :, :H]), f64(si.A[:H]), f64(si.B), f64(si.C), f64(si.D[:H]))
    threads = oracle.default_threads()
    reps, spent = 0, 0.0
    while spent < min_seconds and (reps == 0 or spent * (reps + 1) / reps < max_seconds):
        t0 = time.perf_counter()
        oracle.recurrence(*args, nthreads=threads)
        spent += time.perf_counter() - t0
        reps += 1
    tokens = reps * w.batch * w.seqlen * (H / w.nheads)
    desc = f"{reps} x fp64 recurrence over {H} of {w.nheads} heads x {w.seqlen} tokens (full layer = {w.nheads} heads)"
    return tokens / spent, desc, threads, spent


def oracle_decode_rate(w, seed, min_seconds=10.0, max_seconds=30.0):
    """Oracle decode steps/s of the whole batch, from repeated steps on all heads."""
    import oracle
    from selective_state_space_10_b200 import inputs
    tok = inputs.decode_token(w, 0, seed=seed)
    rng = np.random.default_rng(seed)
    state = rng.standard_normal((w.batch, w.nheads, w.headdim, w.dstate)) * 0.1
    args = [np.ascontiguousarray(a, dtype=np.float64) for a in (tok.x, tok.dt, tok.A, tok.B, tok.C, tok.D)]
    threads = oracle.default_threads()
    reps, spent = 0, 0.0
    while spent < min_seconds and (reps == 0 or spent * (reps + 1) / reps < max_seconds):
        t0 = time.perf_counter()
        _, state = oracle.recurrence(*args, state=state, nthreads=threads)
        spent += time.perf_counter() - t0
        reps += 1
    return reps / spent, f"{reps} fp64 decode steps over all {w.batch}x{w.nheads} heads", threads, spent


# ------------------------------------------------------------------------ GPU legs

def upload(si, dev):
    import torch
    def inp(name):
        if si.dtype == "bf16":
            return torch.from_numpy(si.bits[name].view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(getattr(si, name))).to(dev)
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
    return dict(x=inp("x"), dt=f(si.dt), A=f(si.A), B=inp("B"), C=inp("C"), D=f(si.D))


def prefill_leg(args, dev, rank, world, peaks, sampler):
    import torch
    from selective_state_space_10_b200 import inputs, ssd
    w = inputs.BY_NAME[args.workload]
    si = inputs.workload_sequence(w, seed=rank_seed(w.seed, rank))
    t = upload(si, dev)
    dims = ssd.dims_of_prefill(t["x"], t["B"])
    dtype = ssd.BF16 if w.dtype == "bf16" else ssd.F32
    names = ssd.prefill_kernel_names(dims, dtype, w.chunk)
    nk = len(names)
    ws = torch.empty(ssd.prefill_workspace_size(dims, dtype, w.chunk), dtype=torch.uint8, device=dev)
    y = torch.empty((w.batch, w.seqlen, w.nheads, w.headdim), dtype=torch.float32, device=dev)
    fs = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    K, W = args.steps, args.warmup
    mk = lambda: torch.cuda.Event(enable_timing=True)
    kev = [[mk() for _ in range(nk + 1)] for _ in range(K)]
    outer = [(mk(), mk()) for _ in range(K)]
    for evs in kev:          # create the underlying CUDA events before handing them over
        for e in evs:
            e.record(stream)
    for a, b in outer:
        a.record(stream)
        b.record(stream)
    call = lambda events=None: ssd.prefill(**t, chunk=w.chunk, y=y, final_state=fs, workspace=ws,
                                           stream=stream, events=events)
    # The headline: K prefills back to back (as a model runs one layer after another), their
    # inputs rotated over enough device copies that together they exceed twice the L2, so no
    # step finds its inputs in L2; timed between two events.  Each call's first kernel is a
    # programmatic dependent of the previous call's last one, as in a model's layer sequence.
    # Each copy has its own y and final state as well, as each layer of a model would.
    in_bytes = sum(v.numel() * v.element_size() for v in t.values())
    nsets = max(2, -(-2 * L2_BYTES // in_bytes))
    sets = [t] + [{k_: v.clone() for k_, v in t.items()} for _ in range(nsets - 1)]
    outs = [(y, fs)] + [(torch.empty_like(y), torch.empty_like(fs)) for _ in range(nsets - 1)]
    calls = [lambda s_=s_, o_=o_: ssd.prefill(**s_, chunk=w.chunk, y=o_[0], final_state=o_[1], workspace=ws,
                                              stream=stream)
             for s_, o_ in zip(sets, outs)]
    for i in range(max(W, nsets)):
        calls[i % nsets]()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    sampler.active(True)
    ha, hb = mk(), mk()
    ha.record(stream)
    tq = time.perf_counter()
    for k in range(K):
        calls[k % nsets]()
    host_us = (time.perf_counter() - tq) / K * 1e6  # enqueue time per call (the GPU runs behind)
    hb.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    rotated_same = all(torch.equal(o[0], y) and torch.equal(o[1], fs) for o in outs[1:])
    del sets, outs, calls
    # Context: single steps, each after a 256 MiB write that evicts L2, with an event on each
    # side (each step then also pays its first kernel's launch after the event).
    for i in range(W):
        flush.fill_(i & 0xFF)
        call()
    torch.cuda.synchronize(dev)
    for k in range(K):
        flush.fill_((k + 7) & 0xFF)
        outer[k][0].record(stream)
        call()
        outer[k][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    # Per-kernel durations: the same K steps again with an event between kernels.  Events in
    # the stream keep each kernel from starting before the previous one ends, so this pass
    # runs the kernels serially; the step time above is the one with their overlap.
    for k in range(K):
        flush.fill_((k + 7) & 0xFF)
        call(events=kev[k])
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    # Context only, not the headline: the same steps (overlapped, then serial) after a flush
    # that also reads a second buffer larger than L2, so that the step starts with none of
    # the flush buffer's dirty lines in L2 waiting to be written back to DRAM.
    clean = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    cev = [[mk() for _ in range(nk + 1)] for _ in range(K)]
    couter = [(mk(), mk()) for _ in range(K)]
    for evs in cev:
        for e in evs:
            e.record(stream)
    for a, b in couter:
        a.record(stream)
        b.record(stream)
    for k in range(K):
        flush.fill_((k + 7) & 0xFF)
        torch.sum(clean, dim=0, out=sink)
        couter[k][0].record(stream)
        call()
        couter[k][1].record(stream)
    for k in range(K):
        flush.fill_((k + 7) & 0xFF)
        torch.sum(clean, dim=0, out=sink)
        call(events=cev[k])
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    del clean
    sampler.active(False)
    clean_ctx = {
        "ms_per_step": statistics.mean(a.elapsed_time(b) for a, b in couter),
        "serial_ms_per_step": statistics.mean(cev[k][0].elapsed_time(cev[k][nk]) for k in range(K)),
        "kernels_avg_ms": {n: statistics.mean(cev[k][i].elapsed_time(cev[k][i + 1]) for k in range(K))
                           for i, n in enumerate(names)},
        "flush": "256 MiB written, then another 256 MiB buffer read: L2 holds neither inputs nor dirty lines",
        "note": "context for the kernel fractions; value and ms_per_step use the write-only flush",
    }
    step_ms = [a.elapsed_time(b) for a, b in outer]
    kern_ms = [[kev[k][i].elapsed_time(kev[k][i + 1]) for k in range(K)] for i in range(nk)]
    serial_ms = statistics.mean(kev[k][0].elapsed_time(kev[k][nk]) for k in range(K))
    total_ms = max_over_ranks(ha.elapsed_time(hb), world, dev)
    ms_per_step = total_ms / K
    tokens = w.batch * w.seqlen
    value = world * tokens * K / (total_ms / 1e3)
    fl_dense, fl_causal, min_bytes = prefill_work(w)
    secs = ms_per_step / 1e3
    avg = {n: statistics.mean(kern_ms[i]) for i, n in enumerate(names)}
    tot = sum(avg.values())
    dom = max(avg, key=avg.get)
    res = {
        "value": value, "ms_per_step": ms_per_step, "tokens_per_step_per_gpu": tokens,
        "tflops": {"dense_tile": fl_dense / secs / 1e12, "causal_only": fl_causal / secs / 1e12,
                   "frac_of_bf16_peak_dense_tile": fl_dense / secs / 1e12 / peaks["bf16_tflops"],
                   "peak": peaks["bf16_tflops"], "peak_source": f"{peaks['source']} bf16_tflops (burst)"},
        "hbm": {"min_bytes": min_bytes, "GB/s": min_bytes / secs / 1e9,
                "frac": min_bytes / secs / 1e9 / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"]},
        "serial_ms_per_step": serial_ms,
        "rotated_copies_outputs_identical": bool(rotated_same),
        "host_enqueue_us_per_call": host_us,
        "single_step_l2_flushed": {"ms_per_step": statistics.mean(step_ms),
                                   "what": "one prefill after a 256 MiB write that evicts L2, an event on each side"},
        "kernels": {n: {"avg_ms": avg[n], "share": avg[n] / tot,
                        "roofline": roofline_entry(n, w, w.chunk, avg[n], peaks, profile_traffic(n, w.name))}
                    for n in names},
        "roofline": dict(roofline_entry(dom, w, w.chunk, avg[dom], peaks, profile_traffic(dom, w.name)),
                         layer={"tensor_frac": fl_dense / secs / 1e12 / peaks["bf16_tflops"],
                                "hbm_frac_min_bytes": min_bytes / secs / 1e9 / peaks["hbm_gbs"],
                                "what": "the whole prefill step (all kernels, overlapped): dense-tile FLOPs and "
                                        "the layer's minimum bytes over ms_per_step"}),
        "gpu_launches": K * nk,
        "l2_clean_context": clean_ctx,
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups, "chunk": w.chunk,
                   "input_dtype": w.dtype, "y_dtype": "f32",
                   "l2": f"inputs and outputs rotated over {nsets} device copies (inputs {nsets * in_bytes / 2**20:.0f} "
                         "MiB, more than twice the L2); steps back to back",
                   "parallelism": f"{world} GPU(s), one independent sequence per GPU, no collective"},
    }
    # End to end through the C ABI's host-buffer call: pinned host inputs -> device copies ->
    # prefill -> y and final state -> pinned host, all enqueued by ssd_prefill_host.  Each step
    # is an independent sequence, so consecutive steps alternate between two streams (each with
    # its own device buffer and host outputs): one step's y copy back overlaps the next step's
    # input copies and kernels, as two requests would in a server.
    host = {k: v.cpu().pin_memory() for k, v in t.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y.numel() * 4 + fs.numel() * 4
    ke = max(3, min(K, 20))
    lanes = [torch.cuda.Stream(dev) for _ in range(2)]
    lane_y = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in lanes]
    lane_fs = [torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True) for _ in lanes]
    lane_buf = [torch.empty(ssd.prefill_host_buffer_size(dims, dtype, w.chunk), dtype=torch.uint8, device=dev)
                for _ in lanes]

    def e2e_step(k):
        j = k % len(lanes)
        ssd.prefill_host(**host, chunk=w.chunk, y=lane_y[j], final_state=lane_fs[j], device_buffer=lane_buf[j],
                         stream=lanes[j])
    torch.cuda.synchronize(dev)
    for k in range(2):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    a, b = mk(), mk()
    a.record(stream)
    for s_ in lanes:
        s_.wait_event(a)
    for k in range(ke):
        e2e_step(k)
    for s_ in lanes:
        stream.wait_stream(s_)
    b.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e2e_ms = max_over_ranks(a.elapsed_time(b), world, dev)
    call()  # the device-only call on the same inputs: the host outputs must equal it bit for bit
    torch.cuda.synchronize(dev)
    y_ref, fs_ref = y.cpu(), fs.cpu()
    same = all(torch.equal(yl, y_ref) and torch.equal(fl, fs_ref) for yl, fl in zip(lane_y, lane_fs))
    res["e2e"] = {"value": world * tokens * ke / (e2e_ms / 1e3), "unit": "tokens/s", "steps": ke,
                  "outputs_match_device_call": bool(same),
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                  "path": "ssd_prefill_host (C ABI): pinned host x, dt, A, B, C, D -> device copies -> prefill -> "
                          "y, final_state -> pinned host; consecutive sequences on two streams"}
    return res


def decode_workload(args):
    """The batched decode workload, or the same shapes at another batch (--decode-batch:
    a smaller state for profiling captures that must fit a few GB)."""
    from dataclasses import replace
    from selective_state_space_10_b200 import inputs
    w = inputs.BY_NAME[DECODE_WORKLOAD]
    if args.decode_batch and args.decode_batch != w.batch:
        w = replace(w, batch=args.decode_batch, name=f"{w.name}@batch{args.decode_batch}")
    return w


def decode_leg(args, dev, rank, world, peaks, sampler):
    import torch
    from selective_state_space_10_b200 import inputs, ssd
    w = decode_workload(args)
    seed = rank_seed(w.seed, rank)
    nsteps = args.decode_steps
    state = torch.from_numpy(inputs.decode_initial_state(w, seed=seed)).to(dev)
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    xs = torch.empty((nsteps, b, H, P), dtype=torch.bfloat16, device=dev)
    dts = torch.empty((nsteps, b, H), dtype=torch.float32, device=dev)
    Bs = torch.empty((nsteps, b, G, N), dtype=torch.bfloat16, device=dev)
    Cs = torch.empty((nsteps, b, G, N), dtype=torch.bfloat16, device=dev)
    A = D = None
    for k in range(nsteps):
        tok = inputs.decode_token(w, k, seed=seed)
        bf = lambda n: torch.from_numpy(tok.bits[n].view(np.int16)).view(torch.bfloat16)
        xs[k].copy_(bf("x")[:, 0])
        dts[k].copy_(torch.from_numpy(tok.dt[:, 0]))
        Bs[k].copy_(bf("B")[:, 0])
        Cs[k].copy_(bf("C")[:, 0])
        if A is None:
            A = torch.from_numpy(tok.A).to(dev)
            D = torch.from_numpy(tok.D).to(dev)
    y = torch.empty((b, H, P), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    step = lambda k: ssd.decode_step(state, xs[k], dts[k], A, Bs[k], Cs[k], D, y=y, stream=stream)
    for k in range(args.warmup):
        step(k % nsteps)
    torch.cuda.synchronize(dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)
    # (1) plain launches, back to back
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    sampler.active(True)
    a, e = mk(), mk()
    a.record(stream)
    for k in range(nsteps):
        step(k)
    e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    sampler.active(False)
    plain_ms = max_over_ranks(a.elapsed_time(e), world, dev)
    # (2) the same steps captured once in a CUDA graph and replayed
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            for k in range(nsteps):
                ssd.decode_step(state, xs[k], dts[k], A, Bs[k], Cs[k], D, y=y, stream=cap)
    torch.cuda.synchronize(dev)
    g.replay()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    sampler.active(True)
    a, e = mk(), mk()
    a.record(stream)
    g.replay()
    e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    sampler.active(False)
    graph_ms = max_over_ranks(a.elapsed_time(e), world, dev)
    del g
    # (3) windowed (ReplaySSM-style) decode of the same steps: the state read every step,
    # written once per window of W tokens
    Wn = 16
    bufs = ssd.window_buffers(state, Wn, dtype=torch.bfloat16, ngroups=G)
    def wstep(k):
        ssd.decode_window_step(state, bufs, k % Wn, xs[k], dts[k], A, Bs[k], Cs[k], D, y=y, stream=stream)
        if k % Wn == Wn - 1:
            ssd.decode_window_flush(state, bufs, Wn, A, stream=stream)
    for k in range(Wn):
        wstep(k)
    torch.cuda.synchronize(dev)
    nw = nsteps - nsteps % Wn
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    sampler.active(True)
    a, e = mk(), mk()
    a.record(stream)
    for k in range(nw):
        wstep(k)
    e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    sampler.active(False)
    win_plain_ms = max_over_ranks(a.elapsed_time(e), world, dev)
    # the same windowed steps from a CUDA graph (host launch overhead removed)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            for k in range(nw):
                ssd.decode_window_step(state, bufs, k % Wn, xs[k], dts[k], A, Bs[k], Cs[k], D, y=y, stream=cap)
                if k % Wn == Wn - 1:
                    ssd.decode_window_flush(state, bufs, Wn, A, stream=cap)
    torch.cuda.synchronize(dev)
    g.replay()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    sampler.active(True)
    a, e = mk(), mk()
    a.record(stream)
    g.replay()
    e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    sampler.active(False)
    win_graph_ms = max_over_ranks(a.elapsed_time(e), world, dev)
    del g
    win_ms = min(win_plain_ms, win_graph_ms)
    state_bytes = b * H * P * N * 4
    step_bytes = 2 * state_bytes + b * H * P * (2 + 4) + b * H * 4 + 2 * b * G * N * 2 + 2 * H * 4
    best_ms = min(plain_ms, graph_ms) / nsteps
    gbs = step_bytes / (best_ms / 1e3) / 1e9
    res = {
        "workload": w.name, "value": world * nsteps / (min(plain_ms, graph_ms) / 1e3), "unit": "steps/s",
        "ms_per_step": best_ms, "steps": nsteps, "plain_ms_per_step": plain_ms / nsteps,
        "graph_ms_per_step": graph_ms / nsteps, "bytes_per_step": step_bytes, "GB/s": gbs,
        "frac_of_hbm_peak": gbs / peaks["hbm_gbs"],
        "roofline": {"kernel": "decode_step", "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "traffic": profile_traffic("decode_step", w.name),
                     "peak_source": f"{peaks['source']} hbm_gbs",
                     "duration": "per-launch average over back-to-back launches (CUDA graph replay if faster)"},
        "gpu_launches": nsteps,
        "windowed": {"window": Wn, "steps": nw, "value": world * nw / (win_ms / 1e3), "unit": "steps/s",
                     "ms_per_step": win_ms / nw, "plain_ms_per_step": win_plain_ms / nw,
                     "graph_ms_per_step": win_graph_ms / nw,
                     "speedup_vs_standard_step": (min(plain_ms, graph_ms) / nsteps)
                     / (win_ms / nw),
                     "state_bytes_per_step": state_bytes * (1 + 2.0 / Wn),
                     "state_GB/s": state_bytes * (1 + 2.0 / Wn) / (win_ms / nw / 1e3) / 1e9,
                     "note": "per step the state is read once; every W steps one flush reads and writes it "
                             "(ReplaySSM, SketchSSM Table 4: read D, write D/W)"},
        "config": {"workload": w.name, "batch": b, "nheads": H, "headdim": P, "dstate": N, "ngroups": G,
                   "input_dtype": "bf16", "state_dtype": "f32", "y_dtype": "f32",
                   "l2": "state (671 MB) larger than L2; no flush"},
    }
    # End to end: per step, the step's inputs from pinned host memory and y back.  The steps
    # are sequential (each continues from the state the one before wrote), but their copies
    # need not wait for the compute: step k+1's inputs go up on one copy stream while step k
    # runs, and step k's y comes back on another while step k+1 runs (device inputs and y
    # double-buffered, the reuse of each buffer ordered by events).
    ke = min(nsteps, 64)
    hx = xs[:ke].cpu().pin_memory()
    hdt = dts[:ke].cpu().pin_memory()
    hB = Bs[:ke].cpu().pin_memory()
    hC = Cs[:ke].cpu().pin_memory()
    y_h = torch.empty((ke,) + tuple(y.shape), dtype=y.dtype, pin_memory=True)
    nbuf = 2
    dx = [torch.empty_like(xs[0]) for _ in range(nbuf)]
    ddt = [torch.empty_like(dts[0]) for _ in range(nbuf)]
    dB = [torch.empty_like(Bs[0]) for _ in range(nbuf)]
    dC = [torch.empty_like(Cs[0]) for _ in range(nbuf)]
    dy = [torch.empty_like(y) for _ in range(nbuf)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    snapshot = state.clone()  # to replay the same steps in order afterwards, as a check
    ev_in = [torch.cuda.Event() for _ in range(ke)]
    ev_done = [torch.cuda.Event() for _ in range(ke)]
    ev_out = [torch.cuda.Event() for _ in range(ke)]
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    a, e = mk(), mk()
    a.record(stream)
    up.wait_event(a)
    down.wait_event(a)
    for k in range(ke):
        j = k % nbuf
        with torch.cuda.stream(up):
            if k >= nbuf:
                up.wait_event(ev_done[k - nbuf])  # the step that last read these inputs has run
            dx[j].copy_(hx[k], non_blocking=True)
            ddt[j].copy_(hdt[k], non_blocking=True)
            dB[j].copy_(hB[k], non_blocking=True)
            dC[j].copy_(hC[k], non_blocking=True)
            ev_in[k].record(up)
        stream.wait_event(ev_in[k])
        if k >= nbuf:
            stream.wait_event(ev_out[k - nbuf])  # this y buffer's last copy back has finished
        ssd.decode_step(state, dx[j], ddt[j], A, dB[j], dC[j], D, y=dy[j], stream=stream)
        ev_done[k].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[k])
            y_h[k].copy_(dy[j], non_blocking=True)
            ev_out[k].record(down)
    stream.wait_stream(down)
    e.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e2e_ms = max_over_ranks(a.elapsed_time(e), world, dev)
    # the overlapped copies must not change what the steps compute: replay them in order on
    # one stream from the same state and compare every y bit for bit
    state.copy_(snapshot)
    del snapshot
    same = True
    for k in range(ke):
        yk = ssd.decode_step(state, xs[k], dts[k], A, Bs[k], Cs[k], D, stream=stream)
        same = same and torch.equal(yk.cpu(), y_h[k])
    res["e2e"] = {"value": world * ke / (e2e_ms / 1e3), "unit": "steps/s", "steps": ke,
                  "outputs_match_in_order_steps": bool(same),
                  "h2d_bytes_per_step": dx[0].numel() * 2 + ddt[0].numel() * 4 + dB[0].numel() * 2
                  + dC[0].numel() * 2,
                  "d2h_bytes_per_step": y.numel() * 4,
                  "path": "pinned host x, dt, B, C -> device -> ssd_decode_step -> y -> pinned host; inputs up "
                          "and y back on two copy streams, overlapping the neighbouring steps"}
    return res


def frontend_leg(dev, peaks, w):
    """The fused front end (conv + SiLU + split, softplus dt) on the prefill workload's
    shapes: bf16 xbc [b, L, H*P + 2*G*N] -> x, B, C (bf16) and dt (fp32), conv state
    carried.  HBM-bound: bytes = xbc + x, B, C + dt_raw + dt + the conv state in and out."""
    import torch
    from selective_state_space_10_b200 import ssd
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    CH = H * P + 2 * G * N
    g = torch.Generator(device=dev).manual_seed(7)
    xbc = torch.randn((b, L, CH), device=dev, generator=g).bfloat16()
    cw = torch.randn((CH, 4), device=dev, generator=g) * 0.5
    cb = torch.randn((CH,), device=dev, generator=g) * 0.1
    dtr = torch.randn((b, L, H), device=dev, generator=g)
    dtb = torch.full((H,), -2.0, device=dev)
    st = torch.zeros((b, 3, CH), device=dev)
    x = torch.empty((b, L, H, P), dtype=torch.bfloat16, device=dev)
    Bo = torch.empty((b, L, G, N), dtype=torch.bfloat16, device=dev)
    Co = torch.empty_like(Bo)
    dt = torch.empty((b, L, H), device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda: ssd.frontend(xbc, cw, dtr, dtb, H, P, G, N, conv_b=cb, conv_state_in=st, conv_state_out=st,
                                x=x, B=Bo, C=Co, dt=dt, stream=stream)
    for _ in range(3):
        call()
    # The headline: calls back to back, their inputs and outputs rotated over enough copies
    # that together they exceed twice the L2 (so no call finds its input in L2), captured as
    # one CUDA graph of one call per copy and replayed, the replays timed between two events.
    in_bytes = xbc.numel() * xbc.element_size()
    ncopy = max(2, -(-2 * L2_BYTES // in_bytes))
    ins = [xbc] + [xbc.clone() for _ in range(ncopy - 1)]
    outs = [(x, Bo, Co, dt)] + [(torch.empty_like(x), torch.empty_like(Bo), torch.empty_like(Co), torch.empty_like(dt))
                                for _ in range(ncopy - 1)]
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        for i in range(ncopy):  # warm-up on the capture stream
            ssd.frontend(ins[i], cw, dtr, dtb, H, P, G, N, conv_b=cb, conv_state_in=st, conv_state_out=st,
                         x=outs[i][0], B=outs[i][1], C=outs[i][2], dt=outs[i][3], stream=cap)
        with torch.cuda.graph(graph, stream=cap):
            for i in range(ncopy):
                ssd.frontend(ins[i], cw, dtr, dtb, H, P, G, N, conv_b=cb, conv_state_in=st, conv_state_out=st,
                             x=outs[i][0], B=outs[i][1], C=outs[i][2], dt=outs[i][3], stream=cap)
    torch.cuda.synchronize(dev)
    reps = 10
    graph.replay()
    torch.cuda.synchronize(dev)
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        graph.replay()
    e.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(e) / (reps * ncopy)
    same = all(torch.equal(o[0], x) and torch.equal(o[1], Bo) and torch.equal(o[2], Co) for o in outs[1:])
    del graph, ins, outs
    # context only: one call at a time from a one-call graph, after a 256 MiB write that
    # evicts L2 (and, second, after a flush that also reads another 256 MiB buffer, so that no
    # dirty flush lines wait in L2), an event on each side
    graph = torch.cuda.CUDAGraph()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            ssd.frontend(xbc, cw, dtr, dtb, H, P, G, N, conv_b=cb, conv_state_in=st, conv_state_out=st,
                         x=x, B=Bo, C=Co, dt=dt, stream=cap)
    torch.cuda.synchronize(dev)
    clean = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    times, ctimes = [], []
    for k in range(10):
        for out, read_clean in ((times, False), (ctimes, True)):
            flush.fill_(k)
            if read_clean:
                torch.sum(clean, dim=0, out=sink)
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            e.record(stream)
            torch.cuda.synchronize(dev)
            out.append(a.elapsed_time(e))
    del graph, clean
    nbytes = b * L * CH * 2 * 2 + b * L * H * 4 * 2 + 2 * b * 3 * CH * 4 + CH * 4 * 5
    return {"workload": w.name, "us": ms * 1e3, "bytes": nbytes, "GB/s": nbytes / (ms / 1e3) / 1e9,
            "frac_of_hbm_peak": nbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], "launches": 2,
            "l2": f"inputs and outputs rotated over {ncopy} copies (inputs {ncopy * in_bytes / 2**20:.0f} MiB, more "
                  "than twice the L2); calls back to back",
            "timing": f"{reps} replays of a CUDA graph of {ncopy} calls between two events",
            "rotated_copies_outputs_identical": bool(same),
            "single_call_l2_flushed_us": statistics.median(times) * 1e3,
            "l2_clean_context": {"us": statistics.median(ctimes) * 1e3,
                                 "flush": "256 MiB written, then another 256 MiB buffer read"}}


def decode_vs_recompute_leg(dev, context=4096):
    """The cost of one new token two ways, with libssd's own calls ("Compiler-First State
    Space Duality ..." abstract compares cached decode with full-prefix recomputation at a
    4096-token context): one cached ssd_decode_step from the prefill's final state, against
    an ssd_prefill of the whole context plus the new token.  Batch 1, bf16 inputs, both
    timed back to back on one stream (the decode state, 0.8-2.6 MB, stays in L2 as in a
    decode loop).  Also checks that both give the new token the same output."""
    import torch
    from selective_state_space_10_b200 import inputs, ssd
    stream = torch.cuda.current_stream(dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)
    out = {"context": context, "batch": 1, "chunk": 256,
           "pages": "27-36x faster cached decode than full-prefix recompute (full models, TPU v6e)"}
    for name, H in (("mamba2_130m", 24), ("mamba2_2.7b", 80)):
        si = inputs.sequence(1, context + 1, H, 64, 128, 1, "bf16", seed=20261000 + H)
        t = upload(si, dev)
        ctx = {k: (v[:, :context].contiguous() if v.dim() > 1 else v) for k, v in t.items()}
        tok = {"x": t["x"][:, context].contiguous(), "dt": t["dt"][:, context].contiguous(), "A": t["A"],
               "B": t["B"][:, context].contiguous(), "C": t["C"][:, context].contiguous(), "D": t["D"]}
        _, cache = ssd.prefill(**ctx, chunk=256)
        state = cache.clone()
        y_dec = ssd.decode_step(state, **tok)
        y_full, _ = ssd.prefill(**t, chunk=256)
        torch.cuda.synchronize(dev)
        ref = y_full[:, context]
        rms = float(ref.pow(2).mean().sqrt())
        agree = float((y_dec - ref).abs().max()) / max(rms, 1e-30)
        y = torch.empty_like(y_dec)
        ws = torch.empty(ssd.prefill_workspace_size(ssd.dims_of_prefill(t["x"], t["B"]), ssd.BF16, 256),
                         dtype=torch.uint8, device=dev)
        yf = torch.empty_like(y_full)
        fs = torch.empty_like(cache)
        nd, nr = 200, 20
        for _ in range(10):
            ssd.decode_step(state, **tok, y=y, stream=stream)
        # the decode steps are replayed from a CUDA graph, as a decode loop would, so that
        # host launch overhead does not stand in for the step's device time
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap):
                for _ in range(nd):
                    ssd.decode_step(state, **tok, y=y, stream=cap)
        torch.cuda.synchronize(dev)
        g.replay()
        torch.cuda.synchronize(dev)
        a, e = mk(), mk()
        a.record(stream)
        g.replay()
        e.record(stream)
        torch.cuda.synchronize(dev)
        del g
        dec_us = a.elapsed_time(e) * 1e3 / nd
        for _ in range(3):
            ssd.prefill(**t, chunk=256, y=yf, final_state=fs, workspace=ws, stream=stream)
        a, e = mk(), mk()
        a.record(stream)
        for _ in range(nr):
            ssd.prefill(**t, chunk=256, y=yf, final_state=fs, workspace=ws, stream=stream)
        e.record(stream)
        torch.cuda.synchronize(dev)
        rec_us = a.elapsed_time(e) * 1e3 / nr
        out[name] = {"nheads": H, "decode_us": dec_us, "recompute_us": rec_us, "ratio": rec_us / dec_us,
                     "new_token_output_agreement_max_over_rms": agree}
    return out


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world != args.gpus:
        if args.gpus > 1 and world == 1:
            print(json.dumps({"error": f"--gpus {args.gpus} needs torchrun with {args.gpus} processes"}))
            return 2
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device: libssd has no CPU path"}))
        return 2
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl", dev)
    peaks = load_peaks()
    sampler = ClockSampler(local)
    sampler.start()
    try:
        pre = prefill_leg(args, dev, rank, world, peaks, sampler)
        dec = None if args.skip_decode else decode_leg(args, dev, rank, world, peaks, sampler)
        dvr = None if args.skip_recompute else decode_vs_recompute_leg(dev)
        from selective_state_space_10_b200 import inputs as _inp
        fe = frontend_leg(dev, peaks, _inp.BY_NAME[args.workload])
    finally:
        sampler.stop()
    from selective_state_space_10_b200 import inputs
    out = {
        "metric": METRIC, "value": pre["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": pre["ms_per_step"], "serial_ms_per_step": pre["serial_ms_per_step"],
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; value recipe in inputs.py)",
        "config": pre["config"], "tflops": pre["tflops"], "hbm": pre["hbm"], "kernels": pre["kernels"],
        "roofline": pre["roofline"], "gpu_launches": pre["gpu_launches"] + (dec["gpu_launches"] if dec else 0),
        "gpu_launches_prefill_timed_region": pre["gpu_launches"], "e2e": pre["e2e"],
        "single_step_l2_flushed": pre["single_step_l2_flushed"],
        "rotated_copies_outputs_identical": pre["rotated_copies_outputs_identical"],
        "host_enqueue_us_per_call": pre["host_enqueue_us_per_call"],
        "l2_clean_context": pre["l2_clean_context"], "peaks": peaks, "clocks": sampler.summary(), "impl": "ours",
    }
    if dec:
        out["decode"] = dec
    if dvr:
        out["decode_vs_recompute"] = dvr
    out["frontend"] = fe
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        w = inputs.BY_NAME[args.workload]
        rate, desc, threads, secs = oracle_prefill_rate(w, w.seed)
        out["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                               "sample": desc, "seconds": secs}
        if dec:
            wd = decode_workload(args)
            drate, ddesc, dthreads, dsecs = oracle_decode_rate(wd, wd.seed)
            out["decode"]["cpu_baseline"] = {"value": drate, "unit": "steps/s", "cores": dthreads,
                                             "kind": "oracle", "sample": ddesc, "seconds": dsecs}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_reference(args):
    """The fp64 CPU oracle as the reference arm: rank 0 only, K timed steps of a bounded
    sample (16 of 80 heads, all 4096 tokens) of the prefill workload per step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from selective_state_space_10_b200 import inputs
    w = inputs.BY_NAME[args.workload]
    si = inputs.workload_sequence(w)
    Hs = min(16, w.nheads)
    f64 = lambda a: np.ascontiguousarray(a, dtype=np.float64)
    a = (f64(si.x[:, :, :Hs]), f64(si.dt[:, :, :Hs]), f64(si.A[:Hs]), f64(si.B), f64(si.C), f64(si.D[:Hs]))
    threads = oracle.default_threads()
    for _ in range(args.warmup):
        oracle.recurrence(*a, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrence(*a, nthreads=threads)
    secs = time.perf_counter() - t0
    tokens = args.steps * w.batch * w.seqlen * Hs / w.nheads
    value = tokens / secs
    sample = f"per step: fp64 recurrence over {Hs} of {w.nheads} heads x {w.seqlen} tokens; value scaled to the full layer"
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3 * w.nheads / Hs, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups, "chunk": w.chunk},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=PREFILL_WORKLOAD)
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="decode batch (default: the workload's 256); for small profiling captures")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-recompute", action="store_true",
                    help="skip the cached-decode vs full-prefix-recompute comparison")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
