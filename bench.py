#!/usr/bin/env python
"""Benchmark: one step of multi-head latent attention on the paged latent
cache -- append the new tokens, then attend -- timed on the device with CUDA
events.  The default workload is the DeepSeek-V2-like decode (B=64, n_h=128,
d_c=512, d_r=64, 8192 cached tokens + 1 new token per sequence, bf16); the
other named workloads (synth.WORKLOADS) run with --workload.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is latent-cache GB/s (each sequence's
cache counted once per step) for decode workloads and attention TFLOP/s for
prefill.  The default run adds two objects to the same line, measured the same
way: `prefill` (the causal prefill, B=4, S=4096, attention TFLOP/s) and
`ragged` (the ragged paged decode, B=128, 2 new tokens per sequence).
Multi-GPU runs are independent replicas (the path shards by sequence; there is
no collective on the data path), so `value` is the sum over ranks of what each
rank processed divided by the slowest rank's time.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode latent-cache GB/s + tokens/s; prefill TFLOPS (vs B200 roofline)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


# Clock-event reason bits (NVML): name in the JSON line, NVML constant suffix, value.
NVML_REASONS = (("hw_slowdown", "HwSlowdown", 0x8), ("hw_thermal_slowdown", "HwThermalSlowdown", 0x40),
                ("sw_thermal_slowdown", "SwThermalSlowdown", 0x20), ("sw_power_cap", "SwPowerCap", 0x4))


def summarize_nvml(samples, max_mhz):
    """(sm_mhz, reason bitmask) samples -> the line's clocks object, or None."""
    if not samples:
        return None
    seen = 0
    for _, bits in samples:
        seen |= bits
    return {"sm_mhz": statistics.median(m for m, _ in samples), "sm_max_mhz": max_mhz,
            "reasons": sorted(name for name, _, bit in NVML_REASONS if seen & bit), "samples": len(samples),
            "source": "NVML, every 2 ms during the timed region"}


class NvmlPoller:
    """Reads the SM clock and the clock-event reasons through NVML (read-only)
    from a host thread every ~2 ms while a timed region runs: the regions
    here last milliseconds, well under nvidia-smi's 200 ms period.  Any NVML
    failure leaves it without samples; it never raises."""

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.dev = device_index
        self.period = period_s
        self.nv = None
        self.h = None
        self.max_mhz = None
        self.samples = []
        self.thread = None
        self.stop_evt = threading.Event()

    def _handle(self, nv):
        import torch
        props = torch.cuda.get_device_properties(self.dev)
        try:
            return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:
            pass
        try:
            return nv.nvmlDeviceGetHandleByPciBusId(
                "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id))
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = self._handle(nv)
            self.reasons = (getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None)
                            or nv.nvmlDeviceGetCurrentClocksThrottleReasons)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception:
            self._shutdown()
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                self.samples.append((float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)),
                                     int(self.reasons(self.h))))
            except Exception:
                return
            self.stop_evt.wait(self.period)

    def _shutdown(self):
        if self.nv is not None:
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass
            self.nv = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=2.0)
        self._shutdown()
        return summarize_nvml(list(self.samples), self.max_mhz)


def dist_setup():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return ws, rank, local


def max_over_ranks(x: float, ws: int, device: str = "cuda") -> float:
    """Largest value of x over all ranks (x is each rank's device time)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, ms_local: float, ws: int, device: str = "cuda", scale: float = 1e9):
    """Whole-job throughput of N independent replicas: every rank processes
    units_per_rank (bytes, or flops) per step; the job's step time is the
    slowest rank's.  Returns (ms, units / s / scale)."""
    ms = max_over_ranks(ms_local, ws, device)
    return ms, ws * units_per_rank / (ms * 1e-3) / scale


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def kernel_code_hash(files) -> str:
    """sha256 of the listed csrc files' code, concatenated in order, with
    comments and whitespace removed (a comment edit does not change the
    kernel)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "head_latent_attention_append_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("".join(text.split()).encode())
    return h.hexdigest()


def measured_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    capture (profiles/traffic.json), or None when there is none for this
    workload or the kernel's code changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        rec = json.load(fh).get(workload)
    if not rec:
        return None
    return rec["traffic_bytes"] if kernel_code_hash(rec["source_files"]) == rec["source_sha256"] else None


def e2e_pipelined(s, step_on, h_host, args, ws, stream) -> float:
    """ms per step of the public-API loop with each step's host->device copy
    of its inputs and device->host copy of its outputs on two copy streams,
    double-buffered, so that they overlap the neighbouring steps' compute.
    The timed region runs from the first copy in to the last copy out."""
    import torch
    cs_in, cs_out = torch.cuda.Stream(), torch.cuda.Stream()
    h_dev = [s.h_new, s.h_new.clone()]
    out_dev = [s.out, torch.empty_like(s.out)]
    out_host = [torch.empty(s.out.shape, dtype=s.out.dtype).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            j = i & 1
            if i >= 2:
                cs_in.wait_event(ev_c[j])      # step i-2 no longer reads h_dev[j]
            with torch.cuda.stream(cs_in):
                h_dev[j].copy_(h_host, non_blocking=True)
            ev_in[j].record(cs_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])   # step i-2's outputs have left out_dev[j]
            s.h_new, s.out = h_dev[j], out_dev[j]
            step_on(i)
            ev_c[j].record(stream)
            cs_out.wait_event(ev_c[j])
            with torch.cuda.stream(cs_out):
                out_host[j].copy_(out_dev[j], non_blocking=True)
            ev_out[j].record(cs_out)

    run(args.warmup)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs_in)
    run(args.steps)
    e1.record(cs_out)
    torch.cuda.synchronize()
    s.h_new, s.out = h_dev[0], out_dev[0]
    return max_over_ranks(e0.elapsed_time(e1) / args.steps, ws)


PREFILL_SAMPLE_TOKENS = 1024   # causal prefix of one sequence per oracle prefill sample


def blas_threads() -> int:
    """Threads the oracle's BLAS actually runs with."""
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(name: str, k: int = 0):
    """Times the fp64 oracle on one bounded unit of the workload: the k-th
    sequence (in a seeded order) of a decode workload, with its whole history
    and its new tokens, or the causal prefix of PREFILL_SAMPLE_TOKENS tokens
    of one sequence of a prefill workload.  Returns a dict with the seconds,
    the unique cache bytes, the attention flops, the query tokens and a
    description."""
    import numpy as np
    import oracle as O
    from head_latent_attention_append_b200 import synth
    wl = synth.WORKLOADS[name]
    kv = synth.kv_lengths(wl)
    med = int(np.argsort(kv)[len(kv) // 2])   # the median-length sequence first, then a seeded order
    order = [med] + [int(i) for i in np.random.default_rng(wl.wid).permutation(len(kv)) if i != med]
    b = order[k % len(order)]
    hw = synth.make_weights(wl)
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base,
                  rope_per_head=wl.rope_per_head)
    w = O.Weights(**hw.as_dict())
    if wl.mode == "prefill":
        L = nq = min(PREFILL_SAMPLE_TOKENS, int(kv[b]))
        what = f"causal prefix of {L} tokens of sequence {b} of {wl.B} (S={int(kv[b])})"
    else:
        L, nq = int(kv[b]), wl.n_q
        what = f"sequence {b} of {wl.B} ({L} keys, {nq} new token(s))"
    H = synth.make_hidden(wl, b, L)
    t0 = time.perf_counter()
    O.mla_decode(dims, w, H, nq)
    dt = time.perf_counter() - t0
    esz = 2 if wl.dtype == "bf16" else 4
    pairs = sum(L - nq + 1 + q for q in range(nq))
    return {"seconds": dt, "bytes": L * wl.d_cr * esz, "flops": pairs * wl.flops_per_pair(),
            "tokens": nq, "what": what}


def binding_roof(mode: str, n_q: int) -> str:
    """The roof the attention kernel is held to.  A decode step with one new
    token per sequence does 242 flop per cache byte (d_c = 512, d_r = 64),
    about the ridge of the measured peaks, and is read as HBM-bound; with
    n_q >= 2 new tokens per sequence every cache byte feeds n_q query tokens
    (>= 484 flop per byte), and a causal prefill far more, so those are
    tensor-bound."""
    return "tensor" if mode == "prefill" or n_q >= 2 else "hbm"


def metric_of(mode: str, nbytes: float, flops: float, seconds: float):
    """The workload's headline figure: latent-cache GB/s for decode, attention
    TFLOP/s for prefill."""
    if mode == "prefill":
        return flops / seconds / 1e12, "TFLOP/s"
    return nbytes / seconds / 1e9, "GB/s"


def cpu_baseline(name: str, min_seconds: float = 10.0, max_samples: int = 16):
    """The oracle on successive bounded samples until about min_seconds of
    CPU work; returns the line's cpu_baseline object."""
    from head_latent_attention_append_b200 import synth
    mode = synth.WORKLOADS[name].mode
    tot = {"seconds": 0.0, "bytes": 0, "flops": 0, "tokens": 0}
    whats = []
    k = 0
    while k < max_samples and (k == 0 or tot["seconds"] < min_seconds):
        r = oracle_sample(name, k)
        for key in tot:
            tot[key] += r[key]
        whats.append(r["what"])
        k += 1
    val, unit = metric_of(mode, tot["bytes"], tot["flops"], tot["seconds"])
    return {"value": val, "unit": unit, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{k} sample(s), {tot['seconds']:.1f} s of fp64 oracle work: " + "; ".join(whats),
            "seconds": tot["seconds"], "tokens_per_s": tot["tokens"] / tot["seconds"]}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, one bounded sample
    per step, on the same metric and unit as the GPU line."""
    from head_latent_attention_append_b200 import synth
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    mode = synth.WORKLOADS[args.workload].mode
    for i in range(args.warmup):
        oracle_sample(args.workload, i)
    tot = {"seconds": 0.0, "bytes": 0, "flops": 0, "tokens": 0}
    whats = []
    for i in range(args.steps):
        r = oracle_sample(args.workload, i)
        for key in tot:
            tot[key] += r[key]
        whats.append(r["what"])
    val, unit = metric_of(mode, tot["bytes"], tot["flops"], tot["seconds"])
    sample = f"one bounded sample per step ({whats[0]}{', ...' if len(whats) > 1 else ''})"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": unit, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot["seconds"] / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.workload},
            "tokens_per_s": tot["tokens"] / tot["seconds"],
            "cpu_baseline": {"value": val, "unit": unit, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


REGION_TARGET_S = 0.5     # timed regions are repeated until about this much device time
MIN_REGIONS, MAX_REGIONS = 5, 200


def l2_plan(unique_bytes: int, l2_bytes: int):
    """How a workload keeps L2 from serving the timed steps: the number of
    distinct copies of its latent cache the steps rotate through, and the
    line's note.  A cache larger than L2 needs no copy; a smaller one is
    rotated over enough copies to exceed 4x L2."""
    if unique_bytes > l2_bytes:
        return 1, (f"inputs larger than L2: {unique_bytes / 1e6:.0f} MB of latent cache read per step "
                   f"(L2 {l2_bytes / 1e6:.0f} MB)")
    n = -(-4 * l2_bytes // max(1, unique_bytes)) + 1
    return n, (f"L2 defeated by rotation: each step reads one of {n} distinct caches of "
               f"{unique_bytes / 1e6:.1f} MB ({n * unique_bytes / 1e6:.0f} MB in all, > 4x the "
               f"{l2_bytes / 1e6:.0f} MB L2)")


def with_batch(name: str, batch: int) -> str:
    """Registers (once) and returns a copy of workload `name` with `batch`
    sequences, for profiling the same kernels on a smaller case."""
    import dataclasses
    from head_latent_attention_append_b200 import synth
    if batch <= 0 or batch == synth.WORKLOADS[name].B:
        return name
    key = f"{name}_b{batch}"
    if key not in synth.WORKLOADS:
        synth.WORKLOADS[key] = dataclasses.replace(synth.WORKLOADS[name], name=key, B=batch)
    return key


def measure_workload(name, args, ws, local, peaks, with_cpu_baseline):
    """Every figure of one workload: the device-timed step (median of repeated
    regions of `steps` graph replays), the attention kernel's own time and its
    roofline, the end-to-end figure through the public API with host buffers,
    the clocks seen and, on request, the oracle's CPU baseline."""
    import torch
    from head_latent_attention_append_b200 import mla, synth, workload
    s = workload.setup(name, device=f"cuda:{local}", checked_count=0, check_all=False)
    wl = s.wl
    prefill = wl.mode == "prefill"
    unique_bytes = s.cache_bytes_unique()    # the latent cache, each key once
    streamed_bytes = s.cache_bytes_read()    # what the kernel streams (once per query row block)
    flops = s.attention_flops()
    units, scale, unit = (flops, 1e12, "TFLOP/s") if prefill else (unique_bytes, 1e9, "GB/s")
    stream = torch.cuda.current_stream()
    l2_bytes = torch.cuda.get_device_properties(local).L2_cache_size
    if prefill:
        n_rot = 1
        l2_note = (f"inputs larger than L2: {wl.B * wl.n_q * wl.d_model * 2 / 1e6:.0f} MB of hidden states in and "
                   f"{s.out.numel() * 4 / 1e6:.0f} MB out per step (L2 {l2_bytes / 1e6:.0f} MB)")
    else:
        n_rot, l2_note = l2_plan(unique_bytes, l2_bytes)
    caches = [s.cache] + [s.cache.clone() for _ in range(n_rot - 1)]

    def step_on(i):
        s.cache = caches[i % n_rot]
        return workload.step(s)

    # Launch accounting for one step, then eager warm-up.
    launches = step_on(0)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    for i in range(args.warmup):
        step_on(i)
    torch.cuda.synchronize()

    # Attention-kernel time, bracketed by CUDA events inside the library on
    # the launching stream (eager launches).
    mla.profile_begin(args.steps)
    for i in range(args.steps):
        step_on(i)
    torch.cuda.synchronize()
    attn_ms, attn_n = mla.profile_end()

    # One CUDA graph per cache copy (the library allocates nothing and only
    # enqueues on the caller's stream, so the whole step captures).
    graphs = []
    for i in range(n_rot):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step_on(i)
        graphs.append(g)
    for i in range(args.warmup):
        graphs[i % n_rot].replay()
    torch.cuda.synchronize()

    # Device-timed regions of exactly `steps` replays each, repeated until
    # about REGION_TARGET_S of device time so the clock record has substance;
    # the step time is the median region's.
    barrier(ws)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    poller = NvmlPoller(local)
    poller.start()
    region_ms = []
    n_regions = MIN_REGIONS
    r = 0
    while r < n_regions:
        barrier(ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            graphs[i % n_rot].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        region_ms.append(e0.elapsed_time(e1))
        if r == 0:   # every rank takes the same count (the slowest rank's first region decides)
            first = max_over_ranks(region_ms[0], ws)
            n_regions = min(MAX_REGIONS, max(MIN_REGIONS, int(REGION_TARGET_S * 1e3 / max(first, 1e-3)) + 1))
        r += 1
    in_region = poller.stop()
    barrier(ws)
    ms_step, value = aggregate(units, statistics.median(region_ms) / args.steps, ws, scale=scale)
    smi = clocks.stop()
    clk = dict(in_region, nvidia_smi=smi) if in_region else smi
    assert mla.get_error(s.ws) == mla.MLA_OK

    # End to end through the public API with host buffers: every step copies
    # its hidden states in from pinned host memory, calls the C ABI, and
    # copies the fp32 outputs back.  Eager (each step's host-side work --
    # argument checks, tensor-map encoding, launches -- included) and as a
    # replayed graph of the same three operations.
    h_host = s.h_new.cpu().pin_memory()
    out_host = torch.empty(s.out.shape, dtype=s.out.dtype).pin_memory()

    def e2e_step(i):
        s.h_new.copy_(h_host, non_blocking=True)
        step_on(i)
        out_host.copy_(s.out, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    e3.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3) / args.steps, ws)
    g2s = []
    for i in range(n_rot):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            e2e_step(i)
        g2s.append(g)
    for i in range(args.warmup):
        g2s[i % n_rot].replay()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e2.record(stream)
    for i in range(args.steps):
        g2s[i % n_rot].replay()
    e3.record(stream)
    torch.cuda.synchronize()
    ms_e2e_graph = max_over_ranks(e2.elapsed_time(e3) / args.steps, ws)
    del graphs, g2s

    # The same end-to-end steps as a serving loop runs them: step i's inputs
    # go up on a copy stream while step i-1 computes, and its outputs come
    # down on another while step i+1 computes (two device and two pinned
    # host buffers; every step's copies are still inside the timed region,
    # which runs from the first copy in to the last copy out).
    ms_e2e_pipe = e2e_pipelined(s, step_on, h_host, args, ws, stream)

    tokens = wl.B * wl.n_q
    attn_avg_ms = attn_ms / max(1, attn_n)
    hbm_gbs = unique_bytes / (attn_avg_ms * 1e-3) / 1e9
    tc_tflops = flops / (attn_avg_ms * 1e-3) / 1e12
    # The attention kernel runs inside a step of several kernels, back to
    # back: the sustained tensor peak applies; the burst ratio rides along.
    tc_peak = peaks["bf16_tflops_sustained"]
    hbm_roof = {"bound": "hbm", "achieved": hbm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": hbm_gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": unique_bytes}
    tc_roof = {"bound": "tensor", "achieved": tc_tflops, "peak": tc_peak, "unit": "TFLOP/s",
               "frac": tc_tflops / tc_peak, "algorithmic_flops_per_launch": flops,
               "peak_kind": "bf16 sustained", "frac_of_burst_peak": tc_tflops / peaks["bf16_tflops"]}
    main_roof, other_roof = ((tc_roof, hbm_roof) if binding_roof(wl.mode, wl.n_q) == "tensor"
                             else (hbm_roof, tc_roof))
    roofline = dict(main_roof, traffic=measured_traffic(wl.name), kernel="latent attention (split-KV)",
                    peak_src=peaks["src"], avg_kernel_ms=attn_avg_ms,
                    streamed_cache_bytes_per_launch=streamed_bytes, other_roof=other_roof)
    if wl.materialised:
        # The same causal prefill as the absorbed form: its flops over this
        # path's time compare the two forms on one clock.
        absorbed = s.attention_pairs() * wl.n_h * (2 * wl.d_cr + 2 * wl.d_c)
        roofline["absorbed_equivalent_tflops"] = absorbed / (attn_avg_ms * 1e-3) / 1e12
    h2d = s.h_new.numel() * s.h_new.element_size()
    d2h = s.out.numel() * s.out.element_size()
    res = {
        "workload": wl.name, "value": value, "unit": unit, "ms_per_step": ms_step,
        "cache_bytes_per_token": wl.d_cr * (2 if wl.dtype == "bf16" else 4),
        "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "config": {"workload": wl.name, "B": wl.B, "n_q": wl.n_q, "kv_len": int(s.kv_len_host.max()),
                   "n_h": wl.n_h, "d_c": wl.d_c, "d_r": wl.d_r, "d_model": wl.d_model, "d_cq": wl.d_cq,
                   "page_size": synth.PAGE_SIZE, "parallelism": f"replicas{ws}" if ws > 1 else "single",
                   "l2": l2_note,
                   "timing": (f"CUDA graph of one step, replayed; median of {len(region_ms)} regions of "
                              f"{args.steps} steps; CUDA events on the launching stream")},
        "regions": {"count": len(region_ms), "ms_per_step_min": min(region_ms) / args.steps,
                    "ms_per_step_max": max(region_ms) / args.steps},
        "tokens_per_s": ws * tokens / (ms_step * 1e-3),
        "cache_gbs": ws * unique_bytes / (ms_step * 1e-3) / 1e9,
        "attention_tflops": ws * flops / (ms_step * 1e-3) / 1e12,
        "form": "materialised" if wl.materialised else "absorbed",
        "roofline": roofline,
        "e2e": {"value": ws * units / (ms_e2e_pipe * 1e-3) / scale, "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e_pipe,
                "timing": ("eager C-ABI calls every step, each step's copy in and copy out included, on copy "
                           "streams overlapping the neighbouring steps' compute (double-buffered)"),
                "serial": {"value": ws * units / (ms_e2e * 1e-3) / scale, "ms_per_step": ms_e2e,
                           "timing": "copy in, step, copy out one after another on one stream"},
                "graph": {"value": ws * units / (ms_e2e_graph * 1e-3) / scale, "ms_per_step": ms_e2e_graph,
                          "timing": "the serial form as a replayed graph"}},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }
    if with_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(name)
    del s, caches
    torch.cuda.empty_cache()
    return res


# The workloads the default run reports beside the headline decode: the
# causal prefill (the prefill TFLOP/s half of the metric) and the ragged
# paged decode.
EXTRA = {"prefill": "dsv2_bf16_prefill", "ragged": "dsv2_ragged_decode",
         "prefill_materialised": "dsv2_bf16_prefill_mat", "page": "page_bf16_decode",
         "page_per_head_rope": "page_bf16_decode_rph", "spec4": "dsv2_spec4_decode"}


def run_ours(args):
    import torch
    ws, rank, local = dist_setup()
    peaks = load_peaks()
    want_cpu = rank == 0 and ws == 1 and not args.no_cpu_baseline
    head = measure_workload(with_batch(args.workload, args.batch), args, ws, local, peaks, want_cpu)
    line = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"], "data": "synthetic"}
    for k in ("config", "regions", "tokens_per_s", "cache_gbs", "attention_tflops", "roofline", "e2e",
              "gpu_launches", "clocks", "cpu_baseline"):
        if k in head:
            line[k] = head[k]
    if not args.no_extra and args.workload == "dsv2_bf16_decode":
        for key, name in EXTRA.items():
            line[key] = measure_workload(name, args, ws, local, peaks, want_cpu)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dsv2_bf16_decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="report only the headline workload (no prefill / ragged objects)")
    ap.add_argument("--batch", type=int, default=0,
                    help="run the workload with this many sequences instead of its own B (smaller profiling cases)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
