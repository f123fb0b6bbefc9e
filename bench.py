#!/usr/bin/env python
"""Benchmark: one decode step of multi-head latent attention on the paged
latent cache (append the new tokens, then attend), on the DeepSeek-V2-like
workload (B=64, n_h=128, d_c=512, d_r=64, 8192 cached tokens + 1 new token per
sequence, bf16), timed on the device with CUDA events.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU runs are independent replicas (the
path shards by sequence; there is no collective on the data path), so
`value` is the sum over ranks of the bytes each rank streamed divided by the
slowest rank's time.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
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


def aggregate(bytes_per_rank: int, ms_local: float, ws: int, device: str = "cuda"):
    """Whole-job throughput of N independent replicas: every rank streams
    bytes_per_rank per step; the job's step time is the slowest rank's."""
    ms = max_over_ranks(ms_local, ws, device)
    return ms, ws * bytes_per_rank / (ms * 1e-3) / 1e9


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def oracle_sample(name: str):
    """Times the fp64 oracle on one sequence of the workload (its full
    history and its new tokens): returns (seconds, cache bytes, tokens)."""
    import numpy as np
    import oracle as O
    from head_latent_attention_append_b200 import synth
    wl = synth.WORKLOADS[name]
    kv = synth.kv_lengths(wl)
    b = int(np.argsort(kv)[len(kv) // 2])
    hw = synth.make_weights(wl)
    dims = O.Dims(wl.n_h, wl.d_h, wl.d_v, wl.d_c, wl.d_r, wl.d_model, wl.d_cq, wl.rope_base)
    w = O.Weights(**hw.as_dict())
    L = int(kv[b])
    H = synth.make_hidden(wl, b, L)
    t0 = time.perf_counter()
    O.mla_decode(dims, w, H, wl.n_q)
    dt = time.perf_counter() - t0
    esz = 2 if wl.dtype == "bf16" else 4
    keys = sum(L - wl.n_q + 1 + q for q in range(wl.n_q))
    return dt, keys * wl.d_cr * esz, wl.n_q, f"1 of {wl.B} sequences ({L} keys, {wl.n_q} new token(s))"


def run_reference(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = os.cpu_count()
    for _ in range(args.warmup):
        oracle_sample(args.workload)
    tot_t = tot_b = tot_tok = 0.0
    sample = ""
    for _ in range(args.steps):
        dt, nb, ntok, sample = oracle_sample(args.workload)
        tot_t += dt
        tot_b += nb
        tot_tok += ntok
    val = tot_b / tot_t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.workload},
            "tokens_per_s": tot_tok / tot_t,
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step: {sample}"},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    from head_latent_attention_append_b200 import mla, synth, workload
    ws, rank, local = dist_setup()
    peaks = load_peaks()
    s = workload.setup(args.workload, device=f"cuda:{local}", checked_count=0, check_all=False)
    wl = s.wl
    cache_bytes = s.cache_bytes_read()
    flops = s.attention_flops()
    stream = torch.cuda.current_stream()

    # Launch accounting for one step.
    launches = workload.step(s)
    torch.cuda.synchronize()
    assert mla.get_error(s.ws) == mla.MLA_OK
    for _ in range(args.warmup):
        workload.step(s)
    torch.cuda.synchronize()

    # Attention-kernel time, bracketed by CUDA events inside the library on
    # the launching stream (eager launches).
    mla.profile_begin(args.steps)
    for _ in range(args.steps):
        workload.step(s)
    torch.cuda.synchronize()
    attn_ms, attn_n = mla.profile_end()

    # The step as one CUDA graph (the library allocates nothing and only
    # enqueues on the caller's stream, so the whole step captures).
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        workload.step(s)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    # Device-timed region.
    barrier(ws)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    ms_step, value = aggregate(cache_bytes, e0.elapsed_time(e1) / args.steps, ws)
    clk = clocks.stop()
    assert mla.get_error(s.ws) == mla.MLA_OK

    # End to end through the public API with host buffers: pinned h_new in,
    # the fp32 outputs back, both copies inside the timed region (captured in
    # the same graph as the step).
    h_host = s.h_new.cpu().pin_memory()
    out_host = torch.empty(s.out.shape, dtype=s.out.dtype).pin_memory()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2):
        s.h_new.copy_(h_host, non_blocking=True)
        workload.step(s)
        out_host.copy_(s.out, non_blocking=True)
    for _ in range(args.warmup):
        g2.replay()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(args.steps):
        g2.replay()
    e3.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3) / args.steps, ws)
    del graph, g2

    tokens = wl.B * (wl.n_q if wl.mode == "decode" else wl.n_q)
    attn_avg_ms = attn_ms / max(1, attn_n)
    achieved = cache_bytes / (attn_avg_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "n_q": wl.n_q, "kv_len": int(s.kv_len_host.max()),
                   "n_h": wl.n_h, "d_c": wl.d_c, "d_r": wl.d_r, "d_model": wl.d_model, "d_cq": wl.d_cq,
                   "page_size": synth.PAGE_SIZE, "parallelism": f"replicas{ws}" if ws > 1 else "single",
                   "l2": f"inputs larger than L2: {cache_bytes / 1e6:.0f} MB of cache read per step",
                   "timing": "CUDA graph of one step, replayed; CUDA events on the launching stream"},
        "tokens_per_s": ws * tokens / (ms_step * 1e-3),
        "attention_tflops": ws * flops / (ms_step * 1e-3) / 1e12,
        "roofline": {"bound": "hbm", "kernel": "latent attention (split-KV)", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": None, "peak_src": peaks["src"], "avg_kernel_ms": attn_avg_ms,
                     "algorithmic_bytes_per_launch": cache_bytes},
        "e2e": {"value": ws * cache_bytes / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": s.h_new.numel() * s.h_new.element_size(),
                "d2h_bytes_per_step": s.out.numel() * s.out.element_size(), "ms_per_step": ms_e2e},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        dt, nb, _, sample = oracle_sample(args.workload)
        line["cpu_baseline"] = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
                                "sample": sample, "seconds": dt}
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
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
