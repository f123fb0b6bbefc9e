"""bench.py's multi-replica accounting on two gloo ranks (CPU): the step time
is the slowest rank's, and the job's value sums the ranks' bytes."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    ms_local = [2.0, 3.0][rank]
    ms, value = bench.aggregate(1_000_000_000, ms_local, ws, device="cpu")
    q.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_report_slowest_time_and_summed_bytes():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for _, ms, value in res:
        assert ms == 3.0
        assert value == pytest.approx(2 * 1e9 / 3e-3 / 1e9)


def test_single_rank_is_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.aggregate(604_053_504, 0.5, 1)
    assert ms == 0.5 and value == pytest.approx(604_053_504 / 0.5e-3 / 1e9)


def test_measured_traffic_follows_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from a recorded ncu capture only while the
    kernel sources still hash to what was captured."""
    import hashlib
    import json
    import bench
    csrc = tmp_path / "head_latent_attention_append_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cuh").write_text("int kernel_v1;  // first\n")
    digest = hashlib.sha256(b"intkernel_v1;").hexdigest()  # code only: no comments, no whitespace
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"wl": {"traffic_bytes": 1234, "source_files": ["k.cuh"], "source_sha256": digest}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("wl") == 1234
    assert bench.measured_traffic("other") is None
    (csrc / "k.cuh").write_text("/* reworded */ int  kernel_v1;  // second\n")
    assert bench.measured_traffic("wl") == 1234  # a comment edit is not a kernel change
    (csrc / "k.cuh").write_text("int kernel_v2;\n")
    assert bench.measured_traffic("wl") is None


def test_binding_roof_follows_flops_per_cache_byte():
    sys.path.insert(0, ROOT)
    import bench
    from head_latent_attention_append_b200 import synth
    assert bench.binding_roof("decode", 1) == "hbm"
    assert bench.binding_roof("decode", 2) == "tensor"
    assert bench.binding_roof("prefill", 4096) == "tensor"
    # Flops per unique cache byte of a decode step: every key feeds n_q query
    # tokens (less the causal triangle of the new tokens themselves).
    wl = synth.WORKLOADS["dsv2_bf16_decode"]
    per_key = wl.n_h * (2 * wl.d_cr + 2 * wl.d_c)
    assert abs(per_key / (wl.d_cr * 2) - 241.8) < 0.1
    for name in ("dsv2_ragged_decode", "dsv2_spec4_decode"):
        w = synth.WORKLOADS[name]
        kv = synth.kv_lengths(w)
        pairs = sum(int(L) - w.n_q + 1 + q for L in kv for q in range(w.n_q))
        intensity = pairs * per_key / (int(kv.sum()) * w.d_cr * 2)
        assert intensity >= 1.99 * 241.8, (name, intensity)
        assert bench.binding_roof(w.mode, w.n_q) == "tensor"


def test_nvml_poller_summarises_in_region_samples(monkeypatch):
    """The clock poller against a fake NVML (no GPU here): samples taken on a
    thread, reasons OR-ed over the samples, and a broken NVML yields None."""
    import types
    import time as _time
    sys.path.insert(0, ROOT)
    import bench
    clocks = iter([1965.0, 1965.0, 1800.0] * 1000)
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1, nvmlInit=lambda: None, nvmlShutdown=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda u: "h", nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: next(clocks),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(uuid="abc", pci_domain_id=0, pci_bus_id=1, pci_device_id=0))
    p = bench.NvmlPoller(0, period_s=0.001)
    p.start()
    _time.sleep(0.05)
    out = p.stop()
    assert out["samples"] >= 3 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["sm_mhz"] in (1965.0, 1800.0)
    assert bench.summarize_nvml([(1900.0, 0x8 | 0x40), (1950.0, 0)], 1965) == {
        "sm_mhz": 1925.0, "sm_max_mhz": 1965, "reasons": ["hw_slowdown", "hw_thermal_slowdown"], "samples": 2,
        "source": "NVML, every 2 ms during the timed region"}
    # NVML that fails to start leaves no samples and raises nothing.
    broken = types.SimpleNamespace(nvmlInit=lambda: (_ for _ in ()).throw(RuntimeError("no driver")),
                                   nvmlShutdown=lambda: None)
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    q = bench.NvmlPoller(0)
    q.start()
    assert q.stop() is None
