"""The replica timing of bench.py on several ranks, without a GPU: two gloo
processes on the CPU take the max over ranks and the whole-job rate the way
the benchmark does under torchrun."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank               # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world, device="cpu")
        out[rank] = (ms_max, bench.job_rate(100, world, ms_max))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_on_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        ms_max, rate = out[r]
        assert ms_max == 15.0                # every rank sees the slowest time
        assert rate == pytest.approx(world * 100 / 0.015)


def test_job_rate_single_rank():
    import bench
    assert bench.job_rate(4000, 1, 80.0) == pytest.approx(50_000.0)


def test_reference_arm_prints_the_contract_line_on_rank_0_only():
    """`bench.py --impl reference` (the CPU oracle timed on the host cores)
    prints one JSON line with the metric, the reference tag, its CPU
    baseline and an end-to-end entry without copies; a rank other than 0
    exits 0 without work.  Needs no GPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"]
    p = subprocess.run(cmd, cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "layer_fwd/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["warmup"] == 3
    assert d["config"]["workload"].startswith("moe_layer_int4_batch1")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    p1 = subprocess.run(cmd, cwd=root, env=dict(env, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1"), capture_output=True,
                        text=True, timeout=600)
    assert p1.returncode == 0 and not any(l.startswith("{") for l in p1.stdout.splitlines())


def test_clock_sampler_reads_clocks_and_decodes_reasons_from_nvml(monkeypatch):
    """The benchmark's clock record against a fake NVML (no GPU): the
    median SM clock of the samples, the maximum clock, and the names of the
    active clock-event reason bits (sw_power_cap kept, slowdowns named)."""
    import sys
    import types

    import bench
    clocks = iter([1965, 1800, 1965, 1965, 1500] + [1965] * 1000)
    reasons = iter([0x0, 0x4, 0x8 | 0x40] + [0x0] * 1000)
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByPciBusId=lambda bus: "h",
        nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
        nvmlDeviceGetClockInfo=lambda h, kind: next(clocks),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: next(reasons))
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler(0, period=3600.0)  # samples at entry and exit only
    assert s.ok
    with s:
        pass
    s._sample()
    s._sample()
    out = s.summary()
    assert out["sm_max_mhz"] == 1965 and out["samples"] == 4
    assert out["sm_mhz"] == 1965  # median of 1965, 1800, 1965, 1965
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]


def test_roofline_denominator_and_traffic_record(monkeypatch, tmp_path):
    """The roofline's peak comes from the measured-peaks file when there is
    one (else the stated fallback), and the recorded DRAM traffic is
    reported only while the kernel sources match the digest it was taken
    with."""
    import json

    import bench
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6123.5}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak() == (6123.5, "measured")
    (tmp_path / "MEASURED_PEAKS.json").unlink()
    assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    monkeypatch.undo()
    rec = bench.TRAFFIC_PER_LAYER
    assert bench.measured_traffic(20) in (20 * rec["bytes"], None)
    monkeypatch.setattr(bench, "TRAFFIC_PER_LAYER", dict(rec, sources_sha256_16="0" * 16))
    assert bench.measured_traffic(20) is None
