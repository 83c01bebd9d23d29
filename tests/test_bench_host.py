"""Host logic of bench.py, on CPU: the replica aggregation across ranks (two
gloo processes), the reference arm (its JSON line on rank 0, silence on the
others), the algorithmic byte/FLOP counts behind the roofline fields, the
traffic lookup and the clock record."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(times[rank], torch.device("cpu"), world)
        out[rank] = (ms, bench.aggregate_value(16384, ms, world))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    times = [0.30, 0.45]
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, times, out), nprocs=world, join=True)
    for r in range(world):
        ms, value = out[r]
        assert ms == pytest.approx(0.45)
        assert value == pytest.approx(2 * 16384 / 0.45e-3)


def test_single_rank_aggregate():
    assert bench.max_over_ranks(0.3, torch.device("cpu"), 1) == 0.3
    assert bench.aggregate_value(1000, 2.0, 1) == pytest.approx(5e5)


def test_reference_arm_exits_quietly_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line():
    """Rank 0 of the reference arm prints one JSON line with the bench
    contract's keys: the oracle timed on the host cores, its own line doubling
    as cpu_baseline and e2e (no host-device copies)."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["steps"] == 1 and d["warmup"] == 1 and d["n_gpus"] == 1 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "prefill_bf16_B4_T4096_hk16_hv32_d128_C64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert "whole workload" in cb["sample"] and cb["cpu_model"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert abs(d["ms_per_step"] - 1e3 * 4 * 4096 / d["value"]) <= 1e-6 * d["ms_per_step"]


def test_roofline_counts():
    from linear_attention_sequence_sm_b200 import inputs as I
    # 6 d^2 + 3 C d + 2 C d / G at d = 128, C = 64, G = 2
    assert bench.USEFUL_FLOPS_PER_VHEAD_TOKEN == 131072
    w = I.prefill_bf16()
    # q + k (16 heads) and v + o (32 heads) in bf16, g and beta fp32, the final state fp32
    assert bench.prefill_bytes(w) == 16384 * (16 * 128 * 2 * 2 + 32 * 128 * 2 * 2 + 32 * 8) + 4 * 32 * 128 * 128 * 4
    assert bench.decode_bytes(I.decode_bf16()) == 1080098816


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    prof = tmp_path / "profiles"
    prof.mkdir()
    entry = {"k": {"source": "k.cu", "source_sha256": hashlib.sha256(b"kernel v1").hexdigest(),
                   "bytes_per_launch": 123}}
    (prof / "traffic.json").write_text(json.dumps(entry))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("k") == 123
    src.write_text("kernel v2")
    assert bench.kernel_traffic("k") is None
    assert bench.kernel_traffic("missing") is None


def test_clock_sampler_against_a_fake_nvml(monkeypatch):
    """The clock record of the bench line, from a fake NVML: the median SM
    clock, the maximum, and the clock-event reasons decoded from NVML's bit
    values (idle and applications-clock bits are not slowdowns and are not
    reported); without NVML the record is empty, not an error."""
    import types
    clocks = iter([1965, 1500, 1965, 1965, 1200])
    bits = iter([0x0, 0x4, 0x4 | 0x40, 0x1 | 0x2, 0x8 | 0x20])
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0, nvmlInit=lambda: None, nvmlDeviceGetHandleByIndex=lambda i: ("gpu", i),
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965, nvmlDeviceGetClockInfo=lambda h, c: next(clocks),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: next(bits))
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    cs = bench.ClockSampler(0)
    for _ in range(5):
        cs._sample()
    s = cs.summary()
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["samples"] == 5
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap", "sw_thermal_slowdown"]

    def no_nvml():
        raise RuntimeError("no driver")

    monkeypatch.setitem(sys.modules, "pynvml", types.SimpleNamespace(nvmlInit=no_nvml))
    empty = bench.ClockSampler(0)
    with empty:
        pass
    assert empty.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_cpu_baseline_times_the_whole_workload():
    """The GPU arm's CPU baseline runs the same oracle pass as the reference
    arm: the whole workload, no extrapolation; tokens/s = tokens / seconds per
    pass."""
    from linear_attention_sequence_sm_b200 import inputs as I
    w = I.custom("cpu_base", batch=2, seq_len=256, hk=2, hv=4, d=32, chunk=64, dtype="bf16", seed=5)
    cb = bench.cpu_baseline(w, I.make_prefill_inputs(w), target_s=0.0)
    assert cb["kind"] == "oracle" and "not extrapolated" in cb["sample"] and "all 8" in cb["sample"]
    assert cb["value"] == pytest.approx(w.total_tokens / cb["seconds_per_pass"])
