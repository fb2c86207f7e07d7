"""CPU tests of bench.py's clock record (no GPU needed).

bench.py samples the SM clock and the clock-event reasons through NVML while
its timed region runs, reads only, and reports the median clock and every
reason seen.  Here NVML is a fake module with scripted readings; the reason
bits are checked against the installed NVML binding's named constants; and
two gloo ranks check the whole-job record (slowest rank's clock, reasons of
any rank).
"""
from __future__ import annotations

import multiprocessing as mp
import os
import socket
import sys
import time
import types

import pytest

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def fake_nvml(clocks, reasons, fail_init=False, old_name=False):
    """A stand-in for pynvml: device i has UUID "GPU-fake-i"; the SM clock
    and the reason word step through the given lists (then repeat the last
    value).  Records every call that is not a read."""
    it = {"clock": iter(clocks), "reason": iter(reasons)}
    last = {"clock": clocks[-1], "reason": reasons[-1]}
    writes = []

    def step(kind):
        try:
            last[kind] = next(it[kind])
        except StopIteration:
            pass
        return last[kind]

    def init():
        if fail_init:
            raise RuntimeError("NVML unavailable")

    nv = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=init,
        nvmlDeviceGetCount=lambda: 2,
        nvmlDeviceGetHandleByIndex=lambda i: ("handle", i),
        nvmlDeviceGetUUID=lambda h: f"GPU-fake-{h[1]}",
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
        nvmlDeviceGetClockInfo=lambda h, kind: step("clock"),
        writes=writes,
    )
    getter = lambda h: step("reason")  # noqa: E731
    if old_name:
        nv.nvmlDeviceGetCurrentClocksThrottleReasons = getter
    else:
        nv.nvmlDeviceGetCurrentClocksEventReasons = getter
    for name in ("nvmlDeviceSetGpuLockedClocks", "nvmlDeviceResetGpuLockedClocks",
                 "nvmlDeviceSetPowerManagementLimit", "nvmlDeviceSetApplicationsClocks"):
        setattr(nv, name, lambda *a, _n=name: writes.append(_n))
    return nv


def sample(monkeypatch, nv, seconds=0.08):
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    s = bench.ClockSampler(0, period_s=0.002)
    with s:
        time.sleep(seconds)
    n = len(s.samples)
    time.sleep(0.02)
    assert len(s.samples) == n, "sampling went on after the timed region"
    return s.summary()


def test_reason_bits_are_nvml_named_constants():
    pynvml = pytest.importorskip("pynvml")
    names = {"sw_power_cap": "SwPowerCap", "hw_slowdown": "HwSlowdown",
             "sw_thermal_slowdown": "SwThermalSlowdown",
             "hw_thermal_slowdown": "HwThermalSlowdown",
             "hw_power_brake_slowdown": "HwPowerBrakeSlowdown"}
    for bit, name in bench.ClockSampler.REASONS.items():
        const = getattr(pynvml, "nvmlClocksEventReason" + names[name], None)
        if const is None:
            const = getattr(pynvml, "nvmlClocksThrottleReason" + names[name])
        assert const == bit, name


def test_median_clock_and_reasons_seen(monkeypatch):
    clocks = [1965, 1965, 1800, 1650, 1965]
    # 0x4 power cap; 0x10 (sync boost) and 0x1 (idle) are not throttle reasons
    reasons = [0x0, 0x4, 0x10, 0x1, 0x0]
    nv = fake_nvml(clocks, reasons)
    got = sample(monkeypatch, nv)
    assert got["samples"] >= 5
    assert got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"]
    assert got["sm_mhz"] == 1965  # most samples repeat the last value
    assert nv.writes == [], "the sampler changed a GPU setting"


def test_throttle_reasons_are_all_reported(monkeypatch):
    nv = fake_nvml([1200], [0x8 | 0x40, 0x20, 0x80, 0x0], old_name=True)
    got = sample(monkeypatch, nv)
    assert got["reasons"] == ["hw_power_brake_slowdown", "hw_slowdown", "hw_thermal_slowdown",
                              "sw_thermal_slowdown"]
    assert got["sm_mhz"] == 1200


def test_no_nvml_gives_an_empty_record(monkeypatch):
    got = sample(monkeypatch, fake_nvml([1965], [0], fail_init=True))
    assert got == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_single_rank_record_is_unchanged():
    rec = {"sm_mhz": 1900, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 7}
    assert bench.clocks_over_ranks(rec, 1) is rec


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench as b

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = [{"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 10},
                {"sm_mhz": 1500, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"], "samples": 8},
                {"sm_mhz": None, "sm_max_mhz": 1965, "reasons": [], "samples": 0}][rank]
        q.put((rank, b.clocks_over_ranks(mine, world)))
    finally:
        dist.destroy_process_group()


def test_three_gloo_ranks_report_the_slowest_clock_and_every_reason():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted((q.get(timeout=10) for _ in range(3)), key=lambda x: x[0])
    for rank, rec in res:
        assert rec == {"sm_mhz": 1500, "sm_max_mhz": 1965,
                       "reasons": ["hw_slowdown", "sw_power_cap"], "samples": 18,
                       "per_rank_sm_mhz": [1965, 1500, None]}, rank
