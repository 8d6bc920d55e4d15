"""Host logic of bench.py that needs no GPU: the clock sampler against a fake
NVML (device matched by PCI address, reasons named from NVML's bits)."""
import os
import sys
import time
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _fake_nvml(reason_bits):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    for k, b in dict(GpuIdle=0x1, ApplicationsClocksSetting=0x2, SwPowerCap=0x4, HwSlowdown=0x8,
                     SyncBoost=0x10, SwThermalSlowdown=0x20, HwThermalSlowdown=0x40,
                     HwPowerBrakeSlowdown=0x80, DisplayClockSetting=0x100).items():
        setattr(nv, "nvmlClocksEventReason" + k, b)
    pcis = [types.SimpleNamespace(domain=0, bus=0x18, device=0), types.SimpleNamespace(domain=0, bus=0x2a, device=0)]
    calls = {"shutdown": 0}
    nv.nvmlInit = lambda: None
    nv.nvmlShutdown = lambda: calls.__setitem__("shutdown", calls["shutdown"] + 1)
    nv.nvmlDeviceGetCount = lambda: len(pcis)
    nv.nvmlDeviceGetHandleByIndex = lambda i: i
    nv.nvmlDeviceGetPciInfo = lambda h: pcis[h]
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    nv.nvmlDeviceGetClockInfo = lambda h, c: 1965 if h == 1 else 300      # only the matched GPU is busy
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reason_bits if h == 1 else 0x1
    nv.nvmlDeviceGetPowerUsage = lambda h: 700_000
    return nv, calls


@pytest.mark.parametrize("bits,want", [(0x0, []), (0x1, []), (0x4, ["sw_power_cap"]),
                                       (0x10, ["sync_boost"]), (0x20, ["sw_thermal_slowdown"]),
                                       (0x48, ["hw_slowdown", "hw_thermal_slowdown"])])
def test_clock_sampler_matches_by_pci_and_names_reasons(monkeypatch, bits, want):
    import bench
    nv, calls = _fake_nvml(bits)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x2a, pci_device_id=0)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: props)
    with bench.ClockSampler(0) as clk:
        time.sleep(0.02)
    s = clk.summary()
    assert s["samples"] >= 2
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["power_w"] == 700.0
    assert s["reasons"] == want
    assert calls["shutdown"] == 1


def test_clock_sampler_without_nvml_reports_why(monkeypatch):
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", None)         # import fails
    with bench.ClockSampler(0) as clk:
        pass
    s = clk.summary()
    assert "error" in s and "sm_mhz" not in s


def test_backward_flops_counts_visible_pairs():
    """A 3-block sequence, block size 4, D = 2: query block 0 selects only
    itself (10 pairs), block 1 nothing, block 2 selects block 0 (remote: 16
    pairs), block 5 (past it: nothing) and itself (10 pairs).  Four products
    of 2*D flops per pair."""
    import numpy as np
    import bench
    sel = np.array([[[[-1, -1, 0], [-1, -1, -1], [0, 5, 2]]]])       # [B=1, Hq=1, nb=3, nsel=3]
    assert bench.backward_flops(sel, 4, 2) == 8 * 2 * (10 + 16 + 10)


def test_loglog_exponent_of_power_laws():
    import bench
    S = [4096, 8192, 16384, 32768]
    assert abs(bench.loglog_exponent(S, [3e-3 * x for x in S]) - 1.0) < 1e-12
    assert abs(bench.loglog_exponent(S, [2.0 * x ** 1.5 for x in S]) - 1.5) < 1e-12


def test_oracle_index_route_timing_runs_on_a_small_workload():
    import bench
    from workloads import scaling
    t = bench.oracle_route_seconds(scaling(4096), 0, 2)
    assert len(t) == 2 and min(t) > 0


def test_forward_bytes_follow_the_byte_model():
    """Summary pass: q and k read once; attention: q read, K and V of every
    valid selected block gathered, output written (per route)."""
    import bench
    from workloads import SCALING_32K as w
    by = bench.forward_bytes(w, 23803, 2)
    assert by["summaries"] == (8 + 8) * 32768 * 128 * 2
    assert by["attention"] == 8 * 512 * 2 * 64 * 128 * 2 + 23803 * 64 * 2 * 128 * 2 == 914194432
    assert by["path"] == by["summaries"] + by["attention"]


def test_gqa_union_counts_distinct_blocks_per_group():
    """Two query heads per KV head: head 0 selects {0, 2}, head 1 selects
    {2, 3} for query block 3 -> union 3 of 4; -1 pads count in neither."""
    import types
    import bench
    w = types.SimpleNamespace(B=1, Hq=2, Hkv=1, nb=4, R=2, L=1)
    sel = torch.full((1, 2, 4, 3), -1, dtype=torch.int32)
    sel[0, 0, 3] = torch.tensor([0, 2, 3])
    sel[0, 1, 3] = torch.tensor([2, -1, 3])
    sel[0, 0, 0, 2] = 0
    sel[0, 1, 0, 2] = 0
    u = bench.gqa_union(sel, w)
    assert u == {"group_size": 2, "per_head_blocks": 7, "union_blocks": 4, "union_fraction": 4 / 7}


def test_cpu_baseline_reports_each_thread_setting(monkeypatch):
    import bench
    from workloads import TINY
    seen = []
    monkeypatch.setattr(bench, "oracle_sample", lambda w, seed, max_seconds: (seen.append(1) or (100.0, 0.1, 1)))
    monkeypatch.setattr(os, "cpu_count", lambda: 16)
    c = bench.cpu_baseline(TINY, 3.0)
    assert sorted(c["by_threads"], key=int) == ["1", "4", "16"] and len(seen) == 3
    assert c["cores"] == 16 and c["kind"] == "oracle" and c["value"] == 100.0


def test_reference_arm_prints_whole_steps(monkeypatch, capsys):
    """Each step of the reference arm is one whole forward (every KV-head
    group) when warm-up + steps fit the budget, else a scaled sample."""
    import argparse
    import json
    import bench
    from workloads import TINY
    calls = []
    monkeypatch.setattr(bench, "oracle_group_seconds", lambda w, inp, h: (calls.append(h) or 0.5))
    args = argparse.Namespace(gpus=1, steps=3, warmup=1)
    bench.run_reference(args, TINY)
    line = json.loads(capsys.readouterr().out)
    assert line["impl"] == "reference" and line["ms_per_step"] == 500.0 and "whole forward" in line["cpu_baseline"]["sample"]
    monkeypatch.setattr(bench, "REF_BUDGET_S", 1.0)
    bench.run_reference(args, TINY.with_(Hq=8, Hkv=8))
    line = json.loads(capsys.readouterr().out)
    assert "scaled" in line["cpu_baseline"]["sample"] and line["ms_per_step"] == 8 * 500.0
