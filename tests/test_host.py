"""Host-side consistency: the binding's constants against the header, and the
bench's use of recorded DRAM traffic."""
import json
import os
import re
import sys

import pytest

from mixture_experts_layer_64_b200 import lmoe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lmoe.h")


def header_defines():
    text = open(HEADER).read()
    return {m.group(1): int(m.group(2), 0)
            for m in re.finditer(r"^#define\s+LMOE_(\w+)\s+(0x[0-9a-fA-F]+|\d+)u?\b", text, re.M)}


def test_binding_flags_and_limits_match_the_header():
    defs = header_defines()
    flags = {k: v for k, v in defs.items()
             if k in ("SKIP_PROJ", "DEBUG_CHECKS", "FORCE_SIMT", "FORCE_SWAP", "FORCE_NOSWAP",
                      "FORCE_NOPAIR", "FORCE_WS_PAIR", "ROUTE_FULL_SOFTMAX", "ROUTE_BIAS_SELECT",
                      "EXPERTS_FP8", "SINGLE_STREAM", "NO_PDL", "LOAD_SPLIT",
                      "NO_STREAM_K", "SORTED_ROWS", "EXPERTS_FP4", "FC2_SPLIT")}
    assert len(flags) == 17, sorted(flags)
    for name, value in flags.items():
        assert getattr(lmoe, name) == value, name
    # flags are distinct single bits
    assert len(set(flags.values())) == len(flags)
    assert all(v & (v - 1) == 0 for v in flags.values())
    assert lmoe.MAX_EXPERTS == defs["MAX_EXPERTS"] and lmoe.MAX_TOPK == defs["MAX_TOPK"]
    assert lmoe.DEVERR_WAIT_TIMEOUT == defs["DEVERR_WAIT_TIMEOUT"]
    assert lmoe.DEVERR_RANGE == defs["DEVERR_RANGE"]
    assert lmoe.DEVERR_NONFINITE == defs["DEVERR_NONFINITE"]


def test_binding_stage_ids_match_the_header():
    text = open(HEADER).read()
    enum = {m.group(1).lower(): int(m.group(2))
            for m in re.finditer(r"LMOE_STAGE_(\w+)\s*=\s*(\d+)", text)}
    assert enum == lmoe.STAGES


def test_recorded_traffic_is_used_only_on_the_captured_sources(monkeypatch):
    import bench

    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        recorded = json.load(fh)
    entries = [(wl, st, rec) for wl, stages in recorded.items() if not wl.startswith("_")
               for st, rec in stages.items()]
    assert entries
    for wl, st, rec in entries:
        assert rec["dram_bytes_per_launch"] > 0 and os.path.exists(os.path.join(ROOT, rec["source"]))
        monkeypatch.setattr(bench, "kernel_source_hash", lambda stage, h=rec["kernel_sources"]: h)
        assert bench.recorded_traffic(wl, st) == rec["dram_bytes_per_launch"]
        monkeypatch.setattr(bench, "kernel_source_hash", lambda stage: "0" * 16)
        assert bench.recorded_traffic(wl, st) is None
    assert bench.recorded_traffic("no-such-workload", "expert_fc1") is None


def test_variant_sweep_costs_follow_the_paper():
    """The sweep's cost columns for the paper's variants (LatentMoE, Section 3,
    Table 1): per token, l-MoE_eff activates 1/alpha of the standard layer's
    expert weight bytes and dispatches 1/alpha of its bytes at 1/alpha of its
    expert FLOPs; l-MoE_acc matches the standard layer in all three."""
    import bench
    from mixture_experts_layer_64_b200 import workloads

    for batch, *names in workloads.VARIANT_SWEEP:
        pts = []
        for variant, name in zip(("standard", "l-MoE_eff", "l-MoE_acc"), names):
            w = workloads.WORKLOADS[name]
            r = {"w": w, "expert_loads": {"touched": w.N}, "value": 1.0, "ms_per_step": 1.0,
                 "stage_ms": {"expert_fc1": {"p50": 0.5}, "expert_fc2": {"p50": 0.25}}}
            pts.append(bench.sweep_point(variant, r))
        out = bench.variant_sweep(pts)["points"]
        alpha = out[0]["d"] / out[1]["l"]
        assert alpha == 4
        for key in ("active_weight_bytes_per_token", "dispatch_bytes_per_token",
                    "expert_flops_per_token"):
            assert out[0]["vs_standard"][key] == 1.0
            assert out[1]["vs_standard"][key] == 1 / alpha, (batch, key)
            assert out[2]["vs_standard"][key] == 1.0, (batch, key)
        # every expert touched: all three load the same expert set (alpha N
        # experts of 1 / alpha the size)
        assert [p["vs_standard"]["expert_weight_bytes"] for p in out] == [1.0, 1.0, 1.0]
        assert out[1]["N"] == out[2]["N"] == alpha * out[0]["N"]
        assert out[2]["k"] == alpha * out[1]["k"] == alpha * out[0]["k"]


def test_clock_sampler_reads_nvml_in_a_thread(monkeypatch):
    """The bench's clock record from a fake NVML (read-only queries): the
    median SM clock of the samples under load (the top half by power), the
    maximum clock, and the throttle reasons active under load by name."""
    import time
    import types
    import bench

    fake = types.ModuleType("pynvml")
    fake.NVMLError = type("NVMLError", (Exception,), {})
    fake.NVML_CLOCK_SM = 1
    fake.nvmlClocksEventReasonSwPowerCap = 0x4
    fake.nvmlClocksEventReasonHwSlowdown = 0x8
    fake.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    fake.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    state = {"n": 0}

    def clock(h, kind):
        state["n"] += 1
        return 1800 if state["n"] % 2 else 1965  # alternating samples

    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByUUID = lambda u: ("uuid", u)
    fake.nvmlDeviceGetHandleByIndex = lambda i: ("index", i)
    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    # power follows the clock: the 1965 MHz samples are the loaded ones
    fake.nvmlDeviceGetPowerUsage = lambda h: 900000 if state["n"] % 2 == 0 else 300000
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 if state["n"] % 2 == 0 else 0x0
    monkeypatch.setitem(sys.modules, "pynvml", fake)

    s = bench.ClockSampler(0, None, "00000000-0000-0000-0000-000000000000")
    s.start()
    time.sleep(0.15)
    rec = s.stop()
    assert rec["source"] == "nvml"
    assert rec["samples"] >= 3 and rec["samples_under_load"] == max(1, rec["samples"] // 2)
    assert rec["sm_max_mhz"] == 1965
    assert rec["sm_mhz"] == 1965 and rec["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvml_or_nvidia_smi(monkeypatch, tmp_path):
    """Without NVML the sampler falls back to the nvidia-smi query loop; if
    that command is missing too, the record is None (and start/stop neither
    raise nor wait long)."""
    import time
    import bench

    monkeypatch.setitem(sys.modules, "pynvml", None)  # import pynvml raises ImportError
    monkeypatch.setenv("PATH", str(tmp_path))          # no nvidia-smi on the path
    s = bench.ClockSampler(0, str(tmp_path / "clocks.csv"))
    t0 = time.time()
    s.start()
    rec = s.stop()
    assert rec is None and time.time() - t0 < 5.0
