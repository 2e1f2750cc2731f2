"""bench.py's host logic, without a GPU.

- The roofline numerators at the workloads' full sizes. The units, sweep instructions and
  accumulation bytes that the bench divides by its measured times are checked against
  figures worked out by hand from the shapes, so a change to the shapes or to the byte
  accounting cannot move a reported fraction unnoticed. The layers are shape-only stand-ins
  (nothing is generated), since the formula reads only sizes and routing.
- The reference arm's JSON line, and the silence of its non-zero ranks.
- The clock sampler, against a fake NVML (it only reads).
"""
import types

import numpy as np
import pytest

import bench
from scale_calibration_lh_b200 import synth


def _shape_only(name):
    tokens, cin, rows, groups = synth.FULL_SIZES[name]
    routed = groups > 1
    return types.SimpleNamespace(
        tokens=tokens, cin=cin, rows=rows, groups=groups, mode=synth.MODES[name],
        dtype="f32" if name == "tiny" else "bf16",
        token_ids=np.empty(tokens * synth.MOE_TOP_K, np.int32) if routed else None,
        group_offsets=np.empty(groups + 1, np.int32) if routed else None)


# name: (units, FP32 instructions per unit, accumulation bytes). Units = groups x rows x cin/16.
# Per candidate: 136 FMA for the symmetric 16x16 quadratic (80 is the diagonal form's 32), 48 for
# scale, dequantise and subtract, 16 for the cross term; times 126 candidates. Bytes: X once
# (bf16, or fp32 for the tiny layer), each statistic written once (16x16 or 16 fp32 per block
# and group), plus the CSR routing for the grouped layer. The activation-aware layer reads X
# alone, its X_q being derived in the kernel, and writes H and P.
EXPECTED = {
    "tiny": (32 * 4, 126 * 184, 256 * 64 * 4 + 4 * 1024),
    "dense": (4096 * 256, 126 * 184, 16384 * 4096 * 2 + 256 * 1024),
    "act": (12288 * 256, 126 * 200, 32768 * 4096 * 2 + 2 * 256 * 1024),
    "wmse": (4096 * 768, 126 * 80, 65536 * 12288 * 2 + 768 * 64),
    "moe": (512 * 1280 * 160, 126 * 184, 16384 * 2560 * 2 + 512 * 160 * 1024 + 163840 * 4 + 513 * 4),
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_roofline_numerators_at_full_size(name):
    assert bench.algorithmic(_shape_only(name)) == EXPECTED[name]


def test_numerators_in_the_units_quoted_for_each_workload():
    # Per-workload figures as quoted: 1.05 M / 3.15 M / 3.15 M / 104.9 M units; 134.5 MB,
    # 1.611 GB and 168.4 MB of accumulation traffic (the activation-aware figure is X alone).
    u, _, b = bench.algorithmic(_shape_only("dense"))
    assert (u, b) == (1_048_576, 134_479_872)
    u, _, b = bench.algorithmic(_shape_only("wmse"))
    assert (u, b) == (3_145_728, 1_610_661_888)
    u, _, b = bench.algorithmic(_shape_only("moe"))
    assert (u, b) == (104_857_600, 168_429_572)
    u, _, b = bench.algorithmic(_shape_only("act"))
    assert (u, b) == (3_145_728, 268_959_744)


def _run_bench(args, env_extra=None):
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, capture_output=True, text=True,
                          timeout=600, cwd=root, env=env)


def test_reference_arm_prints_one_contract_line():
    """The reference arm times the oracle on a bounded sample and prints one JSON line with the
    keys the benchmark contract names, in the native arm's metric and unit."""
    import json

    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["vs_baseline"] is None
    assert d["dtype"] == "f64" and d["data"] == "synthetic" and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "3"],
                   {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0 and "warmup" in r.stderr


def _fake_nvml(clocks, reasons, seen, fail=False):
    import itertools

    ck, rs = itertools.cycle(clocks), itertools.cycle(reasons)

    def init():
        if fail:
            raise RuntimeError("driver not loaded")

    def handle(i):
        seen.append(i)
        return ("handle", i)

    return types.SimpleNamespace(
        NVML_CLOCK_SM=0, nvmlInit=init, nvmlDeviceGetHandleByIndex=handle,
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: next(ck),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: next(rs),
        nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonHwThermalSlowdown=0x40,
        nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonHwPowerBrakeSlowdown=0x80,
        nvmlClocksEventReasonSwPowerCap=0x4)


def _sample(sampler, n=12):
    import time

    sampler.start()
    t0 = time.time()
    while len(sampler.samples) < n and time.time() - t0 < 10:
        time.sleep(0.005)
    return sampler.stop()


def test_clock_sampler_reports_median_clock_and_decoded_reasons(monkeypatch):
    """Read-only NVML polling, checked against a fake NVML: median and minimum SM clock, the
    union of the active reasons by name, and the physical index behind CUDA_VISIBLE_DEVICES."""
    import sys

    seen = []
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1800, 1965, 1965], [0x4, 0x0, 0x4 | 0x8], seen))
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5")
    out = _sample(bench.ClockSampler(1, period_s=0.001))
    assert seen == [5]
    assert out["sm_mhz"] == 1965 and out["sm_min_mhz"] == 1800 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"] and out["samples"] >= 12


def test_clock_sampler_without_nvml_says_so(monkeypatch):
    import sys

    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965], [0], [], fail=True))
    out = _sample(bench.ClockSampler(0), n=0)
    assert out["sm_mhz"] is None and out["reasons"][0].startswith("nvml unavailable")


def test_clock_reason_names_exist_in_the_installed_nvml_binding():
    pynvml = pytest.importorskip("pynvml")
    for _, const in bench.ClockSampler.REASONS:
        assert isinstance(getattr(pynvml, const, None), int), const
    assert callable(pynvml.nvmlDeviceGetCurrentClocksEventReasons)


def test_headline_is_the_largest_workload_and_all_run_by_default():
    """With no --workload every workload runs, and the line's headline is the one with the most
    sweep units (the fused-MoE layer), so the largest single-GPU configuration is the number."""
    import argparse

    units = {n: bench.algorithmic(_shape_only(n))[0] for n in synth.WORKLOADS}
    assert bench.HEADLINE == max(units, key=units.get) == "moe"
    assert tuple(bench.ORDER) == tuple(synth.WORKLOADS)
    assert bench.headline_name(argparse.Namespace(workload="all")) == "moe"
    assert bench.headline_name(argparse.Namespace(workload="dense")) == "dense"


def test_median_of_stage_times():
    assert bench.median([3, 1, 2]) == 2 and bench.median([4, 1, 3, 2]) == 2.5


def test_search_multipliers_are_the_stated_grid():
    # 38 multipliers 0.25 + 0.1 i: an amax range of 0.25x to 3.95x, ascending (so that the search's
    # first-best rule and the lowest-code rule agree).
    m = np.array(bench.SEARCH_MULTIPLIERS)
    assert len(m) == 38 and np.all(np.diff(m) > 0)
    np.testing.assert_allclose(m, 0.25 + 0.1 * np.arange(38))


def test_search_fractions_count_38_direct_evaluations_per_unit():
    # The multiplier search's numerator: units x 38 x the direct method's lane-ops per candidate.
    units = 1_048_576
    assert units * len(bench.SEARCH_MULTIPLIERS) * bench.OPS_PER_CANDIDATE["full"] == 7_331_643_392
