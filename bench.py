#!/usr/bin/env python
"""Benchmark: local-Hessian NVFP4 weight-scale calibration of synthetic layers, one per GPU.

One step = the whole hot path over one layer: Hessian accumulation (OVERWRITE), token
counts, finalisation, per-group global scale, and the exhaustive 126-candidate FP8 scale
sweep writing codes, fake-quantized weights and losses. Inputs are resident in HBM when
the timed region starts.

By default every workload runs, in the order tiny, dense, act, wmse, moe, each timed over
the same --steps after the same --warmup; the JSON line's headline (value, ms_per_step,
roofline, e2e, cpu_baseline) is the largest, the fused-MoE gate_up layer, and "workloads"
holds one record per workload. --workload NAME runs one.

Per workload:
  * the step loop, K steps back to back between two events (inputs above the 126 MB L2: no
    flush), or, when the inputs fit in L2 (the tiny layer), each step bracketed by its own
    events with an L2 flush between steps outside them; per-stage events give medians;
  * roofline: the sweep's FP32 lane-ops of the direct method over its median in-step time,
    against 148 SMs x 128 lanes x the max SM clock;
  * roofline_accum: the accumulation launched alone, max(20, K) times, each after a read of a
    256 MB buffer (which leaves the L2 clean and holding none of X), median of the event times;
    the in-step accumulation time is reported beside it;
  * e2e: the same path through calibrate_host from pinned host buffers, inputs copied in and
    the whole output copied out every step: codes, global scales, losses and the bf16
    fake-quantized weights; e2e_scales_only leaves the weights on the device;
  * cpu_baseline (rank 0, one GPU): the CPU oracle timed on a bounded sample.

  python bench.py [--gpus N --steps K --warmup W --workload all|tiny|dense|act|wmse|moe]
  python bench.py --impl reference ...   (the CPU oracle, timed on a bounded sample)

N > 1 runs under torchrun, one independent layer per rank (weak scaling, no collective
on the data path); the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "weight blocks swept/s (126 cand.); Hessian accum GB/s; % of roofline"
UNIT = "blocks/s"
# FP32 lane operations per (unit, candidate) of the direct method: symmetric quadratic
# (136 FMA) or diagonal (32) loss, plus scale-multiply, dequant-multiply and subtract per
# element (48), plus 16 for the cross term.
OPS_PER_CANDIDATE = {"full": 184, "act": 200, "diag": 80}
N_SMS = 148
FP32_LANES_PER_SM = 128
FALLBACK_HBM_GBS = 6650.0
FALLBACK_SM_MHZ = 1965.0
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024
ORDER = ("tiny", "dense", "act", "wmse", "moe")
HEADLINE = "moe"  # the largest workload: 104.9 M sweep units
WORKLOAD_TEXT = {
    "tiny": "tiny linear local_hessian: X fp32 [256,64] N(0,1), W fp32 [32,64] N(0,0.02), 4 blocks, full 16x16 H, "
            "126-candidate FP8 sweep (parity-sized; launch-latency-bound)",
    "dense": "dense projection local_hessian: X bf16 [16384,4096] (lognormal column std, 1% outliers x20), "
             "W bf16 [4096,4096], full 16x16 H per block, 126-candidate FP8 sweep",
    "act": "activation-aware gate_up: X bf16 [32768,4096] through the fused NVFP4 input quantizer (X_q derived "
           "in the kernel; its global scale calibrated beforehand), W bf16 [12288,4096], H and P, cross term",
    "wmse": "WMSE down_proj: X bf16 [65536,12288], W bf16 [4096,12288], diagonal Imp [768,16]",
    "moe": "fused-MoE gate_up: 512 experts, X bf16 [16384,2560] top-10 routed, W bf16 [512,1280,2560], "
           "grouped full H, per-expert global scale",
}
# dram__bytes_read.sum + dram__bytes_write.sum per launch from one ncu capture of the named
# kernel on the workload (the kernels as they are now), as committed with its summary; reported
# as traffic_from_profile, never as a measurement of the run (the bench cannot read DRAM
# counters). The fused-MoE sweep was captured with 128 rows per expert and is scaled to the
# 1280 rows of the workload (its traffic, W in and Wq out, grows with the rows).
PROFILED_TRAFFIC = {
    ("dense", "sweep_tc_kernel"): {"bytes": 33_956_352 + 28_585_216},
    ("act", "sweep_tc_kernel"): {"bytes": 101_255_168 + 177_749_248},
    ("moe", "sweep_tc_kernel"): {"bytes": 10 * (420_230_912 + 702_877_440), "scaled": "x10 from 128 rows per expert"},
    ("wmse", "sweep_diag_kernel"): {"bytes": 100_873_216 + 163_058_176},
    ("dense", "accum"): {"bytes": 134_267_904 + 3_960_064},
    ("act", "accum"): {"bytes": 268_599_552 + 3_796_736},
    ("moe", "accum"): {"bytes": 84_716_032 + 49_333_248},
    ("wmse", "accum"): {"bytes": 1_610_622_000 + 7_723_264, "note": "accum_diag_kernel only"},
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("sm_max_mhz", FALLBACK_SM_MHZ)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_SM_MHZ, "fallback"


def rank_max(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_scaling_value(units_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's step time."""
    return units_per_rank * world / (ms_per_step_max / 1e3)


def median(xs):
    s = sorted(float(x) for x in xs)
    n = len(s)
    return s[n // 2] if n % 2 else 0.5 * (s[n // 2 - 1] + s[n // 2])


# ------------------------------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls the SM clock and clock-event reasons (NVML, read-only) every 5 ms in a thread."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.device_index = device_index
        self.period_s = period_s
        self.samples = []
        self._stop = None
        self._thread = None
        self.error = None

    def start(self):
        import threading

        try:
            import pynvml

            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self.device_index
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if idx < len(ids) and ids[idx].isdigit():
                    idx = int(ids[idx])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.error = f"nvml unavailable: {e}"
            return
        self._stop = threading.Event()

        def poll():
            nv, h = self._nv, self._h
            while not self._stop.is_set():
                try:
                    self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                         nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception:
                    pass
                time.sleep(self.period_s)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "not sampled"]}
        self._stop.set()
        self._thread.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": ["no samples"]}
        sm = sorted(c for c, _ in self.samples)
        reasons = sorted({name for _, bits in self.samples for name, const in self.REASONS
                          if bits & getattr(self._nv, const, 0)})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.sm_max, "sm_min_mhz": sm[0], "reasons": reasons,
                "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------ helpers

def algorithmic(layer):
    """(units, sweep ops per unit, accumulation bytes) of one step on this layer."""
    G, R, C, T = layer.groups, layer.rows, layer.cin, layer.tokens
    nblk = C // 16
    units = G * R * nblk
    ops = 126 * OPS_PER_CANDIDATE[layer.mode]
    hsz = G * nblk * (16 if layer.mode == "diag" else 256) * 4
    xb = T * C * (4 if layer.dtype == "f32" else 2)
    if layer.mode == "act":  # X read once: X_q is derived from it inside the kernel
        acc_bytes = xb + 2 * hsz
    elif layer.token_ids is not None:
        acc_bytes = xb + hsz + layer.token_ids.nbytes + layer.group_offsets.nbytes
    else:
        acc_bytes = xb + hsz
    return units, ops, acc_bytes


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return 1


def _as_f32(a, layer):
    from scale_calibration_lh_b200 import synth

    return a if layer.dtype == "f32" else synth.bf16_bits_to_f32(a)


def oracle_sample_step(layer, frac_tokens: float, n_units: int, seed: int = 0):
    """Time the CPU oracle on a bounded sample; returns estimated seconds for the whole layer."""
    import numpy as np

    from oracle import lhcal_oracle as O

    T = layer.tokens
    ts = max(1, int(T * frac_tokens))
    if layer.mode == "act" and "act_gx_oracle" not in layer.meta:
        layer.meta["act_gx_oracle"] = O.global_scale(_as_f32(layer.x, layer))
    t0 = time.perf_counter()
    if layer.token_ids is not None:
        # Grouped: the first groups' routed rows, about ts rows in total.
        off = layer.group_offsets
        gcount = int(np.searchsorted(off, ts, side="right")) - 1
        gcount = max(1, min(gcount, layer.groups))
        x32 = _as_f32(layer.x, layer)
        O.accumulate(layer.mode, x32, None, off[:gcount + 1], layer.token_ids[:off[gcount]])
        frac = gcount / layer.groups
    else:
        xs = _as_f32(layer.x[:ts], layer)
        # Activation-aware: the oracle derives X_q with the input quantizer's global scale,
        # computed once over the whole X before the timing starts.
        O.accumulate(layer.mode, xs, None, act_gx=layer.meta.get("act_gx_oracle"))
        frac = ts / T
    t_acc = (time.perf_counter() - t0) / frac
    rng = np.random.default_rng(seed)
    G, R, C = layer.groups, layer.rows, layer.cin
    nb = C // 16
    n_units = min(n_units, 4 * G * R * nb)
    # Global scale: the first groups (at most 8), scaled to all groups.
    gs = min(G, 8)
    t0 = time.perf_counter()
    g = np.array([O.global_scale(_as_f32(layer.w[e], layer)) for e in range(gs)], np.float32)
    t_g = (time.perf_counter() - t0) * G / gs
    # Sweep: n_units random (row, block) units in one call, as a one-group layer of the sampled rows.
    rows = rng.integers(0, R, n_units)
    blks = rng.integers(0, nb, n_units)
    grp = rng.integers(0, gs, n_units)
    w_s = _as_f32(layer.w[grp, rows], layer)[None]  # [1, U, C]
    if layer.mode == "diag":
        h = np.abs(rng.normal(size=(1, nb, 16))) + 1.0
    else:
        a = rng.normal(size=(nb, 16, 16))
        h = (a @ a.transpose(0, 2, 1))[None] / 16
    p = (0.01 * rng.normal(size=h.shape)) if layer.mode == "act" else None
    units = np.stack([np.zeros(n_units, np.int64), np.arange(n_units), blks], 1)
    t1 = time.perf_counter()
    O.sweep(layer.mode, w_s, h, p, g[:1], units=units)
    t_sweep = (time.perf_counter() - t1) / n_units * (G * R * nb) + t_g
    return t_acc + t_sweep, {"tokens": ts if layer.token_ids is None else f"{frac:.4f} of groups", "units": n_units}


# ------------------------------------------------------------------------------------------ arms

def headline_name(args) -> str:
    return HEADLINE if args.workload == "all" else args.workload


def run_reference(args, rank, world):
    """The CPU oracle (the deliberately slow reference program) on a bounded sample per step, on
    the workload that the native arm's headline measures."""
    if rank != 0:
        return
    from scale_calibration_lh_b200 import synth

    name = headline_name(args)
    layer = synth.make_layer(name, 0)
    units, _, _ = algorithmic(layer)
    frac, n_units = 1.0 / 64, 512
    for _ in range(args.warmup):
        oracle_sample_step(layer, frac, 64)
    t = 0.0
    for s in range(args.steps):
        est, sample = oracle_sample_step(layer, frac, n_units, seed=s)
        t += est
    ms = t / args.steps * 1e3
    value = units / (ms / 1e3)
    cores = cpu_threads()
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_estimated": True, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[name], "name": name},
        "estimate": f"each step times the oracle on a sample (accumulation over {sample['tokens']} tokens, the "
                    f"sweep of {sample['units']} random units) and scales each stage to the whole layer",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"per step: accumulation over {sample['tokens']} tokens and the sweep of "
                                   f"{sample['units']} random units, each scaled to the whole layer"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


class L2Flush:
    """Reads a 256 MB device buffer: dirty L2 lines are written back on the way and the L2 is
    left holding clean lines of this buffer only (a read, not a write, so nothing stays dirty)."""

    def __init__(self, device):
        import torch

        self.buf = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self):
        self.buf.sum()


def measure_workload(name, args, rank, world, dev, flusher):
    """Time one workload as the module docstring describes; returns its record (rank 0's view,
    times already the maximum over ranks)."""
    import numpy as np
    import torch

    import scale_calibration_lh_b200 as L
    from scale_calibration_lh_b200 import synth

    dist = world > 1

    def barrier():
        if dist:
            torch.distributed.barrier()

    layer = synth.make_layer(name, rank, rows=args.rows)
    d = synth.layer_to_device(layer, dev)
    mode = L.MODE_IDS[layer.mode]
    G, R, C, T = layer.groups, layer.rows, layer.cin, layer.tokens
    xdt = L.BF16 if layer.dtype == "bf16" else L.F32
    buf = L.Buffers(mode, T, C, R, G, xdt, dev)
    stream = torch.cuda.current_stream()
    act_gx = None
    if layer.mode == "act":
        # The input quantizer's global scale, fp32(amax|X| / 2688): calibrated once before the
        # capture (by max calibration in the pages' flow), so it is set up outside the timing.
        act_gx = torch.empty(1, dtype=torch.float32, device=dev)
        L.lhcal_global_scale(d["x"].view(1, T, C), act_gx)

    def accumulate(b):
        if act_gx is not None:
            L.lhcal_accumulate_act_quant(d["x"], b.h, b.p, act_gx, flags=L.ACCUM_OVERWRITE, workspace=b.workspace)
        else:
            L.lhcal_accumulate(mode, d["x"], b.h, xq=d["xq"], p=b.p, group_offsets=d["offs"], token_ids=d["ids"],
                               flags=L.ACCUM_OVERWRITE, workspace=b.workspace)

    def step(e):
        e[0].record(stream)
        accumulate(buf)
        e[1].record(stream)
        L.lhcal_count_tokens(buf.counts, tokens=T, group_offsets=d["offs"], flags=L.ACCUM_OVERWRITE)
        L.lhcal_finalize(mode, buf.counts, buf.h, p=buf.p)
        e[2].record(stream)
        L.lhcal_global_scale(d["w"], buf.g)
        e[3].record(stream)
        L.lhcal_scale_sweep(mode, d["w"], buf.h, buf.g, buf.codes, wq=buf.wq, loss=buf.loss, p=buf.p)
        e[4].record(stream)

    def events(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    input_bytes = sum(t.numel() * t.element_size() for t in (d["x"], d["w"], d["offs"], d["ids"]) if t is not None)
    small = input_bytes < L2_BYTES
    K = args.steps
    for _ in range(args.warmup):
        if small:
            flusher()
        step(events(5))
    torch.cuda.synchronize()

    # ---- the step loop
    clocks = ClockSampler(torch.cuda.current_device())
    ev = [events(5) for _ in range(K)]
    start, end = events(2)
    barrier()
    torch.cuda.synchronize()
    L.lhcal_launch_count(reset=True)
    clocks.start()
    start.record(stream)
    for k in range(K):
        if small:
            flusher()  # outside the step's own events
        step(ev[k])
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    launches = L.lhcal_launch_count()
    ms_total = sum(e[0].elapsed_time(e[4]) for e in ev) if small else start.elapsed_time(end)
    stage = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in ev])  # ms
    med = [median(stage[:, i]) for i in range(4)]
    mean = [float(v) for v in stage.mean(0)]
    ms_total, t_acc_step, t_sweep = rank_max([ms_total, med[0], med[3]], dev)
    ms = ms_total / K
    units, ops, acc_bytes = algorithmic(layer)

    # ---- the accumulation alone, each launch after an L2 flush (median of max(20, K))
    reps = max(20, K)
    acc_ev = [events(2) for _ in range(reps)]
    torch.cuda.synchronize()
    for a, b in acc_ev:
        flusher()
        a.record(stream)
        accumulate(buf)
        b.record(stream)
    torch.cuda.synchronize()
    (t_acc,) = rank_max([median(a.elapsed_time(b) for a, b in acc_ev)], dev)

    # ---- activation-aware: the two-tensor accumulation for comparison. When the capture records
    # X_q next to X (the input-quantizer hook), X_q is already in HBM and the accumulation reads
    # both. X_q is materialised once here, outside every timed region; each launch is timed after
    # an L2 flush and the median taken, as above; the step (and its value) uses the fused path.
    two_tensor = None
    if act_gx is not None:
        xq_res = torch.empty_like(d["x"])
        L.lhcal_act_fake_quant(d["x"], act_gx, xq_res)
        torch.cuda.synchronize()
        ev3 = [events(2) for _ in range(reps)]
        for a3, b3 in ev3:
            flusher()
            a3.record(stream)
            L.lhcal_accumulate(mode, d["x"], buf.h, xq=xq_res, p=buf.p, flags=L.ACCUM_OVERWRITE,
                               workspace=buf.workspace)
            b3.record(stream)
        torch.cuda.synchronize()
        (t3,) = rank_max([median(a3.elapsed_time(b3) for a3, b3 in ev3)], dev)
        two_tensor = {"ms": t3, "bytes": 2 * T * C * 2 + 2 * C // 16 * 256 * 4, "launches": reps}
        del xq_res

    # ---- end to end through the public API from pinned host buffers
    def pinned(t):
        if t is None:
            return None
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    hx = hxq = hw = hoffs = hids = None
    e2e = {}
    if not args.no_e2e:
        hx, hxq, hw = pinned(d["x"]), pinned(d["xq"]), pinned(d["w"])
        hoffs, hids = pinned(d["offs"]), pinned(d["ids"])
    K2 = max(3, min(K, 10))
    for label, want_wq16 in (() if args.no_e2e else (("e2e", True), ("e2e_scales_only", False))):
        # The whole output: codes, global scales and losses, plus the bf16 fake-quantized weights
        # (lhcal_apply_scales of the chosen codes) unless the weights stay on the device.
        b2 = L.Buffers(mode, T, C, R, G, xdt, dev, want_wq=False, want_wq16=want_wq16)
        out_host = L.HostOutputs(b2, want_wq=False)

        def e2e_step():
            L.calibrate_host(mode, hx, hw, b2, d, hxq=hxq, group_offsets=hoffs, token_ids=hids, out=out_host,
                             act_gx=act_gx)

        e2e_step()  # warm
        torch.cuda.synchronize()
        barrier()
        e2s, e2e_end = events(2)
        e2s.record(stream)
        for _ in range(K2):
            e2e_step()
        e2e_end.record(stream)
        torch.cuda.synchronize()
        (ms_e2e,) = rank_max([e2s.elapsed_time(e2e_end) / K2], dev)
        h2d = sum(t.numel() * t.element_size() for t in (hx, hw, hxq, hoffs, hids) if t is not None)
        e2e[label] = {"value": weak_scaling_value(units, world, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": out_host.nbytes(), "ms_per_step": ms_e2e, "steps": K2,
                      "outputs": "codes, global scales, losses" + (", bf16 fake-quantized weights" if want_wq16
                                                                   else "; fake-quantized weights stay on the device")}
        del b2, out_host

    hbm_gbs, sm_mhz, peak_src = load_peaks()
    peak_ops = N_SMS * FP32_LANES_PER_SM * sm_mhz * 1e6
    achieved_ops = units * ops / (t_sweep / 1e3)
    achieved_gbs = acc_bytes / (t_acc / 1e3) / 1e9
    sweep_kernel = "sweep_diag_kernel" if layer.mode == "diag" else "sweep_tc_kernel"
    acc_kernel = {"diag": "accum_diag_kernel + reduce_partials_kernel"}.get(layer.mode, "accum_mma_kernel")
    if layer.dtype == "f32":
        acc_kernel = "accum_generic_kernel + reduce_partials_kernel"
    rec = {
        "name": name, "workload": WORKLOAD_TEXT[name], "tokens": T, "cin": C, "rows": R, "groups": G,
        "mode": layer.mode, "input_dtype": layer.dtype,
        "value": weak_scaling_value(units, world, ms), "unit": UNIT, "ms_per_step": ms, "steps": K,
        "units_per_step": units,
        "l2": ("inputs fit in the L2: an L2 flush between timed steps, outside each step's events" if small else
               f"no flush: each step's inputs ({input_bytes / 1e6:.0f} MB of X and W) exceed the 126 MB L2"),
        "stages_ms": dict(zip(("accumulate", "count_finalize", "global_scale", "sweep"), med)),
        "stages_ms_mean": dict(zip(("accumulate", "count_finalize", "global_scale", "sweep"), mean)),
        "roofline": {"kernel": sweep_kernel, "bound": "alu", "achieved": achieved_ops / 1e12,
                     "peak": peak_ops / 1e12, "unit": "Tops/s", "frac": achieved_ops / peak_ops, "traffic": None,
                     "traffic_from_profile": PROFILED_TRAFFIC.get((name, sweep_kernel)),
                     "note": f"FP32 lane-ops of the direct method ({ops // 126}/candidate) over the median in-step "
                             f"sweep time; peak = {N_SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x {sm_mhz:.0f} MHz "
                             f"(max clock, {peak_src})"},
        "roofline_accum": {"kernel": acc_kernel + (", input quantizer fused" if act_gx is not None else ""),
                           "bound": "hbm", "achieved": achieved_gbs, "peak": hbm_gbs, "unit": "GB/s",
                           "frac": achieved_gbs / hbm_gbs, "traffic": None,
                           "traffic_from_profile": PROFILED_TRAFFIC.get((name, "accum")),
                           "bytes_per_step": acc_bytes, "ms": t_acc, "in_step_ms": t_acc_step,
                           "in_step_frac": acc_bytes / (t_acc_step / 1e3) / 1e9 / hbm_gbs,
                           "note": f"algorithmic bytes over the median of {reps} launches, each after an L2 flush "
                                   f"(peak {peak_src}); in_step_ms is the same stage inside the step loop, where it "
                                   f"follows the previous step's sweep"},
        "gpu_launches": launches,
        "clocks": clk,
    }
    rec.update(e2e)
    rec["searches"] = measure_searches(L, mode, layer, d, buf, units, stream, dev, peak_ops, events, rank_max, flusher)
    if small:
        rec["latency_bound"] = True
    if two_tensor is not None:
        gbs = two_tensor["bytes"] / (two_tensor["ms"] / 1e3) / 1e9
        rec["accumulate_two_tensor"] = {
            "ms": two_tensor["ms"], "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
            "note": "X and X_q both read (X_q materialised beforehand, as the input-quantizer hook provides it); "
                    f"median of {two_tensor['launches']} launches, each after an L2 flush; not part of value"}
    if world == 1 and not args.no_cpu_baseline:
        est, sample = oracle_sample_step(layer, 1.0 / 16, 16384)
        rec["cpu_baseline"] = {"value": units / est, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                               "sample": f"accumulation over {sample['tokens']} tokens and the sweep of "
                                         f"{sample['units']} random units, each scaled to the whole layer"}
    del d, buf, hx, hxq, hw, hoffs, hids
    torch.cuda.empty_cache()
    return rec


# The amax-multiplier search's multipliers: the pages name a step size and multipliers but give no
# values, so the bench takes 38 of them, 0.25 + 0.1 i (an amax range of 0.25x to 3.95x).
SEARCH_MULTIPLIERS = [0.25 + 0.1 * i for i in range(38)]


def measure_searches(L, mode, layer, d, buf, units, stream, dev, peak_ops, events, rank_max, flusher):
    """The non-sweep searches on the workload's finalized statistics, timed alone: the
    amax-multiplier search in the workload's mode, and (one-group layers) the plain MSE sweep
    (H = I). Each is the median of 5 launches after one untimed launch and an L2 flush before
    each; the fraction is the FP32 lane peak against the direct method's lane-ops per evaluated
    scale (the search evaluates at most one scale per multiplier and skips repeated codes)."""
    import torch

    out = {}
    mult = torch.tensor(SEARCH_MULTIPLIERS, dtype=torch.float32, device=dev)
    codes = torch.empty_like(buf.codes)

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        evs = [events(2) for _ in range(reps)]
        for a, b in evs:
            flusher()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        (ms,) = rank_max([median(a.elapsed_time(b) for a, b in evs)], dev)
        return ms

    ms = timed(lambda: L.lhcal_multiplier_search(mode, d["w"], buf.h, buf.g, mult, codes, p=buf.p))
    ops = units * len(SEARCH_MULTIPLIERS) * OPS_PER_CANDIDATE[layer.mode]
    out["multiplier_search"] = {
        "kernel": "msearch_kernel", "mode": layer.mode, "multipliers": len(SEARCH_MULTIPLIERS), "ms": ms,
        "units_per_s": units / (ms / 1e3), "bound": "alu", "achieved": ops / (ms / 1e3) / 1e12,
        "peak": peak_ops / 1e12, "unit": "Tops/s", "frac": ops / (ms / 1e3) / peak_ops,
        "note": "multipliers 0.25 + 0.1 i, i < 38; outputs: codes only"}
    if layer.groups == 1 and layer.mode != "diag":
        g = torch.empty_like(buf.g)
        L.lhcal_global_scale(d["w"], g)
        ms2 = timed(lambda: L.lhcal_scale_sweep("mse", d["w"], None, g, codes))
        ops2 = units * 126 * OPS_PER_CANDIDATE["diag"]
        out["mse_sweep"] = {
            "kernel": "sweep_diag_kernel (importance 1)", "ms": ms2, "units_per_s": units / (ms2 / 1e3),
            "bound": "alu", "achieved": ops2 / (ms2 / 1e3) / 1e12, "peak": peak_ops / 1e12, "unit": "Tops/s",
            "frac": ops2 / (ms2 / 1e3) / peak_ops, "note": "126 candidates, H = I; outputs: codes only"}
    return out


def measure_sharded(name, args, rank, world, dev):
    """One layer shared by the ranks (scale_calibration_lh_b200.sharded): each rank accumulates its
    token shard, one all-reduce (SUM) of the raw statistics and counts, each rank finalizes and
    sweeps its row shard (the global scale is the all-reduce MAX of the shards'). A step is one
    such calibration without gathering the results; value = the layer's units over the slowest
    rank's step time (strong scaling)."""
    import torch

    import scale_calibration_lh_b200 as L
    from scale_calibration_lh_b200 import sharded as S
    from scale_calibration_lh_b200 import synth

    layer = synth.make_layer(name, 0, rows=args.rows)
    G, R, C, T = layer.groups, layer.rows, layer.cin, layer.tokens
    t0, t1 = S.token_range(T, rank, world)
    r0, r1 = S.row_range(R, rank, world)
    kind = "bf16" if layer.dtype == "bf16" else "f32"
    x = synth.to_device(layer.x[t0:t1], kind, dev)
    w = synth.to_device(layer.w[:, r0:r1], kind, dev)
    offs = ids = None
    if layer.group_offsets is not None:
        o, i = S.shard_routing(torch.from_numpy(layer.group_offsets), torch.from_numpy(layer.token_ids), t0, t1)
        offs, ids = o.to(dev), i.to(dev)
    mode = L.MODE_IDS[layer.mode]
    buf = L.Buffers(mode, t1 - t0, C, r1 - r0, G, L.BF16 if kind == "bf16" else L.F32, dev)
    act_gx = None
    if layer.mode == "act":  # the input quantizer's scale, calibrated once: MAX over the ranks' shards
        act_gx = torch.empty(1, dtype=torch.float32, device=dev)
        L.lhcal_global_scale(x.view(1, t1 - t0, C), act_gx)
        torch.distributed.all_reduce(act_gx, op=torch.distributed.ReduceOp.MAX)

    def step():
        S.calibrate_sharded(layer.mode, x, w, group_offsets=offs, token_ids=ids, act_gx=act_gx, buffers=buf,
                            gather=False)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.distributed.barrier()
    torch.cuda.synchronize()
    L.lhcal_launch_count(reset=True)
    clocks.start()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    torch.distributed.barrier()
    (ms_total,) = rank_max([start.elapsed_time(end)], dev)
    ms = ms_total / args.steps
    units, _, _ = algorithmic(layer)
    return {"name": name, "workload": WORKLOAD_TEXT[name], "tokens": T, "cin": C, "rows": R, "groups": G,
            "mode": layer.mode, "value": units / (ms / 1e3), "ms_per_step": ms, "units_per_step": units,
            "gpu_launches": L.lhcal_launch_count(), "clocks": clk,
            "shard": {"tokens": [t0, t1], "rows": [r0, r1]}}


def run_sharded(args, rank, world, local_rank):
    import torch

    import scale_calibration_lh_b200 as L
    from scale_calibration_lh_b200 import build as B

    B.build()
    L.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    rec = measure_sharded(headline_name(args), args, rank, world, dev)
    if rank != 0:
        return
    out = {
        "metric": METRIC, "value": rec["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": rec["workload"], "name": rec["name"], "tokens": rec["tokens"], "cin": rec["cin"],
                   "rows": rec["rows"], "groups": rec["groups"], "mode": rec["mode"],
                   "l2": "no flush: each rank's inputs exceed the 126 MB L2 at the full sizes",
                   "parallelism": f"one layer over {world} GPUs: tokens and rows sharded, NCCL all-reduce of "
                                  "the raw statistics and counts, MAX of the global scales"},
        "e2e": {"value": None, "unit": UNIT, "note": "not measured in the sharded mode"},
        "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"], "shard_of_rank0": rec["shard"],
    }
    print(json.dumps(out), flush=True)


def run_lhcal(args, rank, world, local_rank):
    import torch

    import scale_calibration_lh_b200 as L
    from scale_calibration_lh_b200 import build as B

    B.build()
    L.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    flusher = L2Flush(dev)
    names = ORDER if args.workload == "all" else (args.workload,)
    recs = {n: measure_workload(n, args, rank, world, dev, flusher) for n in names}
    if rank != 0:
        return
    head = recs[headline_name(args)]
    out = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": head["workload"], "name": head["name"], "tokens": head["tokens"], "cin": head["cin"],
                   "rows": head["rows"], "groups": head["groups"], "mode": head["mode"],
                   "input_dtype": head["input_dtype"], "l2": head["l2"],
                   "parallelism": f"{world} independent layers, one per GPU (no collective)",
                   "workloads_run": list(names)},
        "roofline": head["roofline"], "roofline_accum": head["roofline_accum"], "stages_ms": head["stages_ms"],
        "e2e": head.get("e2e", {"value": None, "unit": UNIT, "note": "not measured (--no-e2e)"}),
        "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
    }
    if "cpu_baseline" in head:
        out["cpu_baseline"] = head["cpu_baseline"]
    out["workloads"] = recs
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lhcal", "reference"], default="lhcal")
    ap.add_argument("--workload", choices=["all"] + list(ORDER), default="all")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--shard", action="store_true",
                    help="one layer sharded over the ranks (tokens and rows; strong scaling) instead of one "
                         "layer per rank; runs the headline workload or --workload")
    ap.add_argument("--rows", type=int, default=None,
                    help="weight rows per group instead of the workload's (smaller captures for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1 or args.shard:
        import torch

        torch.cuda.set_device(local_rank)
        if world == 1:  # one rank: a local store, no rendezvous
            torch.distributed.init_process_group("nccl", store=torch.distributed.HashStore(), rank=0, world_size=1,
                                                 device_id=torch.device("cuda", local_rank))
        else:
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                                 device_id=torch.device("cuda", local_rank))
    try:
        if args.shard:
            run_sharded(args, rank, world, local_rank)
        else:
            run_lhcal(args, rank, world, local_rank)
    finally:
        if world > 1 or args.shard:
            import torch

            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
