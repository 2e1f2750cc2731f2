#!/usr/bin/env python
"""Benchmark: local-Hessian NVFP4 weight-scale calibration of one synthetic layer per GPU.

One step = the whole hot path over one layer: Hessian accumulation (OVERWRITE), token
counts, finalisation, per-group global scale, and the exhaustive 126-candidate FP8 scale
sweep writing codes, fake-quantized weights and losses. Inputs are resident in HBM when
the timed region starts; each step's inputs (X and W together) exceed the 126 MB L2 for
every bench workload, so no L2 flush runs between steps.

e2e: the same step through calibrate_host from pinned host buffers, inputs copied in and
the result (codes and losses) copied out every step. The activation-aware workload also
reports the two-tensor accumulation (X_q resident) beside its fused step.

  python bench.py [--gpus N --steps K --warmup W --workload dense|act|wmse|moe]
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
WORKLOAD_TEXT = {
    "dense": "dense projection local_hessian: X bf16 [16384,4096] (lognormal column std, 1% outliers x20), "
             "W bf16 [4096,4096], full 16x16 H per block, 126-candidate FP8 sweep",
    "act": "activation-aware gate_up: X bf16 [32768,4096] through the fused NVFP4 input quantizer (X_q derived "
           "in the kernel; its global scale calibrated beforehand), W bf16 [12288,4096], H and P, cross term",
    "wmse": "WMSE down_proj: X bf16 [65536,12288], W bf16 [4096,12288], diagonal Imp [768,16]",
    "moe": "fused-MoE gate_up: 512 experts, X bf16 [16384,2560] top-10 routed, W bf16 [512,1280,2560], "
           "grouped full H, per-expert global scale",
}
# dram__bytes_read.sum + dram__bytes_write.sum per launch, from one ncu capture of the current
# kernel on this workload (summaries in profiles/); workloads without a capture report null.
SWEEP_TRAFFIC_BYTES = {
    "dense": 33_938_176 + 30_059_264,    # sweep_tc_kernel, profiles/sweep_tc_kernel_dense.md
    "wmse": 101_393_408 + 167_207_936,   # sweep_diag_kernel, profiles/sweep_diag_kernel_wmse.md
}
ACCUM_TRAFFIC_BYTES = {
    "dense": 134_265_344 + 3_774_464,    # accum_mma_kernel (clusters), profiles/accum_mma_kernel_dense.md
    "act": 268_573_696 + 5_457_664,      # accum_mma_kernel (quantizer fused), profiles/accum_mma_kernel_act.md
    "wmse": 1_610_820_000 + 8_041_472,   # accum_diag_kernel (+ the partial reduction, not captured)
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


def oracle_sample_step(layer, frac_tokens: float, n_units: int, seed: int = 0):
    """Time the CPU oracle on a bounded sample; returns estimated seconds for the whole layer."""
    import numpy as np

    from oracle import lhcal_oracle as O
    from scale_calibration_lh_b200 import synth

    T = layer.tokens
    ts = max(1, int(T * frac_tokens))
    if layer.mode == "act" and "act_gx_oracle" not in layer.meta:
        layer.meta["act_gx_oracle"] = O.global_scale(synth.bf16_bits_to_f32(layer.x))
    t0 = time.perf_counter()
    if layer.token_ids is not None:
        # Grouped: the first groups' routed rows, about ts rows in total.
        off = layer.group_offsets
        gcount = int(np.searchsorted(off, ts, side="right")) - 1
        gcount = max(1, min(gcount, layer.groups))
        x32 = synth.bf16_bits_to_f32(layer.x)
        O.accumulate(layer.mode, x32, None, off[:gcount + 1], layer.token_ids[:off[gcount]])
        frac = gcount / layer.groups
    else:
        xs = synth.bf16_bits_to_f32(layer.x[:ts])
        # Activation-aware: the oracle derives X_q with the input quantizer's global scale,
        # computed once over the whole X before the timing starts.
        O.accumulate(layer.mode, xs, None, act_gx=layer.meta.get("act_gx_oracle"))
        frac = ts / T
    t_acc = (time.perf_counter() - t0) / frac
    rng = np.random.default_rng(seed)
    G, R, C = layer.groups, layer.rows, layer.cin
    nb = C // 16
    # Global scale: the first groups (at most 8), scaled to all groups.
    gs = min(G, 8)
    t0 = time.perf_counter()
    g = np.array([O.global_scale(synth.bf16_bits_to_f32(layer.w[e])) for e in range(gs)], np.float32)
    t_g = (time.perf_counter() - t0) * G / gs
    # Sweep: n_units random (row, block) units in one call, as a one-group layer of the sampled rows.
    rows = rng.integers(0, R, n_units)
    blks = rng.integers(0, nb, n_units)
    grp = rng.integers(0, gs, n_units)
    w_s = synth.bf16_bits_to_f32(layer.w[grp, rows])[None]  # [1, U, C]
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

def run_reference(args, rank, world):
    """The CPU oracle (the deliberately slow reference program) on a bounded sample per step."""
    if rank != 0:
        return
    from scale_calibration_lh_b200 import synth

    layer = synth.make_layer(args.workload, 0)
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
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"per step: accumulation over {sample['tokens']} tokens and the sweep of "
                                   f"{n_units} random units, each scaled to the whole layer"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_lhcal(args, rank, world, local_rank):
    import numpy as np
    import torch

    import scale_calibration_lh_b200 as L
    from scale_calibration_lh_b200 import build as B
    from scale_calibration_lh_b200 import synth
    from tests import parity as P

    B.build()
    L.load_library()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = world > 1
    layer = synth.make_layer(args.workload, rank, rows=args.rows)
    d = P.layer_to_device(layer, dev)
    mode = L.MODE_IDS[layer.mode]
    G, R, C, T = layer.groups, layer.rows, layer.cin, layer.tokens
    buf = L.Buffers(mode, T, C, R, G, L.BF16, dev)
    stream = torch.cuda.current_stream()
    act_gx = None
    if layer.mode == "act":
        # The input quantizer's global scale, fp32(amax|X| / 2688): calibrated once before the
        # capture (by max calibration in the pages' flow), so it is set up outside the timing.
        act_gx = torch.empty(1, dtype=torch.float32, device=dev)
        L.lhcal_global_scale(d["x"].view(1, T, C), act_gx)

    def step():
        L.calibrate(mode, d["x"], d["w"], xq=d["xq"], group_offsets=d["offs"], token_ids=d["ids"], buffers=buf,
                    act_gx=act_gx)

    def barrier():
        if dist:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-resident timed region, with per-stage events on the launching stream
    clocks = ClockSampler(torch.cuda.current_device())
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    L.lhcal_launch_count(reset=True)
    clocks.start()
    start.record(stream)
    for k in range(K):
        e = ev[k]
        e[0].record(stream)
        if act_gx is not None:
            L.lhcal_accumulate_act_quant(d["x"], buf.h, buf.p, act_gx, flags=L.ACCUM_OVERWRITE,
                                         workspace=buf.workspace)
        else:
            L.lhcal_accumulate(mode, d["x"], buf.h, xq=d["xq"], p=buf.p, group_offsets=d["offs"],
                               token_ids=d["ids"], flags=L.ACCUM_OVERWRITE, workspace=buf.workspace)
        e[1].record(stream)
        L.lhcal_count_tokens(buf.counts, tokens=T, group_offsets=d["offs"], flags=L.ACCUM_OVERWRITE)
        L.lhcal_finalize(mode, buf.counts, buf.h, p=buf.p)
        e[2].record(stream)
        L.lhcal_global_scale(d["w"], buf.g)
        e[3].record(stream)
        L.lhcal_scale_sweep(mode, d["w"], buf.h, buf.g, buf.codes, wq=buf.wq, loss=buf.loss, p=buf.p)
        e[4].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    launches = L.lhcal_launch_count()
    ms_total = start.elapsed_time(end)
    stage = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in ev])  # ms
    t_acc, t_fin, t_g, t_sweep = (float(v) for v in stage.mean(0))
    ms_total, t_acc, t_sweep = rank_max([ms_total, t_acc, t_sweep], dev)
    ms = ms_total / K
    units, ops, acc_bytes = algorithmic(layer)
    value = weak_scaling_value(units, world, ms)

    # ---- activation-aware: the two-tensor accumulation for comparison. When the capture records
    # X_q next to X (the input-quantizer hook), X_q is already in HBM and the accumulation reads
    # both. X_q is materialised once here, outside every timed region, and the kernel is timed
    # launch by launch; the step above (and its value) uses the fused path.
    two_tensor = None
    if act_gx is not None:
        xq_res = torch.empty_like(d["x"])
        L.lhcal_act_fake_quant(d["x"], act_gx, xq_res)
        torch.cuda.synchronize()
        K3 = max(3, min(K, 20))
        ev3 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K3)]
        for a3, b3 in ev3:
            a3.record(stream)
            L.lhcal_accumulate(mode, d["x"], buf.h, xq=xq_res, p=buf.p, flags=L.ACCUM_OVERWRITE,
                               workspace=buf.workspace)
            b3.record(stream)
        torch.cuda.synchronize()
        t3 = float(np.mean([a3.elapsed_time(b3) for a3, b3 in ev3]))
        (t3,) = rank_max([t3], dev)
        two_tensor = {"ms": t3, "bytes": 2 * T * C * 2 + 2 * C // 16 * 256 * 4, "launches": K3}
        del xq_res

    # ---- end to end through the public API from pinned host buffers
    hx = torch.empty(d["x"].shape, dtype=d["x"].dtype, pin_memory=True)
    hx.copy_(d["x"])
    hxq = None
    if d["xq"] is not None:
        hxq = torch.empty(d["xq"].shape, dtype=d["xq"].dtype, pin_memory=True)
        hxq.copy_(d["xq"])
    hw = torch.empty(d["w"].shape, dtype=d["w"].dtype, pin_memory=True)
    hw.copy_(d["w"])
    # The step's result read back: the codes (the chosen scales) and the winning losses; the
    # fake-quantized weights stay on the device (lhcal_apply_scales derives them from the codes).
    out_host = L.HostOutputs(buf, want_wq=False)
    hoffs = None if d["offs"] is None else d["offs"].cpu().pin_memory()
    hids = None if d["ids"] is None else d["ids"].cpu().pin_memory()
    K2 = max(3, min(K, 10))

    def e2e_step():
        L.calibrate_host(mode, hx, hw, buf, d, hxq=hxq, group_offsets=hoffs, token_ids=hids, out=out_host,
                         act_gx=act_gx)

    e2e_step()  # warm
    torch.cuda.synchronize()
    barrier()
    e2s, e2e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2s.record(stream)
    for _ in range(K2):
        e2e_step()
    e2e_.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e2s.elapsed_time(e2e_) / K2
    (ms_e2e,) = rank_max([ms_e2e], dev)
    h2d = sum(t.numel() * t.element_size() for t in (hx, hw, hxq, hoffs, hids) if t is not None)
    d2h = out_host.nbytes()

    if rank != 0:
        return
    hbm_gbs, sm_mhz, peak_src = load_peaks()
    peak_ops = N_SMS * FP32_LANES_PER_SM * sm_mhz * 1e6
    sweep_units = units
    achieved_ops = sweep_units * ops / (t_sweep / 1e3)
    traffic = SWEEP_TRAFFIC_BYTES.get(args.workload)
    achieved_gbs = acc_bytes / (t_acc / 1e3) / 1e9
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload], "name": args.workload, "tokens": T, "cin": C,
                   "rows": R, "groups": G, "mode": layer.mode, "input_dtype": layer.dtype,
                   "l2": "no flush: each step's inputs (X and W) exceed the 126 MB L2",
                   "parallelism": f"{world} independent layers, one per GPU (no collective)"},
        "roofline": {"kernel": "sweep_diag_kernel" if layer.mode == "diag" else "sweep_tc_kernel", "bound": "alu", "achieved": achieved_ops / 1e12,
                     "peak": peak_ops / 1e12, "unit": "Tops/s", "frac": achieved_ops / peak_ops,
                     "traffic": traffic,
                     "note": f"FP32 lane-ops of the direct method ({ops // 126}/candidate) over the measured sweep "
                             f"time; peak = {N_SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x {sm_mhz:.0f} MHz "
                             f"(max clock, {peak_src})"},
        "roofline_accum": {"kernel": "accumulate (incl. partial reduction)" + (
                               ", input quantizer fused" if act_gx is not None else ""), "bound": "hbm",
                           "achieved": achieved_gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": achieved_gbs / hbm_gbs,
                           "traffic": ACCUM_TRAFFIC_BYTES.get(args.workload), "bytes_per_step": acc_bytes,
                           "note": f"algorithmic bytes over the measured accumulation time; peak {peak_src}"},
        "stages_ms": {"accumulate": t_acc, "count_finalize": t_fin, "global_scale": t_g, "sweep": t_sweep},
        "e2e": {"value": weak_scaling_value(units, world, ms_e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if two_tensor is not None:
        gbs = two_tensor["bytes"] / (two_tensor["ms"] / 1e3) / 1e9
        out["accumulate_two_tensor"] = {
            "ms": two_tensor["ms"], "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": gbs / hbm_gbs,
            "note": "X and X_q both read (X_q materialised beforehand, as the input-quantizer hook provides it); "
                    f"mean of {two_tensor['launches']} launches timed one by one; not part of value"}
    if world == 1 and not args.no_cpu_baseline:
        est, sample = oracle_sample_step(layer, 1.0 / 16, 16384)
        cb_value = units / est
        out["cpu_baseline"] = {"value": cb_value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                               "sample": f"accumulation over {sample['tokens']} tokens and the sweep of "
                                         f"{sample['units']} random units, each scaled to the whole layer"}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lhcal", "reference"], default="lhcal")
    ap.add_argument("--workload", choices=list(WORKLOAD_TEXT), default="dense")
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
    if world > 1:
        import torch

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_lhcal(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch

            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
