"""Comparators and device helpers shared by the GPU parity tests.

Tolerances (the parity bar for the GPU path):
  * Hessians H / P: relative Frobenius error per 16x16 block <= 1e-4; importance per block
    (16 values) <= 1e-4; an all-zero oracle block requires an exactly zero GPU block.
  * Sweep: codes and fake-quant weights bit-exact for every unit whose oracle gap
    (L2 - L*) / max(|L*|, S) exceeds 1e-5, where S = |w|^T |H| |w| (+ 2 |w|^T |P| |w|) is
    the scale of the rounding error of any finite-precision evaluation of the block's loss
    (S >= E0 = w^T H w, and S ~ E0 for a well-conditioned H); winning loss within
    1e-4 * max(|L*|, S) for every unit.
  * Near-tie units (gap <= 1e-5, where several codes are correct): the GPU's code must be one
    of the oracle's tied candidates {k : L_k - L* <= 1e-5 * max(|L*|, S)}, its fake-quant
    weights bit-exact to the oracle's at that code, and its loss within 1e-4 of the oracle's
    loss at that code.
"""
from __future__ import annotations

import numpy as np

from scale_calibration_lh_b200.synth import layer_to_device, to_device  # noqa: F401 (re-exported)

H_TOL = 1e-4
LOSS_TOL = 1e-4
GAP_TOL = 1e-5


def act_inputs(layer):
    """The input quantizer's side of an activation-aware layer, from the oracle: its global
    scale gx = fp32(amax|X| / 2688) (meta["act_gx"]) and X_q = act_fake_quant(X, gx) (layer.xq).
    The unfused entry point reads this X_q; the fused one derives it from X and gx itself."""
    from oracle import lhcal_oracle as O
    from scale_calibration_lh_b200 import synth

    x = layer.x_f32()
    gx = O.global_scale(x)
    layer.meta["act_gx"] = gx
    xq = O.act_fake_quant(x, gx)
    layer.xq = synth.f32_to_bf16_bits(xq) if layer.dtype == "bf16" else xq
    return layer


def make_layer(name: str, seed: int = 0, **kw):
    """synth.make_layer plus, for the activation-aware workload, the input quantizer's data."""
    from scale_calibration_lh_b200 import synth

    layer = synth.make_layer(name, seed, **kw)
    return act_inputs(layer) if layer.mode == "act" else layer


def check_hessians(gpu: np.ndarray, ref: np.ndarray, what: str, tol: float = H_TOL):
    """Per-block relative Frobenius error; blocks are the trailing (16,16) or (16,)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    axes = tuple(range(2, ref.ndim))
    num = np.sqrt(np.sum((gpu - ref) ** 2, axis=axes))
    den = np.sqrt(np.sum(ref ** 2, axis=axes))
    zero = den == 0
    assert np.all(num[zero] == 0), f"{what}: non-zero GPU block where the oracle block is zero"
    rel = np.where(zero, 0.0, num / np.where(zero, 1.0, den))
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= tol, f"{what}: worst per-block relative Frobenius error {worst:.3e} > {tol}"
    return worst


def attach_candidates(ref: dict, mode: str, w, h, p, g, units=None) -> dict:
    """Give an oracle sweep result the hook that check_sweep uses on near-tie units: for the
    units at positions ``sel`` it returns every candidate's code [S, 126], loss [S, 126] and
    fake-quant weights [S, 126, 16], from the oracle's own functions."""
    from oracle import lhcal_oracle as O

    w = np.asarray(w, dtype=np.float32)
    units = all_units(w.shape[0], w.shape[1], w.shape[2] // 16) if units is None else np.asarray(units, np.int64)

    def candidates(sel):
        wb, hb, pb, gu = O.gather_units(mode, w, h, p, g, units[sel])
        n = len(sel)
        codes = np.broadcast_to(O.candidate_codes(), (n, O.N_CANDIDATES))
        loss = np.empty((n, O.N_CANDIDATES))
        wq = np.empty((n, O.N_CANDIDATES, 16), np.float32)
        for gv in np.unique(gu):
            s = np.nonzero(gu == gv)[0]
            loss[s], wq[s], _ = O.candidate_losses(mode, wb[s], None if hb is None else hb[s],
                                                   None if pb is None else pb[s], gv)
        return codes, loss, wq

    ref["candidates"] = candidates
    return ref


def oracle_sweep(mode: str, w, h, p, g, units=None) -> dict:
    """The oracle's sweep of the given units (default: all), ready for check_sweep."""
    from oracle import lhcal_oracle as O

    w = np.asarray(w, dtype=np.float32)
    units = all_units(w.shape[0], w.shape[1], w.shape[2] // 16) if units is None else np.asarray(units, np.int64)
    return attach_candidates(O.sweep(mode, w, h, p, g, units), mode, w, h, p, g, units)


def oracle_multiplier_search(mode: str, w, h, p, g, multipliers, units=None) -> dict:
    """The oracle's amax-multiplier search, with a near-tie hook over the multipliers: each
    multiplier's code (0 = zero scale), its loss and its fake-quant weights."""
    from oracle import lhcal_oracle as O

    w = np.asarray(w, dtype=np.float32)
    units = all_units(w.shape[0], w.shape[1], w.shape[2] // 16) if units is None else np.asarray(units, np.int64)
    ref = O.multiplier_search(mode, w, h, p, g, multipliers, units)

    def candidates(sel):
        wb, hb, pb, gu = O.gather_units(mode, w, h, p, g, units[sel])
        n, m = len(sel), len(multipliers)
        codes = np.empty((n, m), np.int64)
        loss = np.empty((n, m))
        wq = np.empty((n, m, 16), np.float32)
        for gv in np.unique(gu):
            s = np.nonzero(gu == gv)[0]
            c = O.multiplier_codes(wb[s], gv, multipliers)
            sc = np.where(c > 0, O.candidate_scales(gv)[np.maximum(c, 1) - 1], np.float32(0))
            codes[s] = c
            loss[s], wq[s] = O.losses_for_scales(mode, wb[s], None if hb is None else hb[s],
                                                 None if pb is None else pb[s], sc)
        return codes, loss, wq

    ref["candidates"] = candidates
    return ref


def check_sweep(codes, wq, loss, ref: dict, what: str):
    """codes [U] uint8, wq [U, 16] fp32, loss [U] fp32 from the GPU vs the oracle's result
    (from oracle_sweep, oracle_multiplier_search or attach_candidates).

    Decided units (gap > GAP_TOL): code and Wq bit-exact. Near-tie units: the GPU's code is one
    of the oracle's tied candidates, its Wq is bit-exact to the oracle's at that code and its
    loss within LOSS_TOL of the oracle's loss at that code. Every unit: the winning loss within
    LOSS_TOL of the oracle's. Returns counts and worst errors under both denominators,
    max(|L*|, S) (the gate's) and max(|L*|, E0) (E0 = w^T H w, reported only)."""
    assert "candidates" in ref, f"{what}: the oracle result needs its near-tie hook (oracle_sweep)"
    codes = np.asarray(codes).astype(np.int64)
    wq = np.ascontiguousarray(np.asarray(wq, dtype=np.float32))
    loss = np.asarray(loss, dtype=np.float64)
    best, second = ref["loss"], ref["second"]
    scale = np.maximum(np.maximum(np.abs(best), ref["escale"]), 1e-30)
    gap = (second - best) / scale
    strict = gap > GAP_TOL
    bad_code = strict & (codes != ref["codes"].astype(np.int64))
    assert not bad_code.any(), (
        f"{what}: {int(bad_code.sum())} codes differ on non-tied units; first at {np.nonzero(bad_code)[0][:5]}: "
        f"gpu {codes[bad_code][:5]} oracle {ref['codes'][bad_code][:5]} gap {gap[bad_code][:5]}")
    same_bits = np.all(wq.view(np.int32) == ref["wq"].astype(np.float32).view(np.int32), axis=1)
    bad_wq = strict & ~same_bits
    assert not bad_wq.any(), f"{what}: {int(bad_wq.sum())} units with fake-quant weights not bit-exact"
    err = np.abs(loss - best) / scale
    worst = float(err.max()) if err.size else 0.0
    assert worst <= LOSS_TOL, f"{what}: worst loss error {worst:.3e} (relative to max(|L|, S))"
    ex = np.nonzero(~strict)[0]
    worst_tied = 0.0
    if len(ex):
        cc, cl, cw = ref["candidates"](ex)
        tied = (cl - best[ex, None]) <= GAP_TOL * scale[ex, None]
        match = tied & (cc == codes[ex, None])
        outside = ~match.any(axis=1)
        assert not outside.any(), (
            f"{what}: {int(outside.sum())} near-tie units whose GPU code is not among the oracle's tied "
            f"candidates; first at {ex[outside][:5]}: gpu {codes[ex][outside][:5]}")
        j = match.argmax(axis=1)
        rows = np.arange(len(ex))
        ok = np.all(wq[ex].view(np.int32) == cw[rows, j].view(np.int32), axis=1)
        assert ok.all(), (f"{what}: {int((~ok).sum())} near-tie units with fake-quant weights not bit-exact "
                          f"to the oracle's at the GPU's code; first at {ex[~ok][:5]}")
        terr = np.abs(loss[ex] - cl[rows, j]) / scale[ex]
        worst_tied = float(terr.max())
        assert worst_tied <= LOSS_TOL, f"{what}: near-tie loss error {worst_tied:.3e} at the GPU's code"
    scale0 = np.maximum(np.maximum(np.abs(best), ref["e0"]), 1e-30)
    err0 = np.abs(loss - best) / scale0
    return {"units": int(len(codes)), "exempt": int(len(ex)),
            "exempt_e0": int(np.sum((second - best) / scale0 <= GAP_TOL)),
            "worst_loss_err": worst, "worst_loss_err_e0": float(err0.max()) if err0.size else 0.0,
            "worst_tied_loss_err": worst_tied}


def gather_gpu_units(codes, wq, loss, units):
    """Pick units (g, r, n) out of whole GPU outputs (torch tensors or numpy); returns numpy."""
    u = np.asarray(units, dtype=np.int64)
    ge, r, n = u[:, 0], u[:, 1], u[:, 2]
    cols = n[:, None] * 16 + np.arange(16)[None, :]
    import torch

    if isinstance(codes, torch.Tensor):
        dev = codes.device
        tg, tr, tn = (torch.from_numpy(a).to(dev) for a in (ge, r, n))
        tc = torch.from_numpy(cols).to(dev)
        return (codes[tg, tr, tn].cpu().numpy(), wq[tg[:, None], tr[:, None], tc].cpu().numpy(),
                loss[tg, tr, tn].cpu().numpy())
    return codes[ge, r, n], wq[ge[:, None], r[:, None], cols], loss[ge, r, n]


def all_units(groups, rows, nblk):
    ge, r, n = np.meshgrid(np.arange(groups), np.arange(rows), np.arange(nblk), indexing="ij")
    return np.stack([ge.ravel(), r.ravel(), n.ravel()], axis=1)


def sample_units(groups, rows, nblk, count, seed=0):
    """Random units plus the corner units of the layer (first/last group, row and block)."""
    rng = np.random.default_rng(seed)
    u = np.stack([rng.integers(0, groups, count), rng.integers(0, rows, count), rng.integers(0, nblk, count)], 1)
    corners = np.array([[g, r, n] for g in {0, groups - 1} for r in {0, rows - 1} for n in {0, nblk - 1}])
    return np.concatenate([corners, u])


def _sweep_rows_worker(args):
    """One task of oracle_sweep_parallel (runs in a spawned process)."""
    from threadpoolctl import threadpool_limits

    from oracle import lhcal_oracle as O

    mode, w_rows, h, p, g = args
    with threadpool_limits(1):
        return O.sweep(mode, w_rows, h, p, g)


def oracle_sweep_parallel(mode: str, w, h, p, g, rows_per_task: int = 64, processes: int | None = None) -> dict:
    """The oracle's sweep of every unit of a layer (row-major unit order, as all_units), computed
    by a pool of spawned processes over row chunks; with the near-tie hook for check_sweep."""
    import os
    from concurrent.futures import ProcessPoolExecutor
    from multiprocessing import get_context

    w = np.asarray(w, dtype=np.float32)
    G, R, C = w.shape
    tasks = [(mode, w[:, r:r + rows_per_task], h, p, g) for r in range(0, R, rows_per_task)]
    n = processes or max(1, (os.cpu_count() or 2) - 1)
    with ProcessPoolExecutor(max_workers=n, mp_context=get_context("spawn")) as ex:
        parts = list(ex.map(_sweep_rows_worker, tasks))
    # Each part is [G, rows_chunk, N] in unit order; reassemble to [G, R, N].
    out = {}
    for k in parts[0]:
        if k == "all_losses":
            continue
        arrs = [pt[k].reshape((G, -1, C // BLOCK) + pt[k].shape[1:]) for pt in parts]
        out[k] = np.concatenate(arrs, axis=1).reshape((G * R * (C // BLOCK),) + parts[0][k].shape[1:])
    return attach_candidates(out, mode, w, h, p, g)


BLOCK = 16
