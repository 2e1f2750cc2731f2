"""Comparators and device helpers shared by the GPU parity tests.

Tolerances (the parity bar for the GPU path):
  * Hessians H / P: relative Frobenius error per 16x16 block <= 1e-4; importance per block
    (16 values) <= 1e-4; an all-zero oracle block requires an exactly zero GPU block.
  * Sweep: codes and fake-quant weights bit-exact for every unit whose oracle gap
    (L2 - L*) / max(|L*|, S) exceeds 1e-5, where S = |w|^T |H| |w| (+ 2 |w|^T |P| |w|) is
    the scale of the rounding error of any finite-precision evaluation of the block's loss
    (S >= E0 = w^T H w, and S ~ E0 for a well-conditioned H); winning loss within
    1e-4 * max(|L*|, S) for every unit.
"""
from __future__ import annotations

import numpy as np

H_TOL = 1e-4
LOSS_TOL = 1e-4
GAP_TOL = 1e-5


def to_device(a: np.ndarray | None, kind: str, device="cuda"):
    """kind: 'bf16' (uint16 bits), 'f32', 'i32'."""
    import torch

    if a is None:
        return None
    if kind == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    if kind == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    if kind == "i32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    raise ValueError(kind)


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


def layer_to_device(layer, device="cuda"):
    import torch

    kind = "bf16" if layer.dtype == "bf16" else "f32"
    gx = layer.meta.get("act_gx")
    return {
        "x": to_device(layer.x, kind, device),
        "xq": to_device(layer.xq, kind, device),
        "w": to_device(layer.w, kind, device),
        "offs": to_device(layer.group_offsets, "i32", device),
        "ids": to_device(layer.token_ids, "i32", device),
        "act_gx": None if gx is None else torch.tensor([float(gx)], dtype=torch.float32, device=device),
    }


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


def check_sweep(codes, wq, loss, ref: dict, what: str):
    """codes [U] uint8, wq [U, 16] fp32, loss [U] fp32 from the GPU vs the oracle's sweep output."""
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
    return {"units": int(len(codes)), "exempt": int((~strict).sum()), "worst_loss_err": worst}


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
