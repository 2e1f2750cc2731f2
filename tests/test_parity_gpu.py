"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Small cases span several tiles and ragged tails (tokens not a multiple of the 64-token
tile, cin not a multiple of the 128-column slab or the 2048-column DIAG slab, rows not a
multiple of the 128-row sweep tile, experts with no tokens). Full-size workloads compare
all Hessian blocks and a sample of sweep units (plus the layer's corner units).
"""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import scale_calibration_lh_b200 as L  # noqa: E402
from scale_calibration_lh_b200 import synth  # noqa: E402
from oracle import lhcal_oracle as O  # noqa: E402
from tests import parity as P  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from scale_calibration_lh_b200 import build

    build.build()
    L.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _sync():
    torch.cuda.synchronize()


def _oracle_hessians(layer, fused=False):
    if fused:  # the oracle derives X_q from X with the input quantizer's global scale
        return O.accumulate("act", layer.x_f32(), None, layer.group_offsets, layer.token_ids,
                            act_gx=layer.meta["act_gx"])
    xq = layer.xq_f32() if layer.xq is not None else None
    hs, ps, counts = O.accumulate(layer.mode, layer.x_f32(), xq, layer.group_offsets, layer.token_ids)
    return hs, ps, counts


def _run_and_check(layer, units=None, check_raw=True, fused=False):
    """fused: activation-aware layer through the fused input quantizer (X and gx, no X_q)."""
    d = P.layer_to_device(layer)
    mode = L.MODE_IDS[layer.mode]
    G, R, C = layer.groups, layer.rows, layer.cin
    nblk = C // 16
    # Raw sums first (OVERWRITE into fresh buffers), compared before finalisation.
    b = L.Buffers(mode, layer.tokens, C, R, G, L.BF16 if layer.dtype == "bf16" else L.F32, "cuda")
    if fused:
        L.lhcal_accumulate_act_quant(d["x"], b.h, b.p, d["act_gx"], group_offsets=d["offs"], token_ids=d["ids"],
                                     flags=L.ACCUM_OVERWRITE, workspace=b.workspace)
    else:
        L.lhcal_accumulate(mode, d["x"], b.h, xq=d["xq"], p=b.p, group_offsets=d["offs"], token_ids=d["ids"],
                           flags=L.ACCUM_OVERWRITE, workspace=b.workspace)
    _sync()
    hs, ps, counts = _oracle_hessians(layer, fused)
    report = {}
    if check_raw:
        report["h_raw"] = P.check_hessians(b.h.cpu().numpy(), hs, f"{layer.name} raw H")
        if ps is not None:
            report["p_raw"] = P.check_hessians(b.p.cpu().numpy(), ps, f"{layer.name} raw P")
    b2 = L.calibrate(mode, d["x"], d["w"], xq=None if fused else d["xq"], group_offsets=d["offs"],
                     token_ids=d["ids"], buffers=b, act_gx=d["act_gx"] if fused else None)
    _sync()
    h, p = O.finalize(layer.mode, hs, ps, counts)
    report["h"] = P.check_hessians(b2.h.cpu().numpy(), h, f"{layer.name} H")
    if p is not None:
        report["p"] = P.check_hessians(b2.p.cpu().numpy(), p, f"{layer.name} P")
    np.testing.assert_array_equal(b2.counts.cpu().numpy(), counts)
    w32 = layer.w_f32()
    g = np.array([O.global_scale(w32[e]) for e in range(G)], np.float32)
    np.testing.assert_array_equal(b2.g.cpu().numpy().view(np.int32), g.view(np.int32))
    if units is None:
        units = P.all_units(G, R, nblk)
    ref = P.oracle_sweep(layer.mode, w32, h, p, g, units)
    gc, gw, gl = P.gather_gpu_units(b2.codes, b2.wq, b2.loss, units)
    report["sweep"] = P.check_sweep(gc, gw, gl, ref, layer.name)
    return report


# ----------------------------------------------------------------------------- small cases

def test_tiny_full_size_end_to_end():
    r = _run_and_check(P.make_layer("tiny", 0))
    assert r["sweep"]["units"] == 128


@pytest.mark.parametrize("tokens,cin,rows", [(1000, 272, 300), (64, 128, 128), (1, 16, 1), (130, 400, 257)])
def test_dense_full_bf16(tokens, cin, rows):
    _run_and_check(P.make_layer("dense", 1, tokens=tokens, cin=cin, rows=rows))


@pytest.mark.parametrize("tokens,cin,rows", [(777, 160, 200), (65, 48, 129)])
def test_act_aware_bf16(tokens, cin, rows):
    _run_and_check(P.make_layer("act", 2, tokens=tokens, cin=cin, rows=rows))


@pytest.mark.parametrize("tokens,cin,rows", [(1500, 2064, 130), (9, 32, 3)])
def test_wmse_diag_bf16(tokens, cin, rows):
    _run_and_check(P.make_layer("wmse", 3, tokens=tokens, cin=cin, rows=rows))


def test_moe_grouped_with_empty_experts():
    layer = P.make_layer("moe", 4, tokens=40, cin=160, rows=40, groups=64, top_k=3)
    counts = np.diff(layer.group_offsets)
    assert (counts == 0).any() and (counts > 1).any()
    _run_and_check(layer)


def test_moe_grouped_full_rank_experts():
    layer = P.make_layer("moe", 13, tokens=600, cin=272, rows=150, groups=24, top_k=4)
    assert np.diff(layer.group_offsets).min() >= 32
    r = _run_and_check(layer)
    assert r["sweep"]["exempt"] < 0.05 * r["sweep"]["units"]


@pytest.mark.parametrize("variant", ["full", "act", "act_fused"])
def test_moe_grouped_tile_boundaries(variant):
    """Experts with 0, 1, 63, 64, 65, 127, 128, 129 and 200 routed rows (the 64-row tiles of the
    grouped accumulation full, ragged and empty) over cin = 160 (one full 128-column slab and a
    partial one): the loader's unpredicated copies for full tiles and predicated ones for ragged
    tiles and out-of-range columns, against the oracle."""
    counts = [0, 1, 63, 64, 65, 127, 128, 129, 200]
    T = 300
    layer = synth.make_layer("moe", 41, tokens=T, cin=160, rows=20, groups=len(counts), top_k=2)
    rng = np.random.default_rng(42)
    ids = [np.sort(rng.choice(T, size=c, replace=False)) for c in counts]
    layer.group_offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    layer.token_ids = np.concatenate(ids).astype(np.int32)
    if variant != "full":
        layer.mode = "act"
        P.act_inputs(layer)
    assert np.array_equal(np.diff(layer.group_offsets), counts)
    _run_and_check(layer, fused=variant == "act_fused")


def test_moe_grouped_diag_bf16_generic_path():
    layer = P.make_layer("moe", 5, tokens=50, cin=48, rows=20, groups=8, top_k=2)
    layer.mode = "diag"
    _run_and_check(layer)


@pytest.mark.parametrize("mode", ["full", "act", "diag"])
@pytest.mark.parametrize("grouped", [False, True])
def test_fp32_inputs_all_modes(mode, grouped):
    rng = np.random.default_rng(6)
    T, C, R, G = 100, 48, 20, (5 if grouped else 1)
    x = rng.normal(size=(T, C)).astype(np.float32)
    w = rng.normal(0, 0.02, (G, R, C)).astype(np.float32)
    layer = synth.Layer("f32-" + mode, mode, "f32", x, w)
    if mode == "act":
        layer.xq = (x + rng.normal(0, 0.05, x.shape)).astype(np.float32)
    if grouped:
        layer.group_offsets, layer.token_ids = synth.moe_routing(T, G, 2, 7)
    _run_and_check(layer)


# ----------------------------------------------------------------------------- sweep special cases

def _sweep_gpu(mode, w, h, p, g, w_bf16=False):
    """w fp32 [G,R,C] (bf16-exact values when w_bf16: the kernel then reads bf16 weights); h/p/g
    from the oracle side (fp32-rounded) -> GPU outputs (numpy)."""
    G, R, C = w.shape
    dw = P.to_device((w.view(np.uint32) >> 16).astype(np.uint16), "bf16") if w_bf16 else P.to_device(w, "f32")
    dh = None if h is None else P.to_device(np.asarray(h, np.float32), "f32")
    dp = None if p is None else P.to_device(np.asarray(p, np.float32), "f32")
    dg = P.to_device(g, "f32")
    codes = torch.empty((G, R, C // 16), dtype=torch.uint8, device="cuda")
    wq = torch.empty((G, R, C), dtype=torch.float32, device="cuda")
    loss = torch.empty((G, R, C // 16), dtype=torch.float32, device="cuda")
    L.lhcal_scale_sweep(mode, dw, dh, dg, codes, wq=wq, loss=loss, p=dp)
    _sync()
    return codes.cpu().numpy(), wq.cpu().numpy(), loss.cpu().numpy()


def _special_weights(seed=8):
    """Blocks with exact E2M1 ties, neighbours of ties, zeros, -0.0, a lone outlier, tiny values."""
    rng = np.random.default_rng(seed)
    G, R, C = 3, 40, 64
    w = rng.normal(0, 0.02, (G, R, C)).astype(np.float32)
    g0 = O.global_scale(w[0])
    s = O.candidate_scales(g0)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    for r in range(0, 20):
        k = rng.integers(0, 126)
        t = (mids[rng.integers(0, 7, 16)] * np.float64(s[k])).astype(np.float32)  # may round: then a near-tie
        sign = np.where(rng.random(16) < 0.5, -1, 1).astype(np.float32)
        w[0, r, :16] = t * sign
        w[0, r, 16:32] = np.nextafter(t, np.float32(1)) * sign
        w[0, r, 32:48] = np.nextafter(t, np.float32(0)) * sign
    w[0, 0, :] = np.float32(0.0)             # all-zero block row
    w[0, 1, 16:32] = np.float32(-0.0)        # negative zeros
    w[0, 2, 48:64] = 0.0
    w[0, 2, 50] = 0.5                        # lone outlier
    w[1] = rng.normal(0, 1e-3, (R, C)).astype(np.float32) * (rng.random((R, C)) < 0.3)
    w[2] = 0.0                               # whole group zero: g = 0
    return w


@pytest.mark.parametrize("mode", ["full", "act", "diag"])
def test_sweep_special_weights_with_oracle_hessians(mode):
    w = _special_weights()
    G, R, C = w.shape
    nblk = C // 16
    rng = np.random.default_rng(9)
    x = (rng.normal(size=(200, C)) * rng.lognormal(0, 1, C)).astype(np.float32)
    if mode == "diag":
        h = np.broadcast_to(O.importance_sum(x), (G, nblk, 16)).astype(np.float32)
        p = None
    elif mode == "act":
        xq = (x * 0.95 + rng.normal(0, 0.05, x.shape)).astype(np.float32)
        hs, ps = O.hessian_sum_act(x, xq)
        h = np.broadcast_to(hs / 200, (G, nblk, 16, 16)).astype(np.float32)
        p = np.broadcast_to(ps / 200, (G, nblk, 16, 16)).astype(np.float32)
    else:
        h = np.broadcast_to(O.hessian_sum_full(x) / 200, (G, nblk, 16, 16)).astype(np.float32)
        p = None
    g = np.array([O.global_scale(w[e]) for e in range(G)], np.float32)
    assert g[2] == 0
    codes, wq, loss = _sweep_gpu(L.MODE_IDS[mode], w, h, p, g)
    units = P.all_units(G, R, nblk)
    ref = P.oracle_sweep(mode, w, h.astype(np.float64), None if p is None else p.astype(np.float64), g, units)
    gc, gw, gl = P.gather_gpu_units(codes, wq, loss, units)
    P.check_sweep(gc, gw, gl, ref, f"special {mode}")
    # Degenerate units: every candidate ties, the lowest code wins, outputs are signed zeros.
    assert np.all(codes[2] == 1) and np.all(codes[0, 0] == 1)
    assert np.all(wq[2] == 0) and np.all(wq[0, 1, 16:32].view(np.int32) == np.float32(-0.0).view(np.int32))


def _bf16_step(t: np.ndarray, up: bool) -> np.ndarray:
    """The neighbouring bf16 value of positive bf16 values t (as fp32), above or below."""
    b = (t.view(np.uint32) >> 16).astype(np.int64) + (1 if up else -1)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _bf16_tie_weights(seed=12):
    """bf16 weights whose group 0 has the global scale 2^-12 (its largest |w| is 2688 * 2^-12), so
    that every E2M1 midpoint times a candidate scale (at most 7 significant bits) is a bf16 value:
    rows of exact ties, their bf16 neighbours above and below, and ordinary weights. Group 1 has
    an arbitrary global scale, where the rounded midpoints are near-ties."""
    rng = np.random.default_rng(seed)
    G, R, C = 2, 48, 64
    w = rng.normal(0, 0.02, (G, R, C)).astype(np.float32)
    w = ((w.view(np.uint32) >> 16) << 16).view(np.float32)  # bf16 values
    w[0, 0, 0] = np.float32(2688.0 * 2.0 ** -12)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    for e in range(G):
        s = O.candidate_scales(O.global_scale(w[e]))
        for r in range(1, 41):
            k = rng.integers(0, 126)
            t = (mids[rng.integers(0, 7, 16)] * np.float64(s[k])).astype(np.float32)
            t = ((t.view(np.uint32) >> 16) << 16).view(np.float32)  # exact in group 0
            sign = np.where(rng.random(16) < 0.5, -1, 1).astype(np.float32)
            w[e, r, :16] = t * sign
            w[e, r, 16:32] = _bf16_step(t, True) * sign
            w[e, r, 32:48] = _bf16_step(t, False) * sign
    return w


@pytest.mark.parametrize("mode", ["full", "act", "diag", "mse"])
def test_sweep_bf16_weights_at_exact_ties(mode):
    """bf16 weights at exact E2M1 ties (round half to even) and their bf16 neighbours against the
    oracle, in every sweep mode; the tensor-core sweep decides their levels on bf16 thresholds,
    two elements per packed compare."""
    w = _bf16_tie_weights()
    G, R, C = w.shape
    g = np.array([O.global_scale(w[e]) for e in range(G)], np.float32)
    assert g[0] == np.float32(2.0 ** -12)
    s0 = O.candidate_scales(g[0]).astype(np.float64)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    a = np.abs(w[0, 1:41, :16]).astype(np.float64)
    assert np.isin(a, np.outer(mids, s0)).all()  # every one an exact tie for some candidate
    nblk = C // 16
    rng = np.random.default_rng(13)
    x = (rng.normal(size=(200, C)) * rng.lognormal(0, 1, C)).astype(np.float32)
    p = None
    if mode == "act":
        xq = (x * 0.95 + rng.normal(0, 0.05, x.shape)).astype(np.float32)
        hs, ps = O.hessian_sum_act(x, xq)
        h = np.broadcast_to(hs / 200, (G, nblk, 16, 16)).astype(np.float32)
        p = np.broadcast_to(ps / 200, (G, nblk, 16, 16)).astype(np.float32)
    elif mode == "diag":
        h = np.broadcast_to(O.importance_sum(x), (G, nblk, 16)).astype(np.float32)
    elif mode == "mse":
        h = None  # every importance 1
    else:
        h = np.broadcast_to(O.hessian_sum_full(x) / 200, (G, nblk, 16, 16)).astype(np.float32)
    codes, wq, loss = _sweep_gpu(L.MODE_IDS[mode], w, h, p, g, w_bf16=True)
    units = P.all_units(G, R, nblk)
    href = None if h is None else h.astype(np.float64)
    ref = P.oracle_sweep(mode, w, href, None if p is None else p.astype(np.float64), g, units)
    gc, gw, gl = P.gather_gpu_units(codes, wq, loss, units)
    rep = P.check_sweep(gc, gw, gl, ref, f"bf16 ties {mode}")
    assert rep["units"] == G * R * nblk
    # The same weights as fp32: identical codes, weights and losses (the FULL and activation-aware
    # bf16 paths decide on bf16 thresholds, the others share the fp32 code).
    c32, w32, l32 = _sweep_gpu(L.MODE_IDS[mode], w, h, p, g)
    assert np.array_equal(codes, c32)
    assert np.array_equal(wq.view(np.int32), w32.view(np.int32))
    assert np.array_equal(loss.view(np.int32), l32.view(np.int32))


@pytest.mark.parametrize("mode", ["full", "act", "diag"])
def test_sweep_codes_invariant_under_power_of_two_statistics(mode):
    """Scaling H (and P, or the importances) by a power of two scales every loss exactly, so the
    codes and fake-quantized weights must not change. The extreme factors take the sweeps'
    clamped-prefix window out of range (its curvature beyond 2^100, or below 2^-100 times the
    squared smallest scale), so the full prefix is evaluated there and the window elsewhere."""
    layer = P.make_layer("dense" if mode != "act" else "act", 43, tokens=600, cin=64, rows=256)
    x = layer.x_f32()
    G, R, C = layer.groups, layer.rows, layer.cin
    nblk = C // 16
    w = layer.w_f32()
    g = np.array([O.global_scale(w[e]) for e in range(G)], np.float32)
    p = None
    if mode == "act":
        hs, ps = O.hessian_sum_act(x, layer.xq_f32())
        h = (hs / x.shape[0]).reshape(G, nblk, 16, 16)
        p = (ps / x.shape[0]).reshape(G, nblk, 16, 16)
    elif mode == "diag":
        h = O.importance_sum(x).reshape(G, nblk, 16)
    else:
        h = (O.hessian_sum_full(x) / x.shape[0]).reshape(G, nblk, 16, 16)
    base = _sweep_gpu(L.MODE_IDS[mode], w, h, p, g, w_bf16=True)
    for f in (2.0 ** -90, 2.0 ** -40, 2.0 ** 40, 2.0 ** 90):
        got = _sweep_gpu(L.MODE_IDS[mode], w, h * f, None if p is None else p * f, g, w_bf16=True)
        assert np.array_equal(got[0], base[0]), (mode, f)
        assert np.array_equal(got[1].view(np.int32), base[1].view(np.int32)), (mode, f)
        np.testing.assert_allclose(got[2], base[2] * np.float32(f), rtol=1e-6)


def test_sweep_identity_hessian_is_plain_mse():
    rng = np.random.default_rng(10)
    w = rng.normal(0, 0.05, (1, 64, 96)).astype(np.float32)
    h = np.broadcast_to(np.eye(16, dtype=np.float32), (1, 6, 16, 16)).copy()
    g = np.array([O.global_scale(w[0])], np.float32)
    codes, wq, loss = _sweep_gpu(L.FULL, w, h, None, g)
    # Plain block MSE of the GPU's own fake-quant output equals its reported loss.
    mse = ((wq.astype(np.float64) - w.astype(np.float64)) ** 2).reshape(1, 64, 6, 16).sum(-1)
    np.testing.assert_allclose(loss, mse, rtol=1e-5)
    ref = P.oracle_sweep("full", w, h.astype(np.float64), None, g)
    P.check_sweep(codes.reshape(-1), wq.reshape(-1, 16), loss.reshape(-1), ref, "identity H")


def test_act_aware_negative_winning_losses():
    """Activation-aware losses may be negative: the best loss starts at +inf and the argmin must
    handle negative values ("Add activation-aware local Hessian scale calibration", PR #1976,
    both review comments). With X_q = bf16(0.9 X), H ~ 0.81 M and P ~ -0.09 M (M = X^T X / B);
    each weight block lies at 0.9 x (E2M1 grid value x s_k) for a random candidate k, so at k
    dW = w / 9 and the objective is about 0.01 w^T M w - 0.02 w^T M w < 0. The whole path (two-tensor
    accumulation, finalize, global scale, sweep) must match the oracle, and most winning losses
    must be negative on both sides."""
    rng = np.random.default_rng(77)
    T, C, R = 700, 64, 150
    x = synth.f32_to_bf16_bits((rng.normal(size=(T, C)) * rng.lognormal(0, 1, C)).astype(np.float32))
    xq = synth.f32_to_bf16_bits(np.float32(0.9) * synth.bf16_bits_to_f32(x))
    g0 = np.float32(2.0 ** -10)
    s = O.candidate_scales(g0)
    grid = np.array([0.5, 1, 1.5, 2, 3, 4, 6])
    nblk = C // 16
    k = rng.integers(40, 126, (R, nblk))
    q = grid[rng.integers(0, len(grid), (R, nblk, 16))]
    sign = np.where(rng.random((R, nblk, 16)) < 0.5, -1.0, 1.0)
    w = (0.9 * q * s[k][..., None].astype(np.float64) * sign).astype(np.float32).reshape(1, R, C)
    w[0, 0, 0] = np.float32(2688.0 * 2.0 ** -10)  # amax: the global scale is exactly g0
    assert O.global_scale(w[0]) == g0
    dev = {"x": synth.to_device(x, "bf16"), "xq": synth.to_device(xq, "bf16"), "w": synth.to_device(w, "f32")}
    b = L.calibrate("act", dev["x"], dev["w"], xq=dev["xq"])
    _sync()
    hs, ps, counts = O.accumulate("act", synth.bf16_bits_to_f32(x), synth.bf16_bits_to_f32(xq))
    h, p = O.finalize("act", hs, ps, counts)
    P.check_hessians(b.h.cpu().numpy(), h, "negative-loss layer H")
    P.check_hessians(b.p.cpu().numpy(), p, "negative-loss layer P")
    np.testing.assert_array_equal(b.g.cpu().numpy(), [g0])
    units = P.all_units(1, R, nblk)
    ref = P.oracle_sweep("act", w, h, p, np.array([g0], np.float32), units)
    gc, gw, gl = P.gather_gpu_units(b.codes, b.wq, b.loss, units)
    rep = P.check_sweep(gc, gw, gl, ref, "negative-loss layer")
    assert rep["units"] == R * nblk
    neg = ref["loss"] < 0
    assert neg.mean() > 0.9, f"only {neg.mean():.2f} of the oracle's winning losses are negative"
    assert np.all(gl[neg] < 0), "the GPU's winning loss is not negative where the oracle's is"


# ----------------------------------------------------------------------------- accumulate semantics

def test_accumulate_add_equals_one_pass_and_is_deterministic():
    layer = P.make_layer("act", 11, tokens=700, cin=96, rows=8)
    d = P.layer_to_device(layer)
    x, xq = d["x"], d["xq"]
    nb = 96 // 16
    ws_bytes = max(L.lhcal_accumulate_workspace("act", L.BF16, 700, 96, 1), 4)
    ws = torch.empty(ws_bytes // 4, dtype=torch.float32, device="cuda")
    h1 = torch.empty((1, nb, 16, 16), dtype=torch.float32, device="cuda")
    p1 = torch.empty_like(h1)
    L.lhcal_accumulate("act", x[:300], h1, xq=xq[:300], p=p1, flags=L.ACCUM_OVERWRITE, workspace=ws)
    L.lhcal_accumulate("act", x[300:], h1, xq=xq[300:], p=p1, flags=L.ACCUM_ADD, workspace=ws)
    h2 = torch.empty_like(h1)
    p2 = torch.empty_like(h1)
    h3 = torch.empty_like(h1)
    p3 = torch.empty_like(h1)
    L.lhcal_accumulate("act", x, h2, xq=xq, p=p2, flags=L.ACCUM_OVERWRITE, workspace=ws)
    L.lhcal_accumulate("act", x, h3, xq=xq, p=p3, flags=L.ACCUM_OVERWRITE, workspace=ws)
    _sync()
    hs, ps, _ = _oracle_hessians(layer)
    P.check_hessians(h1.cpu().numpy(), hs, "two-call H")
    P.check_hessians(p1.cpu().numpy(), ps, "two-call P")
    assert torch.equal(h2.view(torch.int32), h3.view(torch.int32))
    assert torch.equal(p2.view(torch.int32), p3.view(torch.int32))


@pytest.mark.parametrize("cin", [4096, 4000])
@pytest.mark.parametrize("name", ["dense", "act"])
def test_accumulate_cluster_path_overwrite_and_add(name, cin):
    """Wide layers (32 column slabs; with cin = 4000 the last holds 32 columns) reduce token
    splits inside CTA clusters, with no workspace."""
    layer = P.make_layer(name, 14, tokens=3001, cin=cin, rows=2)
    mode = layer.mode
    assert L.lhcal_accumulate_workspace(mode, L.BF16, layer.tokens, layer.cin, 1) == 0
    d = P.layer_to_device(layer)
    shape = (1, cin // 16, 16, 16)
    h = torch.full(shape, 3.0, dtype=torch.float32, device="cuda")
    p = torch.full(shape, 3.0, dtype=torch.float32, device="cuda") if mode == "act" else None
    L.lhcal_accumulate(mode, d["x"], h, xq=d["xq"], p=p, flags=L.ACCUM_OVERWRITE)
    h2 = h.clone()
    p2 = None if p is None else p.clone()
    L.lhcal_accumulate(mode, d["x"], h2, xq=d["xq"], p=p2, flags=L.ACCUM_ADD)
    _sync()
    hs, ps, _ = _oracle_hessians(layer)
    P.check_hessians(h.cpu().numpy(), hs, f"{name} cluster H")
    P.check_hessians(h2.cpu().numpy(), 2 * hs, f"{name} cluster H added twice")
    if p is not None:
        P.check_hessians(p.cpu().numpy(), ps, f"{name} cluster P")
        P.check_hessians(p2.cpu().numpy(), 2 * ps, f"{name} cluster P added twice")


def test_accumulate_strided_rows_and_zero_tokens():
    layer = P.make_layer("dense", 12, tokens=333, cin=64, rows=4)
    d = P.layer_to_device(layer)
    wide = torch.zeros((333, 96), dtype=torch.bfloat16, device="cuda")
    wide[:, :64] = d["x"]
    xs = wide[:, :64]  # row stride 96 elements
    h = torch.full((1, 4, 16, 16), 7.0, dtype=torch.float32, device="cuda")
    ws_bytes = L.lhcal_accumulate_workspace("full", L.BF16, 333, 64, 1)
    ws = torch.empty(ws_bytes // 4, dtype=torch.float32, device="cuda")
    L.lhcal_accumulate("full", xs, h, flags=L.ACCUM_OVERWRITE, workspace=ws)
    _sync()
    hs, _, _ = _oracle_hessians(layer)
    P.check_hessians(h.cpu().numpy(), hs, "strided H")
    # Zero tokens: OVERWRITE zeroes the sums, ADD leaves them.
    h0 = torch.full((1, 4, 16, 16), 3.0, dtype=torch.float32, device="cuda")
    L.lhcal_accumulate("full", xs[:0], h0, flags=L.ACCUM_ADD)
    _sync()
    assert torch.all(h0 == 3.0)
    L.lhcal_accumulate("full", xs[:0], h0, flags=L.ACCUM_OVERWRITE)
    _sync()
    assert torch.all(h0 == 0.0)


def test_device_and_host_pointer_errors():
    w = torch.zeros((1, 4, 32), dtype=torch.bfloat16)
    g = torch.zeros(1, dtype=torch.float32)
    with pytest.raises(L.LhcalError) as e:
        L.lhcal_global_scale(w, g)  # host tensors
    assert e.value.status == L.ERR_INVALID_ARG
    flat = torch.zeros(256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LhcalError) as e:
        L.lhcal_global_scale(flat[4:68].view(1, 2, 32), g.cuda())  # 8-byte offset: misaligned
    assert e.value.status == L.ERR_INVALID_ARG


# ----------------------------------------------------------------------------- full-size workloads

@pytest.mark.parametrize("name", ["dense", "act", "wmse", "moe"])
def test_full_size_workload(name):
    layer = P.make_layer(name, 0)
    G, R, C = layer.groups, layer.rows, layer.cin
    units = P.sample_units(G, R, C // 16, 3000, seed=1)
    if name == "wmse":
        _run_and_check_wmse_full(layer, units)
    else:  # the activation-aware workload runs with the input quantizer fused, as benchmarked
        _run_and_check(layer, units=units, check_raw=False, fused=name == "act")


def _run_and_check_wmse_full(layer, units):
    """Full-size WMSE: the oracle's importance is accumulated over row chunks (fp64 sums)."""
    d = P.layer_to_device(layer)
    b = L.calibrate("diag", d["x"], d["w"])
    _sync()
    imp = np.zeros((layer.cin // 16, 16))
    for lo in range(0, layer.tokens, 4096):
        imp += O.importance_sum(synth.bf16_bits_to_f32(layer.x[lo:lo + 4096]))
    h, _ = O.finalize("diag", imp[None], None, np.array([layer.tokens]))
    P.check_hessians(b.h.cpu().numpy(), h, "wmse Imp")
    w32 = layer.w_f32()
    g = np.array([O.global_scale(w32[0])], np.float32)
    np.testing.assert_array_equal(b.g.cpu().numpy().view(np.int32), g.view(np.int32))
    ref = P.oracle_sweep("diag", w32, h, None, g, units)
    gc, gw, gl = P.gather_gpu_units(b.codes, b.wq, b.loss, units)
    P.check_sweep(gc, gw, gl, ref, "wmse full")


# ----------------------------------------------------------------------------- more edge cases

def test_grouped_add_mode_over_two_batches():
    """Two routed batches added into the same per-expert sums equal one pass over both."""
    layer = P.make_layer("moe", 15, tokens=200, cin=96, rows=8, groups=16, top_k=3)
    d = P.layer_to_device(layer)
    x = d["x"]
    off = layer.group_offsets
    ids = layer.token_ids
    # Batch 1: tokens < 100, batch 2: tokens >= 100 (ids renumbered into each batch's rows).
    batches = []
    for lo, hi in ((0, 100), (100, 200)):
        o, t = [0], []
        for e in range(16):
            sel = [int(v) - lo for v in ids[off[e]:off[e + 1]] if lo <= v < hi]
            t += sel
            o.append(len(t))
        batches.append((lo, hi, np.array(o, np.int32), np.array(t, np.int32)))
    h = torch.full((16, 6, 16, 16), 9.0, dtype=torch.float32, device="cuda")
    counts = torch.empty(16, dtype=torch.int64, device="cuda")
    for j, (lo, hi, o, t) in enumerate(batches):
        flags = L.ACCUM_OVERWRITE if j == 0 else L.ACCUM_ADD
        do, dt = P.to_device(o, "i32"), P.to_device(t, "i32")
        L.lhcal_accumulate("full", x[lo:hi], h, group_offsets=do, token_ids=dt, flags=flags)
        L.lhcal_count_tokens(counts, group_offsets=do, flags=flags)
    L.lhcal_finalize("full", counts, h)
    _sync()
    hs, _, c = _oracle_hessians(layer)
    hf, _ = O.finalize("full", hs, None, c)
    np.testing.assert_array_equal(counts.cpu().numpy(), c)
    P.check_hessians(h.cpu().numpy(), hf, "two-batch grouped H")


@pytest.mark.parametrize("mode", ["full", "act", "diag"])
def test_sweep_optional_outputs_and_determinism(mode):
    name = {"full": "dense", "act": "act", "diag": "wmse"}[mode]
    layer = P.make_layer(name, 16, tokens=300, cin=128, rows=200)
    d = P.layer_to_device(layer)
    b = L.calibrate(mode, d["x"], d["w"], xq=d["xq"])
    codes1 = b.codes.clone()
    wq1 = b.wq.clone()
    loss1 = b.loss.clone()
    codes2 = torch.empty_like(codes1)
    L.lhcal_scale_sweep(mode, d["w"], b.h, b.g, codes2, wq=None, loss=None, p=b.p)
    codes3 = torch.empty_like(codes1)
    wq3 = torch.empty_like(wq1)
    loss3 = torch.empty_like(loss1)
    L.lhcal_scale_sweep(mode, d["w"], b.h, b.g, codes3, wq=wq3, loss=loss3, p=b.p)
    _sync()
    assert torch.equal(codes1, codes2) and torch.equal(codes1, codes3)
    assert torch.equal(wq1.view(torch.int32), wq3.view(torch.int32))
    assert torch.equal(loss1.view(torch.int32), loss3.view(torch.int32))


def test_diag_sweep_multiple_groups():
    layer = P.make_layer("moe", 17, tokens=120, cin=64, rows=70, groups=6, top_k=2)
    layer.mode = "diag"
    _run_and_check(layer)


def test_graph_replay_matches_eager_calls():
    layer_a = P.make_layer("dense", 18, tokens=700, cin=512, rows=96)
    layer_b = P.make_layer("dense", 19, tokens=700, cin=512, rows=96)
    da, db = P.layer_to_device(layer_a), P.layer_to_device(layer_b)
    x, w = da["x"].clone(), da["w"].clone()
    graph = L.CalibrationGraph("full", x, w)
    for d in (db, da):
        x.copy_(d["x"])
        w.copy_(d["w"])
        out = graph.replay()
        eager = L.calibrate("full", d["x"], d["w"])
        _sync()
        assert torch.equal(out.codes, eager.codes)
        assert torch.equal(out.wq.view(torch.int32), eager.wq.view(torch.int32))
        assert torch.equal(out.h.view(torch.int32), eager.h.view(torch.int32))


@pytest.mark.parametrize("mode", ["act", "mse"])
def test_graph_replay_fused_quantizer_and_mse(mode):
    """The captured path with the input quantizer fused (X and gx in; the token splits reduce
    through the workspace), and the statistics-free MSE sweep."""
    layers = [P.make_layer("act" if mode == "act" else "dense", s, tokens=900, cin=256, rows=64) for s in (31, 32)]
    devs = [P.layer_to_device(ly) for ly in layers]
    x, w = devs[0]["x"].clone(), devs[0]["w"].clone()
    gx = devs[0]["act_gx"].clone() if mode == "act" else None
    graph = L.CalibrationGraph(mode, None if mode == "mse" else x, w, act_gx=gx)
    for d in (devs[1], devs[0]):
        x.copy_(d["x"])
        w.copy_(d["w"])
        if gx is not None:
            gx.copy_(d["act_gx"])
        out = graph.replay()
        eager = L.calibrate(mode, None if mode == "mse" else d["x"], d["w"], act_gx=d["act_gx"] if gx is not None else None)
        _sync()
        assert torch.equal(out.codes, eager.codes)
        assert torch.equal(out.loss.view(torch.int32), eager.loss.view(torch.int32))
        if mode == "act":
            assert torch.equal(out.p.view(torch.int32), eager.p.view(torch.int32))


# ----------------------------------------------------------------------------- input quantizer

def _act_x(tokens, cin, seed):
    """bf16 activations drawn like the dense workload, plus blocks that stress the quantizer:
    all-zero, negative-zero, tiny (small and subnormal scale codes) and huge outlier blocks."""
    rng = np.random.default_rng(seed)
    sig = np.exp(rng.normal(0, 1, cin))
    sig[rng.choice(cin, max(1, cin // 100), replace=False)] *= 20
    x = rng.normal(size=(tokens, cin)) * sig
    if tokens >= 4 and cin >= 32:
        x[0, :16] = 0.0
        x[1, 16:32] = -0.0
        x[2, :16] *= 1e-30
        x[3, 16:32] *= 1e4
    return synth.f32_to_bf16_bits(x.astype(np.float32))


@pytest.mark.parametrize("tokens,cin,pad,gx_factor", [(1, 16, 0, 1.0), (37, 48, 8, 1.0), (300, 4096, 0, 1.0),
                                                       (129, 256, 24, 1e-3), (129, 256, 0, 1e3),
                                                       (64, 64, 0, 0.0), (0, 32, 0, 1.0)])
def test_act_fake_quant_kernel_bit_exact(tokens, cin, pad, gx_factor):
    xb = _act_x(tokens, cin, 40 + tokens)
    x32 = synth.bf16_bits_to_f32(xb)
    gx = np.float32(O.global_scale(x32) * gx_factor) if tokens else np.float32(1.0)
    want = synth.f32_to_bf16_bits(O.act_fake_quant(x32, gx)) if tokens else np.zeros((0, cin), np.uint16)
    ld = cin + pad
    xfull = np.zeros((tokens, ld), np.uint16)
    xfull[:, :cin] = xb
    dx = P.to_device(xfull, "bf16")[:, :cin]
    dq_full = torch.full((tokens, ld), 7.0, dtype=torch.bfloat16, device="cuda")
    dq = dq_full[:, :cin]
    L.lhcal_act_fake_quant(dx, torch.tensor([float(gx)], device="cuda"), dq)
    _sync()
    got = dq_full.cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got[:, :cin], want)
    assert np.all(got[:, cin:] == np.uint16(0x40E0))  # the padding columns (7.0) are untouched


@pytest.mark.parametrize("tokens,cin,rows", [(1000, 256, 40), (70, 48, 24), (2500, 4096, 16), (1, 16, 8)])
def test_fused_act_quant_accumulation(tokens, cin, rows):
    """X and gx in, no X_q: split (few slabs), cluster (4096 wide) and ragged cases."""
    _run_and_check(P.make_layer("act", 31, tokens=tokens, cin=cin, rows=rows), fused=True)


def test_fused_act_quant_grouped():
    layer = synth.make_layer("moe", 32, tokens=300, cin=96, rows=24, groups=12, top_k=3)
    layer.mode = "act"
    P.act_inputs(layer)
    _run_and_check(layer, fused=True)


@pytest.mark.parametrize("tokens,cin,grouped,same_order", [(3000, 512, False, True), (2048, 4096, False, False),
                                                            (400, 160, True, True)])
def test_fused_equals_quantizer_then_unfused(tokens, cin, grouped, same_order):
    """The fused kernel's sums equal the standalone quantizer's X_q fed to the two-tensor
    accumulation: bit for bit where both split the tokens alike (the 512-wide layer, grouped
    sums), else up to the fp32 summation order (the 4096-wide layer: clusters vs splits)."""
    if grouped:
        layer = synth.make_layer("moe", 33, tokens=tokens, cin=cin, rows=4, groups=10, top_k=3)
        layer.mode = "act"
        P.act_inputs(layer)
    else:
        layer = P.make_layer("act", 33, tokens=tokens, cin=cin, rows=4)
    d = P.layer_to_device(layer)
    G = layer.groups
    shape = (G, cin // 16, 16, 16)
    ws_bytes = max(L.lhcal_accumulate_workspace("act", L.BF16, tokens, cin, G),
                   L.lhcal_accumulate_act_quant_workspace(L.BF16, tokens, cin, G))
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device="cuda")
    hf, pf = (torch.full(shape, 1.0, device="cuda") for _ in range(2))
    L.lhcal_accumulate_act_quant(d["x"], hf, pf, d["act_gx"], group_offsets=d["offs"], token_ids=d["ids"],
                                 flags=L.ACCUM_OVERWRITE, workspace=ws)
    xq = torch.empty_like(d["x"])
    L.lhcal_act_fake_quant(d["x"], d["act_gx"], xq)
    hu, pu = (torch.full(shape, 2.0, device="cuda") for _ in range(2))
    L.lhcal_accumulate("act", d["x"], hu, xq=xq, p=pu, group_offsets=d["offs"], token_ids=d["ids"],
                       flags=L.ACCUM_OVERWRITE, workspace=ws)
    _sync()
    if same_order:
        assert torch.equal(hf.view(torch.int32), hu.view(torch.int32))
        assert torch.equal(pf.view(torch.int32), pu.view(torch.int32))
    else:
        P.check_hessians(hf.cpu().numpy(), hu.cpu().numpy().astype(np.float64), "fused vs unfused H", tol=1e-5)
        P.check_hessians(pf.cpu().numpy(), pu.cpu().numpy().astype(np.float64), "fused vs unfused P", tol=1e-5)
    # and the GPU quantizer's X_q is the oracle's
    np.testing.assert_array_equal(xq.cpu().view(torch.int16).numpy().view(np.uint16), layer.xq)


def test_fused_act_quant_rejects_fp32_and_missing_scale():
    x = torch.zeros((8, 32), dtype=torch.float32, device="cuda")
    h = torch.zeros((1, 2, 16, 16), device="cuda")
    p = torch.zeros_like(h)
    gx = torch.ones(1, device="cuda")
    with pytest.raises(L.LhcalError) as e:
        L.lhcal_accumulate_act_quant(x, h, p, gx, flags=L.ACCUM_OVERWRITE)
    assert e.value.status == L.ERR_UNSUPPORTED
    with pytest.raises(L.LhcalError) as e:
        L.lhcal_accumulate_act_quant(x.bfloat16(), h, p, None, flags=L.ACCUM_OVERWRITE)
    assert e.value.status == L.ERR_INVALID_ARG


# ----------------------------------------------------------------------------- mse, 4/6 scale, outputs

@pytest.mark.parametrize("name,kw", [("dense", dict(tokens=16, cin=272, rows=300)), ("tiny", dict()),
                                     ("moe", dict(tokens=16, cin=64, rows=40, groups=5, top_k=2))])
def test_mse_sweep(name, kw):
    """Plain block MSE (H = I): no statistics, the diagonal kernel with unit weights."""
    layer = synth.make_layer(name, 41, **kw)
    d = P.layer_to_device(layer)
    b = L.calibrate("mse", None, d["w"])
    _sync()
    assert b.h is None
    w32 = layer.w_f32()
    G, R, C = layer.groups, layer.rows, layer.cin
    g = np.array([O.global_scale(w32[e]) for e in range(G)], np.float32)
    np.testing.assert_array_equal(b.g.cpu().numpy().view(np.int32), g.view(np.int32))
    units = P.all_units(G, R, C // 16)
    ref = P.oracle_sweep("mse", w32, None, None, g, units)
    gc, gw, gl = P.gather_gpu_units(b.codes, b.wq, b.loss, units)
    P.check_sweep(gc, gw, gl, ref, f"{name} mse")


def test_mse_sweep_full_size_weights():
    layer = synth.make_layer("dense", 0, tokens=16)
    d = P.layer_to_device(layer)
    b = L.calibrate("mse", None, d["w"])
    _sync()
    w32 = layer.w_f32()
    g = np.array([O.global_scale(w32[0])], np.float32)
    units = P.sample_units(1, layer.rows, layer.cin // 16, 3000, seed=2)
    ref = P.oracle_sweep("mse", w32, None, None, g, units)
    gc, gw, gl = P.gather_gpu_units(b.codes, b.wq, b.loss, units)
    P.check_sweep(gc, gw, gl, ref, "dense mse full size")


@pytest.mark.parametrize("name", ["dense", "tiny", "moe"])
def test_global_scale_fp8_max(name):
    layer = synth.make_layer(name, 42, tokens=16, rows=64, cin=64, **({"groups": 7, "top_k": 2} if name == "moe" else {}))
    d = P.layer_to_device(layer)
    w32 = layer.w_f32()
    for fp8_max in (448.0, 256.0):
        g = torch.empty(layer.groups, dtype=torch.float32, device="cuda")
        L.lhcal_global_scale(d["w"], g, fp8_max=fp8_max)
        _sync()
        want = np.array([O.global_scale(w32[e], fp8_max) for e in range(layer.groups)], np.float32)
        np.testing.assert_array_equal(g.cpu().numpy().view(np.int32), want.view(np.int32))
    g = torch.empty(layer.groups, dtype=torch.float32, device="cuda")
    for bad in (0.0, 500.0, 1.0 / 3.0):
        with pytest.raises(L.LhcalError) as e:
            L.lhcal_global_scale(d["w"], g, fp8_max=bad)
        assert e.value.status == L.ERR_INVALID_ARG


@pytest.mark.parametrize("name,kw", [("dense", dict(tokens=400, cin=256, rows=96)), ("tiny", dict()),
                                     ("moe", dict(tokens=80, cin=96, rows=24, groups=6, top_k=2))])
def test_apply_scales_bit_exact(name, kw):
    """Fake-quantized weights (fp32, bf16) and per-block amax for the sweep's codes and for
    arbitrary codes (zero, every candidate, out of range), against the oracle."""
    layer = synth.make_layer(name, 43, **kw)
    d = P.layer_to_device(layer)
    mode = layer.mode
    b = L.calibrate(mode, d["x"], d["w"], group_offsets=d["offs"], token_ids=d["ids"])
    G, R, C = layer.groups, layer.rows, layer.cin
    rng = np.random.default_rng(7)
    crafted = rng.integers(0, 256, (G, R, C // 16)).astype(np.uint8)
    crafted.flat[:128] = np.arange(128, dtype=np.uint8)
    w32 = layer.w_f32()
    g_host = b.g.cpu().numpy()
    for codes in (b.codes, P.to_device(crafted, "i32").to(torch.uint8)):
        wq = torch.empty((G, R, C), dtype=torch.float32, device="cuda")
        wq16 = torch.empty((G, R, C), dtype=torch.bfloat16, device="cuda")
        amax = torch.empty((G, R, C // 16), dtype=torch.float32, device="cuda")
        L.lhcal_apply_scales(d["w"], b.g, codes, wq=wq, wq16=wq16, amax=amax)
        _sync()
        rw, rw16, ra = O.apply_scales(w32, g_host, codes.cpu().numpy())
        np.testing.assert_array_equal(wq.cpu().numpy().view(np.int32), rw.view(np.int32))
        np.testing.assert_array_equal(wq16.float().cpu().numpy().view(np.int32), rw16.view(np.int32))
        np.testing.assert_array_equal(amax.cpu().numpy().view(np.int32), ra.view(np.int32))
    # The sweep's own fake-quantized weights are the apply_scales output for its codes.
    wq = torch.empty((G, R, C), dtype=torch.float32, device="cuda")
    L.lhcal_apply_scales(d["w"], b.g, b.codes, wq=wq)
    _sync()
    assert torch.equal(wq.view(torch.int32), b.wq.view(torch.int32))


# ----------------------------------------------------------------------------- amax-multiplier search

@pytest.mark.parametrize("mode,name,kw", [
    ("full", "dense", dict(tokens=500, cin=96, rows=150)),
    ("act", "act", dict(tokens=400, cin=64, rows=130)),
    ("diag", "wmse", dict(tokens=300, cin=80, rows=140)),
    ("mse", "dense", dict(tokens=16, cin=48, rows=200)),
    ("full", "tiny", dict()),
    ("full", "moe", dict(tokens=60, cin=64, rows=40, groups=5, top_k=2)),
])
def test_multiplier_search(mode, name, kw):
    """Both sides get the oracle's finalized H (and P) rounded to fp32, the same global scales
    and multipliers 0.5, 0.55, ..., 2.0 (plus 0 and one that reaches the 448 saturation)."""
    layer = P.make_layer(name, 51, **kw)
    G, R, C = layer.groups, layer.rows, layer.cin
    w32 = layer.w_f32()
    g = np.array([O.global_scale(w32[e]) for e in range(G)], np.float32)
    h = p = None
    if mode != "mse":
        xq = layer.xq_f32() if mode == "act" else None
        hs, ps, counts = O.accumulate(mode, layer.x_f32(), xq, layer.group_offsets, layer.token_ids)
        h, p = O.finalize(mode, hs, ps, counts)
        h = h.astype(np.float32).astype(np.float64)
        p = None if p is None else p.astype(np.float32).astype(np.float64)
    mult = np.concatenate([np.arange(0.5, 2.0001, 0.05), [0.0, 5000.0]]).astype(np.float32)
    d = P.layer_to_device(layer)
    codes = torch.empty((G, R, C // 16), dtype=torch.uint8, device="cuda")
    wq = torch.empty((G, R, C), dtype=torch.float32, device="cuda")
    loss = torch.empty((G, R, C // 16), dtype=torch.float32, device="cuda")
    L.lhcal_multiplier_search(mode, d["w"], None if h is None else P.to_device(h, "f32"), P.to_device(g, "f32"),
                              P.to_device(mult, "f32"), codes, wq=wq, loss=loss,
                              p=None if p is None else P.to_device(p, "f32"))
    _sync()
    units = P.all_units(G, R, C // 16)
    ref = P.oracle_multiplier_search(mode, w32, h, p, g, mult, units)
    gc, gw, gl = P.gather_gpu_units(codes, wq, loss, units)
    rep = P.check_sweep(gc, gw, gl, ref, f"{name} {mode} multiplier search")
    assert rep["units"] == len(units)
    # Optional outputs: codes alone give the same codes.
    codes2 = torch.empty_like(codes)
    L.lhcal_multiplier_search(mode, d["w"], None if h is None else P.to_device(h, "f32"), P.to_device(g, "f32"),
                              P.to_device(mult, "f32"), codes2, p=None if p is None else P.to_device(p, "f32"))
    _sync()
    assert torch.equal(codes, codes2)


def test_multiplier_search_rejects_bad_counts():
    w = torch.zeros((1, 4, 32), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(1, device="cuda")
    codes = torch.empty((1, 4, 2), dtype=torch.uint8, device="cuda")
    for n in (0, 1025):
        m = torch.ones(max(n, 1), device="cuda")
        lib = L.load_library()
        st = lib.lhcal_multiplier_search(3, 1, L._ptr(w), 1, 4, 32, None, None, L._ptr(g), L._ptr(m), n,
                                         L._ptr(codes), None, None, None)
        assert st == L.ERR_INVALID_ARG


# ----------------------------------------------------------------------------- host path

@pytest.mark.parametrize("name,kw,chunks", [
    ("dense", dict(tokens=500, cin=128, rows=64), 8),
    ("dense", dict(tokens=500, cin=128, rows=300), 8),  # row chunks 0, 128, 256, 300
    ("moe", dict(tokens=300, cin=96, rows=24, groups=20, top_k=3), 8),
    ("moe", dict(tokens=300, cin=96, rows=24, groups=20, top_k=3), 3),
    ("moe", dict(tokens=300, cin=96, rows=24, groups=20, top_k=3), None),  # chunks sized by bytes
    ("act", dict(tokens=300, cin=64, rows=40), 8),
    ("act", dict(tokens=300, cin=64, rows=520), 2),  # row chunks 0, 256, 520
    ("wmse", dict(tokens=200, cin=64, rows=260), 8),
    ("mse", dict(), 1),
])
def test_calibrate_host_matches_the_device_path(name, kw, chunks):
    """calibrate_host (pinned host inputs; grouped layers pipelined over chunks of groups, one-group
    layers over chunks of rows, on side streams) returns exactly the codes, global scales, losses
    and fake-quantized weights (fp32, and bf16 when the buffers hold them) of calibrate."""
    mse = name == "mse"
    layer = P.make_layer("dense" if mse else name, 61, **(dict(tokens=16, cin=64, rows=48) if mse else kw))
    mode = "mse" if mse else layer.mode
    d = P.layer_to_device(layer)
    fused = mode == "act"
    ref = L.calibrate(mode, d["x"], d["w"], group_offsets=d["offs"], token_ids=d["ids"],
                      act_gx=d["act_gx"] if fused else None, xq=None)
    wq16 = torch.empty(ref.wq.shape, dtype=torch.bfloat16, device="cuda")
    L.lhcal_apply_scales(d["w"], ref.g, ref.codes, wq16=wq16)
    _sync()
    want = (ref.codes.cpu(), ref.loss.cpu(), ref.wq.cpu(), ref.g.cpu(), wq16.cpu())
    staging = {k: (torch.empty_like(v) if isinstance(v, torch.Tensor) else None) for k, v in d.items()}
    pin = lambda t: None if t is None else t.cpu().pin_memory()  # noqa: E731
    xdt = L.BF16 if layer.dtype == "bf16" else L.F32
    buf = L.Buffers(mode, layer.tokens, layer.cin, layer.rows, layer.groups, xdt, "cuda")
    args = dict(group_offsets=pin(d["offs"]), token_ids=pin(d["ids"]), act_gx=d["act_gx"] if fused else None,
                group_chunks=chunks, row_chunks=chunks or 8)
    out = L.calibrate_host(mode, pin(d["x"]), pin(d["w"]), buf, staging, **args)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(out.codes, want[0])
    assert torch.equal(out.loss.view(torch.int32), want[1].view(torch.int32))
    assert torch.equal(out.wq.view(torch.int32), want[2].view(torch.int32))
    assert torch.equal(out.g.view(torch.int32), want[3].view(torch.int32))
    out2 = L.calibrate_host(mode, pin(d["x"]), pin(d["w"]), buf, staging, out=L.HostOutputs(buf, want_wq=False),
                            **args)
    torch.cuda.current_stream().synchronize()
    assert out2.wq is None and torch.equal(out2.codes, want[0])
    # The bf16 fake-quantized weights, without the fp32 ones (what the e2e measurement copies out).
    buf16 = L.Buffers(mode, layer.tokens, layer.cin, layer.rows, layer.groups, xdt, "cuda", want_wq=False,
                      want_wq16=True)
    out3 = L.calibrate_host(mode, pin(d["x"]), pin(d["w"]), buf16, staging, out=L.HostOutputs(buf16), **args)
    torch.cuda.current_stream().synchronize()
    assert out3.wq is None and torch.equal(out3.codes, want[0])
    assert torch.equal(out3.wq16.view(torch.int16), want[4].view(torch.int16))


@pytest.mark.slow
def test_dense_whole_layer_every_unit():
    """All 1,048,576 units of the dense workload (X [16384, 4096], W [4096, 4096]) against the
    oracle, not a sample: codes and Wq bit-exact outside near-ties, near-ties within the oracle's
    tie set, every winning loss within 1e-4. The oracle runs in spawned worker processes."""
    layer = P.make_layer("dense", 0)
    d = synth.layer_to_device(layer)
    b = L.calibrate("full", d["x"], d["w"])
    _sync()
    hs, _, counts = O.accumulate("full", layer.x_f32())
    h, _ = O.finalize("full", hs, None, counts)
    P.check_hessians(b.h.cpu().numpy(), h, "dense whole-layer H")
    w32 = layer.w_f32()
    g = np.array([O.global_scale(w32[0])], np.float32)
    ref = P.oracle_sweep_parallel("full", w32, h, None, g)
    rep = P.check_sweep(b.codes.cpu().numpy().reshape(-1), b.wq.cpu().numpy().reshape(-1, 16),
                        b.loss.cpu().numpy().reshape(-1), ref, "dense whole layer")
    assert rep["units"] == 4096 * 256
    print("dense whole layer:", rep)


def test_sweep_hessian_with_2e20_diagonal_dynamic_range():
    """The tensor-core sweep scales H by a power of two into fp16 range and splits it into fp16
    hi + lo: entries far below the largest keep an absolute accuracy (the lo part reaches fp16
    subnormals), not a relative one. A block Hessian whose diagonal spans 2^0 .. 2^20, with
    off-diagonal coupling, against the oracle in FULL and activation-aware modes."""
    rng = np.random.default_rng(12)
    G, R, C = 1, 256, 64
    nblk = C // 16
    w = (rng.normal(0, 0.05, (G, R, C)) * np.exp2(rng.uniform(-6, 0, (G, R, C)))).astype(np.float32)
    scale = np.exp2(np.linspace(0, 20, 16))  # the diagonal's dynamic range: 2^20
    h = np.zeros((G, nblk, 16, 16))
    p = np.zeros((G, nblk, 16, 16))
    for n in range(nblk):
        a = rng.normal(size=(16, 16)) * np.sqrt(scale)[:, None] * 0.2
        h[0, n] = np.diag(scale[rng.permutation(16)]) + a @ a.T / 16
        p[0, n] = 0.01 * rng.normal(size=(16, 16)) * np.sqrt(np.outer(np.diag(h[0, n]), np.diag(h[0, n])))
    h32, p32 = h.astype(np.float32), p.astype(np.float32)
    g = np.array([O.global_scale(w[0])], np.float32)
    for mode, pp in (("full", None), ("act", p32)):
        codes, wq, loss = _sweep_gpu(L.MODE_IDS[mode], w, h32, pp, g)
        units = P.all_units(G, R, nblk)
        ref = P.oracle_sweep(mode, w, h32.astype(np.float64), None if pp is None else pp.astype(np.float64), g, units)
        gc, gw, gl = P.gather_gpu_units(codes, wq, loss, units)
        rep = P.check_sweep(gc, gw, gl, ref, f"2^20 dynamic range {mode}")
        assert rep["units"] == R * nblk


# ----------------------------------------------------------------------------- more edge cases (2)

def test_fused_act_quant_grouped_with_empty_experts():
    """20 tokens routed to 2 of 16 experts each: most experts get no token and fall back to
    H = I, P = 0 after finalisation; their raw sums must be exact zeros."""
    layer = synth.make_layer("moe", 71, tokens=20, cin=48, rows=16, groups=16, top_k=2)
    assert np.any(np.diff(layer.group_offsets) == 0)
    layer.mode = "act"
    P.act_inputs(layer)
    _run_and_check(layer, fused=True)


@pytest.mark.parametrize("n_mult", [1, 1024])
def test_multiplier_search_counts(n_mult):
    layer = P.make_layer("dense", 72, tokens=300, cin=64, rows=50)
    G, R, C = layer.groups, layer.rows, layer.cin
    w32 = layer.w_f32()
    g = np.array([O.global_scale(w32[0])], np.float32)
    hs, _, counts = O.accumulate("full", layer.x_f32())
    h, _ = O.finalize("full", hs, None, counts)
    h = h.astype(np.float32).astype(np.float64)
    mult = (np.float32([1.0]) if n_mult == 1 else np.linspace(0.01, 3.0, n_mult).astype(np.float32))
    d = P.layer_to_device(layer)
    codes = torch.empty((G, R, C // 16), dtype=torch.uint8, device="cuda")
    wq = torch.empty((G, R, C), dtype=torch.float32, device="cuda")
    loss = torch.empty((G, R, C // 16), dtype=torch.float32, device="cuda")
    L.lhcal_multiplier_search("full", d["w"], P.to_device(h, "f32"), P.to_device(g, "f32"), P.to_device(mult, "f32"),
                              codes, wq=wq, loss=loss)
    _sync()
    units = P.all_units(G, R, C // 16)
    ref = P.oracle_multiplier_search("full", w32, h, None, g, mult, units)
    gc, gw, gl = P.gather_gpu_units(codes, wq, loss, units)
    P.check_sweep(gc, gw, gl, ref, f"multiplier search, {n_mult} multipliers")


def test_golden_sweep_winners_on_the_gpu():
    """The hand-derived sweep winners of tests/golden (plain block MSE, one block per group, each
    group with its own g): the CUDA sweep returns the same codes, zero losses and Wq = W."""
    from tests import test_golden as G

    cases = G._cases()["sweep"]
    gs, ws, want = [], [], []
    for rest in cases:
        lhs, rhs = rest.split("->")
        vals = lhs.split()
        gs.append(np.float32(vals[0]))
        ws.append(np.array([float(v) for v in vals[1:]], np.float32))
        code, loss = rhs.split()
        want.append((int(code, 16), float(loss)))
    n = len(cases)
    w = P.to_device(np.stack(ws)[:, None, :], "f32")  # [groups, 1 row, 16]
    g = P.to_device(np.array(gs, np.float32), "f32")
    codes = torch.empty((n, 1, 1), dtype=torch.uint8, device="cuda")
    wq = torch.empty((n, 1, 16), dtype=torch.float32, device="cuda")
    loss = torch.empty((n, 1, 1), dtype=torch.float32, device="cuda")
    L.lhcal_scale_sweep("mse", w, None, g, codes, wq=wq, loss=loss)
    _sync()
    assert codes.flatten().tolist() == [c for c, _ in want]
    assert loss.flatten().tolist() == [v for _, v in want]
    np.testing.assert_array_equal(wq.cpu().numpy().reshape(n, 16).view(np.int32), np.stack(ws).view(np.int32))



@pytest.mark.parametrize("name,kw", [
    ("dense", dict(tokens=700, cin=256, rows=300)),
    ("act", dict(tokens=500, cin=128, rows=130)),
    ("moe", dict(tokens=300, cin=128, rows=40, groups=9, top_k=3)),
])
def test_sharded_path_on_one_nccl_rank_equals_calibrate(name, kw):
    """scale_calibration_lh_b200.sharded (token-sharded statistics, all-reduce, row-sharded sweep,
    all-gather) run by one NCCL rank through the C ABI: every collective is then an identity, so
    the results equal calibrate()'s bit for bit. The partition and reductions over two ranks are
    covered on the CPU (tests/test_sharded_cpu.py)."""
    import torch.distributed as dist

    from scale_calibration_lh_b200 import sharded as S

    layer = P.make_layer(name, 23, **kw)
    d = synth.layer_to_device(layer)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        b, res = S.calibrate_sharded(layer.mode, d["x"], d["w"], group_offsets=d["offs"], token_ids=d["ids"],
                                     act_gx=None)
        ref = L.calibrate(layer.mode, d["x"], d["w"], group_offsets=d["offs"], token_ids=d["ids"],
                          act_gx=d["act_gx"] if name == "act" else None)
        _sync()
    finally:
        dist.destroy_process_group()
    for k in ("h", "p", "counts", "g"):
        if getattr(ref, k) is not None:
            assert torch.equal(getattr(b, k), getattr(ref, k)), k
    assert torch.equal(res["codes"], ref.codes) and torch.equal(res["loss"], ref.loss)
    assert torch.equal(res["wq"].view(torch.int32), ref.wq.view(torch.int32))
