"""Pins for the CPU oracle: format facts, closed forms, brute force and invariants.

Each test ties the oracle to something other than itself: a library's own
number-format conversion, exact rational arithmetic, an identity the pages
state, or a brute-force evaluation on a tiny input.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import lhcal_oracle as O

E2M1 = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]


# --------------------------------------------------------------------------- formats

def test_e4m3_candidates_match_torch_float8():
    codes = O.candidate_codes()
    assert len(codes) == 126 and codes[0] == 1 and codes[-1] == 0x7E
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(O.e4m3_value(codes), lib[codes])
    v = O.e4m3_value(codes)
    assert np.all(np.diff(v) > 0)
    assert v[0] == 2.0 ** -9 and v[-1] == 448.0
    # The set is every positive finite non-zero E4M3 value.
    finite = lib[np.isfinite(lib) & (lib > 0)]
    assert sorted(finite.tolist()) == v.tolist()


@pytest.mark.parametrize("u,q", [(0.25, 0), (0.75, 1), (1.25, 1), (1.75, 2), (2.5, 2), (3.5, 4), (5.0, 4),
                                 (6.0, 6), (7.0, 6), (100.0, 6), (0.0, 0), (0.2499, 0), (0.2501, 0.5)])
def test_e2m1_midpoints_ties_to_even(u, q):
    assert O.e2m1_round(np.array([u]))[0] == q


def test_e2m1_matches_ml_dtypes_on_fp32_values():
    rng = np.random.default_rng(1)
    u = np.concatenate([rng.uniform(0, 8, 200000), np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])])
    u = u.astype(np.float32)
    lib = u.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(O.e2m1_round(u.astype(np.float64)), lib)


def _fq_exact(w: float, s: float) -> float:
    """Fake quant by exact rationals: nearest grid point to |w|/s, ties to even code."""
    if s == 0:
        return float(np.copysign(0.0, w))
    u = min(Fraction(abs(w)) / Fraction(s), Fraction(6))
    d = [abs(u - g) for g in E2M1]
    m = min(d)
    idx = [i for i, x in enumerate(d) if x == m]
    i = idx[0] if len(idx) == 1 else [j for j in idx if j % 2 == 0][0]
    mag = np.float32(float(E2M1[i] * Fraction(s)))  # exact product rounded once to fp32
    return float(np.copysign(mag, w))


def test_fake_quant_exact_ties_and_neighbours():
    # s with few mantissa bits so m * s is an exact fp32 midpoint.
    rng = np.random.default_rng(2)
    ws, ss = [], []
    for s in (np.float32(0.0078125), np.float32(3.0 * 2 ** -12), np.float32(0.1)):
        for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
            t = np.float32(m * float(s))
            for w in (t, np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(1))):
                for sign in (1, -1):
                    ws.append(np.float32(sign * w))
                    ss.append(s)
    ws += list(rng.normal(0, 0.05, 2000).astype(np.float32))
    ss += list(np.float32(rng.uniform(1e-4, 1e-2, 2000)))
    ws, ss = np.array(ws, np.float32), np.array(ss, np.float32)
    got = O.fake_quant(ws, ss)
    want = np.array([_fq_exact(float(w), float(s)) for w, s in zip(ws, ss)], np.float32)
    np.testing.assert_array_equal(got.view(np.int32), want.view(np.int32))


def test_fake_quant_negative_zero_and_zero_scale():
    out = O.fake_quant(np.array([-1e-6, 1e-6, -0.5], np.float32), np.float32(1.0))
    assert out.view(np.int32)[0] == np.float32(-0.0).view(np.int32)
    assert out[1] == 0.0 and out[2] == -0.5
    z = O.fake_quant(np.array([0.3, -0.3], np.float32), np.float32(0.0))
    assert z.view(np.int32).tolist() == [0, np.float32(-0.0).view(np.int32)]


def test_global_scale_is_448_normalized():
    w = np.array([[0.5, -1.75, 0.25]], np.float32)
    assert O.global_scale(w) == np.float32(1.75 / 2688.0)
    s = O.candidate_scales(O.global_scale(w))
    # The largest candidate maps amax onto the top of the FP4 grid: 448 * g * 6 ~ amax.
    assert abs(float(s[-1]) * 6 - 1.75) < 1e-6
    assert O.global_scale(np.zeros((2, 3), np.float32)) == 0.0


# --------------------------------------------------------------------------- activation fake quant

E4M3_ALL = [Fraction(0)] + [Fraction(float(v)) for v in O.e4m3_value(O.candidate_codes())]


def _round_binary(y: Fraction, bits: int, emin: int) -> Fraction:
    """Round y >= 0 to `bits` significant bits (exponents below emin: fixed ulp), half to even."""
    if y == 0:
        return y
    e = y.numerator.bit_length() - y.denominator.bit_length()
    if Fraction(2) ** e > y:
        e -= 1
    ulp = Fraction(2) ** (max(e, emin) - (bits - 1))
    return round(y / ulp) * ulp  # Fraction.__round__ rounds half to even


def _e4m3_code_brute(r: Fraction) -> int:
    """Nearest of all 127 non-negative finite E4M3 values, ties to the even code; > 448 -> 448."""
    if r > 448:
        return 126
    return min(range(127), key=lambda k: (abs(E4M3_ALL[k] - r), k % 2))


def _act_quant_brute(block, gx) -> list:
    """One 16-value block by exact rationals and exhaustive nearest-value searches."""
    g = Fraction(float(np.float32(gx)))
    amax = max(abs(Fraction(float(v))) for v in block)
    code = _e4m3_code_brute(amax / (6 * g)) if g > 0 else 0
    s = _round_binary(E4M3_ALL[code] * g, 24, -126)
    out = []
    for v in block:
        a = abs(Fraction(float(v)))
        i = min(range(8), key=lambda j: (abs(E2M1[j] * s - a), j % 2))
        mag = _round_binary(_round_binary(E2M1[i] * s, 24, -126), 8, -126)
        out.append(float(np.copysign(float(mag), float(v))))
    return out


def _bf16_values(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def test_e4m3_round_brute_force_and_library():
    rng = np.random.default_rng(11)
    vals = np.array([float(v) for v in E4M3_ALL])
    mids = (vals[:-1] + vals[1:]) / 2
    r = np.concatenate([rng.uniform(0, 460, 3000), np.exp2(rng.uniform(-14, 9, 3000)), vals, mids,
                        np.nextafter(mids, 0), np.nextafter(mids, 1e9), [0.0, 2.0 ** -10, 448.0, 463.9, 500.0, 1e30]])
    got = O.e4m3_round(r)
    want = np.array([_e4m3_code_brute(Fraction(float(v))) for v in r])
    np.testing.assert_array_equal(got, want)
    # ml_dtypes' float8_e4m3fn conversion (nearest, ties to even) agrees below its NaN range.
    ok = r < 464
    lib = r[ok].astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    exact32 = r[ok] == r[ok].astype(np.float32)  # compare where the fp32 cast loses nothing
    np.testing.assert_array_equal(got[ok][exact32], lib[exact32])


@pytest.mark.parametrize("gx_factor", [1.0, 1e-3, 1e3, 0.0])
def test_act_fake_quant_brute_force(gx_factor):
    rng = np.random.default_rng(12)
    sig = np.exp(rng.normal(0, 1.5, 64))
    sig[[3, 40]] *= 20
    x = _bf16_values(rng.normal(size=(5, 64)) * sig)
    x[1, 16:32] = 0.0  # an all-zero block
    x[2, 0:16] = -0.0
    x[3, 32:48] *= 1e-30  # a tiny block: small and subnormal scale codes
    gx = np.float32(O.global_scale(x) * gx_factor)
    got = O.act_fake_quant(x, gx)
    want = np.array([_act_quant_brute(x[t, 16 * n:16 * n + 16], gx) for t in range(5) for n in range(4)],
                    np.float32).reshape(5, 4, 16).reshape(5, 64)
    np.testing.assert_array_equal(got.view(np.int32), want.view(np.int32))
    assert np.all(got == _bf16_values(got))  # bf16-exact values


def test_act_fake_quant_hand_worked_ties():
    # gx = 1: amax 6.375 -> 6.375 / 6 = 1.0625, midway between E4M3 1.0 (0x38) and 1.125 (0x39):
    # the even code wins, s = 1.0. amax 7.125 -> 1.1875, midway between 1.125 (0x39) and
    # 1.25 (0x3A): s = 1.25. With s = 1.25 every E2M1 midpoint m * 1.25 is bf16-exact.
    blk_a = np.zeros(16, np.float32)
    blk_a[0], blk_a[1], blk_a[2] = 6.375, -0.75, 0.25
    blk_b = np.array([7.125, 0.3125, 0.9375, 1.5625, 2.1875, 3.125, 4.375, 6.25,
                      -0.3125, -0.9375, -1.5625, -2.1875, -3.125, -4.375, -6.25, 0.0], np.float32)
    x = np.stack([np.concatenate([blk_a, blk_b])])
    got = O.act_fake_quant(x, np.float32(1.0))[0]
    # s = 1.0: 6.375 -> 6 (clamped), 0.75 -> tie 0.5 | 1 -> 1, 0.25 -> tie 0 | 0.5 -> 0.
    assert got[:3].tolist() == [6.0, -1.0, 0.0]
    # s = 1.25: ties go to the even E2M1 code: .25->0, .75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4.
    want_b = [7.5, 0.0, 1.25, 1.25, 2.5, 2.5, 5.0, 5.0, -0.0, -1.25, -1.25, -2.5, -2.5, -5.0, -5.0, 0.0]
    np.testing.assert_array_equal(got[16:].view(np.int32), np.array(want_b, np.float32).view(np.int32))


def test_act_fake_quant_saturates_and_zero_global_scale():
    x = np.full((1, 16), 3.0, np.float32)
    # gx so small that amax / (6 gx) is far above 448: the code saturates at 448 and every
    # value lands on the top of the grid at s = fp32(448 gx): 6 * s.
    gx = np.float32(1e-6)
    s = np.float32(448.0 * np.float64(gx))
    np.testing.assert_array_equal(O.act_fake_quant(x, gx), _bf16_values(np.full((1, 16), np.float32(6 * np.float64(s)))))
    assert np.all(O.act_fake_quant(x, np.float32(0.0)) == 0.0)


# --------------------------------------------------------------------------- Hessians

def _tiny_x(t=7, c=32, seed=3):
    return np.random.default_rng(seed).normal(size=(t, c)).astype(np.float32)


def test_full_hessian_brute_force():
    x = _tiny_x()
    h = O.hessian_sum_full(x)
    for n in range(2):
        for i in range(16):
            for j in range(16):
                ref = sum(Fraction(float(x[t, 16 * n + i])) * Fraction(float(x[t, 16 * n + j])) for t in range(x.shape[0]))
                assert abs(h[n, i, j] - float(ref)) <= 1e-12 * max(1.0, abs(float(ref)))


def test_act_hessians_brute_force_and_properties():
    x = _tiny_x(9, 32, 4)
    xq = (x + np.random.default_rng(5).normal(0, 0.1, x.shape)).astype(np.float32)
    h, p = O.hessian_sum_act(x, xq)
    for n, i, j in [(0, 0, 0), (0, 3, 11), (1, 15, 2), (1, 7, 7)]:
        refh = sum(float(xq[t, 16 * n + i]) * float(xq[t, 16 * n + j]) for t in range(9))
        refp = sum(float(xq[t, 16 * n + i]) * (float(xq[t, 16 * n + j]) - float(x[t, 16 * n + j])) for t in range(9))
        assert abs(h[n, i, j] - refh) < 1e-12 and abs(p[n, i, j] - refp) < 1e-12
    assert not np.allclose(p, p.transpose(0, 2, 1))  # P is not symmetric: its index order matters
    h0, p0 = O.hessian_sum_act(x, x)
    assert np.all(p0 == 0.0)
    np.testing.assert_array_equal(h0, O.hessian_sum_full(x))


def test_hessian_symmetric_psd_and_diag_is_importance():
    x = _tiny_x(40, 64, 6)
    h = O.hessian_sum_full(x)
    np.testing.assert_array_equal(h, h.transpose(0, 2, 1))
    ev = np.linalg.eigvalsh(h)
    assert ev.min() >= -1e-12 * np.abs(ev).max()
    np.testing.assert_allclose(np.diagonal(h, axis1=1, axis2=2), O.importance_sum(x), rtol=1e-14)


def test_grouped_accumulate_and_zero_group_fallback():
    x = _tiny_x(12, 32, 7)
    off = np.array([0, 3, 3, 8], np.int32)
    ids = np.array([0, 5, 11, 1, 2, 3, 4, 9], np.int32)
    h, _, counts = O.accumulate("full", x, group_offsets=off, token_ids=ids)
    assert counts.tolist() == [3, 0, 5]
    np.testing.assert_array_equal(h[0], O.hessian_sum_full(x[[0, 5, 11]]))
    np.testing.assert_array_equal(h[2], O.hessian_sum_full(x[[1, 2, 3, 4, 9]]))
    assert np.all(h[1] == 0)
    hf, _ = O.finalize("full", h, None, counts)
    np.testing.assert_array_equal(hf[1], np.broadcast_to(np.eye(16), (2, 16, 16)))
    np.testing.assert_allclose(hf[2], h[2] / 5.0, rtol=1e-15)
    hd, _, cd = O.accumulate("diag", x, group_offsets=off, token_ids=ids)
    hdf, _ = O.finalize("diag", hd, None, cd)
    assert np.all(hdf[1] == 1.0)
    np.testing.assert_array_equal(hdf[0], hd[0])  # importance stays a raw sum


def test_grouped_calibrate_is_each_expert_on_its_own():
    """A grouped layer is its experts calibrated one by one: each on its routed rows (PR #2864 /
    #2840), with a global scale from its own weights, since every expert has its own weight
    quantizer. Expert 1 gets no token and falls back to H = I."""
    rng = np.random.default_rng(15)
    x = rng.normal(size=(20, 32)).astype(np.float32)
    w = (rng.normal(0, 0.05, (3, 4, 32)) * np.array([1.0, 7.0, 0.2])[:, None, None]).astype(np.float32)
    off = np.array([0, 6, 6, 13], np.int32)
    ids = np.concatenate([np.sort(rng.permutation(20)[:6]), np.sort(rng.permutation(20)[:7])]).astype(np.int32)
    out = O.calibrate("full", x, w, group_offsets=off, token_ids=ids)
    per = 4 * 2  # units per expert: rows x blocks
    for e in range(3):
        one = O.calibrate("full", x[ids[off[e]:off[e + 1]]], w[e:e + 1])
        assert out["g"][e] == one["g"][0] == O.global_scale(w[e])
        np.testing.assert_array_equal(out["h"][e], one["h"][0])
        sl = slice(e * per, (e + 1) * per)
        np.testing.assert_array_equal(out["codes"][sl], one["codes"])
        np.testing.assert_array_equal(out["wq"][sl].view(np.int32), one["wq"].view(np.int32))
        np.testing.assert_array_equal(out["loss"][sl], one["loss"])
    assert len(set(out["g"].tolist())) == 3
    np.testing.assert_array_equal(out["h"][1], np.broadcast_to(np.eye(16), (2, 16, 16)))


# --------------------------------------------------------------------------- losses and sweep

def _layer(seed, rows=6, cin=16, t=64):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(t, cin)).astype(np.float32) * rng.lognormal(0, 1, cin).astype(np.float32)
    w = rng.normal(0, 0.05, (1, rows, cin)).astype(np.float32)
    return x, w


def test_act_expanded_loss_equals_output_mse_including_negative():
    """On one block (cin = 16): L_k + w^T D^T D w / B == ||X_q wq_k - X w||^2 / B for every k."""
    x, w = _layer(8, rows=1)
    t = x.shape[0]
    g = O.global_scale(w[0])
    s = O.candidate_scales(g)
    # X_q = 0.9 X and w chosen so that one candidate's quantized weights equal w / 0.9:
    # the output error then vanishes and the expanded objective is negative there.
    k0 = 100
    qv = np.array([6, 4, 3, 2, 1.5, 1, 0.5, 6, 4, 3, 2, 1.5, 1, 0.5, 6, 4], np.float64)
    sign = np.where(np.arange(16) % 3 == 0, -1.0, 1.0)
    wrow = (0.9 * qv * float(s[k0]) * sign).astype(np.float32)
    xq = (0.9 * x.astype(np.float64)).astype(np.float32)
    for wr in (w[0, 0], wrow):
        hs, ps = O.hessian_sum_act(x, xq)
        h, p = hs[0] / t, ps[0] / t
        loss, wq, _ = O.candidate_losses("act", wr[None], h[None], p[None], g)
        d = xq.astype(np.float64) - x.astype(np.float64)
        const = float(np.sum((d @ wr.astype(np.float64)) ** 2)) / t
        for k in range(126):
            out = xq.astype(np.float64) @ wq[0, k].astype(np.float64) - x.astype(np.float64) @ wr.astype(np.float64)
            mse = float(np.sum(out ** 2)) / t
            assert abs(loss[0, k] + const - mse) <= 1e-9 * max(mse, const, 1e-30)
    assert loss[0, k0] < 0  # the deliberately negative objective of the last row


def test_act_with_xq_equal_x_is_local_hessian():
    x, w = _layer(9, rows=20, cin=48)
    full = O.calibrate("full", x, w)
    act = O.calibrate("act", x, w, xq=x)
    np.testing.assert_array_equal(full["codes"], act["codes"])
    np.testing.assert_array_equal(full["wq"].view(np.int32), act["wq"].view(np.int32))
    np.testing.assert_array_equal(full["loss"], act["loss"])


def test_wmse_equals_full_with_diagonal_hessian():
    x, w = _layer(10, rows=20, cin=48)
    d = O.calibrate("diag", x, w)
    imp = O.importance_sum(x)[None]
    hdiag = np.zeros((1, imp.shape[1], 16, 16))
    hdiag[0, :, np.arange(16), np.arange(16)] = imp[0].T
    f = O.sweep("full", w, hdiag, None, d["g"])
    np.testing.assert_array_equal(f["codes"], d["codes"])
    np.testing.assert_allclose(f["loss"], d["loss"], rtol=1e-13)


def test_identity_hessian_is_plain_block_mse_by_exact_rationals():
    _, w = _layer(11, rows=3, cin=16)
    g = O.global_scale(w[0])
    s = O.candidate_scales(g)
    h = np.eye(16)[None].repeat(3, 0)
    loss, _, _ = O.candidate_losses("full", w[0], h, None, g)
    for r in range(3):
        for k in range(0, 126, 5):
            ref = sum((Fraction(_fq_exact(float(wi), float(s[k]))) - Fraction(float(wi))) ** 2 for wi in w[0, r])
            assert abs(loss[r, k] - float(ref)) <= 1e-12 * float(ref)


def test_mse_mode_is_plain_block_mse_by_exact_rationals_and_equals_identity_hessian():
    _, w = _layer(12, rows=4, cin=32)
    g = O.global_scale(w[0])
    s = O.candidate_scales(g)
    wb = w[0].reshape(8, 16)
    loss, _, e0 = O.candidate_losses("mse", wb, None, None, g)
    for u in range(0, 8, 3):
        for k in range(0, 126, 7):
            ref = sum((Fraction(_fq_exact(float(wi), float(s[k]))) - Fraction(float(wi))) ** 2 for wi in wb[u])
            assert abs(loss[u, k] - float(ref)) <= 1e-12 * float(ref)
        assert e0[u] == pytest.approx(float(sum(Fraction(float(v)) ** 2 for v in wb[u])), rel=1e-14)
    a = O.sweep("mse", w, None, None, np.array([g], np.float32))
    b = O.sweep("full", w, np.eye(16)[None, None].repeat(2, 1), None, np.array([g], np.float32))
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["wq"].view(np.int32), b["wq"].view(np.int32))


def test_global_scale_four_over_six_is_256_normalized():
    w = np.array([[0.5, -1.75, 0.25]], np.float32)
    assert O.global_scale(w, 256.0) == np.float32(1.75 / 1536.0)
    assert O.global_scale(w) == O.global_scale(w, 448.0) == np.float32(1.75 / 2688.0)


def test_apply_scales_matches_the_sweep_and_exact_amax():
    _, w = _layer(13, rows=6, cin=48)
    g = np.array([O.global_scale(w[0])], np.float32)
    out = O.sweep("mse", w, None, None, g)
    codes = out["codes"].reshape(1, 6, 3).astype(np.int64)
    codes[0, 0, 0] = 0    # zero scale: every weight becomes +-0
    codes[0, 1, 1] = 200  # above 126: taken as 126
    wq, wq16, amax = O.apply_scales(w, g, codes)
    ref = out["wq"].reshape(1, 6, 3, 16).copy()
    ref[0, 0, 0] = np.copysign(np.float32(0.0), w[0, 0, :16])
    ref[0, 1, 1] = O.fake_quant(w[0, 1, 16:32], O.candidate_scales(g[0])[125])
    np.testing.assert_array_equal(wq.view(np.int32), ref.reshape(1, 6, 48).view(np.int32))
    gq = Fraction(float(g[0]))
    for r in range(6):
        for n in range(3):
            c = min(int(codes[0, r, n]), 126)
            exact = 6 * E4M3_ALL[c] * gq
            assert amax[0, r, n] == np.float32(float(_round_binary(exact, 24, -126)))
            for i in range(0, 16, 5):
                v = Fraction(float(wq[0, r, 16 * n + i]))
                mag = float(_round_binary(abs(v), 8, -126))
                assert wq16[0, r, 16 * n + i] == np.copysign(mag, float(wq[0, r, 16 * n + i]))


def test_sweep_is_exhaustive_lowest_code_on_ties():
    x, w = _layer(12, rows=8, cin=32)
    hs, _, c = O.accumulate("full", x)
    h, _ = O.finalize("full", hs, None, c)
    g = np.array([O.global_scale(w[0])], np.float32)
    out = O.sweep("full", w, h, None, g)
    losses = O.sweep("full", w, h, None, g)["all_losses"] if "all_losses" in out else None
    for u, (r, n) in enumerate([(r, n) for r in range(8) for n in range(2)]):
        wb = w[0, r, 16 * n:16 * n + 16]
        all_l, _, _ = O.candidate_losses("full", wb[None], h[0, n][None], None, g[0])
        brute = min(range(126), key=lambda k: (all_l[0, k], k))
        assert out["codes"][u] == brute + 1
        assert out["loss"][u] == all_l[0, brute]
    assert losses is None or losses.shape[1] == 126
    # An all-zero block ties every candidate: code 1 wins.
    w0 = w.copy()
    w0[0, 0, :16] = 0
    z = O.sweep("full", w0, h, None, g)
    assert z["codes"][0] == 1 and z["loss"][0] == 0.0


def test_sweep_invariances():
    x, w = _layer(13, rows=16, cin=32)
    hs, _, c = O.accumulate("full", x)
    h, _ = O.finalize("full", hs, None, c)
    g = np.array([O.global_scale(w[0])], np.float32)
    base = O.sweep("full", w, h, None, g)
    scaled = O.sweep("full", w, 4.0 * h, None, g)
    np.testing.assert_array_equal(base["codes"], scaled["codes"])
    np.testing.assert_allclose(scaled["loss"], 4.0 * base["loss"], rtol=1e-14)
    neg = O.sweep("full", -w, h, None, g)
    np.testing.assert_array_equal(base["codes"], neg["codes"])
    np.testing.assert_array_equal(base["wq"], -neg["wq"])
    np.testing.assert_allclose(neg["loss"], base["loss"], rtol=1e-14)
    perm = np.random.default_rng(0).permutation(16)
    wp = w.copy()
    wp[0, :, :16] = w[0, :, :16][:, perm]
    hp = h.copy()
    hp[0, 0] = h[0, 0][np.ix_(perm, perm)]
    pb = O.sweep("full", wp, hp, None, g)
    np.testing.assert_array_equal(pb["codes"], base["codes"])
    np.testing.assert_allclose(pb["loss"], base["loss"], rtol=1e-12)
    imp = np.random.default_rng(1).uniform(0.5, 2, (1, 2, 16))
    d1 = O.sweep("diag", w, imp, None, g)
    d2 = O.sweep("diag", -w, imp, None, g)
    np.testing.assert_array_equal(d1["codes"], d2["codes"])
    np.testing.assert_array_equal(d1["loss"], d2["loss"])


def test_power_of_two_scaling_is_exact():
    """W -> 2^k W with g -> 2^k g scales every candidate scale exactly, so each quotient |w| / s_k
    and every E2M1 decision is unchanged: the same codes, Wq scaled by 2^k bit for bit, and
    losses by 4^k (ACT: H and P fixed, the cross term scales with dW and w alike)."""
    rng = np.random.default_rng(17)
    w = (rng.normal(0, 0.05, (1, 24, 32)) * np.exp(rng.normal(0, 1, (1, 24, 1)))).astype(np.float32)
    a = rng.normal(size=(1, 2, 16, 16))
    h = a @ a.transpose(0, 1, 3, 2) / 16
    p = 0.2 * rng.normal(size=(1, 2, 16, 16))
    imp = np.abs(rng.normal(size=(1, 2, 16))) + 0.1
    g = np.array([O.global_scale(w[0])], np.float32)
    for mode, hh, pp in (("full", h, None), ("act", h, p), ("diag", imp, None), ("mse", None, None)):
        base = O.sweep(mode, w, hh, pp, g)
        for k in (-3, 1, 5):
            f = np.float32(2.0 ** k)
            sc = O.sweep(mode, w * f, hh, pp, g * f)
            np.testing.assert_array_equal(sc["codes"], base["codes"])
            np.testing.assert_array_equal(sc["wq"].view(np.int32), (base["wq"] * f).view(np.int32))
            np.testing.assert_allclose(sc["loss"], base["loss"] * 4.0 ** k, rtol=1e-12, atol=0)


def test_loss_scale_bounds_e0_and_equals_it_for_diagonal_h():
    rng = np.random.default_rng(14)
    w = rng.normal(0, 0.05, (50, 16)).astype(np.float32)
    a = rng.normal(size=(50, 16, 16))
    h = a @ a.transpose(0, 2, 1)
    _, _, e0 = O.candidate_losses("full", w, h, None, O.global_scale(w))
    s = O.loss_scale("full", w, h, None)
    assert np.all(s >= e0 - 1e-12 * s)
    hd = np.zeros_like(h)
    idx = np.arange(16)
    hd[:, idx, idx] = np.abs(rng.normal(size=(50, 16)))
    _, _, e0d = O.candidate_losses("full", w, hd, None, O.global_scale(w))
    np.testing.assert_allclose(O.loss_scale("full", w, hd, None), e0d, rtol=1e-13)
    imp = hd[:, idx, idx]
    np.testing.assert_allclose(O.loss_scale("diag", w, imp, None), e0d, rtol=1e-13)


def test_loss_scale_bounds_every_candidate_and_sees_only_magnitudes():
    """Rounding to the nearest E2M1 point, or saturating, never moves a weight by more than its
    magnitude: |dW_i| <= |w_i| for every candidate. Hence |L_k| <= |w|^T |H| |w| (+ 2 |w|^T |P| |w|)
    = S for all 126 k. S depends on magnitudes only: flipping the signs of weights or of H and P
    entries leaves it unchanged; and the cross term adds to it whenever P is not zero."""
    rng = np.random.default_rng(16)
    w = rng.normal(0, 0.05, (40, 16)).astype(np.float32)
    a = rng.normal(size=(40, 16, 16))
    h = a @ a.transpose(0, 2, 1) / 16
    p = 0.3 * rng.normal(size=(40, 16, 16))
    g = O.global_scale(w)
    for mode, pp in (("full", None), ("act", p)):
        loss, wq, _ = O.candidate_losses(mode, w, h, pp, g)
        dw = wq.astype(np.float64) - w.astype(np.float64)[:, None, :]
        assert np.all(np.abs(dw) <= np.abs(w.astype(np.float64))[:, None, :])
        s = O.loss_scale(mode, w, h, pp)
        assert np.all(np.abs(loss) <= s[:, None] * (1 + 1e-12))
        flip = rng.choice([-1.0, 1.0], w.shape).astype(np.float32)
        hs = h * rng.choice([-1.0, 1.0], h.shape)
        ps = None if pp is None else pp * rng.choice([-1.0, 1.0], pp.shape)
        np.testing.assert_array_equal(O.loss_scale(mode, w * flip, hs, ps), s)
    assert np.all(O.loss_scale("act", w, h, p) > O.loss_scale("full", w, h, None))


# --------------------------------------------------------------------------- amax-multiplier search

@pytest.mark.parametrize("mode", ["full", "act", "diag", "mse"])
def test_losses_for_scales_is_candidate_losses_at_the_candidate_scales(mode):
    rng = np.random.default_rng(21)
    w = rng.normal(0, 0.05, (9, 16)).astype(np.float32)
    a = rng.normal(size=(9, 16, 16))
    h = a @ a.transpose(0, 2, 1) / 16 if mode in ("full", "act") else (np.abs(rng.normal(size=(9, 16))) + 0.5)
    p = 0.05 * rng.normal(size=(9, 16, 16)) if mode == "act" else None
    g = O.global_scale(w)
    ref, wq_ref, _ = O.candidate_losses(mode, w, None if mode == "mse" else h, p, g)
    s = np.broadcast_to(O.candidate_scales(g), (9, 126))
    got, wq = O.losses_for_scales(mode, w, None if mode == "mse" else h, p, s)
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(wq.view(np.int32), wq_ref.view(np.int32))


def test_multiplier_codes_by_exact_rationals():
    rng = np.random.default_rng(22)
    w = (rng.normal(0, 0.05, (6, 16)) * np.exp(rng.normal(0, 2, (6, 1)))).astype(np.float32)
    w[5] = 0.0
    g = np.float32(O.global_scale(w) * 0.7)
    m = np.concatenate([np.linspace(0.05, 3.0, 40), [0.0, -1.0, np.nan, 1e30]]).astype(np.float32)
    codes = O.multiplier_codes(w, g, m)
    gq = Fraction(float(g))
    for u in range(6):
        amax = max(abs(Fraction(float(v))) for v in w[u])
        for i, mi in enumerate(m):
            if not np.isfinite(mi):
                want = 0
            else:
                a = _round_binary(abs(Fraction(float(mi)) * amax), 24, -126) * (1 if mi >= 0 else -1)
                if a > Fraction(float(np.finfo(np.float32).max)):
                    want = 126  # the fp32 product overflows to +inf
                else:
                    want = 0 if a <= 0 else _e4m3_code_brute(a / (6 * gq))
            assert codes[u, i] == want, (u, i, float(mi))
    assert np.all(O.multiplier_codes(w, np.float32(0.0), m) == 0)


def test_multiplier_codes_round_the_candidate_amax_to_fp32():
    """The candidate amax is the fp32 product m * amax, as the quantizer holds its amax in fp32.
    Worked by hand: g = 2^-3, so 6g = 0.75 and the E4M3 tie 1.0625 (between 1.0 = 0x38 and
    1.125 = 0x39) is a candidate amax of 0.796875. With amax = 1 + 2^-22 and
    m = 0.796875 - 3 * 2^-24 the exact product is 0.796875 + (0.1875 - 6 * 2^-23) * 2^-24, above
    the tie by less than half an fp32 ulp (2^-25). It rounds to 0.796875 exactly, and the tie
    goes to the even code 0x38; the unrounded product would give 0x39."""
    amax, m = np.float32(1 + 2 ** -22), np.float32(0.796875 - 3 * 2 ** -24)
    assert float(amax) == 1 + 2 ** -22 and float(m) == 0.796875 - 3 * 2 ** -24
    w = np.zeros((1, 16), np.float32)
    w[0, 3] = -amax
    assert O.multiplier_codes(w, np.float32(0.125), np.array([m, 1.0], np.float32)).tolist() == [[0x38, 0x3B]]


@pytest.mark.parametrize("mode", ["full", "diag", "mse"])
def test_dense_multipliers_reproduce_the_sweep(mode):
    """Multipliers so dense that every code 1..126 is some multiplier's code: the search then
    scores every sweep candidate, in ascending code order, so it finds the sweep's winner."""
    _, w = _layer(23, rows=5, cin=32)
    g = np.array([O.global_scale(w[0])], np.float32)
    h = None
    if mode == "full":
        a = np.random.default_rng(3).normal(size=(2, 16, 16))
        h = (a @ a.transpose(0, 2, 1))[None] / 16
    elif mode == "diag":
        h = np.abs(np.random.default_rng(3).normal(size=(1, 2, 16))) + 0.5
    mult = np.exp(np.linspace(np.log(1e-7), np.log(1e4), 9000)).astype(np.float32)
    ms = O.multiplier_search(mode, w, h, None, g, mult)
    sw = O.sweep(mode, w, h, None, g)
    wb = w[0].reshape(10, 16)
    cover = np.array([set(range(1, 127)) <= set(O.multiplier_codes(wb[u:u + 1], g[0], mult)[0].tolist())
                      for u in range(10)])
    assert cover.all()
    np.testing.assert_array_equal(ms["codes"], sw["codes"])
    np.testing.assert_array_equal(ms["wq"].view(np.int32), sw["wq"].view(np.int32))
    np.testing.assert_array_equal(ms["loss"], sw["loss"])
