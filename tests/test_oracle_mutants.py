"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in the oracle, on the CPU, by wrapping one of its functions: a
dropped factor, a transposed or negated operand, another tie rule, a missing normalisation, an
off-by-one candidate set. It then runs the pins named for that mistake. At least one pin must
fail with an AssertionError; a crash does not count. The oracle resolves its helpers through
the module at call time, so a mistake planted in ``e2m1_round`` also reaches ``fake_quant``,
the sweep and the input quantizer. The pins' own references (exact rationals, ml_dtypes,
torch's float8 decode) are built apart from the oracle and stay as they are.
"""
import numpy as np
import pytest

from oracle import lhcal_oracle as O
from tests import test_golden as golden
from tests import test_oracle_pins as pins

# E2M1 midpoints and the two grid values around each.
_MID = {0.25: (0.0, 0.5), 0.75: (0.5, 1.0), 1.25: (1.0, 1.5), 1.75: (1.5, 2.0), 2.5: (2.0, 3.0),
        3.5: (3.0, 4.0), 5.0: (4.0, 6.0)}


def _e2m1_on_ties(choose):
    """E2M1 rounding whose exact ties take choose(lo, hi, even_choice) instead of the even value."""
    def factory(orig):
        def mutant(u):
            u64 = np.minimum(np.asarray(u, dtype=np.float64), 6.0)
            out = np.array(orig(u), dtype=np.float64, copy=True)
            for m, (lo, hi) in _MID.items():
                out = np.where(u64 == m, choose(lo, hi, out), out)
            return out
        return mutant
    return factory


def _e2m1_of_fp32_quotient(orig):
    return lambda u: orig(np.asarray(u, dtype=np.float64).astype(np.float32).astype(np.float64))


def _e4m3_ties_up(orig):
    vals = np.concatenate([[0.0], O.e4m3_value(O.candidate_codes())])

    def mutant(r):
        r64 = np.asarray(r, dtype=np.float64)
        out = np.asarray(orig(r))
        hi = np.clip(np.searchsorted(vals, r64, side="left"), 1, len(vals) - 1)
        return np.where(r64 == (vals[hi - 1] + vals[hi]) / 2, hi, out).astype(np.int64)
    return mutant


def _e4m3_truncating(orig):
    vals = np.concatenate([[0.0], O.e4m3_value(O.candidate_codes())])

    def mutant(r):
        r64 = np.asarray(r, dtype=np.float64)
        down = np.clip(np.searchsorted(vals, r64, side="right") - 1, 0, len(vals) - 1)
        return np.where(r64 >= 448.0, len(vals) - 1, down).astype(np.int64)
    return mutant


def _act_hessians(change):
    def factory(orig):
        def mutant(x, xq):
            h, p = orig(x, xq)
            return change(h, p, x, orig)
        return mutant
    return factory


def _cross_term(change):
    def factory(orig):
        def mutant(mode, w_blk, h_blk, p_blk, g):
            if mode == "act":
                p_blk = change(np.asarray(p_blk, dtype=np.float64))
            return orig(mode, w_blk, h_blk, p_blk, g)
        return mutant
    return factory


def _finalize(change):
    def factory(orig):
        def mutant(mode, h, p, counts):
            hf, pf = orig(mode, h, p, counts)
            hf = np.array(hf, copy=True)
            for e, b in enumerate(np.asarray(counts)):
                change(mode, hf, np.asarray(h, dtype=np.float64), e, int(b))
            return hf, pf
        return mutant
    return factory


def _raw_sums(mode, hf, h, e, b):
    if b > 0 and mode != "diag":
        hf[e] = h[e]


def _diag_divided(mode, hf, h, e, b):
    if b > 0 and mode == "diag":
        hf[e] = h[e] / b


def _no_fallback(mode, hf, h, e, b):
    if b == 0:
        hf[e] = 0.0


def _highest_code_on_ties(orig):
    def mutant(loss):
        k, best, second = orig(np.asarray(loss)[:, ::-1])
        return loss.shape[1] - 1 - k, best, second
    return mutant


def _gather_from_group_zero(which):
    def factory(orig):
        def mutant(mode, w, h, p, g, units):
            wb, hb, pb, gu = orig(mode, w, h, p, g, units)
            n = np.asarray(units, dtype=np.int64)[:, 2]
            if which == "g":
                gu = np.full_like(gu, np.asarray(g)[0])
            elif h is not None:
                hb = np.asarray(h)[0, n]
            return wb, hb, pb, gu
        return mutant
    return factory


def _routing_ignored(orig):
    def mutant(mode, x, xq=None, group_offsets=None, token_ids=None, act_gx=None):
        if token_ids is not None:
            token_ids = np.arange(len(token_ids)) % np.asarray(x).shape[0]
        return orig(mode, x, xq, group_offsets, token_ids, act_gx)
    return mutant


def _multiplier_codes(fp32_product=True, signed=True):
    """The multiplier codes with one step changed; otherwise as the oracle states them."""
    def factory(orig):
        def mutant(w_blk, g, multipliers):
            amax = np.abs(np.asarray(w_blk, dtype=np.float32).astype(np.float64)).max(axis=1)
            m = np.asarray(multipliers, dtype=np.float32).astype(np.float64)
            with np.errstate(invalid="ignore"):
                a = m[None, :] * amax[:, None]
                if fp32_product:
                    a = a.astype(np.float32).astype(np.float64)
            a = np.abs(a) if not signed else np.where(np.isnan(a) | (a < 0), 0.0, a)
            a = np.where(np.isnan(a), 0.0, a)
            g64 = np.float64(np.float32(g))
            return np.zeros(a.shape, dtype=np.int64) if g64 == 0 else O.e4m3_round(a / (6.0 * g64))
        return mutant
    return factory


def _loss_scale_signed(orig):
    def mutant(mode, w_blk, h_blk, p_blk):
        if mode not in ("full", "act"):
            return orig(mode, w_blk, h_blk, p_blk)
        w = np.asarray(w_blk, dtype=np.float64)
        s = np.einsum("ui,uij,uj->u", w, np.asarray(h_blk, dtype=np.float64), w)
        if mode == "act":
            s = s + 2.0 * np.abs(np.einsum("ui,uij,uj->u", w, np.asarray(p_blk, dtype=np.float64), w))
        return s
    return mutant


def _quadratic_of_wq(orig):
    def mutant(mode, w_blk, h_blk, p_blk, g):
        loss, wq, e0 = orig(mode, w_blk, h_blk, p_blk, g)
        if mode in ("full", "act"):
            w64, q64 = np.asarray(w_blk, dtype=np.float64), wq.astype(np.float64)
            loss = np.einsum("uki,uij,ukj->uk", q64, np.asarray(h_blk, dtype=np.float64), q64)
            if mode == "act":
                pw = np.einsum("uij,uj->ui", np.asarray(p_blk, dtype=np.float64), w64)
                loss = loss + 2.0 * np.einsum("uki,ui->uk", q64 - w64[:, None, :], pw)
        return loss, wq, e0
    return mutant


def _act_quant_amax_over_32(orig):
    """The input quantizer with its block amax taken over two neighbouring blocks (32 values)."""
    def mutant(x, gx, rows_per_chunk=1024):
        x64 = np.asarray(x, dtype=np.float64)
        t, c = x64.shape
        gx64 = np.float64(np.float32(gx))
        blk = np.abs(x64).reshape(t, c // 16, 16).max(axis=-1)
        n2 = blk.shape[1] - blk.shape[1] % 2  # pairs of neighbouring blocks; a lone last block keeps its own
        pm = np.maximum(blk[:, 0:n2:2], blk[:, 1:n2:2])
        blk[:, 0:n2:2], blk[:, 1:n2:2] = pm, pm
        amax = blk[..., None]
        code = O.e4m3_round(amax / (6.0 * gx64)) if gx64 > 0 else np.zeros(amax.shape, np.int64)
        v = np.where(code > 0, O.e4m3_value(np.maximum(code, 1)), 0.0)
        s = (v * gx64).astype(np.float32).astype(np.float64)
        xb = x64.reshape(t, c // 16, 16)
        with np.errstate(divide="ignore", invalid="ignore"):
            u = np.where(s > 0, np.abs(xb) / np.where(s > 0, s, 1.0), 0.0)
        mag = O.f32_to_bf16_values((O.e2m1_round(u) * s).astype(np.float32))
        return np.copysign(mag, xb).reshape(t, c).astype(np.float32)
    return mutant


def _apply_scales_amax_without_six(orig):
    def mutant(w, g, codes):
        wq, wq16, amax = orig(w, g, codes)
        return wq, wq16, amax / 6.0
    return mutant


MUTANTS = {
    "E2M1 ties to the odd value": (
        "e2m1_round", _e2m1_on_ties(lambda lo, hi, even: lo + hi - even),
        [lambda: pins.test_e2m1_midpoints_ties_to_even(0.25, 0), pins.test_fake_quant_exact_ties_and_neighbours,
         golden.test_e2m1_cases]),
    "E2M1 ties away from zero": (
        "e2m1_round", _e2m1_on_ties(lambda lo, hi, even: hi),
        [lambda: pins.test_e2m1_midpoints_ties_to_even(2.5, 2), pins.test_fake_quant_exact_ties_and_neighbours,
         golden.test_e2m1_cases]),
    "E2M1 of the fp32-rounded quotient": (
        "e2m1_round", _e2m1_of_fp32_quotient, [pins.test_fake_quant_exact_ties_and_neighbours]),
    "E4M3 ties to the larger code": (
        "e4m3_round", _e4m3_ties_up,
        [pins.test_e4m3_round_brute_force_and_library, pins.test_act_fake_quant_hand_worked_ties,
         golden.test_e4m3_cases]),
    "E4M3 by truncation": (
        "e4m3_round", _e4m3_truncating, [pins.test_e4m3_round_brute_force_and_library, golden.test_e4m3_cases]),
    "candidate codes shifted down by one": (
        "candidate_codes", lambda orig: (lambda: orig() - 1), [pins.test_e4m3_candidates_match_torch_float8]),
    "X_q left unrounded to bf16": (
        "f32_to_bf16_values", lambda orig: (lambda v: np.asarray(v, dtype=np.float32)),
        [lambda: pins.test_act_fake_quant_brute_force(1.0)]),
    "fake quant drops the sign": (
        "fake_quant", lambda orig: (lambda w, s: np.abs(orig(w, s))),
        [pins.test_fake_quant_negative_zero_and_zero_scale, pins.test_fake_quant_exact_ties_and_neighbours]),
    "fake quant loses -0": (
        "fake_quant", lambda orig: (lambda w, s: orig(w, s) + np.float32(0.0)),
        [pins.test_fake_quant_negative_zero_and_zero_scale]),
    "P transposed": (
        "hessian_sum_act", _act_hessians(lambda h, p, x, orig: (h, p.transpose(0, 2, 1))),
        [pins.test_act_hessians_brute_force_and_properties]),
    "P negated (X_q^T (X - X_q))": (
        "hessian_sum_act", _act_hessians(lambda h, p, x, orig: (h, -p)),
        [pins.test_act_hessians_brute_force_and_properties, pins.test_act_expanded_loss_equals_output_mse_including_negative]),
    "activation-aware H taken from X": (
        "hessian_sum_act", _act_hessians(lambda h, p, x, orig: (orig(x, x)[0], p)),
        [pins.test_act_hessians_brute_force_and_properties, pins.test_act_expanded_loss_equals_output_mse_including_negative]),
    "cross term without its factor 2": (
        "candidate_losses", _cross_term(lambda p: 0.5 * p),
        [pins.test_act_expanded_loss_equals_output_mse_including_negative]),
    "cross term with P^T w": (
        "candidate_losses", _cross_term(lambda p: p.transpose(0, 2, 1)),
        [pins.test_act_expanded_loss_equals_output_mse_including_negative]),
    "cross term negated": (
        "candidate_losses", _cross_term(lambda p: -p),
        [pins.test_act_expanded_loss_equals_output_mse_including_negative]),
    "H and P left as raw sums (no 1/B)": (
        "finalize", _finalize(_raw_sums), [pins.test_grouped_accumulate_and_zero_group_fallback]),
    "importance divided by B": (
        "finalize", _finalize(_diag_divided), [pins.test_grouped_accumulate_and_zero_group_fallback]),
    "no fallback for a zero-token group": (
        "finalize", _finalize(_no_fallback), [pins.test_grouped_accumulate_and_zero_group_fallback]),
    "importance as a mean over tokens": (
        "importance_sum", lambda orig: (lambda x: orig(x) / np.asarray(x).shape[0]),
        [pins.test_hessian_symmetric_psd_and_diag_is_importance]),
    "global scale over 448 instead of 6 * 448": (
        "global_scale", lambda orig: (lambda w, fp8_max=448.0: np.float32(orig(w, fp8_max) * 6)),
        [pins.test_global_scale_is_448_normalized]),
    "global scale ignores the 4/6 normalization": (
        "global_scale", lambda orig: (lambda w, fp8_max=448.0: orig(w)),
        [pins.test_global_scale_four_over_six_is_256_normalized]),
    "highest code wins a tie": (
        "argmin_lowest", _highest_code_on_ties,
        [pins.test_sweep_is_exhaustive_lowest_code_on_ties, golden.test_sweep_winners]),
    "every group swept with group 0's global scale": (
        "gather_units", _gather_from_group_zero("g"), [pins.test_grouped_calibrate_is_each_expert_on_its_own]),
    "every group swept with group 0's H": (
        "gather_units", _gather_from_group_zero("h"), [pins.test_grouped_calibrate_is_each_expert_on_its_own]),
    "grouped accumulation ignores the routing": (
        "accumulate", _routing_ignored,
        [pins.test_grouped_accumulate_and_zero_group_fallback, pins.test_grouped_calibrate_is_each_expert_on_its_own]),
    "candidate amax not rounded to fp32": (
        "multiplier_codes", _multiplier_codes(fp32_product=False),
        [pins.test_multiplier_codes_round_the_candidate_amax_to_fp32]),
    "negative multiplier taken by magnitude": (
        "multiplier_codes", _multiplier_codes(signed=False), [pins.test_multiplier_codes_by_exact_rationals]),
    "loss scale from signed weights and H": (
        "loss_scale", _loss_scale_signed, [pins.test_loss_scale_bounds_every_candidate_and_sees_only_magnitudes]),
    "loss scale without the cross term": (
        "loss_scale", lambda orig: (lambda mode, w, h, p: orig("full" if mode == "act" else mode, w, h, None)),
        [pins.test_loss_scale_bounds_every_candidate_and_sees_only_magnitudes]),
    "input quantizer ignores its global scale": (
        "act_fake_quant", lambda orig: (lambda x, gx, rows_per_chunk=1024: orig(x, np.float32(1.0), rows_per_chunk)),
        [lambda: pins.test_act_fake_quant_brute_force(1e-3), pins.test_act_fake_quant_saturates_and_zero_global_scale]),
    "E4M3 without saturation (NaN code above 448)": (
        "e4m3_round", lambda orig: (lambda r: np.where(np.asarray(r, dtype=np.float64) > 464.0, 127, orig(r))),
        [pins.test_e4m3_round_brute_force_and_library, golden.test_e4m3_cases]),
    "DIAG loss weighted by Imp squared": (
        "candidate_losses",
        lambda orig: (lambda mode, w, h, p, g: orig(mode, w, np.asarray(h) ** 2 if mode == "diag" else h, p, g)),
        [pins.test_wmse_equals_full_with_diagonal_hessian]),
    "MSE loss doubled": (
        "candidate_losses",
        lambda orig: (lambda mode, w, h, p, g: orig("diag", w, np.full(np.shape(w), 2.0), None, g)
                      if mode == "mse" else orig(mode, w, h, p, g)),
        [pins.test_mse_mode_is_plain_block_mse_by_exact_rationals_and_equals_identity_hessian]),
    "quadratic form of Wq instead of dW": (
        "candidate_losses", _quadratic_of_wq,
        [pins.test_act_expanded_loss_equals_output_mse_including_negative,
         pins.test_identity_hessian_is_plain_block_mse_by_exact_rationals]),
    "E4M3 subnormals decoded with the normal exponent bias": (
        "e4m3_value",
        lambda orig: (lambda code: np.where((np.asarray(code) >> 3) == 0, orig(code) * 8.0, orig(code))),
        [pins.test_e4m3_candidates_match_torch_float8]),
    "candidate scales in descending order": (
        "candidate_scales", lambda orig: (lambda g: orig(g)[::-1].copy()),
        [pins.test_global_scale_is_448_normalized]),
    "full Hessian drops the last token": (
        "hessian_sum_full", lambda orig: (lambda x: orig(np.asarray(x)[:-1])),
        [pins.test_full_hessian_brute_force]),
    "codes above 126 applied as zero": (
        "apply_scales",
        lambda orig: (lambda w, g, codes: orig(w, g, np.where(np.asarray(codes) > 126, 0, codes).astype(np.uint8))),
        [pins.test_apply_scales_matches_the_sweep_and_exact_amax]),
    "losses for scales evaluated on reversed scales": (
        "losses_for_scales",
        lambda orig: (lambda mode, w, h, p, s: orig(mode, w, h, p, np.asarray(s)[:, ::-1].copy())),
        [lambda: pins.test_losses_for_scales_is_candidate_losses_at_the_candidate_scales("full")]),
    "input quantizer amax over 32 values": (
        "act_fake_quant", _act_quant_amax_over_32,
        [lambda: pins.test_act_fake_quant_brute_force(1.0), golden.test_activation_blocks]),
    "Hessian kept in fp32": (
        "hessian_sum_full", lambda orig: (lambda x: orig(x).astype(np.float32).astype(np.float64)),
        [pins.test_full_hessian_brute_force]),
    "exported amax without the factor 6": (
        "apply_scales", _apply_scales_amax_without_six, [pins.test_apply_scales_matches_the_sweep_and_exact_amax]),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_fails_a_pin(name, monkeypatch):
    attr, factory, checks = MUTANTS[name]
    monkeypatch.setattr(O, attr, factory(getattr(O, attr)))
    caught = 0
    for check in checks:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught, f"no pin caught: {name}"


def test_the_named_pins_pass_on_the_oracle_as_written():
    for _, _, checks in MUTANTS.values():
        for check in checks:
            check()
