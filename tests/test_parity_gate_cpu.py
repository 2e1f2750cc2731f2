"""The parity gate itself, on the CPU.

Fed the oracle's own results, it accepts them. Fed them with one discrepancy planted, it
rejects each of these:
- a wrong code on a clearly decided unit;
- a flipped bit of a fake-quantized weight;
- a loss, or an H block, off by more than 1e-4;
- anything non-zero where the oracle's block is zero.

It still accepts what it is meant to allow: another code on a tied unit, and an error inside
the tolerance. On a near-tie unit it checks what is unique: the GPU's code must be one of the
oracle's tied candidates and its fake-quantized weights those of that code, bit for bit.
"""
import numpy as np
import pytest

from oracle import lhcal_oracle as O
from tests import parity as P


def _ref():
    rng = np.random.default_rng(31)
    x = rng.normal(size=(64, 32)).astype(np.float32)
    w = rng.normal(0, 0.05, (1, 12, 32)).astype(np.float32)
    w[0, 0, :16] = 0.0  # an all-zero block: every candidate ties, so the unit is exempt
    ref = O.calibrate("full", x, w)
    return P.attach_candidates(ref, "full", w, ref["h"], None, ref["g"])


def _copies(ref):
    return ref["codes"].copy(), ref["wq"].astype(np.float32).copy(), ref["loss"].astype(np.float32)


def _scale(ref):
    return np.maximum(np.maximum(np.abs(ref["loss"]), ref["escale"]), 1e-30)


def test_gate_accepts_the_oracle_and_counts_the_tied_unit():
    ref = _ref()
    rep = P.check_sweep(*_copies(ref), ref, "oracle against itself")
    assert rep["units"] == 24 and rep["exempt"] >= 1 and rep["worst_loss_err"] < 1e-7


def test_gate_rejects_a_wrong_code_or_a_flipped_weight_bit_on_a_decided_unit():
    ref = _ref()
    gap = (ref["second"] - ref["loss"]) / _scale(ref)
    u = int(np.argmax(gap))
    assert gap[u] > P.GAP_TOL
    codes, wq, loss = _copies(ref)
    codes[u] = codes[u] % 126 + 1
    with pytest.raises(AssertionError, match="codes differ"):
        P.check_sweep(codes, wq, loss, ref, "planted code")
    codes, wq, loss = _copies(ref)
    wq.view(np.int32)[u, 5] ^= 1
    with pytest.raises(AssertionError, match="not bit-exact"):
        P.check_sweep(codes, wq, loss, ref, "planted weight bit")


def test_gate_allows_another_code_on_a_tied_unit():
    ref = _ref()
    assert ref["codes"][0] == 1 and ref["second"][0] == ref["loss"][0]
    codes, wq, loss = _copies(ref)
    codes[0] = 77
    P.check_sweep(codes, wq, loss, ref, "tied unit")


def test_gate_loss_tolerance_is_1e4_of_the_loss_scale():
    ref = _ref()
    scale = _scale(ref)
    u = int(np.argmax(ref["escale"]))
    codes, wq, _ = _copies(ref)
    inside = ref["loss"].copy()
    inside[u] += 5e-5 * scale[u]
    P.check_sweep(codes, wq, inside, ref, "loss inside the tolerance")
    outside = ref["loss"].copy()
    outside[u] += 2e-4 * scale[u]
    with pytest.raises(AssertionError, match="worst loss error"):
        P.check_sweep(codes, wq, outside, ref, "loss outside the tolerance")


def test_hessian_gate_per_block_tolerance_and_zero_blocks():
    rng = np.random.default_rng(32)
    x = rng.normal(size=(50, 48)).astype(np.float32)
    h, _, _ = O.accumulate("full", x, group_offsets=np.array([0, 20, 20], np.int32),
                           token_ids=np.arange(20, dtype=np.int32))
    assert np.all(h[1] == 0)  # the second group has no token
    P.check_hessians(h.copy(), h, "oracle against itself")
    e = np.zeros_like(h)
    e[0, 2, 3, 4] = 1.0
    norm = np.sqrt(np.sum(h[0, 2] ** 2))
    P.check_hessians(h + 5e-5 * norm * e, h, "inside the tolerance")
    with pytest.raises(AssertionError, match="relative Frobenius"):
        P.check_hessians(h + 2e-4 * norm * e, h, "outside the tolerance")
    z = h.copy()
    z[1, 0, 0, 0] = 1e-30
    with pytest.raises(AssertionError, match="oracle block is zero"):
        P.check_hessians(z, h, "zero block")


def _near_tie_ref():
    """A seeded layer with near-tie units (gap <= 1e-5) whose tied codes give different Wq."""
    rng = np.random.default_rng(40)
    x = rng.normal(size=(64, 32)).astype(np.float32)
    w = rng.normal(0, 0.05, (1, 300, 32)).astype(np.float32)
    ref = O.calibrate("full", x, w)
    P.attach_candidates(ref, "full", w, ref["h"], None, ref["g"])
    scale = _scale(ref)
    ex = np.nonzero((ref["second"] - ref["loss"]) / scale <= P.GAP_TOL)[0]
    cc, cl, cw = ref["candidates"](ex)
    for i, u in enumerate(ex):
        tied = np.nonzero(cl[i] - ref["loss"][u] <= P.GAP_TOL * scale[u])[0]
        for k in tied:
            if k + 1 != ref["codes"][u] and not np.array_equal(cw[i, k].view(np.int32), ref["wq"][u].view(np.int32)):
                untied = int(np.argmax(cl[i]))  # the worst candidate: far outside the tie
                return ref, int(u), int(k), cw[i, k].copy(), untied, cw[i, untied].copy()
    raise AssertionError("no near-tie unit with distinct tied weights in the seeded layer")


def test_gate_accepts_the_other_tied_code_with_its_own_weights():
    ref, u, k, wq_k, _, _ = _near_tie_ref()
    codes, wq, loss = _copies(ref)
    codes[u], wq[u] = k + 1, wq_k
    rep = P.check_sweep(codes, wq, loss, ref, "other tied code")
    assert rep["exempt"] >= 1 and rep["exempt_e0"] >= 0


def test_gate_rejects_a_tied_code_paired_with_the_other_codes_weights():
    ref, u, k, _, _, _ = _near_tie_ref()
    codes, wq, loss = _copies(ref)
    codes[u] = k + 1  # weights still those of the oracle's winner
    with pytest.raises(AssertionError, match="not bit-exact to the oracle's at the GPU's code"):
        P.check_sweep(codes, wq, loss, ref, "tied code, wrong weights")


def test_gate_rejects_a_code_outside_the_tie_on_a_near_tie_unit():
    ref, u, _, _, bad, wq_bad = _near_tie_ref()
    codes, wq, loss = _copies(ref)
    codes[u], wq[u] = bad + 1, wq_bad
    with pytest.raises(AssertionError, match="not among the oracle's tied candidates"):
        P.check_sweep(codes, wq, loss, ref, "untied code")


def test_gate_needs_the_near_tie_hook():
    ref = O.calibrate("full", np.ones((4, 16), np.float32), np.ones((1, 2, 16), np.float32))
    with pytest.raises(AssertionError, match="near-tie hook"):
        P.check_sweep(*_copies(ref), ref, "no hook")
