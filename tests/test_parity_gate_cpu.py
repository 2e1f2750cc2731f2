"""The parity gate itself, on the CPU.

Fed the oracle's own results, it accepts them. Fed them with one discrepancy planted, it
rejects each of these:
- a wrong code on a clearly decided unit;
- a flipped bit of a fake-quantized weight;
- a loss, or an H block, off by more than 1e-4;
- anything non-zero where the oracle's block is zero.

It still accepts what it is meant to allow: another code on a tied unit, and an error inside
the tolerance.
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
    return O.calibrate("full", x, w)


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
