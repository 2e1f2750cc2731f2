"""Hand-derived NVFP4 cases (tests/golden/nvfp4_rounding.txt, with its derivations and sources)
against the oracle: E2M1 midpoints, E4M3 ties, subnormals and saturation, activation blocks
through the input quantizer, and sweep winners of the plain block-MSE search."""
import os

import numpy as np

from oracle import lhcal_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_rounding.txt")


def _cases():
    out = {"e2m1": [], "e4m3": [], "act": [], "sweep": []}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        kind, rest = line.split(None, 1)
        out[kind].append(rest)
    return out


def test_golden_file_has_all_kinds():
    c = _cases()
    assert len(c["e2m1"]) >= 16 and len(c["e4m3"]) >= 14 and len(c["act"]) >= 3 and len(c["sweep"]) >= 5


def test_e2m1_cases():
    for rest in _cases()["e2m1"]:
        u, q = (float(v) for v in rest.split())
        assert O.e2m1_round(np.array([u]))[0] == q, rest


def test_e4m3_cases():
    for rest in _cases()["e4m3"]:
        r, code = rest.split()
        assert O.e4m3_round(np.array([float(r)]))[0] == int(code, 16), rest


def test_activation_blocks():
    for rest in _cases()["act"]:
        lhs, rhs = rest.split("->")
        vals = lhs.split()
        gx, x = np.float32(vals[0]), np.array([float(v) for v in vals[1:]], np.float32)
        want = np.array([float(v) for v in rhs.split()], np.float32)
        assert x.size == 16 and want.size == 16
        got = O.act_fake_quant(x[None], gx)[0]
        np.testing.assert_array_equal(got.view(np.int32), want.view(np.int32), err_msg=rest)


def test_sweep_winners():
    for rest in _cases()["sweep"]:
        lhs, rhs = rest.split("->")
        vals = lhs.split()
        g, w = np.float32(vals[0]), np.array([float(v) for v in vals[1:]], np.float32)
        code, loss = rhs.split()
        assert w.size == 16
        out = O.sweep("mse", w[None, None, :], None, None, np.array([g], np.float32))
        assert int(out["codes"][0]) == int(code, 16) and out["loss"][0] == float(loss), rest
        if float(loss) == 0.0:  # a zero loss means the fake-quantized weights are the weights
            np.testing.assert_array_equal(out["wq"][0].view(np.int32), w.view(np.int32), err_msg=rest)
