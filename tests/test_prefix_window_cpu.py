"""The sweeps' shortcut for the clamped prefix, checked on the CPU against every candidate.

While all weights of a unit sit at the top E2M1 level, its loss over the candidate scales s_k is
a parabola, f(k) = (pa s_k + pb) s_k (FULL / activation-aware, L - C') or ((pa s_k + pb) s_k + pc)
(WMSE / MSE), evaluated in fp32 with fused multiply-adds. The sweeps evaluate f only at the
candidates within two places of the E4M3 code of s*/g, s* = -pb / (2 pa) the vertex, under the
conditions they test, and rely on the minimum over the whole prefix (lowest k on equal values)
lying in that window. Here that claim is tested directly: random parabolas, global scales and
prefix lengths; f evaluated at every candidate of the prefix with the kernels' arithmetic
(fp32 rounding after each fused multiply-add and product); the argmin must fall in the window.
The candidate scales come from the oracle; E4M3 rounding of s*/g from torch's float8 conversion.
"""
import numpy as np
import torch

from oracle import lhcal_oracle as O

WIN = 2


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma32(a, b, c):
    """fp32 fused multiply-add: the product of two fp32 values is exact in fp64, then the sum
    and the rounding to fp32 (in rare cases the fp64 sum rounds first, which moves a value by
    one fp32 unit at most: far below the margins tested here)."""
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def _window(pa, pb, g, kstart, s, centre=False):
    """The kernels' window [lo, hi) for one unit (FULL form: the conditions before pc's); with
    centre, the candidate the window is centred on."""
    q = np.float32(max(np.float32(-pb) / (np.float32(2.0) * pa), np.float32(0.0))) / np.float32(g)
    q = min(np.float32(q), np.float32(448.0))  # saturating conversion
    code = int(torch.tensor([float(q)], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0]) & 0x7F
    k0 = min(max(code - 1, 0), kstart - 1)
    if centre:
        return k0
    return max(0, k0 - WIN), min(kstart, k0 + WIN + 1)


def _cases(rng, n):
    """Random units: a global scale, a prefix length, a vertex placed anywhere from far below the
    first candidate to far above the prefix, and a curvature over many binades."""
    for _ in range(n):
        g = np.float32(2.0 ** rng.uniform(-24, 2))
        s = O.candidate_scales(g).astype(np.float32)
        kstart = int(rng.integers(2 * WIN + 2, 127))
        pa = np.float32(2.0 ** rng.uniform(-40, 40))
        k_v = rng.uniform(-20, kstart + 20)
        sv = np.float32(s[int(np.clip(k_v, 0, 125))] * 2.0 ** rng.uniform(-0.5, 0.5))
        if k_v < 0:
            sv = np.float32(s[0] * 2.0 ** rng.uniform(-8, 0))
        pb = np.float32(-2.0 * pa * sv)
        yield g, s, kstart, pa, pb


def _fast_path(pa, pb, s, kstart):
    s0 = s[0]
    return (kstart > 2 * WIN + 1 and s0 > 0 and 0 < pa < 2.0 ** 100 and abs(pb) < 2.0 ** 100
            and float(pa) * float(s0) * float(s0) >= 2.0 ** -100 and s[kstart - 1] < 2.0 ** 40)


def test_full_form_minimum_lies_in_the_window():
    rng = np.random.default_rng(20)
    checked = 0
    for g, s, kstart, pa, pb in _cases(rng, 4000):
        if not _fast_path(pa, pb, s, kstart):
            continue
        sk = s[:kstart]
        f = _f32(_fma32(np.full(kstart, pa, np.float32), sk, np.full(kstart, pb, np.float32)) * sk)
        kmin = int(np.argmin(f))  # the first index of the smallest value: the lowest code on ties
        lo, hi = _window(pa, pb, g, kstart, s)
        assert lo <= kmin < hi, (g, kstart, pa, pb, kmin, lo, hi)
        checked += 1
    assert checked > 3000


def test_diagonal_form_with_a_constant_term():
    rng = np.random.default_rng(21)
    checked = 0
    for g, s, kstart, pa, pb in _cases(rng, 4000):
        # pc = sum Imp w^2 >= (sum Imp |w|)^2 / sum Imp = pb^2 / (4 pa): from there up to 2^10 times
        # that, the range the diagonal sweep's extra condition admits.
        depth = float(pb) * float(pb) / (4.0 * float(pa))
        pc = np.float32(depth * 2.0 ** rng.uniform(0, 10))
        if not (_fast_path(pa, pb, s, kstart) and pc < 2.0 ** 100
                and float(pb) * float(pb) >= 2.0 ** -10 * float(pa) * float(pc)):
            continue
        sk = s[:kstart]
        inner = _fma32(np.full(kstart, pa, np.float32), sk, np.full(kstart, pb, np.float32))
        f = _fma32(inner, sk, np.full(kstart, pc, np.float32))
        kmin = int(np.argmin(f))
        lo, hi = _window(pa, pb, g, kstart, s)
        assert lo <= kmin < hi, (g, kstart, pa, pb, pc, kmin, lo, hi)
        checked += 1
    assert checked > 2000


def test_centre_is_the_nearest_candidate_up_to_rounding():
    # The parabola is symmetric about s*, so the candidate nearest s* (in value) is the discrete
    # minimum, and rounding s*/g to the nearest E4M3 value finds it: the window's centre is the
    # minimum, or next to it where s*/g falls on a midpoint or the fp32 evaluation rounds a near
    # tie. The kernels' window of two places each side is the margin for those cases.
    rng = np.random.default_rng(22)
    checked = 0
    for g, s, kstart, pa, pb in _cases(rng, 3000):
        if not _fast_path(pa, pb, s, kstart):
            continue
        sk = s[:kstart]
        f = _f32(_fma32(np.full(kstart, pa, np.float32), sk, np.full(kstart, pb, np.float32)) * sk)
        assert abs(int(np.argmin(f)) - _window(pa, pb, g, kstart, s, centre=True)) <= 1
        checked += 1
    assert checked > 2000
