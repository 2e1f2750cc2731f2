"""CPU oracle for local-Hessian NVFP4 weight-scale calibration (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Only the tests, the package's smoke check and the
benchmark's CPU-baseline / reference arm may import this module. The CUDA
library never calls it, and it shares no code with the CUDA library.

It is the plain definition of what the hot path computes, evaluated in fp64 on
the same host tensors (bf16 or fp32, widened exactly) that the GPU receives.
Sources (PR pages of NVIDIA Model-Optimizer):

* "add local hessian calibration" (PR #788), Overview and the Changes table:
  per-16-wide-input-block Hessians H_n = X_b^T X_b / B weighting the scale
  candidates; an FP8 scale sweep chooses the block scale.
* "Add activation-aware local Hessian scale calibration" (PR #1976), "What does
  this PR do?" and the two review comments: H = X_q^T X_q / B,
  P = X_q^T (X_q - X) / B; loss dW^T H dW + 2 dW^T (P W0) with dW = quant(w) - w;
  best loss starts at +inf and losses may be negative.
* "Add WMSE weight scale search calibration" (PR #2283), "What" and "How":
  Imp_i = ||X[:, i]||^2 in a [n_blocks, 16] buffer; loss sum_i Imp_i dW_i^2;
  126 candidate E4M3 scales.
* "Add composable scale calibration to GPTQ" (PR #2004), "What does this PR do?":
  the NVFP4 global scale is 448-normalized, g = amax / (6 * 448).
* "[2/3] Speed up layerwise GPTQ on MoE models" (PR #2864), the embedded #2840
  description: one Hessian per expert over exactly the tokens routed to it; an
  expert no token reaches gets the plain search.

Readings where the pages are silent:
candidates are E4M3 codes 0x01..0x7E; scale s_k = fp32(v_k * g); E2M1 rounds the
exact quotient |w|/s_k to nearest, ties to even, clamped at 6; the fake-quant value
is fp32(q * s_k) with w's sign; ties in loss go to the lowest code; B is the number
of token rows accumulated; a group with B = 0 gets H = I, P = 0 (DIAG: Imp = 1);
g = 0 makes every q zero. The input quantizer that produces X_q (act_fake_quant) takes a
per-tensor global scale gx = fp32(amax|X| / 2688) as an input, rounds each block's
amax / (6 gx) to the nearest E4M3 code and each value to E2M1 on exact quotients, and
outputs bf16. The "mse" method is the same search with H = I. The 4/6 variant
normalizes the global scale by 256 instead of 448. The exported per-block amax is
fp32(6 v g). The amax-multiplier search maps fp32(m * amax_blk) to the nearest E4M3
code of amax / (6 g), and the first multiplier with the smallest loss wins.
"""
from __future__ import annotations

import os

import numpy as np

BLOCK = 16
N_CANDIDATES = 126
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
FP4_MAX = 6.0
FP8_MAX = 448.0


# ---------------------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------------------

def e4m3_value(code) -> np.ndarray:
    """Value of an E4M3 byte with sign bit 0 (OCP FP8: 4 exponent bits, bias 7, 3 mantissa bits);
    the block-scale format of "Add WMSE weight scale search calibration" (PR #2283), How.

    e = code >> 3, m = code & 7; e == 0 is subnormal m * 2^-9, else (1 + m/8) * 2^(e-7).
    Codes 0x01..0x7E are the 126 positive finite non-zero values (0x7F is NaN).
    """
    code = np.asarray(code, dtype=np.int64)
    e = code >> 3
    m = code & 7
    sub = m.astype(np.float64) * 2.0 ** -9
    nrm = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    return np.where(e == 0, sub, nrm)


def candidate_codes() -> np.ndarray:
    """The sweep's candidates: every positive finite non-zero E4M3 code, ascending (PR #2283, How)."""
    return np.arange(1, N_CANDIDATES + 1, dtype=np.int64)


def e2m1_round(u: np.ndarray) -> np.ndarray:
    """Round non-negative reals to the E2M1 grid {0,.5,1,1.5,2,3,4,6}: nearest, ties to even
    (the FP4 E2M1 weight format of PR #2283, How; the pages state no tie rule, and ties to even
    is the reading taken).

    Values above 6 saturate to 6. "Even" means an even E2M1 code; the grid index
    is the code (exponent << 1 | mantissa), so an even index has mantissa bit 0.
    """
    u = np.minimum(np.asarray(u, dtype=np.float64), FP4_MAX)
    d = np.abs(u[..., None] - E2M1_GRID)
    nearest = d == d.min(axis=-1, keepdims=True)
    even = nearest & (np.arange(8) % 2 == 0)
    idx = np.where(even.any(-1), np.argmax(even, -1), np.argmax(nearest, -1))
    return E2M1_GRID[idx]


# ---------------------------------------------------------------------------------------
# Global scale and candidate scales
# ---------------------------------------------------------------------------------------

def global_scale(w: np.ndarray, fp8_max: float = FP8_MAX) -> np.float32:
    """g = fp32(amax|W| / (6 * fp8_max)) (PR #2004: 448-normalized NVFP4 scaling; the NVFP4
    "4/6" variant of the same page normalizes by 256 instead)."""
    amax = float(np.abs(np.asarray(w, dtype=np.float64)).max()) if np.size(w) else 0.0
    return np.float32(amax / (FP4_MAX * float(fp8_max)))


def candidate_scales(g) -> np.ndarray:
    """s_k = fp32(v_k * g) for the 126 candidates; the fp64 product is exact (candidates of
    PR #2283, How; g of PR #2004, "448-normalized")."""
    return (e4m3_value(candidate_codes()) * np.float64(np.float32(g))).astype(np.float32)


def fake_quant(w: np.ndarray, s) -> np.ndarray:
    """NVFP4 fake quant of fp32 weights with fp32 block scale(s) s (broadcast against w): the
    quant(w) of dW = quant(w) - w in PR #1976, "What does this PR do?".

    q = E2M1(|w| / s) on the exact quotient; result fp32(q * s) with the sign of w
    (a negative weight that rounds to 0 gives -0.0). s == 0 gives q = 0.
    """
    w = np.asarray(w, dtype=np.float32)
    s64 = np.asarray(s, dtype=np.float32).astype(np.float64)
    a = np.abs(w.astype(np.float64))
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.where(s64 > 0, a / np.where(s64 > 0, s64, 1.0), 0.0)
    q = e2m1_round(u)
    mag = (q * s64).astype(np.float32)
    return np.copysign(mag, w)


# ---------------------------------------------------------------------------------------
# Activation fake quant (the input quantizer that produces X_q)
# ---------------------------------------------------------------------------------------

def e4m3_round(r) -> np.ndarray:
    """E4M3 code (0..126) of the value nearest to each real r >= 0: ties to the even code (the
    block-scale rounding of the input quantizer, PR #1976 re-review).

    Code 0 is zero; 1..126 are the positive finite values of ``e4m3_value``, so the even
    code is the one with mantissa bit 0. Anything above 448 saturates to 448 (code 126).
    The decision compares r with the exact midpoint of the two bracketing values.
    """
    r = np.asarray(r, dtype=np.float64)
    vals = np.concatenate([[0.0], e4m3_value(candidate_codes())])
    hi = np.clip(np.searchsorted(vals, r, side="left"), 1, N_CANDIDATES)  # vals[hi-1] < r <= vals[hi]
    lo = hi - 1
    mid = (vals[lo] + vals[hi]) / 2.0
    up = (r > mid) | ((r == mid) & (hi % 2 == 0))
    return np.where(r >= FP8_MAX, N_CANDIDATES, np.where(up, hi, lo)).astype(np.int64)


def f32_to_bf16_values(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns the bf16 values as fp32."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def act_fake_quant(x: np.ndarray, gx, rows_per_chunk: int = 1024) -> np.ndarray:
    """NVFP4 fake quant of activations X [T, C] with the per-tensor global scale gx (fp32).

    The input quantizer whose output the activation-aware capture records ("Add
    activation-aware local Hessian scale calibration", PR #1976, re-review): 16-wide
    blocks along C, an E4M3 block scale and a per-tensor global scale (the NVFP4 layout of
    "Add composable scale calibration to GPTQ", PR #2004). Reading, per (token, block):
    code c = E4M3(amax_blk / (6 gx)) on the exact quotient (nearest, ties to even,
    saturating at 448); s = fp32(v_c gx); each value becomes E2M1(|x| / s) on the exact
    quotient, then bf16(fp32(q s)) with the sign of x. gx == 0 or c == 0 gives a zero
    block. Returns fp32 values that are exactly bf16. Rows are independent; they are
    processed rows_per_chunk at a time (on a thread pool) only to bound memory and time.
    """
    x = np.asarray(x)
    t, c = x.shape
    gx64 = np.float64(np.float32(gx))
    out = np.empty((t, c), dtype=np.float32)

    def rows(lo):
        xb = x[lo:lo + rows_per_chunk].astype(np.float64).reshape(-1, c // BLOCK, BLOCK)
        amax = np.abs(xb).max(axis=-1)
        if gx64 > 0:
            code = e4m3_round(amax / (FP4_MAX * gx64))
        else:
            code = np.zeros(amax.shape, dtype=np.int64)
        v = np.where(code > 0, e4m3_value(np.maximum(code, 1)), 0.0)
        s = (v * gx64).astype(np.float32).astype(np.float64)[..., None]  # exact product, one rounding
        with np.errstate(divide="ignore", invalid="ignore"):
            u = np.where(s > 0, np.abs(xb) / np.where(s > 0, s, 1.0), 0.0)
        q = e2m1_round(u)
        mag = f32_to_bf16_values((q * s).astype(np.float32))
        out[lo:lo + rows_per_chunk] = np.copysign(mag, xb).reshape(-1, c)

    starts = range(0, t, rows_per_chunk)
    if t > rows_per_chunk:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(rows, starts))
    else:
        for lo in starts:
            rows(lo)
    return out


# ---------------------------------------------------------------------------------------
# Hessian accumulation (raw sums) and finalisation
# ---------------------------------------------------------------------------------------

def _blocks(x: np.ndarray) -> np.ndarray:
    """[T, C] -> [C/16, 16, T] fp64 view of the 16-wide input blocks."""
    x = np.asarray(x, dtype=np.float64)
    t, c = x.shape
    return x.reshape(t, c // BLOCK, BLOCK).transpose(1, 2, 0)


def hessian_sum_full(x: np.ndarray) -> np.ndarray:
    """Hsum[n] = sum_t x_{t,n} x_{t,n}^T over 16-wide blocks (PR #788 Overview): [C/16, 16, 16]."""
    xb = _blocks(x)
    return np.matmul(xb, xb.transpose(0, 2, 1))


def hessian_sum_act(x: np.ndarray, xq: np.ndarray):
    """(Hsum, Psum): Hsum = sum x_q x_q^T, Psum[i, j] = sum_t xq_{t,i} (xq - x)_{t,j} (PR #1976)."""
    xqb = _blocks(xq)
    db = _blocks(np.asarray(xq, dtype=np.float64) - np.asarray(x, dtype=np.float64))
    return np.matmul(xqb, xqb.transpose(0, 2, 1)), np.matmul(xqb, db.transpose(0, 2, 1))


def importance_sum(x: np.ndarray) -> np.ndarray:
    """Imp[n, i] = sum_t X[t, 16n + i]^2 (PR #2283 How: x.square().sum into [n_blocks, 16])."""
    x = np.asarray(x, dtype=np.float64)
    t, c = x.shape
    return np.square(x).sum(axis=0).reshape(c // BLOCK, BLOCK)


def accumulate(mode: str, x, xq=None, group_offsets=None, token_ids=None, act_gx=None):
    """Raw per-group sums and token counts.

    Returns (h [G, N, 16, 16] or [G, N, 16] for diag, p or None, counts [G]).
    Grouped: group e sums over rows token_ids[offsets[e]:offsets[e+1]] of x
    (the tokens routed to expert e, PR #2864 / #2840).
    ACT without xq: X_q = act_fake_quant(x, act_gx), the input quantizer's output.
    """
    x = np.asarray(x)
    if mode == "act" and xq is None:
        if act_gx is None:
            raise ValueError("act needs xq or the activation global scale act_gx")
        xq = act_fake_quant(x, act_gx)
    if group_offsets is None:
        sets = [np.arange(x.shape[0])]
    else:
        off = np.asarray(group_offsets, dtype=np.int64)
        ids = np.asarray(token_ids, dtype=np.int64)
        sets = [ids[off[e]:off[e + 1]] for e in range(len(off) - 1)]
    hs, ps, counts = [], [], []
    for rows in sets:
        xs = x[rows]
        counts.append(len(rows))
        if mode == "full":
            hs.append(hessian_sum_full(xs))
        elif mode == "act":
            h, p = hessian_sum_act(xs, np.asarray(xq)[rows])
            hs.append(h)
            ps.append(p)
        elif mode == "diag":
            hs.append(importance_sum(xs))
        else:
            raise ValueError(mode)
    return np.stack(hs), (np.stack(ps) if ps else None), np.asarray(counts, dtype=np.int64)


def finalize(mode: str, h, p, counts):
    """H = Hsum / B, P = Psum / B per group (PR #1976); DIAG keeps the raw sum (PR #2283).

    A group with B = 0 falls back to the plain search (PR #2864 / #2840): H = I, P = 0,
    and for DIAG Imp = 1.
    """
    h = np.array(h, dtype=np.float64, copy=True)
    p = None if p is None else np.array(p, dtype=np.float64, copy=True)
    for e, b in enumerate(np.asarray(counts)):
        if b == 0:
            if mode == "diag":
                h[e] = 1.0
            else:
                h[e] = np.eye(BLOCK)
                if p is not None:
                    p[e] = 0.0
        elif mode != "diag":
            h[e] /= float(b)
            if p is not None:
                p[e] /= float(b)
    return h, p


# ---------------------------------------------------------------------------------------
# Exhaustive FP8 scale sweep
# ---------------------------------------------------------------------------------------

def candidate_losses(mode: str, w_blk: np.ndarray, h_blk: np.ndarray, p_blk, g) -> tuple:
    """Losses of all 126 candidates for U units.

    w_blk: [U, 16] fp32 weights; h_blk: [U, 16, 16] (full/act) or [U, 16] (diag);
    p_blk: [U, 16, 16] (act) or None. Returns (L [U, 126], wq [U, 126, 16] fp32, E0 [U]).
    FULL: L = dW^T H dW; ACT: + 2 dW^T (P w); DIAG: sum Imp dW^2, with dW = wq - w (PR #1976);
    MSE: sum dW^2, the plain block MSE (h_blk unused), i.e. H = I.
    E0 is the q = 0 loss without the cross term, the scale for relative comparisons.
    """
    w = np.asarray(w_blk, dtype=np.float32)
    s = candidate_scales(g)  # [126]
    wq = fake_quant(w[:, None, :], s[None, :, None])  # [U, 126, 16]
    dw = wq.astype(np.float64) - w.astype(np.float64)[:, None, :]
    w64 = w.astype(np.float64)
    if mode == "mse":
        return np.einsum("uki,uki->uk", dw, dw), wq, np.einsum("ui,ui->u", w64, w64)
    h = np.asarray(h_blk, dtype=np.float64)
    if mode == "diag":
        loss = np.einsum("uki,ui->uk", dw * dw, h)
        e0 = np.einsum("ui,ui->u", w64 * w64, h)
    else:
        loss = np.einsum("uki,uij,ukj->uk", dw, h, dw)
        e0 = np.einsum("ui,uij,uj->u", w64, h, w64)
        if mode == "act":
            pw = np.einsum("uij,uj->ui", np.asarray(p_blk, dtype=np.float64), w64)
            loss = loss + 2.0 * np.einsum("uki,ui->uk", dw, pw)
    return loss, wq, e0


def argmin_lowest(loss: np.ndarray):
    """Best candidate per unit scanning codes ascending from best = +inf with strict < (PR #1976
    reviews: the best loss starts at +inf and may end negative).

    Returns (k* index [U], best loss [U], second-best loss [U]).
    """
    u, k = loss.shape
    best = np.full(u, np.inf)
    kbest = np.zeros(u, dtype=np.int64)
    for j in range(k):
        better = loss[:, j] < best
        best = np.where(better, loss[:, j], best)
        kbest = np.where(better, j, kbest)
    masked = loss.copy()
    masked[np.arange(u), kbest] = np.inf
    return kbest, best, masked.min(axis=1)


def sweep_units(mode: str, w_blk, h_blk, p_blk, g):
    """Sweep U independent units over all 126 candidates (PR #2283, How). Returns dict of codes
    (uint8), wq [U,16], loss, second, e0."""
    loss, wq, e0 = candidate_losses(mode, w_blk, h_blk, p_blk, g)
    kbest, best, second = argmin_lowest(loss)
    u = np.arange(len(kbest))
    return {
        "codes": (kbest + 1).astype(np.uint8),
        "wq": wq[u, kbest],
        "loss": best,
        "second": second,
        "e0": e0,
        "escale": loss_scale(mode, w_blk, h_blk, p_blk),
        "all_losses": loss,
    }


def loss_scale(mode: str, w_blk, h_blk, p_blk) -> np.ndarray:
    """|w|^T |H| |w| (+ 2 |w|^T |P| |w| for ACT; sum Imp w^2 for DIAG) per unit. Not a step of
    the method: the denominator of the parity gate, a reading of this project's.

    The magnitude that bounds the rounding error of any Hessian-weighted loss of this block
    evaluated in finite precision; it is >= E0 and equals it for a diagonal H. Parity gaps
    and loss errors are measured relative to max(|L*|, this scale).
    """
    a = np.abs(np.asarray(w_blk, dtype=np.float64))
    if mode == "mse":
        return np.einsum("ui,ui->u", a, a)
    h = np.abs(np.asarray(h_blk, dtype=np.float64))
    if mode == "diag":
        return np.einsum("ui,ui->u", a * a, h)
    s = np.einsum("ui,uij,uj->u", a, h, a)
    if mode == "act":
        s = s + 2.0 * np.einsum("ui,uij,uj->u", a, np.abs(np.asarray(p_blk, dtype=np.float64)), a)
    return s


def gather_units(mode: str, w, h, p, g, units):
    """Slice units (group, row, block) out of whole-layer tensors.

    w [G, R, C] fp32; h [G, N, 16, 16] or [G, N, 16]; p like h or None; g [G].
    units: int array [U, 3]. Returns (w_blk, h_blk, p_blk, g_per_unit).
    """
    units = np.asarray(units, dtype=np.int64)
    ge, r, n = units[:, 0], units[:, 1], units[:, 2]
    cols = n[:, None] * BLOCK + np.arange(BLOCK)[None, :]
    w_blk = np.asarray(w)[ge[:, None], r[:, None], cols]
    h_blk = None if h is None else np.asarray(h)[ge, n]
    p_blk = None if p is None else np.asarray(p)[ge, n]
    return w_blk, h_blk, p_blk, np.asarray(g)[ge]


def sweep(mode: str, w, h, p, g, units=None, chunk: int = 512):
    """Sweep the given units (default: all) of a layer; g has one entry per group (one weight
    quantizer per expert, PR #2864 / #2840).

    Returns dict with codes, wq, loss, second, e0 for each unit, in ``units`` order.
    """
    w = np.asarray(w, dtype=np.float32)
    gcount, rows, cin = w.shape
    if units is None:
        ge, r, n = np.meshgrid(np.arange(gcount), np.arange(rows), np.arange(cin // BLOCK), indexing="ij")
        units = np.stack([ge.ravel(), r.ravel(), n.ravel()], axis=1)
    units = np.asarray(units, dtype=np.int64)
    outs = []
    for lo in range(0, len(units), chunk):
        sub = units[lo:lo + chunk]
        wb, hb, pb, gu = gather_units(mode, w, h, p, g, sub)
        # Units in a chunk may belong to different groups: sweep each group's slice.
        res = {k: [] for k in ("codes", "wq", "loss", "second", "e0", "escale")}
        order = []
        for gv in np.unique(gu):
            sel = np.nonzero(gu == gv)[0]
            o = sweep_units(mode, wb[sel], None if hb is None else hb[sel], None if pb is None else pb[sel], gv)
            for k in res:
                res[k].append(o[k])
            order.append(sel)
        order = np.concatenate(order)
        inv = np.empty_like(order)
        inv[order] = np.arange(len(order))
        outs.append({k: np.concatenate(v)[inv] for k, v in res.items()})
    return {k: np.concatenate([o[k] for o in outs]) for k in outs[0]} if outs else {}


def losses_for_scales(mode: str, w_blk, h_blk, p_blk, s) -> tuple:
    """Losses of given block scales: s [U, K] fp32 (0 allowed) for U units (the losses of
    ``candidate_losses`` at other scales, for the multiplier search of PR #788).

    Same definitions as ``candidate_losses`` (which is this with the 126 candidate scales
    for every unit). Returns (L [U, K], wq [U, K, 16] fp32).
    """
    w = np.asarray(w_blk, dtype=np.float32)
    s = np.asarray(s, dtype=np.float32)
    wq = fake_quant(w[:, None, :], s[:, :, None])
    dw = wq.astype(np.float64) - w.astype(np.float64)[:, None, :]
    if mode == "mse":
        return np.einsum("uki,uki->uk", dw, dw), wq
    h = np.asarray(h_blk, dtype=np.float64)
    if mode == "diag":
        return np.einsum("uki,ui->uk", dw * dw, h), wq
    loss = np.einsum("uki,uij,ukj->uk", dw, h, dw)
    if mode == "act":
        pw = np.einsum("uij,uj->ui", np.asarray(p_blk, dtype=np.float64), w.astype(np.float64))
        loss = loss + 2.0 * np.einsum("uki,ui->uk", dw, pw)
    return loss, wq


def multiplier_codes(w_blk, g, multipliers) -> np.ndarray:
    """Block-scale codes of the amax-multiplier search (PR #788, Changes table: step size and
    multipliers): [U, M].

    For multiplier m the block's candidate amax is fp32(m * amax_blk) (amax_blk = max |w| of
    the block), and it becomes a block scale as in the NVFP4 quantizer: the E4M3 code nearest to
    amax / (6 g) on the exact quotient (ties to the even code, saturating at 448; 0 is a zero
    scale). g == 0 gives code 0.
    """
    w = np.asarray(w_blk, dtype=np.float32)
    amax = np.abs(w.astype(np.float64)).max(axis=1)  # exact
    m = np.asarray(multipliers, dtype=np.float32).astype(np.float64)
    with np.errstate(invalid="ignore"):
        a = (m[None, :] * amax[:, None]).astype(np.float32).astype(np.float64)  # exact product, one rounding
    a = np.where(np.isnan(a) | (a < 0), 0.0, a)  # a negative or NaN candidate amax counts as 0
    g64 = np.float64(np.float32(g))
    if g64 == 0:
        return np.zeros(a.shape, dtype=np.int64)
    return e4m3_round(a / (FP4_MAX * g64))


def multiplier_search_units(mode: str, w_blk, h_blk, p_blk, g, multipliers):
    """Amax-multiplier search on U units (the non-sweep search of the MSE calibrator that
    "add local hessian calibration", PR #788, configures by step size and multipliers).

    Candidates are the multipliers in the given order; each is scored with the loss of
    ``mode`` at the scale of its code (``multiplier_codes``); the first multiplier with the
    smallest loss wins (strict <). Returns codes, wq, loss, index (winning multiplier),
    second (the best loss among candidates with another code; +inf if none), e0, escale.
    """
    w = np.asarray(w_blk, dtype=np.float32)
    codes = multiplier_codes(w, g, multipliers)
    v = np.where(codes > 0, e4m3_value(np.maximum(codes, 1)), 0.0)
    s = (v * np.float64(np.float32(g))).astype(np.float32)
    loss, wq = losses_for_scales(mode, w, h_blk, p_blk, s)
    idx, best, _ = argmin_lowest(loss)
    u = np.arange(len(idx))
    bc = codes[u, idx]
    other = np.where(codes != bc[:, None], loss, np.inf)
    w64 = w.astype(np.float64)  # E0: the q = 0 loss without the cross term
    if mode == "mse":
        e0 = np.einsum("ui,ui->u", w64, w64)
    elif mode == "diag":
        e0 = np.einsum("ui,ui->u", w64 * w64, np.asarray(h_blk, dtype=np.float64))
    else:
        e0 = np.einsum("ui,uij,uj->u", w64, np.asarray(h_blk, dtype=np.float64), w64)
    return {
        "codes": bc.astype(np.uint8),
        "wq": wq[u, idx],
        "loss": best,
        "index": idx,
        "second": other.min(axis=1),
        "e0": e0,
        "escale": loss_scale(mode, w, h_blk, p_blk),
        "all_codes": codes,
    }


def multiplier_search(mode: str, w, h, p, g, multipliers, units=None):
    """``multiplier_search_units`` over the given units (default: all) of a layer."""
    w = np.asarray(w, dtype=np.float32)
    gcount, rows, cin = w.shape
    if units is None:
        ge, r, n = np.meshgrid(np.arange(gcount), np.arange(rows), np.arange(cin // BLOCK), indexing="ij")
        units = np.stack([ge.ravel(), r.ravel(), n.ravel()], axis=1)
    units = np.asarray(units, dtype=np.int64)
    wb, hb, pb, gu = gather_units(mode, w, h, p, g, units)
    keys = ("codes", "wq", "loss", "index", "second", "e0", "escale")
    res = {k: np.empty((len(units),) + ((BLOCK,) if k == "wq" else ()),
                       dtype={"codes": np.uint8, "wq": np.float32, "index": np.int64}.get(k, np.float64))
           for k in keys}
    for gv in np.unique(gu):  # units of one group share g
        sel = np.nonzero(gu == gv)[0]
        o = multiplier_search_units(mode, wb[sel], None if hb is None else hb[sel],
                                    None if pb is None else pb[sel], gv, multipliers)
        for k in keys:
            res[k][sel] = o[k]
    return res


def apply_scales(w, g, codes):
    """Fake-quantized weights and per-block amax for chosen block-scale codes.

    w [G, R, C] fp32 values; g [G]; codes [G, R, C/16] (E4M3 bytes, 0 = zero scale, values
    above 126 taken as 126). Returns (wq fp32 [G, R, C], wq rounded to bf16 [G, R, C] as fp32
    values, amax [G, R, C/16] fp32). The block's amax is the value whose NVFP4 scale is the
    chosen one, fp32(6 v g) ("Add WMSE weight scale search calibration", PR #2283, the
    quantizer state it fingerprints: amax and the per-block _amax); the exact product has at
    most 29 significant bits, so it is rounded once.
    """
    w = np.asarray(w, dtype=np.float32)
    gcount, rows, cin = w.shape
    c = np.minimum(np.asarray(codes, dtype=np.int64), N_CANDIDATES)
    v = np.where(c > 0, e4m3_value(np.maximum(c, 1)), 0.0)  # [G, R, N]
    g64 = np.asarray(g, dtype=np.float32).astype(np.float64)[:, None, None]
    s = (v * g64).astype(np.float32)
    wq = fake_quant(w.reshape(gcount, rows, cin // BLOCK, BLOCK), s[..., None]).reshape(gcount, rows, cin)
    amax = (FP4_MAX * v * g64).astype(np.float32)
    return wq, f32_to_bf16_values(wq), amax


def calibrate(mode: str, x, w, xq=None, group_offsets=None, token_ids=None, units=None, act_gx=None):
    """The whole hot path (PR #788, #1976, #2283, #2004, #2864): accumulate, finalize, global
    scale per group, sweep. MSE has no
    statistics: x is ignored and the sweep uses H = I."""
    if mode == "mse":
        w = np.asarray(w, dtype=np.float32)
        g = np.array([global_scale(w[e]) for e in range(w.shape[0])], dtype=np.float32)
        out = sweep(mode, w, None, None, g, units)
        out.update({"h": None, "p": None, "g": g, "counts": None})
        return out
    hsum, psum, counts = accumulate(mode, x, xq, group_offsets, token_ids, act_gx)
    h, p = finalize(mode, hsum, psum, counts)
    w = np.asarray(w, dtype=np.float32)
    g = np.array([global_scale(w[e]) for e in range(w.shape[0])], dtype=np.float32)
    out = sweep(mode, w, h, p, g, units)
    out.update({"h": h, "p": p, "g": g, "counts": counts})
    return out
