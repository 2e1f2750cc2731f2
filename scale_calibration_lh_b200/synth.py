"""Seeded synthetic inputs for the calibration hot path.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds no step of the calibration method itself (no Hessian,
no scale sweep, no loss): only random draws, their shaping into the layer
workloads below, and bf16 rounding of the drawn values.

Workloads (token-major activations X[T, C], weights W[G, R, C]):

* ``tiny``  : X fp32 [256, 64] ~ N(0, 1); W fp32 [32, 64] ~ N(0, 0.02^2); full H.
* ``dense`` : X bf16 [16384, 4096], per-column std sigma_i = exp(N(0, 1)) with
  round(1% of C) distinct columns (chosen uniformly) multiplied by 20;
  W bf16 [4096, 4096] ~ N(0, (1/sqrt(4096))^2); full H.
* ``act``   : X as ``dense`` at [32768, 4096]; W bf16 [12288, 4096]; activation-aware H
  and P, where X_q is the NVFP4 input quantizer's output of X (derived from X by the
  calibration path itself; this module draws X only).
* ``wmse``  : X bf16 [65536, 12288], sigma_i = exp(N(0, 1.5^2)), no outliers;
  W bf16 [4096, 12288] ~ N(0, 1/12288); diagonal importance.
* ``moe``   : X bf16 [16384, 2560] drawn as ``dense``; each token routed to 10
  distinct experts of 512 chosen uniformly; CSR sorted by expert with token ids
  ascending; W bf16 [512, 1280, 2560] ~ N(0, 1/2560); grouped full H with a
  global scale per expert.

The pages name the workloads' shapes and distributions but never the
calibration data itself, so these draws stand in for captured activations.

Random numbers come from numpy PCG64 streams, one per 2^22-element chunk and per
tensor tag, seeded by ``SeedSequence([seed, tag, chunk])``; chunks are filled on
a thread pool, so the values do not depend on the thread count.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

CHUNK = 1 << 22
_TAGS = {"sigma": 1, "outlier": 2, "x": 3, "w": 4, "route": 5}

WORKLOADS = ("tiny", "dense", "act", "wmse", "moe")

# Full sizes of each workload: (tokens, cin, rows, groups).
FULL_SIZES = {
    "tiny": (256, 64, 32, 1),
    "dense": (16384, 4096, 4096, 1),
    "act": (32768, 4096, 12288, 1),
    "wmse": (65536, 12288, 4096, 1),
    "moe": (16384, 2560, 1280, 512),
}
MODES = {"tiny": "full", "dense": "full", "act": "act", "wmse": "diag", "moe": "full"}
MOE_TOP_K = 10


def _pool():
    return ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1))


def _normal_f32(n: int, seed: int, tag: str) -> np.ndarray:
    """n standard normal float32 draws, chunked into independent streams."""
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + CHUNK - 1) // CHUNK

    def fill(i):
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], i])))
        lo, hi = i * CHUNK, min(n, (i + 1) * CHUNK)
        g.standard_normal(out=out[lo:hi], dtype=np.float32)

    if nchunks == 1:
        fill(0)
    else:
        with _pool() as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def _rng(seed: int, tag: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], 0])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bit patterns.

    Inputs are finite by construction, so NaN handling is not needed.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    flat_u, flat_o = u.reshape(-1), out.reshape(-1)

    def rnd(lo_hi):
        lo, hi = lo_hi
        v = flat_u[lo:hi]
        r = v + np.uint32(0x7FFF) + ((v >> np.uint32(16)) & np.uint32(1))
        flat_o[lo:hi] = (r >> np.uint32(16)).astype(np.uint16)

    spans = [(i, min(flat_u.size, i + CHUNK)) for i in range(0, flat_u.size, CHUNK)]
    if len(spans) <= 1:
        for s in spans:
            rnd(s)
    else:
        with _pool() as ex:
            list(ex.map(rnd, spans))
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _scaled_columns(tokens: int, cin: int, sigma: np.ndarray, seed: int) -> np.ndarray:
    z = _normal_f32(tokens * cin, seed, "x").reshape(tokens, cin)
    # Multiply in place chunk by chunk to bound temporaries.
    rows_per = max(1, CHUNK // max(cin, 1))
    spans = [(r, min(tokens, r + rows_per)) for r in range(0, tokens, rows_per)]

    def mul(span):
        lo, hi = span
        z[lo:hi] *= sigma[None, :]

    with _pool() as ex:
        list(ex.map(mul, spans))
    return z


def _column_sigma(cin: int, seed: int, log_std: float, outlier_frac: float) -> np.ndarray:
    sigma = np.exp(_rng(seed, "sigma").normal(0.0, log_std, size=cin)).astype(np.float32)
    n_out = int(round(outlier_frac * cin))
    if n_out:
        cols = _rng(seed, "outlier").choice(cin, size=n_out, replace=False)
        sigma[cols] *= np.float32(20.0)
    return sigma


# --- workloads ------------------------------------------------------------------------------


@dataclass
class Layer:
    """One synthetic layer. bf16 tensors are uint16 bit patterns."""

    name: str
    mode: str  # "full" | "act" | "diag"
    dtype: str  # "f32" | "bf16"
    x: np.ndarray  # [T, C]
    w: np.ndarray  # [G, R, C]
    xq: np.ndarray | None = None
    group_offsets: np.ndarray | None = None  # int32 [G + 1]
    token_ids: np.ndarray | None = None  # int32 [group_offsets[-1]]
    meta: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return int(self.x.shape[0])

    @property
    def cin(self) -> int:
        return int(self.x.shape[1])

    @property
    def groups(self) -> int:
        return int(self.w.shape[0])

    @property
    def rows(self) -> int:
        return int(self.w.shape[1])

    def x_f32(self) -> np.ndarray:
        return self.x if self.dtype == "f32" else bf16_bits_to_f32(self.x)

    def xq_f32(self) -> np.ndarray:
        return self.xq if self.dtype == "f32" else bf16_bits_to_f32(self.xq)

    def w_f32(self) -> np.ndarray:
        return self.w if self.dtype == "f32" else bf16_bits_to_f32(self.w)


def moe_routing(tokens: int, experts: int, top_k: int, seed: int):
    """Uniform top-k routing: each token picks top_k distinct experts.

    Returns CSR (offsets[experts + 1], token ids sorted by expert, ascending within).
    """
    g = _rng(seed, "route")
    keys = g.random((tokens, experts), dtype=np.float32) if experts > 1 else np.zeros((tokens, 1), np.float32)
    top_k = min(top_k, experts)
    picks = np.argpartition(keys, top_k - 1, axis=1)[:, :top_k] if top_k < experts else np.tile(np.arange(experts), (tokens, 1))
    exp_flat = picks.reshape(-1).astype(np.int64)
    tok_flat = np.repeat(np.arange(tokens, dtype=np.int64), top_k)
    order = np.lexsort((tok_flat, exp_flat))
    token_ids = tok_flat[order].astype(np.int32)
    counts = np.bincount(exp_flat, minlength=experts)
    offsets = np.zeros(experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    return offsets, token_ids


def make_layer(name: str, seed: int = 0, tokens: int | None = None, cin: int | None = None,
               rows: int | None = None, groups: int | None = None, top_k: int = MOE_TOP_K) -> Layer:
    """Build workload ``name`` at its full size, or at the given smaller sizes."""
    if name not in FULL_SIZES:
        raise ValueError(f"unknown workload {name!r}")
    T0, C0, R0, G0 = FULL_SIZES[name]
    T = T0 if tokens is None else tokens
    C = C0 if cin is None else cin
    R = R0 if rows is None else rows
    G = G0 if groups is None else groups
    if C % 16:
        raise ValueError("cin must be a multiple of 16")
    mode = MODES[name]
    if name == "tiny":
        x = _normal_f32(T * C, seed, "x").reshape(T, C)
        w = (_normal_f32(G * R * C, seed, "w") * np.float32(0.02)).reshape(G, R, C)
        return Layer(name, mode, "f32", x, w)
    log_std, outl = (1.5, 0.0) if name == "wmse" else (1.0, 0.01)
    sigma = _column_sigma(C, seed, log_std, outl)
    xf = _scaled_columns(T, C, sigma, seed)
    x = f32_to_bf16_bits(xf)
    del xf
    wf = _normal_f32(G * R * C, seed, "w").reshape(G, R, C)
    wf *= np.float32(1.0 / np.sqrt(C))
    w = f32_to_bf16_bits(wf)
    del wf
    layer = Layer(name, mode, "bf16", x, w, meta={"sigma": sigma})
    if name == "moe":
        layer.group_offsets, layer.token_ids = moe_routing(T, G, top_k, seed)
    return layer


# --- device placement (torch imported lazily; no step of the method) -------------------------


def to_device(a: np.ndarray | None, kind: str, device="cuda"):
    """Copy a host array to a torch device tensor. kind: 'bf16' (uint16 bit patterns, kept
    bit for bit), 'f32' or 'i32'."""
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


def layer_to_device(layer: Layer, device="cuda") -> dict:
    """A layer's tensors on the device: x, xq, w, the CSR routing (offs, ids) and the input
    quantizer's global scale act_gx when the layer carries one (None where absent)."""
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
