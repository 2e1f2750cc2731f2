"""Python binding of liblhcal.so (local-Hessian NVFP4 weight-scale calibration on B200).

Argument marshalling only: every step runs in the CUDA library. Functions carry the C
names (``lhcal_accumulate`` ...) and take torch tensors, passing their device pointers,
sizes and the current CUDA stream. Since the C layer sees only pointers, each wrapper first
checks every tensor's dtype, density and element count against the sizes it passes. A
missing or unloadable library raises at import of the first call; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblhcal.so")

# lhcal_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_DEVICE_MISMATCH, ERR_CUDA, ERR_TIMEOUT = range(6)
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "DEVICE_MISMATCH", 4: "CUDA", 5: "TIMEOUT"}
# lhcal_dtype / lhcal_mode / flags
F32, BF16 = 0, 1
FULL, ACT_AWARE, DIAG, MSE = 0, 1, 2, 3
ACCUM_ADD, ACCUM_OVERWRITE = 0, 1
N_CANDIDATES = 126
BLOCK = 16
MODE_IDS = {"full": FULL, "act": ACT_AWARE, "diag": DIAG, "mse": MSE}

_lib = None


class LhcalError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"lhcal {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblhcal.so (built by ``python -m scale_calibration_lh_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"liblhcal.so not found at {path}; build it with "
                           "`python -m scale_calibration_lh_b200.build`")
    lib = ctypes.CDLL(path)
    i32, i64, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    sigs = {
        "lhcal_accumulate_workspace": [i32, i32, i64, i64, i32, ctypes.POINTER(sz)],
        "lhcal_accumulate": [i32, i32, vp, vp, i64, i64, i64, i32, vp, vp, i32, vp, vp, vp, sz, vp],
        "lhcal_accumulate_noalloc": [i32, i32, vp, vp, i64, i64, i64, i32, vp, vp, i32, vp, vp, vp],
        "lhcal_accumulate_act_quant_workspace": [i32, i64, i64, i32, ctypes.POINTER(sz)],
        "lhcal_accumulate_act_quant": [i32, vp, i64, i64, i64, i32, vp, vp, vp, i32, vp, vp, vp, sz, vp],
        "lhcal_act_fake_quant": [i32, vp, i64, i64, i64, vp, vp, i64, vp],
        "lhcal_count_tokens": [i32, i64, vp, i32, vp, vp],
        "lhcal_finalize": [i32, i32, i64, vp, vp, vp, vp],
        "lhcal_global_scale": [i32, vp, i32, i64, i64, vp, vp],
        "lhcal_global_scale_ex": [i32, vp, i32, i64, i64, ctypes.c_float, vp, vp],
        "lhcal_multiplier_search": [i32, i32, vp, i32, i64, i64, vp, vp, vp, vp, i32, vp, vp, vp, vp],
        "lhcal_apply_scales": [i32, vp, i32, i64, i64, vp, vp, vp, vp, vp, vp],
        "lhcal_scale_sweep": [i32, i32, vp, i32, i64, i64, vp, vp, vp, vp, vp, vp, vp],
    }
    for name, args in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.lhcal_last_error_string.restype = ctypes.c_char_p
    lib.lhcal_last_error_string.argtypes = []
    lib.lhcal_version.restype = ctypes.c_int32
    lib.lhcal_version.argtypes = []
    lib.lhcal_launch_count.restype = ctypes.c_int64
    lib.lhcal_launch_count.argtypes = [ctypes.c_int32]
    _lib = lib
    return lib


def _check(status: int):
    if status != OK:
        msg = load_library().lhcal_last_error_string().decode(errors="replace")
        raise LhcalError(status, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ld(t, cin: int) -> int:
    """Row stride in elements; an empty tensor's stride carries no meaning, so cin is passed."""
    return int(t.stride(0)) if t.shape[0] > 0 else cin


def _need(t, name: str, numel: int, dtype=None, dense: bool = True):
    """Reject a tensor the library would misread. The entry points take bare pointers and
    infer a dense layout from the sizes, so a short, strided or mistyped buffer would be
    read or written past its end without an error. None passes (the C layer decides
    whether the pointer is optional)."""
    if t is None:
        return
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dense and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements; the call needs {numel}")


def _stats_numel(m: int, groups: int, cin: int) -> int:
    """fp32 elements of H (or P): [groups, cin/16, 16, 16], or [groups, cin/16, 16] for DIAG."""
    return groups * (cin // BLOCK) * (BLOCK if m == DIAG else BLOCK * BLOCK)


def _check_xq(x, xq):
    """X_q is read with x's row stride (the two-tensor entry points take one ldx for both)."""
    if xq is None:
        return
    if tuple(xq.shape) != tuple(x.shape) or xq.dtype != x.dtype:
        raise ValueError(f"xq {tuple(xq.shape)} {xq.dtype} must match x {tuple(x.shape)} {x.dtype}")
    if x.numel() and (xq.stride(1) != 1 or xq.stride(0) != x.stride(0)):
        raise ValueError("xq must have x's row stride and unit stride along cin")


def _check_stats(m: int, x, h, p, group_offsets, token_ids, groups: int):
    import torch

    n = _stats_numel(m, groups, int(x.shape[1]))
    _need(h, "h", n, torch.float32)
    if m == ACT_AWARE:
        _need(p, "p", n, torch.float32)
    _need(group_offsets, "group_offsets", groups + 1, torch.int32)
    _need(token_ids, "token_ids", 0, torch.int32)


def _check_sweep_buffers(m: int | None, w, h, p, g, codes, wq, loss, wq16=None, amax=None):
    import torch

    groups, rows, cin = (int(v) for v in w.shape)
    units = groups * rows * (cin // BLOCK)
    _need(w, "w", 0)
    if m is not None and m != MSE:
        n = _stats_numel(m, groups, cin)
        _need(h, "h", n, torch.float32)
        if m == ACT_AWARE:
            _need(p, "p", n, torch.float32)
    _need(g, "g", groups, torch.float32)
    _need(codes, "codes", units, torch.uint8)
    _need(wq, "wq", groups * rows * cin, torch.float32)
    _need(wq16, "wq16", groups * rows * cin, torch.bfloat16)
    _need(loss, "loss", units, torch.float32)
    _need(amax, "amax", units, torch.float32)


def _dtype_id(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _mode_id(mode) -> int:
    return MODE_IDS[mode] if isinstance(mode, str) else int(mode)


def lhcal_version() -> int:
    return int(load_library().lhcal_version())


def lhcal_launch_count(reset: bool = False) -> int:
    """Kernels enqueued by the library from this thread (since the last reset)."""
    return int(load_library().lhcal_launch_count(1 if reset else 0))


def lhcal_accumulate_workspace(mode, dtype: int, tokens: int, cin: int, groups: int = 1) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().lhcal_accumulate_workspace(_mode_id(mode), dtype, tokens, cin, groups, ctypes.byref(out)))
    return int(out.value)


def lhcal_accumulate(mode, x, h, xq=None, p=None, group_offsets=None, token_ids=None,
                     flags: int = ACCUM_ADD, workspace=None, stream=None):
    """x, xq: [tokens, cin] (row stride x.stride(0)); h, p, workspace: fp32 device tensors."""
    m = _mode_id(mode)
    tokens, cin = int(x.shape[0]), int(x.shape[1])
    if x.numel() and x.stride(1) != 1:
        raise ValueError("x must have unit stride along cin")
    groups = 1 if group_offsets is None else int(group_offsets.numel()) - 1
    _check_xq(x, xq)
    _check_stats(m, x, h, p, group_offsets, token_ids, groups)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().lhcal_accumulate(
        m, _dtype_id(x), _ptr(x), _ptr(xq), tokens, cin, _ld(x, cin), groups,
        _ptr(group_offsets), _ptr(token_ids), flags, _ptr(h), _ptr(p), _ptr(workspace), ws_bytes,
        _stream(stream)))


def lhcal_accumulate_act_quant_workspace(dtype: int, tokens: int, cin: int, groups: int = 1) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().lhcal_accumulate_act_quant_workspace(dtype, tokens, cin, groups, ctypes.byref(n)))
    return int(n.value)


def lhcal_accumulate_act_quant(x, h, p, act_gx, group_offsets=None, token_ids=None, flags: int = ACCUM_ADD,
                               workspace=None, stream=None):
    """Activation-aware accumulation with the input quantizer fused: X_q is derived from x (bf16)
    in the kernel with the global scale act_gx (fp32 device scalar); h, p as for ``act``."""
    import torch

    tokens, cin = int(x.shape[0]), int(x.shape[1])
    if x.numel() and x.stride(1) != 1:
        raise ValueError("x must have unit stride along cin")
    groups = 1 if group_offsets is None else int(group_offsets.numel()) - 1
    _check_stats(ACT_AWARE, x, h, p, group_offsets, token_ids, groups)
    _need(act_gx, "act_gx", 1, torch.float32)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().lhcal_accumulate_act_quant(
        _dtype_id(x), _ptr(x), tokens, cin, _ld(x, cin), groups, _ptr(group_offsets), _ptr(token_ids),
        _ptr(act_gx), flags, _ptr(h), _ptr(p), _ptr(workspace), ws_bytes, _stream(stream)))


def lhcal_act_fake_quant(x, act_gx, xq, stream=None):
    """X_q = NVFP4 fake quant of bf16 x [tokens, cin] with global scale act_gx, into bf16 xq."""
    import torch

    tokens, cin = int(x.shape[0]), int(x.shape[1])
    if xq is None or tuple(xq.shape) != tuple(x.shape):
        raise ValueError("xq must be a tensor shaped like x")
    _need(xq, "xq", 0, torch.bfloat16, dense=False)  # its own row stride is passed
    _need(act_gx, "act_gx", 1, torch.float32)
    if x.numel() and (x.stride(1) != 1 or xq.stride(1) != 1):
        raise ValueError("x and xq must have unit stride along cin")
    _check(load_library().lhcal_act_fake_quant(_dtype_id(x), _ptr(x), tokens, cin, _ld(x, cin), _ptr(act_gx),
                                               _ptr(xq), _ld(xq, cin), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


def lhcal_accumulate_noalloc(mode, x, h, xq=None, p=None, group_offsets=None, token_ids=None,
                             flags: int = ACCUM_ADD, stream=None):
    """lhcal_accumulate for callers that cannot allocate: uses the library's fixed scratch.

    For callers whose device memory is owned by someone else (a host framework's memory
    planner, a plugin handed only its inputs and outputs) and who therefore cannot supply
    a workspace. Sizes needing more than NOALLOC_SCRATCH_BYTES of scratch are rejected;
    calls that may overlap on the GPU share the scratch and must be ordered.
    """
    m = _mode_id(mode)
    tokens, cin = int(x.shape[0]), int(x.shape[1])
    if x.numel() and x.stride(1) != 1:
        raise ValueError("x must have unit stride along cin")
    groups = 1 if group_offsets is None else int(group_offsets.numel()) - 1
    _check_xq(x, xq)
    _check_stats(m, x, h, p, group_offsets, token_ids, groups)
    _check(load_library().lhcal_accumulate_noalloc(
        m, _dtype_id(x), _ptr(x), _ptr(xq), tokens, cin, _ld(x, cin), groups,
        _ptr(group_offsets), _ptr(token_ids), flags, _ptr(h), _ptr(p), _stream(stream)))


def lhcal_count_tokens(counts, tokens: int = 0, group_offsets=None, flags: int = ACCUM_ADD, stream=None):
    import torch

    groups = 1 if group_offsets is None else int(group_offsets.numel()) - 1
    _need(counts, "counts", groups, torch.int64)
    _need(group_offsets, "group_offsets", groups + 1, torch.int32)
    _check(load_library().lhcal_count_tokens(groups, tokens, _ptr(group_offsets), flags, _ptr(counts),
                                             _stream(stream)))


def lhcal_finalize(mode, counts, h, p=None, stream=None):
    import torch

    m = _mode_id(mode)
    groups = int(h.shape[0])
    cin = int(h.shape[1]) * BLOCK
    _need(h, "h", _stats_numel(m, groups, cin), torch.float32)
    if m == ACT_AWARE:
        _need(p, "p", _stats_numel(m, groups, cin), torch.float32)
    _need(counts, "counts", groups, torch.int64)
    _check(load_library().lhcal_finalize(m, groups, cin, _ptr(counts), _ptr(h), _ptr(p), _stream(stream)))


def lhcal_global_scale(w, g, stream=None, fp8_max: float | None = None):
    """w: [groups, rows, cin] fp32/bf16; g: fp32 [groups]. fp8_max: 448 (default) or 256 (4/6)."""
    groups, rows, cin = (int(v) for v in w.shape)
    _check_sweep_buffers(None, w, None, None, g, None, None, None)
    if fp8_max is None:
        _check(load_library().lhcal_global_scale(_dtype_id(w), _ptr(w), groups, rows, cin, _ptr(g), _stream(stream)))
    else:
        _check(load_library().lhcal_global_scale_ex(_dtype_id(w), _ptr(w), groups, rows, cin, float(fp8_max),
                                                    _ptr(g), _stream(stream)))


def lhcal_multiplier_search(mode, w, h, g, multipliers, codes, wq=None, loss=None, p=None, stream=None):
    """Amax-multiplier search: multipliers fp32 device [M]; other tensors as lhcal_scale_sweep."""
    import torch

    groups, rows, cin = (int(v) for v in w.shape)
    _check_sweep_buffers(_mode_id(mode), w, h, p, g, codes, wq, loss)
    _need(multipliers, "multipliers", 0, torch.float32)
    _check(load_library().lhcal_multiplier_search(
        _mode_id(mode), _dtype_id(w), _ptr(w), groups, rows, cin, _ptr(h), _ptr(p), _ptr(g), _ptr(multipliers),
        int(multipliers.numel()), _ptr(codes), _ptr(wq), _ptr(loss), _stream(stream)))


def lhcal_apply_scales(w, g, codes, wq=None, wq16=None, amax=None, stream=None):
    """Fake-quantized weights (fp32 wq, bf16 wq16) and per-block amax for chosen codes."""
    groups, rows, cin = (int(v) for v in w.shape)
    _check_sweep_buffers(None, w, None, None, g, codes, wq, None, wq16=wq16, amax=amax)
    _check(load_library().lhcal_apply_scales(_dtype_id(w), _ptr(w), groups, rows, cin, _ptr(g), _ptr(codes),
                                             _ptr(wq), _ptr(wq16), _ptr(amax), _stream(stream)))


def lhcal_scale_sweep(mode, w, h, g, codes, wq=None, loss=None, p=None, stream=None):
    """w [G, R, C]; h/p finalized; g [G]; codes uint8 [G, R, C/16]; wq fp32 [G, R, C]; loss fp32 [G, R, C/16]."""
    groups, rows, cin = (int(v) for v in w.shape)
    _check_sweep_buffers(_mode_id(mode), w, h, p, g, codes, wq, loss)
    _check(load_library().lhcal_scale_sweep(
        _mode_id(mode), _dtype_id(w), _ptr(w), groups, rows, cin, _ptr(h), _ptr(p), _ptr(g), _ptr(codes),
        _ptr(wq), _ptr(loss), _stream(stream)))


# ------------------------------------------------------------------------------------------------
# Buffers and the whole hot path
# ------------------------------------------------------------------------------------------------

class Buffers:
    """Device buffers for one layer's calibration (allocated by torch, owned by the caller)."""

    def __init__(self, mode, tokens: int, cin: int, rows: int, groups: int, x_dtype: int, device,
                 want_wq: bool = True, want_loss: bool = True, want_wq16: bool = False):
        import torch

        self.mode = _mode_id(mode)
        nblk = cin // BLOCK
        hshape = (groups, nblk, BLOCK) if self.mode == DIAG else (groups, nblk, BLOCK, BLOCK)
        # MSE (H = I) needs no statistics.
        self.h = None if self.mode == MSE else torch.empty(hshape, dtype=torch.float32, device=device)
        self.p = torch.empty(hshape, dtype=torch.float32, device=device) if self.mode == ACT_AWARE else None
        self.counts = torch.empty(groups, dtype=torch.int64, device=device)
        self.g = torch.empty(groups, dtype=torch.float32, device=device)
        self.codes = torch.empty((groups, rows, nblk), dtype=torch.uint8, device=device)
        self.wq = torch.empty((groups, rows, cin), dtype=torch.float32, device=device) if want_wq else None
        self.loss = torch.empty((groups, rows, nblk), dtype=torch.float32, device=device) if want_loss else None
        # bf16 fake-quantized weights, derived from the chosen codes by lhcal_apply_scales.
        self.wq16 = torch.empty((groups, rows, cin), dtype=torch.bfloat16, device=device) if want_wq16 else None
        ws = 0 if self.mode == MSE else lhcal_accumulate_workspace(self.mode, x_dtype, tokens, cin, groups)
        if self.mode == ACT_AWARE and x_dtype == BF16:  # either activation-aware entry point
            ws = max(ws, lhcal_accumulate_act_quant_workspace(x_dtype, tokens, cin, groups))
        self.workspace = torch.empty(max(ws // 4, 1), dtype=torch.float32, device=device) if ws else None


def calibrate(mode, x, w, xq=None, group_offsets=None, token_ids=None, buffers: Buffers | None = None,
              stream=None, act_gx=None) -> Buffers:
    """The whole hot path on one layer: accumulate, count, finalize, global scale, sweep.

    x [T, C], w [G, R, C] (and for ``act`` either xq or act_gx, the input quantizer's global
    scale from which the kernel derives X_q; CSR routing for grouped layers) are device
    tensors. Returns the buffers holding h, p, g, codes, wq and loss (and the bf16 fake-quantized
    weights wq16 when the buffers have them).
    """
    if stream is not None:  # enqueue everything on the given stream
        import torch

        with torch.cuda.stream(stream):
            return calibrate(mode, x, w, xq, group_offsets, token_ids, buffers, None, act_gx)
    m = _mode_id(mode)
    groups, rows, cin = (int(v) for v in w.shape)
    if m == MSE:  # plain block MSE: no statistics, x is not read
        b = buffers or Buffers(m, 0, cin, rows, groups, _dtype_id(w), w.device)
        _scales_and_sweep(m, w, b, 0, groups)
        return b
    if buffers is None:
        buffers = Buffers(m, int(x.shape[0]), cin, rows, groups, _dtype_id(x), x.device)
    b = buffers
    _statistics(m, x, b, xq=xq, group_offsets=group_offsets, token_ids=token_ids, act_gx=act_gx)
    _scales_and_sweep(m, w, b, 0, groups)
    return b


class HostOutputs:
    """Pinned host copies of a calibration's results: the codes (the chosen block scales), the
    per-group global scales and the winning losses, plus the fake-quantized weights that the
    buffers hold (fp32 ``wq`` when ``want_wq``, bf16 ``wq16`` when the buffers have it)."""

    def __init__(self, buffers: Buffers, want_wq: bool = True):
        import torch

        self.codes = torch.empty(buffers.codes.shape, dtype=torch.uint8, pin_memory=True)
        self.g = torch.empty(buffers.g.shape, dtype=torch.float32, pin_memory=True)
        self.wq = (torch.empty(buffers.wq.shape, dtype=torch.float32, pin_memory=True)
                   if want_wq and buffers.wq is not None else None)
        self.wq16 = (torch.empty(buffers.wq16.shape, dtype=torch.bfloat16, pin_memory=True)
                     if getattr(buffers, "wq16", None) is not None else None)
        self.loss = None if buffers.loss is None else torch.empty(buffers.loss.shape, dtype=torch.float32,
                                                                   pin_memory=True)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.g, self.wq, self.wq16, self.loss)
                   if t is not None)


_side_streams: dict = {}


def _side_stream(device, which: str):
    import torch

    key = (str(device), which)
    if key not in _side_streams:
        _side_streams[key] = torch.cuda.Stream(device=device)
    return _side_streams[key]


def _statistics(m, x, buffers, xq=None, group_offsets=None, token_ids=None, act_gx=None):
    """Accumulate, count and finalize on the current stream (nothing for MSE)."""
    b = buffers
    if m == MSE:
        return
    if m == ACT_AWARE and xq is None and act_gx is not None:
        lhcal_accumulate_act_quant(x, b.h, b.p, act_gx, group_offsets=group_offsets, token_ids=token_ids,
                                   flags=ACCUM_OVERWRITE, workspace=b.workspace)
    else:
        lhcal_accumulate(m, x, b.h, xq=xq, p=b.p, group_offsets=group_offsets, token_ids=token_ids,
                         flags=ACCUM_OVERWRITE, workspace=b.workspace)
    lhcal_count_tokens(b.counts, tokens=int(x.shape[0]), group_offsets=group_offsets, flags=ACCUM_OVERWRITE)
    lhcal_finalize(m, b.counts, b.h, p=b.p)


def _scales_and_sweep(m, w, buffers, e0: int, e1: int):
    """Global scales and sweep of groups [e0, e1) on the current stream, then the bf16
    fake-quantized weights of the chosen codes when the buffers hold wq16."""
    b = buffers
    sl = slice(e0, e1)
    lhcal_global_scale(w[sl], b.g[sl])
    lhcal_scale_sweep(m, w[sl], None if b.h is None else b.h[sl], b.g[sl], b.codes[sl],
                      wq=None if b.wq is None else b.wq[sl], loss=None if b.loss is None else b.loss[sl],
                      p=None if b.p is None else b.p[sl])
    if getattr(b, "wq16", None) is not None:
        lhcal_apply_scales(w[sl], b.g[sl], b.codes[sl], wq16=b.wq16[sl])


PIPELINE_CHUNK_BYTES = 64 << 20  # weights per chunk of calibrate_host's pipeline
SWEEP_TILE_ROWS = 128  # rows of one sweep CTA: row chunks start on multiples of it


def calibrate_host(mode, x, w, buffers: Buffers, staging: dict, hxq=None, group_offsets=None, token_ids=None,
                   out: HostOutputs | None = None, act_gx=None, group_chunks: int | None = None,
                   row_chunks: int = 8) -> HostOutputs:
    """The whole hot path from host tensors (pinned, for asynchronous copies) to host results.

    ``staging`` holds device tensors shaped like the inputs under keys "x", "w" and, when
    used, "xq", "offs", "ids". One side stream copies the activations (and routing) in, then the
    weights in chunks, starting at once: it waits only for what was enqueued before this call (an
    earlier call's kernels may still read the staging). The current stream computes the
    statistics as soon as the activations are in, then, chunk by chunk, it computes global
    scales and sweeps what is resident; each chunk's results are copied out on another side
    stream as soon as they are ready. A grouped layer (groups > 1) is chunked by
    groups: ``group_chunks`` chunks, by default enough for about 64 MB of weights each (at least
    8). A layer with one group needs all of its weights for its scale: it is copied in whole and
    its sweep is split into ``row_chunks`` chunks of rows, starting on multiples of the sweep's
    128-row tile, so every unit is computed exactly as in one sweep. The results land in ``out``
    (codes, global scales, loss, and the fake-quantized weights it was made for: fp32 wq, or
    bf16 wq16 when the buffers hold it); the function returns without synchronising, and the
    current stream waits for every copy it issued.
    """
    import torch

    m = _mode_id(mode)
    if out is None:
        out = HostOutputs(buffers)
    cur = torch.cuda.current_stream()
    dev = staging["w"].device
    s_in, s_out = _side_stream(dev, "in"), _side_stream(dev, "out")
    start = torch.cuda.Event()
    start.record(cur)
    s_in.wait_event(start)
    s_out.wait_event(start)
    groups, rows = int(w.shape[0]), int(w.shape[1])
    if groups > 1:
        n = group_chunks or max(8, -(-w.numel() * w.element_size() // PIPELINE_CHUNK_BYTES))
        n = max(1, min(n, groups))
        bounds = [groups * j // n for j in range(n + 1)]
    else:
        bounds = [0, 1]
    # Host-to-device copies run in the order they are issued, whatever their stream: the
    # activations (and routing) go first, so the statistics start as soon as they are in, and
    # the weight chunks follow on the same stream without a gap.
    ready = []
    with torch.cuda.stream(s_in):
        if m != MSE:
            staging["x"].copy_(x, non_blocking=True)
            if hxq is not None:
                staging["xq"].copy_(hxq, non_blocking=True)
            if group_offsets is not None:
                staging["offs"].copy_(group_offsets, non_blocking=True)
                staging["ids"].copy_(token_ids, non_blocking=True)
            x_in = torch.cuda.Event()
            x_in.record(s_in)
        for e0, e1 in zip(bounds[:-1], bounds[1:]):
            staging["w"][e0:e1].copy_(w[e0:e1], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s_in)
            ready.append(ev)
    if m != MSE:
        cur.wait_event(x_in)
        # X_q is read only when the caller copies it in; otherwise (act_gx) the kernel derives it.
        _statistics(m, staging["x"], buffers, xq=staging["xq"] if hxq is not None else None,
                    group_offsets=staging.get("offs") if group_offsets is not None else None,
                    token_ids=staging.get("ids") if token_ids is not None else None, act_gx=act_gx)

    def copy_out(e0, e1, r0, r1, with_g):
        done = torch.cuda.Event()
        done.record(cur)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            for name in ("codes", "wq16", "loss", "wq"):
                dst = getattr(out, name)
                if dst is not None:
                    dst[e0:e1, r0:r1].copy_(getattr(buffers, name)[e0:e1, r0:r1], non_blocking=True)
            if with_g:
                out.g[e0:e1].copy_(buffers.g[e0:e1], non_blocking=True)

    if groups > 1:
        for (e0, e1), ev in zip(zip(bounds[:-1], bounds[1:]), ready):
            cur.wait_event(ev)
            _scales_and_sweep(m, staging["w"], buffers, e0, e1)
            copy_out(e0, e1, 0, rows, True)
    else:
        cur.wait_event(ready[0])
        b = buffers
        lhcal_global_scale(staging["w"], b.g)
        tiles = -(-rows // SWEEP_TILE_ROWS)
        k = max(1, min(row_chunks, tiles))
        rb = [min(rows, SWEEP_TILE_ROWS * (tiles * j // k)) for j in range(k + 1)]
        for j, (r0, r1) in enumerate(zip(rb[:-1], rb[1:])):
            wr = staging["w"][:, r0:r1]
            lhcal_scale_sweep(m, wr, b.h, b.g, b.codes[:, r0:r1], wq=None if b.wq is None else b.wq[:, r0:r1],
                              loss=None if b.loss is None else b.loss[:, r0:r1], p=b.p)
            if getattr(b, "wq16", None) is not None:
                lhcal_apply_scales(wr, b.g, b.codes[:, r0:r1], wq16=b.wq16[:, r0:r1])
            copy_out(0, 1, r0, r1, j == 0)
    cur.wait_stream(s_in)
    cur.wait_stream(s_out)
    return out


class CalibrationGraph:
    """The whole hot path on fixed device buffers, captured once as a CUDA graph.

    Construction runs the path once eagerly (so that any first-call set-up happens outside the
    capture), then captures accumulate, count, finalize, global scale and sweep on a side
    stream. ``replay()`` re-runs the captured launches on the current contents of the tensors
    given at construction: copy new activations / weights into them between replays. The
    results land in ``self.buffers``.
    """

    def __init__(self, mode, x, w, xq=None, group_offsets=None, token_ids=None, buffers: Buffers | None = None,
                 act_gx=None):
        import torch

        m = _mode_id(mode)
        groups, rows, cin = (int(v) for v in w.shape)
        dev = w.device
        tokens = 0 if x is None else int(x.shape[0])  # MSE reads no activations
        self.buffers = buffers or Buffers(m, tokens, cin, rows, groups, _dtype_id(w if x is None else x), dev)
        args = dict(xq=xq, group_offsets=group_offsets, token_ids=token_ids, buffers=self.buffers, act_gx=act_gx)
        calibrate(m, x, w, **args)
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.graph(self.graph, stream=side, capture_error_mode="thread_local"):
            calibrate(m, x, w, **args)
        torch.cuda.current_stream(dev).wait_stream(side)

    def replay(self):
        self.graph.replay()
        return self.buffers
