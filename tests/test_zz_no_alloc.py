"""lhcal_accumulate_noalloc: the accumulation entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc (a plugin handed only input and output pointers by a
host framework, or a runtime whose memory planner owns all device memory), so they cannot
pass the workspace that lhcal_accumulate takes. This variant keeps its scratch in a fixed
array inside the library. Its results must match lhcal_accumulate's, call after call,
although every call reuses the same scratch.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import scale_calibration_lh_b200 as L  # noqa: E402
from tests import parity as P  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from scale_calibration_lh_b200 import build

    build.build()
    L.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _with_workspace(mode, d, nblk, tokens, cin):
    shape = (1, nblk, 16) if mode == "diag" else (1, nblk, 16, 16)
    h = torch.empty(shape, dtype=torch.float32, device="cuda")
    p = torch.empty_like(h) if mode == "act" else None
    ws_bytes = L.lhcal_accumulate_workspace(mode, L.BF16, tokens, cin, 1)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device="cuda")
    L.lhcal_accumulate(mode, d["x"], h, xq=d["xq"], p=p, flags=L.ACCUM_OVERWRITE, workspace=ws)
    return h, p


def _without_workspace(mode, d, nblk):
    shape = (1, nblk, 16) if mode == "diag" else (1, nblk, 16, 16)
    h = torch.full(shape, 5.0, dtype=torch.float32, device="cuda")
    p = torch.full(shape, 5.0, dtype=torch.float32, device="cuda") if mode == "act" else None
    L.lhcal_accumulate_noalloc(mode, d["x"], h, xq=d["xq"], p=p, flags=L.ACCUM_OVERWRITE)
    return h, p


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # Call 1 (large: many token splits) then call 2 (smaller, different mode and fewer splits):
    # the second must not see the first call's leftovers in the shared scratch.
    cases = [("dense", "full", dict(tokens=16384, cin=2048, rows=4)),
             ("act", "act", dict(tokens=3000, cin=1024, rows=4)),
             ("wmse", "diag", dict(tokens=5000, cin=4096, rows=4))]
    for name, mode, kw in cases:
        layer = P.make_layer(name, 21, **kw)
        d = P.layer_to_device(layer)
        nblk = layer.cin // 16
        assert L.lhcal_accumulate_workspace(mode, L.BF16, layer.tokens, layer.cin, 1) > 0
        h_ref, p_ref = _with_workspace(mode, d, nblk, layer.tokens, layer.cin)
        h_na, p_na = _without_workspace(mode, d, nblk)
        torch.cuda.synchronize()
        P.check_hessians(h_na.cpu().numpy(), h_ref.cpu().numpy().astype(np.float64), f"noalloc {mode} H")
        if mode == "act":
            P.check_hessians(p_na.cpu().numpy(), p_ref.cpu().numpy().astype(np.float64), "noalloc P")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = L.load_library()
    # WMSE over X [65536, 12288]: 196 token splits x 12288 partial sums = 9.6 MB of scratch.
    tokens, cin = 65536, 12288
    need = L.lhcal_accumulate_workspace("diag", L.BF16, tokens, cin, 1)
    assert need > L.NOALLOC_SCRATCH_BYTES
    st = lib.lhcal_accumulate_noalloc(L.DIAG, L.BF16, None, None, tokens, cin, cin, 1, None, None,
                                      L.ACCUM_OVERWRITE, None, None, ctypes.c_void_p(0))
    assert st == L.ERR_INVALID_ARG
    assert b"scratch" in lib.lhcal_last_error_string()
