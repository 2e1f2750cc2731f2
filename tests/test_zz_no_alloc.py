"""lhcal_accumulate_noalloc: the accumulation entry point for callers that cannot allocate.

Some callers cannot call cudaMalloc (a plugin handed only input and output pointers by a
host framework, or a runtime whose memory planner owns all device memory), so they cannot
pass the workspace that lhcal_accumulate takes. This variant keeps its scratch in a fixed
array inside the library. It runs the same kernels with the same split plan and summation
order as lhcal_accumulate, so its results must equal that entry point's bit for bit, call
after call, although every call reuses the same scratch.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import scale_calibration_lh_b200 as L  # noqa: E402
from oracle import lhcal_oracle as O  # noqa: E402
from scale_calibration_lh_b200 import synth  # noqa: E402
from tests import parity as P  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from scale_calibration_lh_b200 import build

    build.build()
    L.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _stats(mode, nblk, fill):
    shape = (1, nblk, 16) if mode == "diag" else (1, nblk, 16, 16)
    h = torch.full(shape, fill, dtype=torch.float32, device="cuda")
    p = torch.full(shape, fill, dtype=torch.float32, device="cuda") if mode == "act" else None
    return h, p


def _with_workspace(mode, d, nblk, tokens, cin):
    h, p = _stats(mode, nblk, 0.0)
    ws_bytes = L.lhcal_accumulate_workspace(mode, L.BF16, tokens, cin, 1)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device="cuda")
    L.lhcal_accumulate(mode, d["x"], h, xq=d["xq"], p=p, flags=L.ACCUM_OVERWRITE, workspace=ws)
    return h, p


def _without_workspace(mode, d, nblk):
    h, p = _stats(mode, nblk, 5.0)  # OVERWRITE must replace these
    L.lhcal_accumulate_noalloc(mode, d["x"], h, xq=d["xq"], p=p, flags=L.ACCUM_OVERWRITE)
    return h, p


@pytest.mark.parametrize("name,mode,kw", [
    ("dense", "full", dict(tokens=16384, cin=2048, rows=4)),  # many token splits
    ("act", "act", dict(tokens=3000, cin=1024, rows=4)),
    ("wmse", "diag", dict(tokens=5000, cin=4096, rows=4)),
])
def test_noalloc_equals_workspace_entry_point_bit_for_bit(name, mode, kw):
    """Two checked calls in a row, each preceded by a call on other activations of the same
    shape: the scratch then holds another batch's partials, and a partial that a checked call
    failed to overwrite would change its sums."""
    layer = P.make_layer(name, 21, **kw)
    other = P.make_layer(name, 22, **kw)
    d, d_other = synth.layer_to_device(layer), synth.layer_to_device(other)
    nblk = layer.cin // 16
    assert L.lhcal_accumulate_workspace(mode, L.BF16, layer.tokens, layer.cin, 1) > 0
    h_ref, p_ref = _with_workspace(mode, d, nblk, layer.tokens, layer.cin)
    for _ in range(2):
        h_other, _ = _without_workspace(mode, d_other, nblk)
        h_na, p_na = _without_workspace(mode, d, nblk)
        torch.cuda.synchronize()
        assert not torch.equal(h_other, h_ref), "the poisoning batch must differ"
        assert torch.equal(h_na, h_ref), f"noalloc {mode} H differs from lhcal_accumulate"
        if mode == "act":
            assert torch.equal(p_na, p_ref), "noalloc P differs from lhcal_accumulate"
    # And within the parity bar against the oracle, so that the equality is not of two wrong results.
    hs, ps, _ = O.accumulate(mode, layer.x_f32(), layer.xq_f32() if mode == "act" else None)
    P.check_hessians(h_na.cpu().numpy(), hs, f"noalloc {mode} H vs oracle")
    if mode == "act":
        P.check_hessians(p_na.cpu().numpy(), ps, "noalloc P vs oracle")


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
