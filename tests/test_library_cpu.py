"""liblhcal.so builds, loads and exports the C ABI; host-side validation needs no GPU."""
import ctypes
import os
import re

import pytest

import scale_calibration_lh_b200 as L
from scale_calibration_lh_b200 import build as B


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load_library()


def declared_functions(root):
    text = open(os.path.join(root, "include", "lhcal.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lhcal_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib, root_dir):
    names = declared_functions(root_dir)
    assert "lhcal_scale_sweep" in names and "lhcal_accumulate" in names
    for n in names:
        assert hasattr(lib, n), n
    assert L.lhcal_version() == 100


def test_status_values_match_header(root_dir):
    text = open(os.path.join(root_dir, "include", "lhcal.h")).read()
    for name, val in [("LHCAL_OK", L.OK), ("LHCAL_ERR_INVALID_ARG", L.ERR_INVALID_ARG),
                      ("LHCAL_ERR_UNSUPPORTED", L.ERR_UNSUPPORTED), ("LHCAL_ERR_DEVICE_MISMATCH", L.ERR_DEVICE_MISMATCH),
                      ("LHCAL_ERR_CUDA", L.ERR_CUDA), ("LHCAL_ERR_TIMEOUT", L.ERR_TIMEOUT),
                      ("LHCAL_F32", L.F32), ("LHCAL_BF16", L.BF16), ("LHCAL_FULL", L.FULL),
                      ("LHCAL_ACT_AWARE", L.ACT_AWARE), ("LHCAL_DIAG", L.DIAG),
                      ("LHCAL_ACCUM_ADD", L.ACCUM_ADD), ("LHCAL_ACCUM_OVERWRITE", L.ACCUM_OVERWRITE),
                      ("LHCAL_N_CANDIDATES", L.N_CANDIDATES)]:
        m = re.search(rf"\b{name}\s*=?\s*(\d+)", text)
        assert m and int(m.group(1)) == val, name


def test_noalloc_scratch_size_in_python_matches_the_header(root_dir):
    """The binding's copy of LHCAL_NOALLOC_SCRATCH_BYTES (used to size-check before the call)
    is the header's value."""
    text = open(os.path.join(root_dir, "include", "lhcal.h")).read()
    m = re.search(r"#define\s+LHCAL_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", text)
    assert m, "LHCAL_NOALLOC_SCRATCH_BYTES not found in lhcal.h"
    assert eval(m.group(1).replace("u", ""), {}) == L.NOALLOC_SCRATCH_BYTES


def test_workspace_query_is_host_only(lib):
    dense = L.lhcal_accumulate_workspace("full", L.BF16, 16384, 2048, 1)
    assert dense > 0 and dense % (128 * 4 * 256) == 0  # whole [splits, N, 16, 16] partials
    act = L.lhcal_accumulate_workspace("act", L.BF16, 16384, 2048, 1)
    assert act > 0 and act % (2 * 128 * 4 * 256) == 0  # H and P partials per split
    # Wide layers reduce their token splits inside CTA clusters and need no workspace.
    assert L.lhcal_accumulate_workspace("full", L.BF16, 16384, 4096, 1) == 0
    diag = L.lhcal_accumulate_workspace("diag", L.BF16, 65536, 12288, 1)
    assert diag % (12288 * 4) == 0
    assert L.lhcal_accumulate_workspace("full", L.BF16, 16384, 2560, 512) == 0
    assert L.lhcal_accumulate_workspace("full", L.BF16, 0, 64, 1) == 0
    with pytest.raises(L.LhcalError) as e:
        L.lhcal_accumulate_workspace("full", L.BF16, 100, 24, 1)
    assert e.value.status == L.ERR_INVALID_ARG and "multiple of 16" in str(e.value)
    with pytest.raises(L.LhcalError) as e:
        L.lhcal_accumulate_workspace(7, L.BF16, 100, 32, 1)
    assert e.value.status == L.ERR_UNSUPPORTED


def _call_accumulate(lib, **kw):
    args = dict(mode=L.FULL, dtype=L.BF16, x=None, xq=None, tokens=10, cin=32, ldx=32, groups=1, offs=None,
                ids=None, flags=0, h=None, p=None, ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    return lib.lhcal_accumulate(args["mode"], args["dtype"], args["x"], args["xq"], args["tokens"], args["cin"],
                                args["ldx"], args["groups"], args["offs"], args["ids"], args["flags"], args["h"],
                                args["p"], args["ws"], args["ws_bytes"], args["stream"])


def test_argument_validation_without_gpu(lib):
    assert _call_accumulate(lib, cin=33) == L.ERR_INVALID_ARG
    assert _call_accumulate(lib, ldx=16) == L.ERR_INVALID_ARG
    assert _call_accumulate(lib, ldx=36) == L.ERR_INVALID_ARG  # 72 bytes: not a multiple of 16
    assert _call_accumulate(lib, flags=5) == L.ERR_INVALID_ARG
    assert _call_accumulate(lib, groups=3) == L.ERR_INVALID_ARG
    assert _call_accumulate(lib, mode=L.ACT_AWARE) == L.ERR_INVALID_ARG  # no xq
    assert _call_accumulate(lib, tokens=-1) == L.ERR_INVALID_ARG
    assert _call_accumulate(lib, dtype=9) == L.ERR_UNSUPPORTED
    assert _call_accumulate(lib, tokens=100000, cin=2048, ldx=2048) == L.ERR_INVALID_ARG  # workspace too small
    assert b"workspace" in lib.lhcal_last_error_string()
    # Sweep / finalize / global scale reject bad sizes before touching memory.
    assert lib.lhcal_scale_sweep(0, 1, None, 1, 0, 32, None, None, None, None, None, None, None) == L.ERR_INVALID_ARG
    assert lib.lhcal_scale_sweep(0, 1, None, 0, 4, 32, None, None, None, None, None, None, None) == L.ERR_INVALID_ARG
    assert lib.lhcal_scale_sweep(1, 1, None, 1, 4, 32, None, None, None, None, None, None, None) == L.ERR_INVALID_ARG
    assert lib.lhcal_finalize(0, 1, 20, None, None, None, None) == L.ERR_INVALID_ARG
    assert lib.lhcal_global_scale(3, None, 1, 4, 32, None, None) == L.ERR_UNSUPPORTED
    assert lib.lhcal_count_tokens(2, 5, None, 0, None, None) == L.ERR_INVALID_ARG
    # A pointer that is not device memory is refused (no GPU here: the query itself fails).
    buf = ctypes.create_string_buffer(4096)
    addr = (ctypes.addressof(buf) + 255) // 256 * 256
    st = lib.lhcal_global_scale(1, ctypes.c_void_p(addr), 1, 4, 32, ctypes.c_void_p(addr), None)
    assert st in (L.ERR_INVALID_ARG, L.ERR_DEVICE_MISMATCH)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(RuntimeError, match="not found"):
        L.load_library(str(tmp_path / "nope.so"))


def test_input_quantizer_entry_points_validate_without_gpu(lib):
    q = lib.lhcal_act_fake_quant
    assert q(L.F32, None, 4, 32, 32, None, None, 32, None) == L.ERR_UNSUPPORTED
    assert q(L.BF16, None, 4, 33, 33, None, None, 33, None) == L.ERR_INVALID_ARG  # cin not a multiple of 16
    assert q(L.BF16, None, 4, 32, 36, None, None, 32, None) == L.ERR_INVALID_ARG  # 72-byte row stride
    assert q(L.BF16, None, 4, 32, 32, None, None, 16, None) == L.ERR_INVALID_ARG  # ldxq < cin
    assert q(L.BF16, None, -1, 32, 32, None, None, 32, None) == L.ERR_INVALID_ARG
    assert q(L.BF16, None, 4, 32, 32, None, None, 32, None) == L.ERR_INVALID_ARG  # act_gx NULL
    a = lib.lhcal_accumulate_act_quant
    assert a(L.F32, None, 4, 32, 32, 1, None, None, None, 0, None, None, None, 0, None) == L.ERR_UNSUPPORTED
    assert a(L.BF16, None, 4, 32, 32, 1, None, None, None, 0, None, None, None, 0, None) == L.ERR_INVALID_ARG
    assert b"act_gx" in lib.lhcal_last_error_string()


def test_mse_scale_and_output_entry_points_validate_without_gpu(lib):
    # MSE takes no statistics.
    assert lib.lhcal_scale_sweep(3, 1, None, 1, 4, 32, ctypes.c_void_p(256), None, None, None, None, None,
                                 None) == L.ERR_INVALID_ARG
    assert b"MSE" in lib.lhcal_last_error_string()
    # MSE is a sweep mode only.
    assert lib.lhcal_finalize(3, 1, 32, None, None, None, None) == L.ERR_UNSUPPORTED
    gs = lib.lhcal_global_scale_ex
    for bad in (0.0, -1.0, 449.0, 1.0 / 3.0, float("nan")):
        assert gs(1, None, 1, 4, 32, bad, None, None) == L.ERR_INVALID_ARG, bad
    assert b"fp8_max" in lib.lhcal_last_error_string()
    assert gs(7, None, 1, 4, 32, 256.0, None, None) == L.ERR_UNSUPPORTED
    ap = lib.lhcal_apply_scales
    assert ap(1, None, 1, 4, 33, None, None, None, None, None, None) == L.ERR_INVALID_ARG
    assert ap(1, None, 1, 0, 32, None, None, None, None, None, None) == L.ERR_INVALID_ARG
    assert ap(5, None, 1, 4, 32, None, None, None, None, None, None) == L.ERR_UNSUPPORTED


def test_multiplier_search_validates_without_gpu(lib):
    f = lib.lhcal_multiplier_search
    assert f(9, 1, None, 1, 4, 32, None, None, None, None, 8, None, None, None, None) == L.ERR_UNSUPPORTED
    assert f(0, 1, None, 1, 4, 33, None, None, None, None, 8, None, None, None, None) == L.ERR_INVALID_ARG
    assert f(0, 1, None, 1, 4, 32, None, None, None, None, 0, None, None, None, None) == L.ERR_INVALID_ARG
    assert f(0, 1, None, 1, 4, 32, None, None, None, None, 2000, None, None, None, None) == L.ERR_INVALID_ARG
    assert b"n_multipliers" in lib.lhcal_last_error_string()
    assert f(1, 1, None, 1, 4, 32, None, None, None, None, 8, None, None, None, None) == L.ERR_INVALID_ARG  # no p


def test_buffers_size_the_workspace_for_either_activation_aware_entry_point(lib):
    """Buffers (host-only sizing, CPU tensors here) cover both the two-tensor and the fused
    activation-aware accumulations, and the statistics-free MSE mode allocates no H."""
    for tokens, cin in ((32768, 4096), (3000, 1024), (700, 96)):
        b = L.Buffers("act", tokens, cin, 8, 1, L.BF16, "cpu")
        need = max(L.lhcal_accumulate_workspace("act", L.BF16, tokens, cin, 1),
                   L.lhcal_accumulate_act_quant_workspace(L.BF16, tokens, cin, 1))
        have = 0 if b.workspace is None else b.workspace.numel() * b.workspace.element_size()
        assert have >= need and b.p is not None
    m = L.Buffers("mse", 0, 64, 8, 2, L.BF16, "cpu")
    assert m.h is None and m.p is None and m.workspace is None
    assert tuple(m.codes.shape) == (2, 8, 4) and tuple(m.wq.shape) == (2, 8, 64)


def test_binding_rejects_buffers_the_library_would_misread(lib):
    """The C entry points take bare pointers, so the binding checks each tensor's dtype, density
    and size against the call. A consistent call (CPU tensors here) reaches the library, which
    refuses host pointers with an LhcalError; an inconsistent one stops in the binding first."""
    import types

    import torch

    s = types.SimpleNamespace(cuda_stream=0)
    x = torch.zeros((8, 32), dtype=torch.bfloat16)
    h = torch.zeros((1, 2, 16, 16))
    p = torch.zeros_like(h)
    xq = torch.zeros_like(x)
    with pytest.raises(L.LhcalError):
        L.lhcal_accumulate("act", x, h, xq=xq, p=p, stream=s)
    wide = torch.zeros((8, 48), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="row stride"):  # one ldx serves x and xq
        L.lhcal_accumulate("act", x, h, xq=wide[:, :32], p=p, stream=s)
    with pytest.raises(ValueError, match="must match"):
        L.lhcal_accumulate("act", x, h, xq=xq.float(), p=p, stream=s)
    with pytest.raises(ValueError, match="needs 512"):
        L.lhcal_accumulate("full", x, h[:, :1], stream=s)
    with pytest.raises(ValueError, match="needs 512"):
        L.lhcal_accumulate_noalloc("act", x, h, xq=xq, p=p[:, :1], stream=s)
    with pytest.raises(TypeError, match="float32"):
        L.lhcal_accumulate("full", x, h.double(), stream=s)
    with pytest.raises(L.LhcalError):  # DIAG statistics are [groups, cin/16, 16]
        L.lhcal_accumulate("diag", x, torch.zeros((1, 2, 16)), stream=s)
    offs = torch.tensor([0, 4, 8], dtype=torch.int32)
    with pytest.raises(ValueError, match="needs 1024"):  # two groups
        L.lhcal_accumulate("full", x, h, group_offsets=offs, token_ids=torch.zeros(8, dtype=torch.int32), stream=s)
    with pytest.raises(TypeError, match="int32"):
        L.lhcal_accumulate("full", x, torch.zeros((2, 2, 16, 16)), group_offsets=offs.long(),
                           token_ids=torch.zeros(8, dtype=torch.int32), stream=s)
    gx = torch.ones(1)
    with pytest.raises(L.LhcalError):
        L.lhcal_accumulate_act_quant(x, h, p, gx, stream=s)
    with pytest.raises(TypeError, match="act_gx"):
        L.lhcal_accumulate_act_quant(x, h, p, gx.double(), stream=s)
    # The quantizer's output carries its own row stride, so a strided xq is fine there.
    with pytest.raises(L.LhcalError):
        L.lhcal_act_fake_quant(x, gx, wide[:, :32], stream=s)
    with pytest.raises(ValueError, match="shaped like x"):
        L.lhcal_act_fake_quant(x, gx, wide, stream=s)
    with pytest.raises(TypeError, match="bfloat16"):
        L.lhcal_act_fake_quant(x, gx, xq.float(), stream=s)
    counts = torch.zeros(1, dtype=torch.int64)
    with pytest.raises(TypeError, match="int64"):
        L.lhcal_count_tokens(counts.int(), tokens=8, stream=s)
    with pytest.raises(TypeError, match="int64"):
        L.lhcal_finalize("full", counts.int(), h, stream=s)
    with pytest.raises(ValueError, match="p has"):
        L.lhcal_finalize("act", counts, h, p=p[:, :1], stream=s)

    w = torch.zeros((2, 4, 32), dtype=torch.bfloat16)
    hw = torch.zeros((2, 2, 16, 16))
    g = torch.zeros(2)
    codes = torch.zeros((2, 4, 2), dtype=torch.uint8)
    wq = torch.zeros((2, 4, 32))
    loss = torch.zeros((2, 4, 2))
    with pytest.raises(L.LhcalError):
        L.lhcal_scale_sweep("full", w, hw, g, codes, wq=wq, loss=loss, stream=s)
    with pytest.raises(ValueError, match="w must be contiguous"):
        L.lhcal_scale_sweep("full", w.transpose(1, 2).contiguous().transpose(1, 2), hw, g, codes, stream=s)
    with pytest.raises(TypeError, match="uint8"):
        L.lhcal_scale_sweep("full", w, hw, g, codes.to(torch.int8), stream=s)
    with pytest.raises(ValueError, match="wq has"):
        L.lhcal_scale_sweep("full", w, hw, g, codes, wq=wq[:1], stream=s)
    with pytest.raises(ValueError, match="h has"):
        L.lhcal_scale_sweep("act", w, hw[:1], g, codes, p=hw, stream=s)
    with pytest.raises(ValueError, match="g has"):
        L.lhcal_global_scale(w, g[:1], stream=s)
    with pytest.raises(L.LhcalError):  # MSE reads no statistics
        L.lhcal_scale_sweep("mse", w, None, g, codes, stream=s)
    with pytest.raises(TypeError, match="multipliers"):
        L.lhcal_multiplier_search("full", w, hw, g, torch.ones(4, dtype=torch.float64), codes, stream=s)
    with pytest.raises(TypeError, match="wq16"):
        L.lhcal_apply_scales(w, g, codes, wq16=wq, stream=s)
    with pytest.raises(ValueError, match="amax has"):
        L.lhcal_apply_scales(w, g, codes, amax=loss[:1], stream=s)
    with pytest.raises(L.LhcalError):
        L.lhcal_apply_scales(w, g, codes, wq=wq, wq16=wq.bfloat16(), amax=loss, stream=s)


def test_zero_token_calls_validate_as_the_header_states(lib):
    """tokens = 0: one group accepts a NULL x (the next check to fail here is h, a host pointer
    without a GPU); a grouped call still needs x; the two-tensor ACT_AWARE call still needs xq."""
    host = ctypes.create_string_buffer(4096)
    addr = ctypes.c_void_p((ctypes.addressof(host) + 255) // 256 * 256)
    st = _call_accumulate(lib, tokens=0, x=None, h=addr, flags=1)
    assert st in (L.ERR_INVALID_ARG, L.ERR_DEVICE_MISMATCH)
    assert lib.lhcal_last_error_string().startswith(b"h")
    st = _call_accumulate(lib, tokens=0, x=None, groups=2, offs=addr, ids=addr, h=addr, flags=1)
    assert st == L.ERR_INVALID_ARG and lib.lhcal_last_error_string() == b"x is NULL"
    st = _call_accumulate(lib, mode=L.ACT_AWARE, tokens=0, x=None, xq=None, h=addr, p=addr, flags=1)
    assert st == L.ERR_INVALID_ARG and b"needs xq" in lib.lhcal_last_error_string()


def test_token_count_and_fused_workspace_errors_as_documented(lib):
    ct = lib.lhcal_count_tokens
    for groups, tokens, flags in ((0, 5, 0), (65536, 5, 0), (2, 5, 0), (1, -1, 0), (1, 5, 7)):
        assert ct(groups, tokens, None, flags, None, None) == L.ERR_INVALID_ARG, (groups, tokens, flags)
    n = ctypes.c_size_t(0)
    q = lib.lhcal_accumulate_act_quant_workspace
    assert q(L.F32, 100, 32, 1, ctypes.byref(n)) == L.ERR_UNSUPPORTED
    assert q(L.BF16, 100, 24, 1, ctypes.byref(n)) == L.ERR_INVALID_ARG
    assert q(L.BF16, 100, 32, 0, ctypes.byref(n)) == L.ERR_INVALID_ARG
    assert q(L.BF16, -1, 32, 1, ctypes.byref(n)) == L.ERR_INVALID_ARG
    assert q(L.BF16, 100, 32, 1, None) == L.ERR_INVALID_ARG
    assert q(L.BF16, 0, 32, 1, ctypes.byref(n)) == L.OK
