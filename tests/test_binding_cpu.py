"""The binding's sequencing of the C calls, on the CPU, against a recording fake of the library.

The binding only reads shapes, strides and data pointers, so CPU tensors stand in for device
memory here. The fake records every call and answers OK; workspace queries return a fixed
size. The checks are:
- each mode's calls, in order: MSE takes no statistics, and ``act`` uses the fused entry point
  only when given the global scale and no X_q;
- the sizes, flags and pointers each call receives;
- the binding's own buffer checks accept everything ``calibrate`` allocates.
"""
import ctypes

import numpy as np
import pytest
import torch

import scale_calibration_lh_b200 as L

WS_BYTES = 4096


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, args))
            if name.endswith("_workspace"):
                args[-1]._obj.value = WS_BYTES
            return L.OK
        return call

    def names(self):
        return [n for n, _ in self.calls]

    def args(self, name):
        return [a for n, a in self.calls if n == name]


@pytest.fixture
def fake(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(L, "_lib", rec)
    monkeypatch.setattr(L, "_stream", lambda stream: ctypes.c_void_p(0))
    return rec


def _ptr(arg):
    return None if arg is None else arg.value


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_full_layer_calls_in_order_with_the_buffers_it_allocated(fake):
    x, w = _bf16(300, 64), _bf16(1, 40, 64)
    b = L.calibrate("full", x, w)
    assert fake.names() == ["lhcal_accumulate_workspace", "lhcal_accumulate", "lhcal_count_tokens", "lhcal_finalize",
                            "lhcal_global_scale", "lhcal_scale_sweep"]
    (acc,) = fake.args("lhcal_accumulate")
    mode, dtype, xp, xqp, tokens, cin, ldx, groups, offs, ids, flags, h, p, ws, ws_bytes, _ = acc
    assert (mode, dtype, tokens, cin, ldx, groups, flags) == (L.FULL, L.BF16, 300, 64, 64, 1, L.ACCUM_OVERWRITE)
    assert _ptr(xp) == x.data_ptr() and xqp is None and offs is None and ids is None and p is None
    assert _ptr(h) == b.h.data_ptr() and _ptr(ws) == b.workspace.data_ptr() and ws_bytes >= WS_BYTES
    (cnt,) = fake.args("lhcal_count_tokens")
    assert cnt[0] == 1 and cnt[1] == 300 and cnt[2] is None and _ptr(cnt[4]) == b.counts.data_ptr()
    (sw,) = fake.args("lhcal_scale_sweep")
    assert sw[:2] == (L.FULL, L.BF16) and sw[3:6] == (1, 40, 64)
    assert [_ptr(a) for a in sw[6:12]] == [b.h.data_ptr(), None, b.g.data_ptr(), b.codes.data_ptr(),
                                          b.wq.data_ptr(), b.loss.data_ptr()]
    assert tuple(b.h.shape) == (1, 4, 16, 16) and tuple(b.codes.shape) == (1, 40, 4)


def test_activation_aware_uses_the_fused_entry_point_only_without_xq(fake):
    x, w = _bf16(100, 32), _bf16(1, 8, 32)
    gx = torch.ones(1)
    b = L.calibrate("act", x, w, act_gx=gx)
    assert "lhcal_accumulate_act_quant" in fake.names() and "lhcal_accumulate" not in fake.names()
    (fused,) = fake.args("lhcal_accumulate_act_quant")
    assert _ptr(fused[8]) == gx.data_ptr() and _ptr(fused[10]) == b.h.data_ptr() and _ptr(fused[11]) == b.p.data_ptr()
    (fin,) = fake.args("lhcal_finalize")
    assert fin[0] == L.ACT_AWARE and _ptr(fin[5]) == b.p.data_ptr()
    (sw,) = fake.args("lhcal_scale_sweep")
    assert _ptr(sw[7]) == b.p.data_ptr()
    fake.calls.clear()
    xq = _bf16(100, 32)
    L.calibrate("act", x, w, xq=xq, act_gx=gx)  # X_q given: the two-tensor kernel reads it
    assert "lhcal_accumulate_act_quant" not in fake.names()
    (acc,) = fake.args("lhcal_accumulate")
    assert acc[0] == L.ACT_AWARE and _ptr(acc[3]) == xq.data_ptr()


def test_mse_takes_no_statistics(fake):
    w = _bf16(2, 8, 48)
    b = L.calibrate("mse", None, w)
    assert fake.names() == ["lhcal_global_scale", "lhcal_scale_sweep"]
    assert b.h is None and b.p is None and b.workspace is None
    (sw,) = fake.args("lhcal_scale_sweep")
    assert sw[0] == L.MSE and sw[6] is None and sw[7] is None and sw[3:6] == (2, 8, 48)


def test_grouped_layer_passes_its_routing_and_group_count(fake):
    x, w = _bf16(50, 32), _bf16(5, 8, 32)
    offs = torch.tensor([0, 3, 3, 10, 12, 20], dtype=torch.int32)
    ids = torch.from_numpy(np.arange(20, dtype=np.int32))
    b = L.calibrate("full", x, w, group_offsets=offs, token_ids=ids)
    (acc,) = fake.args("lhcal_accumulate")
    assert acc[7] == 5 and _ptr(acc[8]) == offs.data_ptr() and _ptr(acc[9]) == ids.data_ptr()
    (cnt,) = fake.args("lhcal_count_tokens")
    assert cnt[0] == 5 and _ptr(cnt[2]) == offs.data_ptr()
    (gs,) = fake.args("lhcal_global_scale")
    assert gs[2] == 5 and tuple(b.g.shape) == (5,) and tuple(b.h.shape) == (5, 2, 16, 16)


def test_diag_statistics_are_one_vector_per_block(fake):
    x, w = _bf16(64, 48), _bf16(1, 4, 48)
    b = L.calibrate("diag", x, w)
    assert tuple(b.h.shape) == (1, 3, 16) and b.p is None
    (sw,) = fake.args("lhcal_scale_sweep")
    assert sw[0] == L.DIAG and _ptr(sw[6]) == b.h.data_ptr()
