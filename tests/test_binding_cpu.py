"""The binding's sequencing of the C calls, on the CPU, against a recording fake of the library.

The binding only reads shapes, strides and data pointers, so CPU tensors stand in for device
memory here. The fake records every call and answers OK; workspace queries return a fixed
size. The checks are:
- each mode's calls, in order: MSE takes no statistics, and ``act`` uses the fused entry point
  only when given the global scale and no X_q;
- the sizes, flags and pointers each call receives;
- the binding's own buffer checks accept everything ``calibrate`` allocates;
- ``calibrate_host`` stages the inputs, takes the statistics once and pipelines global scales,
  sweeps and result copies over chunks of groups, or, with one group, over chunks of rows that
  start on multiples of the sweep's 128-row tile (streams and events faked, copies at once).
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


class _FakeStream:
    def wait_stream(self, other):
        pass

    def wait_event(self, event):
        pass


class _FakeEvent:
    def record(self, stream=None):
        pass


@pytest.fixture
def fake_streams(monkeypatch):
    """Streams and events that only accept the ordering calls; copies run on the CPU at once."""
    import contextlib

    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Stream", lambda device=None: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: _FakeEvent())
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(L, "_side_streams", {})


def _host_outputs(b):
    out = object.__new__(L.HostOutputs)  # plain CPU tensors in place of pinned ones
    out.codes = torch.full(b.codes.shape, 255, dtype=torch.uint8)
    out.loss = torch.full(b.loss.shape, -1.0)
    out.g = torch.full(b.g.shape, -1.0)
    out.wq = None
    out.wq16 = None
    return out


def test_calibrate_host_pipelines_groups_in_chunks(fake, fake_streams):
    G, R, C, T = 10, 4, 32, 40
    x = torch.randn(T, C).bfloat16()
    w = torch.randn(G, R, C).bfloat16()
    offs = torch.tensor([0, 4, 8, 8, 12, 16, 20, 24, 28, 34, 40], dtype=torch.int32)
    ids = torch.from_numpy(np.arange(T, dtype=np.int32))
    b = L.Buffers("full", T, C, R, G, L.BF16, "cpu")
    b.codes.copy_(torch.arange(b.codes.numel(), dtype=torch.int64).remainder(127).to(torch.uint8).view(b.codes.shape))
    b.loss.copy_(torch.arange(b.loss.numel(), dtype=torch.float32).view(b.loss.shape))
    staging = {"x": torch.empty_like(x), "w": torch.empty_like(w), "offs": torch.empty_like(offs),
               "ids": torch.empty_like(ids)}
    fake.calls.clear()  # the workspace query of Buffers
    out = L.calibrate_host("full", x, w, b, staging, group_offsets=offs, token_ids=ids, out=_host_outputs(b),
                           group_chunks=4)
    # Statistics once over all tokens from the staged copies, then scale and sweep per chunk.
    assert fake.names()[:3] == ["lhcal_accumulate", "lhcal_count_tokens", "lhcal_finalize"]
    (acc,) = fake.args("lhcal_accumulate")
    assert _ptr(acc[2]) == staging["x"].data_ptr() and _ptr(acc[8]) == staging["offs"].data_ptr() and acc[7] == G
    assert torch.equal(staging["x"], x) and torch.equal(staging["w"], w) and torch.equal(staging["ids"], ids)
    bounds = [0, 2, 5, 7, 10]  # groups * j // chunks
    scales, sweeps = fake.args("lhcal_global_scale"), fake.args("lhcal_scale_sweep")
    assert [a[2] for a in scales] == [e1 - e0 for e0, e1 in zip(bounds, bounds[1:])]
    for (e0, _), sc, sw in zip(zip(bounds, bounds[1:]), scales, sweeps):
        assert _ptr(sc[1]) == staging["w"][e0].data_ptr() and _ptr(sc[5]) == b.g[e0].data_ptr()
        assert _ptr(sw[2]) == staging["w"][e0].data_ptr() and _ptr(sw[6]) == b.h[e0].data_ptr()
        assert _ptr(sw[9]) == b.codes[e0].data_ptr() and _ptr(sw[11]) == b.loss[e0].data_ptr()
    # Every group's results came back.
    assert torch.equal(out.codes, b.codes) and torch.equal(out.loss, b.loss) and torch.equal(out.g, b.g)


def test_calibrate_host_default_group_chunks(fake, fake_streams):
    G, R, C, T = 10, 4, 32, 40
    x, w = torch.randn(T, C).bfloat16(), torch.randn(G, R, C).bfloat16()
    offs = torch.tensor([0, 4, 8, 8, 12, 16, 20, 24, 28, 34, 40], dtype=torch.int32)
    ids = torch.from_numpy(np.arange(T, dtype=np.int32))
    b = L.Buffers("full", T, C, R, G, L.BF16, "cpu")
    staging = {"x": torch.empty_like(x), "w": torch.empty_like(w), "offs": torch.empty_like(offs),
               "ids": torch.empty_like(ids)}
    fake.calls.clear()
    L.calibrate_host("full", x, w, b, staging, group_offsets=offs, token_ids=ids, out=_host_outputs(b))
    # A few KB of weights: the minimum of 8 chunks, groups * j // 8.
    assert [a[2] for a in fake.args("lhcal_global_scale")] == [1, 1, 1, 2, 1, 1, 1, 2]  # bounds 0 1 2 3 5 6 7 8 10


@pytest.mark.parametrize("rows,row_chunks,expect", [(300, 8, [0, 128, 256, 300]), (1000, 3, [0, 256, 640, 1000]),
                                                    (100, 8, [0, 100]), (640, 1, [0, 640])])
def test_calibrate_host_one_group_sweeps_in_row_chunks_on_tile_boundaries(fake, fake_streams, rows, row_chunks,
                                                                           expect):
    T, C = 24, 32
    x, w = torch.randn(T, C).bfloat16(), torch.randn(1, rows, C).bfloat16()
    b = L.Buffers("full", T, C, rows, 1, L.BF16, "cpu", want_wq16=True)
    b.codes.copy_(torch.arange(b.codes.numel()).remainder(127).to(torch.uint8).view(b.codes.shape))
    b.loss.copy_(torch.arange(b.loss.numel(), dtype=torch.float32).view(b.loss.shape))
    b.wq16.copy_(torch.randn(b.wq16.shape).bfloat16())
    staging = {"x": torch.empty_like(x), "w": torch.empty_like(w)}
    out = _host_outputs(b)
    out.wq16 = torch.zeros(b.wq16.shape, dtype=torch.bfloat16)
    fake.calls.clear()
    L.calibrate_host("full", x, w, b, staging, out=out, row_chunks=row_chunks)
    # One global scale over the whole layer, before any sweep.
    names = fake.names()
    assert names.count("lhcal_global_scale") == 1 and names.index("lhcal_global_scale") < names.index(
        "lhcal_scale_sweep")
    (sc,) = fake.args("lhcal_global_scale")
    assert _ptr(sc[1]) == staging["w"].data_ptr() and sc[3] == rows
    sweeps, apply = fake.args("lhcal_scale_sweep"), fake.args("lhcal_apply_scales")
    assert [a[4] for a in sweeps] == [r1 - r0 for r0, r1 in zip(expect, expect[1:])]
    assert [a[3] for a in apply] == [a[4] for a in sweeps]
    for r0, sw, ap in zip(expect, sweeps, apply):
        assert r0 % 128 == 0  # every chunk starts on a sweep tile
        assert _ptr(sw[2]) == staging["w"][0, r0].data_ptr() and _ptr(sw[6]) == b.h.data_ptr()
        assert _ptr(sw[8]) == b.g.data_ptr() and _ptr(sw[9]) == b.codes[0, r0].data_ptr()
        assert _ptr(sw[11]) == b.loss[0, r0].data_ptr()
        assert _ptr(ap[1]) == staging["w"][0, r0].data_ptr() and _ptr(ap[8]) == b.wq16[0, r0].data_ptr()
    assert torch.equal(out.codes, b.codes) and torch.equal(out.loss, b.loss) and torch.equal(out.g, b.g)
    assert torch.equal(out.wq16, b.wq16)


def test_calibrate_host_reads_xq_only_when_the_caller_copies_it_in(fake, fake_streams):
    T, C, R = 48, 32, 8
    x, w, hxq = torch.randn(T, C).bfloat16(), torch.randn(1, R, C).bfloat16(), torch.randn(T, C).bfloat16()
    b = L.Buffers("act", T, C, R, 1, L.BF16, "cpu")
    staging = {"x": torch.empty_like(x), "w": torch.empty_like(w), "xq": torch.empty_like(hxq)}
    gx = torch.ones(1)
    L.calibrate_host("act", x, w, b, staging, out=_host_outputs(b), act_gx=gx)
    assert "lhcal_accumulate_act_quant" in fake.names() and "lhcal_accumulate" not in fake.names()
    fake.calls.clear()
    L.calibrate_host("act", x, w, b, staging, hxq=hxq, out=_host_outputs(b))
    (acc,) = fake.args("lhcal_accumulate")
    assert _ptr(acc[3]) == staging["xq"].data_ptr() and torch.equal(staging["xq"], hxq)
