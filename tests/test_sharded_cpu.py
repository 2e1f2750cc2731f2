"""Token-sharded statistics and row-sharded sweep on two gloo ranks, without a GPU.

scale_calibration_lh_b200.sharded partitions one layer over the ranks: each accumulates its
tokens, one all-reduce (SUM) of the raw sums and counts, every rank finalizes, the global
scale is the all-reduce (MAX) of the ranks' row shards, each rank sweeps its rows, and the
results are all-gathered. Here the compute calls go to a CPU stand-in built from the oracle
(same call names and buffer semantics as the C-ABI binding), so that the test checks the
partition and the reductions: the gathered result must be the oracle's whole-layer calibration.
Dense, activation-aware with the fused quantizer (whose global scale is the MAX over ranks),
grouped (routing restricted to each rank's tokens) and plain MSE layers; ragged shard sizes.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

CASES = {
    "dense": dict(name="dense", mode="full", kw=dict(tokens=301, cin=48, rows=37)),
    "act": dict(name="act", mode="act", kw=dict(tokens=203, cin=32, rows=21)),
    "moe": dict(name="moe", mode="full", kw=dict(tokens=91, cin=32, rows=13, groups=6, top_k=2)),
    "mse": dict(name="dense", mode="mse", kw=dict(tokens=16, cin=32, rows=25)),
}


class OracleOps:
    """The binding's compute calls on CPU tensors, evaluated by the oracle (fp64, stored in the
    buffers' fp32). Only what calibrate_sharded calls."""

    def __init__(self):
        import scale_calibration_lh_b200 as L

        self.L = L
        for k in ("MODE_IDS", "F32", "BF16", "MSE", "ACT_AWARE", "DIAG", "ACCUM_OVERWRITE", "Buffers"):
            setattr(self, k, getattr(L, k))
        self.names = {v: k for k, v in L.MODE_IDS.items()}

    @staticmethod
    def _np(t):
        return None if t is None else t.detach().double().numpy()

    def lhcal_global_scale(self, w, g):
        from oracle import lhcal_oracle as O

        w64 = w.detach().float().numpy()
        g.copy_(torch.tensor([float(O.global_scale(w64[e])) for e in range(w64.shape[0])], dtype=torch.float32))

    def _accumulate(self, mode, x, xq, h, p, group_offsets, token_ids, act_gx):
        from oracle import lhcal_oracle as O

        offs = None if group_offsets is None else group_offsets.numpy()
        ids = None if token_ids is None else token_ids.numpy()
        hs, ps, _ = O.accumulate(mode, x.float().numpy(), None if xq is None else xq.float().numpy(), offs, ids,
                                 act_gx=act_gx)
        h.copy_(torch.from_numpy(hs).float().view_as(h))
        if p is not None:
            p.copy_(torch.from_numpy(ps).float().view_as(p))

    def lhcal_accumulate(self, m, x, h, xq=None, p=None, group_offsets=None, token_ids=None, flags=None,
                         workspace=None):
        assert flags == self.ACCUM_OVERWRITE
        self._accumulate(self.names[m], x, xq, h, p, group_offsets, token_ids, None)

    def lhcal_accumulate_act_quant(self, x, h, p, act_gx, group_offsets=None, token_ids=None, flags=None,
                                   workspace=None):
        assert flags == self.ACCUM_OVERWRITE
        self._accumulate("act", x, None, h, p, group_offsets, token_ids, np.float32(act_gx.item()))

    def lhcal_count_tokens(self, counts, tokens=0, group_offsets=None, flags=None):
        if group_offsets is None:
            counts.fill_(tokens)
        else:
            counts.copy_((group_offsets[1:] - group_offsets[:-1]).to(torch.int64))

    def lhcal_finalize(self, m, counts, h, p=None):
        from oracle import lhcal_oracle as O

        hf, pf = O.finalize(self.names[m], self._np(h), self._np(p), counts.numpy())
        h.copy_(torch.from_numpy(hf).float())
        if p is not None:
            p.copy_(torch.from_numpy(pf).float())

    def lhcal_scale_sweep(self, m, w, h, g, codes, wq=None, loss=None, p=None):
        from oracle import lhcal_oracle as O

        G, R, C = w.shape
        out = O.sweep(self.names[m], w.float().numpy(), self._np(h), self._np(p), g.numpy())
        codes.copy_(torch.from_numpy(out["codes"].reshape(G, R, C // 16)))
        if wq is not None:
            wq.copy_(torch.from_numpy(out["wq"].astype(np.float32).reshape(G, R, C)))
        if loss is not None:
            loss.copy_(torch.from_numpy(out["loss"].astype(np.float32).reshape(G, R, C // 16)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(case):
    from tests import parity as P

    c = CASES[case]
    return P.make_layer(c["name"], 17, **c["kw"])


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    from scale_calibration_lh_b200 import sharded as S

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        ops = OracleOps()
        for case, c in CASES.items():
            layer = _layer(case)
            bf16 = layer.dtype == "bf16"
            x = torch.from_numpy(layer.x_f32()).to(torch.bfloat16 if bf16 else torch.float32)
            w = torch.from_numpy(layer.w_f32()).to(torch.bfloat16 if bf16 else torch.float32)
            t0, t1 = S.token_range(layer.tokens, rank, world)
            r0, r1 = S.row_range(layer.rows, rank, world)
            offs = ids = None
            if layer.group_offsets is not None:
                offs, ids = S.shard_routing(torch.from_numpy(layer.group_offsets), torch.from_numpy(layer.token_ids),
                                            t0, t1)
            b, res = S.calibrate_sharded(c["mode"], x[t0:t1], w[:, r0:r1].contiguous(), group_offsets=offs,
                                         token_ids=ids, ops=ops)
            out[(rank, case)] = {
                "h": None if b.h is None else b.h.numpy().copy(), "p": None if b.p is None else b.p.numpy().copy(),
                "counts": b.counts.numpy().copy(), "g": b.g.numpy().copy(),
                "codes": res["codes"].numpy().copy(), "wq": res["wq"].numpy().copy(),
                "loss": res["loss"].numpy().copy(), "rows": (r0, r1), "tokens": (t0, t1)}
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def sharded_results():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    return dict(out)


def test_shards_partition_the_tokens_and_rows():
    from scale_calibration_lh_b200 import sharded as S

    for n, world in ((301, 2), (7, 3), (2, 4), (0, 2)):
        parts = [S.token_range(n, r, world) for r in range(world)]
        assert parts[0][0] == 0 and parts[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
        assert max(b - a for a, b in parts) - min(b - a for a, b in parts) <= 1
        assert S.row_range(n, 1, world) == S.token_range(n, 1, world)


def test_routing_restricted_to_a_token_shard():
    from scale_calibration_lh_b200 import sharded as S
    from scale_calibration_lh_b200 import synth

    offs, ids = synth.moe_routing(50, 7, 3, 5)
    t_offs, t_ids = torch.from_numpy(offs), torch.from_numpy(ids)
    pieces = [S.shard_routing(t_offs, t_ids, a, b) for a, b in ((0, 20), (20, 33), (33, 50))]
    for e in range(7):
        whole = sorted(ids[offs[e]:offs[e + 1]].tolist())
        got = []
        for (o, i), t0 in zip(pieces, (0, 20, 33)):
            got += (i[o[e]:o[e + 1]] + t0).tolist()
        assert got == whole  # every routed token once, ascending, in its own shard


@pytest.mark.parametrize("case", sorted(CASES))
def test_sharded_calibration_equals_the_whole_layer(sharded_results, case):
    from oracle import lhcal_oracle as O

    c = CASES[case]
    layer = _layer(case)
    r0 = sharded_results[(0, case)]
    r1 = sharded_results[(1, case)]
    # Every rank ends with the same global statistics and scales.
    mode = c["mode"]
    for k in ("h", "p", "g") + (() if mode == "mse" else ("counts",)):  # MSE takes no statistics
        if r0[k] is not None:
            np.testing.assert_array_equal(r0[k], r1[k])
    x, w = layer.x_f32(), layer.w_f32()
    g = np.array([O.global_scale(w[e]) for e in range(layer.groups)], np.float32)
    np.testing.assert_array_equal(r0["g"].view(np.int32), g.view(np.int32))  # MAX over ranks: exact
    h = p = None
    if mode != "mse":
        act_gx = O.global_scale(x) if mode == "act" else None  # MAX of the shards' scales: exact
        hs, ps, counts = O.accumulate(mode, x, None, layer.group_offsets, layer.token_ids, act_gx=act_gx)
        np.testing.assert_array_equal(r0["counts"], counts)
        hf, pf = O.finalize(mode, hs, ps, counts)
        from tests import parity as P

        P.check_hessians(r0["h"], hf, f"{case} sharded H", tol=1e-6)
        if pf is not None:
            P.check_hessians(r0["p"], pf, f"{case} sharded P", tol=1e-6)
        h = r0["h"].astype(np.float64)
        p = None if r0["p"] is None else r0["p"].astype(np.float64)
    # The gathered rows are the whole layer's sweep with the same statistics, in row order.
    ref = O.sweep(mode, w, h, p, g)
    G, R, C = layer.groups, layer.rows, layer.cin
    np.testing.assert_array_equal(r0["codes"].reshape(-1), ref["codes"])
    np.testing.assert_array_equal(r0["wq"].reshape(-1, 16).view(np.int32), ref["wq"].astype(np.float32).view(np.int32))
    np.testing.assert_array_equal(r0["loss"].reshape(-1), ref["loss"].astype(np.float32))
    assert r0["codes"].shape == (G, R, C // 16)
    assert r0["rows"] != r1["rows"] and r0["tokens"] != r1["tokens"]
