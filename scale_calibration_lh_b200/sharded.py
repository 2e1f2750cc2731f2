"""One layer calibrated by the ranks of a process group: token-sharded statistics, row-sharded sweep.

The accumulation is a sum over tokens and the sweep's units are independent, so the hot path
partitions ("add local hessian calibration", PR #788, Changes table: distributed sync
controls; "[2/3] Speed up layerwise GPTQ on MoE models", PR #2864: data-parallel ranks):

1. every rank accumulates the raw sums over its own token shard (OVERWRITE) and counts its
   tokens (per expert for a grouped layer, whose routing each rank holds for its own tokens);
2. one all-reduce (SUM) of the raw H (and P) sums and of the counts: the path's only exchange;
3. every rank finalizes the same global sums (so the zero-token fallback sees global counts);
4. every rank holds a shard of W's rows (the same rows of every group) and computes the global
   scale of its shard; an all-reduce (MAX) gives the layer's. This is exact: g = fp32(amax /
   2688) is a monotone function of amax, so the maximum of the ranks' g is the g of the
   maximum amax;
5. every rank sweeps its rows; with ``gather`` the codes and losses (and the fake-quantized
   weights, when kept) are all-gathered so that every rank holds the whole layer's results.

For the activation-aware layer with the input quantizer fused, the quantizer's global scale is
likewise the all-reduce (MAX) of the ranks' scales of their token shards, unless given.

The collectives are torch.distributed calls (NCCL between GPUs; any backend the tensors' device
supports). The compute goes through ``ops``, this package's C-ABI binding by default; the tests
pass a stand-in with the same call names to check the partition and the reductions on the CPU.
"""
from __future__ import annotations


def row_range(rows: int, rank: int, world: int) -> tuple[int, int]:
    """Rows [r0, r1) of the row shard of ``rank``: contiguous, sizes differing by at most one."""
    return rows * rank // world, rows * (rank + 1) // world


def token_range(tokens: int, rank: int, world: int) -> tuple[int, int]:
    """Tokens [t0, t1) of the token shard of ``rank`` (contiguous, sizes differing by at most one)."""
    return tokens * rank // world, tokens * (rank + 1) // world


def shard_routing(group_offsets, token_ids, t0: int, t1: int):
    """The CSR routing restricted to tokens [t0, t1), with ids relative to t0.

    group_offsets [G + 1] and token_ids (sorted by expert, ascending within) are host int tensors
    of the whole batch; returns the shard's (offsets, ids) as int32 host tensors."""
    import torch

    offs = group_offsets.to(torch.int64)
    ids = token_ids.to(torch.int64)
    keep = (ids >= t0) & (ids < t1)
    expert = torch.repeat_interleave(torch.arange(offs.numel() - 1), offs[1:] - offs[:-1])
    counts = torch.bincount(expert[keep], minlength=offs.numel() - 1)
    new_offs = torch.zeros(offs.numel(), dtype=torch.int64)
    new_offs[1:] = torch.cumsum(counts, 0)
    return new_offs.to(torch.int32), (ids[keep] - t0).to(torch.int32)


def calibrate_sharded(mode, x_shard, w_shard, group=None, xq_shard=None, group_offsets=None, token_ids=None,
                      act_gx=None, buffers=None, gather: bool = True, ops=None):
    """Calibrate one layer over the ranks of ``group`` (default: the default process group).

    x_shard   : [T_r, C] this rank's tokens (any split of the layer's tokens over the ranks).
    w_shard   : [G, R_r, C] this rank's rows of every group (see ``row_range``).
    xq_shard  : the two-tensor activation-aware input, X_q of this rank's tokens (or None).
    group_offsets, token_ids : grouped layers, the routing of this rank's tokens (``shard_routing``).
    act_gx    : activation-aware with the fused input quantizer: the quantizer's global scale,
                or None to take the all-reduce (MAX) of the ranks' scales of their shards.
    Returns (buffers, results): the rank's Buffers (global H/P/counts/g, its rows' codes, wq and
    loss) and, with ``gather``, a dict of the whole layer's codes and loss (and wq) in row order.
    """
    import torch
    import torch.distributed as dist

    if ops is None:
        import scale_calibration_lh_b200 as ops
    m = ops.MODE_IDS[mode] if isinstance(mode, str) else int(mode)
    G, Rr, C = (int(v) for v in w_shard.shape)
    T = int(x_shard.shape[0]) if x_shard is not None else 0
    dev = w_shard.device
    if buffers is None:
        xdt = ops.F32 if x_shard is None or x_shard.dtype == torch.float32 else ops.BF16
        buffers = ops.Buffers(m, T, C, Rr, G, xdt, dev)
    b = buffers
    if m != ops.MSE:
        fused = m == ops.ACT_AWARE and xq_shard is None
        if fused and act_gx is None:
            act_gx = torch.empty(1, dtype=torch.float32, device=dev)
            if T > 0:
                ops.lhcal_global_scale(x_shard.view(1, T, C), act_gx)
            else:
                act_gx.zero_()
            dist.all_reduce(act_gx, op=dist.ReduceOp.MAX, group=group)
        # 1. raw sums over this rank's tokens
        if fused:
            ops.lhcal_accumulate_act_quant(x_shard, b.h, b.p, act_gx, group_offsets=group_offsets,
                                           token_ids=token_ids, flags=ops.ACCUM_OVERWRITE, workspace=b.workspace)
        else:
            ops.lhcal_accumulate(m, x_shard, b.h, xq=xq_shard, p=b.p, group_offsets=group_offsets,
                                 token_ids=token_ids, flags=ops.ACCUM_OVERWRITE, workspace=b.workspace)
        ops.lhcal_count_tokens(b.counts, tokens=T, group_offsets=group_offsets, flags=ops.ACCUM_OVERWRITE)
        # 2. the exchange: global raw sums and token counts
        dist.all_reduce(b.h, op=dist.ReduceOp.SUM, group=group)
        if b.p is not None:
            dist.all_reduce(b.p, op=dist.ReduceOp.SUM, group=group)
        dist.all_reduce(b.counts, op=dist.ReduceOp.SUM, group=group)
        # 3. the same finalisation on every rank
        ops.lhcal_finalize(m, b.counts, b.h, p=b.p)
    # 4. global scale per group: the maximum of the ranks' scales of their rows
    ops.lhcal_global_scale(w_shard, b.g)
    dist.all_reduce(b.g, op=dist.ReduceOp.MAX, group=group)
    # 5. this rank's rows
    ops.lhcal_scale_sweep(m, w_shard, b.h, b.g, b.codes, wq=b.wq, loss=b.loss, p=b.p)
    if not gather:
        return b, None
    return b, gather_rows(b, G, C, group=group)


def gather_rows(buffers, groups: int, cin: int, group=None) -> dict:
    """All-gather the ranks' row shards of codes and loss (and wq) into whole-layer tensors
    [G, R, ...] in row order (shards of different sizes are padded for the exchange)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    b = buffers
    rr = torch.tensor([int(b.codes.shape[1])], dtype=torch.int64, device=b.codes.device)
    sizes = [torch.zeros_like(rr) for _ in range(world)]
    dist.all_gather(sizes, rr, group=group)
    sizes = [int(s.item()) for s in sizes]
    rmax = max(sizes)
    out = {}
    for name in ("codes", "loss", "wq"):
        t = getattr(b, name)
        if t is None:
            continue
        pad = torch.zeros((t.shape[0], rmax) + tuple(t.shape[2:]), dtype=t.dtype, device=t.device)
        pad[:, :t.shape[1]] = t
        parts = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(parts, pad, group=group)
        out[name] = torch.cat([p[:, :n] for p, n in zip(parts, sizes)], dim=1)
    return out
