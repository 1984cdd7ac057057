"""Data parallelism across GPUs: one process per GPU, utterances sharded.

Utterances of a transducer batch are independent, so the batch is split
across ranks with every rank running the whole fused joint + loss call on its
shard; frame / label gradients (df, dg) stay with the rank that owns the
utterances.  The one exchange is the sum of the weight gradients (dW_f, dW_g,
dW_o, db_o) over ranks: one torch.distributed all-reduce of one flat fp32
buffer (NCCL over NVLink / NVSwitch between GPUs; gloo on CPU for the tests),
fed with the library's unrounded fp32 accumulators and rounded once after
the sum.

The loss of every utterance is -log P of its own alignment lattice
("Sequence Transduction with Recurrent Neural Networks", abstract), so the
sharded result equals the single-device one up to floating-point reassociation
of the weight-gradient sum.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

WEIGHT_GRADS = ("dW_f", "dW_g", "dW_o", "db_o")


def utterance_cost(T_len, U_len) -> list[int]:
    """Lattice cells per utterance, T_len * (U_len + 1): the work of one call scales with it."""
    return [int(t) * (int(u) + 1) for t, u in zip(T_len.tolist(), U_len.tolist())]


def shard_utterances(T_len, U_len, world: int) -> list[list[int]]:
    """Deterministic balanced split of utterance indices over `world` ranks.

    Longest-processing-time first: utterances sorted by cost (ties by index)
    go one by one to the currently lightest rank (ties to the lowest rank).
    Every utterance lands on exactly one rank; each rank's indices are
    returned in increasing order.  Ranks may be empty when world > B."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = utterance_cost(T_len, U_len)
    order = sorted(range(len(cost)), key=lambda i: (-cost[i], i))
    load = [0] * world
    shards: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        shards[r].append(i)
        load[r] += cost[i]
    return [sorted(s) for s in shards]


def take_shard(tensors: dict, idx: list[int], trim: bool = True) -> dict:
    """The shard's rows of every per-utterance tensor (dim 0); weights are shared.

    With ``trim`` the padded frame / label extents shrink to the shard's
    longest utterance, so a rank does not pay for another rank's padding."""
    sel = torch.as_tensor(idx, dtype=torch.long, device=tensors["f"].device)
    out = dict(tensors)
    for k in ("f", "g", "labels", "T_len", "U_len"):
        out[k] = tensors[k].index_select(0, sel).contiguous()
    if trim and len(idx) > 0:
        T = int(out["T_len"].max())
        U = int(out["U_len"].max())
        out["f"] = out["f"][:, :T].contiguous()
        out["g"] = out["g"][:, :U + 1].contiguous()
        out["labels"] = out["labels"][:, :max(U, 1)].contiguous() if U > 0 else out["labels"][:, :0].contiguous()
    return out


def _weight_keys(grads: dict) -> tuple:
    return WEIGHT_GRADS + tuple(k for k in ("dW_d", "db_d") if k in grads)


def _shared_flat(grads: dict, keys) -> torch.Tensor | None:
    """The one contiguous fp32 buffer every weight gradient is a view of
    (frnnt.Outputs with wgrad_f32), else None."""
    base = grads[keys[0]]._base
    if base is None or base.dtype != torch.float32 or not base.is_contiguous() or base.dim() != 1:
        return None
    for k in keys:
        if grads[k]._base is not base or grads[k].dtype != torch.float32:
            return None
    return base


def allreduce_weight_grads(grads: dict, group=None, out_dtype=None) -> dict:
    """Sums dW_f, dW_g, dW_o, db_o (and the duration head's dW_d, db_d when
    present) over the ranks of `group` with ONE all-reduce of one flat fp32
    buffer, then rounds each sum once, to ``out_dtype`` (default: the dtype
    each gradient arrived in).  df / dg are left as they are.

    The partial gradients should arrive in fp32: the library's unrounded
    accumulators, asked for with ``wgrad_f32=True``.  When they are views of
    one flat buffer (frnnt.Outputs with wgrad_f32) that buffer is reduced in
    place; otherwise they are packed (16-bit ones widened) into a new one."""
    keys = _weight_keys(grads)
    flat = _shared_flat(grads, keys)
    views = {}
    if flat is None:
        # at least fp32 (fp64 partials, as the CPU tests' oracle gives, stay fp64)
        acc = torch.float64 if any(grads[k].dtype == torch.float64 for k in keys) else torch.float32
        flat = torch.cat([grads[k].reshape(-1).to(acc) for k in keys])
        off = 0
        for k in keys:
            n = grads[k].numel()
            views[k] = flat[off:off + n].view(grads[k].shape)
            off += n
    else:
        views = {k: grads[k] for k in keys}
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    out = dict(grads)
    for k in keys:
        dt = grads[k].dtype if out_dtype is None else out_dtype
        out[k] = views[k] if dt == views[k].dtype else views[k].to(dt)
    return out


def fwd_bwd_sharded(tensors: dict, compute, rank: int, world: int, group=None, grad_loss=None, out_dtype=None):
    """One data-parallel step.

    ``tensors`` holds the full batch (f, g, W_f, W_g, W_o, b_o, labels, T_len,
    U_len); ``compute(shard_tensors, grad_loss_shard) -> (loss, grads)`` runs
    the single-device call (frnnt.fwd_bwd on the GPU, with fp32 weight
    gradients).  Returns (shard indices, shard losses, grads) where df / dg
    cover the shard's utterances and the weight gradients are summed over all
    ranks in fp32 and rounded once to ``out_dtype`` (default: as computed)."""
    shards = shard_utterances(tensors["T_len"].cpu(), tensors["U_len"].cpu(), world)
    # every rank sees the same shards, so all ranks refuse alike (before any collective)
    if any(len(s) == 0 for s in shards):
        raise ValueError(f"{world} ranks for {tensors['f'].shape[0]} utterances leave a rank without work")
    idx = shards[rank]
    shard = take_shard(tensors, idx)
    w = None if grad_loss is None else grad_loss.index_select(
        0, torch.as_tensor(idx, dtype=torch.long, device=grad_loss.device)).contiguous()
    loss, grads = compute(shard, w)
    grads = allreduce_weight_grads(grads, group=group, out_dtype=out_dtype)
    return idx, loss, grads


def gpu_compute(mode: str = "tiled", durations=None, wgrad_f32: bool = True, **kw):
    """The CUDA library as the per-rank compute of fwd_bwd_sharded (with
    ``durations``: the token-and-duration transducer, whose duration head
    W_d / b_d travels in the tensors dict like the other weights).  By default
    the weight gradients come back as the library's fp32 accumulators, views
    of one flat buffer that the exchange reduces in place."""
    from . import frnnt

    def run(t, w):
        if durations is not None:
            return frnnt.fwd_bwd_tdt(t["f"], t["g"], t["W_f"], t["W_g"], t["W_o"], t["b_o"], t["W_d"], t["b_d"],
                                     t["labels"], t["T_len"], t["U_len"], durations, grad_loss=w, mode=mode,
                                     wgrad_f32=wgrad_f32, **kw)
        return frnnt.fwd_bwd(t["f"], t["g"], t["W_f"], t["W_g"], t["W_o"], t["b_o"], t["labels"], t["T_len"],
                             t["U_len"], grad_loss=w, mode=mode, wgrad_f32=wgrad_f32, **kw)
    return run
