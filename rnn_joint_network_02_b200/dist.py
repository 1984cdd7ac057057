"""Data parallelism across GPUs: one process per GPU, utterances sharded.

Utterances of a transducer batch are independent, so the batch is split
across ranks with every rank running the whole fused joint + loss call on its
shard; frame / label gradients (df, dg) stay with the rank that owns the
utterances.  The one exchange is the sum of the weight gradients (dW_f, dW_g,
dW_o, db_o) over ranks, done by torch.distributed's all-reduce (NCCL over
NVLink / NVSwitch between GPUs; gloo on CPU for the tests).

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


def allreduce_weight_grads(grads: dict, group=None) -> dict:
    """Sums dW_f, dW_g, dW_o, db_o (and the duration head's dW_d, db_d when
    present) over the ranks of `group` in at least fp32 (16-bit gradients are
    widened for the sum, then rounded back).  df / dg are left as they are."""
    out = dict(grads)
    for k in WEIGHT_GRADS + tuple(k for k in ("dW_d", "db_d") if k in grads):
        g = grads[k]
        acc = g.float() if g.element_size() < 4 else g.clone()
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
        out[k] = acc.to(grads[k].dtype)
    return out


def fwd_bwd_sharded(tensors: dict, compute, rank: int, world: int, group=None, grad_loss=None):
    """One data-parallel step.

    ``tensors`` holds the full batch (f, g, W_f, W_g, W_o, b_o, labels, T_len,
    U_len); ``compute(shard_tensors, grad_loss_shard) -> (loss, grads)`` runs
    the single-device call (frnnt.fwd_bwd on the GPU).  Returns
    (shard indices, shard losses, grads) where df / dg cover the shard's
    utterances and the weight gradients are summed over all ranks."""
    shards = shard_utterances(tensors["T_len"].cpu(), tensors["U_len"].cpu(), world)
    # every rank sees the same shards, so all ranks refuse alike (before any collective)
    if any(len(s) == 0 for s in shards):
        raise ValueError(f"{world} ranks for {tensors['f'].shape[0]} utterances leave a rank without work")
    idx = shards[rank]
    shard = take_shard(tensors, idx)
    w = None if grad_loss is None else grad_loss.index_select(
        0, torch.as_tensor(idx, dtype=torch.long, device=grad_loss.device)).contiguous()
    loss, grads = compute(shard, w)
    grads = allreduce_weight_grads(grads, group=group)
    return idx, loss, grads


def gpu_compute(mode: str = "tiled", durations=None, **kw):
    """The CUDA library as the per-rank compute of fwd_bwd_sharded (with
    ``durations``: the token-and-duration transducer, whose duration head
    W_d / b_d travels in the tensors dict like the other weights)."""
    from . import frnnt

    def run(t, w):
        if durations is not None:
            return frnnt.fwd_bwd_tdt(t["f"], t["g"], t["W_f"], t["W_g"], t["W_o"], t["b_o"], t["W_d"], t["b_d"],
                                     t["labels"], t["T_len"], t["U_len"], durations, grad_loss=w, mode=mode, **kw)
        return frnnt.fwd_bwd(t["f"], t["g"], t["W_f"], t["W_g"], t["W_o"], t["b_o"], t["labels"], t["T_len"],
                             t["U_len"], grad_loss=w, mode=mode, **kw)
    return run
