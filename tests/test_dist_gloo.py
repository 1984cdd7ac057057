"""Data-parallel sharding and the weight-gradient exchange, on CPU.

The sharding logic is checked directly; the multi-process path runs as two
gloo ranks on CPU, each computing its shard with the fp64 oracle, and must
reproduce the oracle's single-process result for the whole batch."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rnn_joint_network_02_b200 import dist as rdist
from rnn_joint_network_02_b200 import synth


def test_shards_cover_every_utterance_once_and_balance():
    batch = synth.workload("medium")
    for world in (1, 2, 3, 4, 8):
        shards = rdist.shard_utterances(batch.T_len, batch.U_len, world)
        flat = sorted(i for s in shards for i in s)
        assert flat == list(range(batch.f.shape[0]))
        cost = rdist.utterance_cost(batch.T_len, batch.U_len)
        loads = [sum(cost[i] for i in s) for s in shards]
        # LPT bound: max load <= mean + largest single item
        assert max(loads) <= sum(cost) / world + max(cost)
    assert rdist.shard_utterances(batch.T_len, batch.U_len, 2) == rdist.shard_utterances(batch.T_len, batch.U_len, 2)


def test_more_ranks_than_utterances_leaves_empty_shards():
    T_len = torch.tensor([5, 3], dtype=torch.int32)
    U_len = torch.tensor([1, 2], dtype=torch.int32)
    shards = rdist.shard_utterances(T_len, U_len, 4)
    assert sorted(len(s) for s in shards) == [0, 0, 1, 1]


def test_take_shard_trims_padding():
    batch = synth.make(B=4, T=20, U=6, D_enc=3, D_pred=3, H=4, V=5, dtype="f32", seed=1, T_range=(3, 20),
                       U_range=(0, 6))
    t = {k: getattr(batch, k) for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")}
    sh = rdist.take_shard(t, [1, 3])
    assert sh["f"].shape[1] == int(batch.T_len[[1, 3]].max())
    assert sh["g"].shape[1] == int(batch.U_len[[1, 3]].max()) + 1
    assert torch.equal(sh["W_o"], batch.W_o)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_compute(shard, w):
    import oracle
    f, g, W_f, W_g, W_o, b_o = (shard[k].double().numpy() for k in ("f", "g", "W_f", "W_g", "W_o", "b_o"))
    res = oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, shard["labels"].numpy(), shard["T_len"].numpy(),
                         shard["U_len"].numpy(), grad_loss=None if w is None else w.double().numpy())
    grads = {k: torch.from_numpy(getattr(res, k)) for k in ("df", "dg", "dW_f", "dW_g", "dW_o", "db_o")}
    return torch.from_numpy(res.loss), grads


def _worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        batch = synth.make(B=5, T=7, U=4, D_enc=4, D_pred=3, H=6, V=7, dtype="f32", seed=77, T_range=(2, 7),
                           U_range=(0, 4), bias_std=0.3)
        t = {k: getattr(batch, k) for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")}
        w = torch.linspace(0.5, 1.5, 5)
        idx, loss, grads = rdist.fwd_bwd_sharded(t, _oracle_compute, rank, world, grad_loss=w)
        torch.save({"idx": idx, "loss": loss, "grads": grads}, f"{out_path}.{rank}")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_single_process(tmp_path):
    world = 2
    out = str(tmp_path / "res")
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    import oracle
    batch = synth.make(B=5, T=7, U=4, D_enc=4, D_pred=3, H=6, V=7, dtype="f32", seed=77, T_range=(2, 7),
                       U_range=(0, 4), bias_std=0.3)
    w = np.linspace(0.5, 1.5, 5)
    f, g, W_f, W_g, W_o, b_o = (x.numpy() for x in batch.float64())
    ref = oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(),
                         grad_loss=w)
    seen = []
    for r in range(world):
        d = torch.load(f"{out}.{r}")
        idx = d["idx"]
        seen += idx
        np.testing.assert_allclose(d["loss"].numpy(), ref.loss[idx], rtol=1e-12)
        for k in ("dW_f", "dW_g", "dW_o", "db_o"):
            np.testing.assert_allclose(d["grads"][k].numpy(), getattr(ref, k), rtol=1e-10, atol=1e-12)
        for j, b in enumerate(idx):
            Tb, Ub = int(batch.T_len[b]), int(batch.U_len[b])
            np.testing.assert_allclose(d["grads"]["df"][j, :Tb].numpy(), ref.df[b, :Tb], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(d["grads"]["dg"][j, :Ub + 1].numpy(), ref.dg[b, :Ub + 1], rtol=1e-10,
                                       atol=1e-12)
    assert sorted(seen) == list(range(5))


TDT_D = (0, 1, 2)


def _tdt_batch():
    batch = synth.make(B=5, T=7, U=4, D_enc=4, D_pred=3, H=6, V=7, dtype="f32", seed=78, T_range=(2, 7),
                       U_range=(0, 4), bias_std=0.3)
    W_d, b_d = synth.duration_head(batch, len(TDT_D), seed=4)
    return batch, W_d, b_d


def _oracle_tdt_compute(shard, w):
    import oracle
    f, g, W_f, W_g, W_o, b_o, W_d, b_d = (shard[k].double().numpy()
                                          for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "W_d", "b_d"))
    res = oracle.tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d, b_d, shard["labels"].numpy(), shard["T_len"].numpy(),
                             shard["U_len"].numpy(), TDT_D, grad_loss=None if w is None else w.double().numpy())
    grads = {k: torch.from_numpy(getattr(res, k))
             for k in ("df", "dg", "dW_f", "dW_g", "dW_o", "db_o", "dW_d", "db_d")}
    return torch.from_numpy(res.loss), grads


def _tdt_worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        batch, W_d, b_d = _tdt_batch()
        t = {k: getattr(batch, k) for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")}
        t["W_d"], t["b_d"] = W_d, b_d
        idx, loss, grads = rdist.fwd_bwd_sharded(t, _oracle_tdt_compute, rank, world,
                                                 grad_loss=torch.linspace(0.5, 1.5, 5))
        torch.save({"idx": idx, "loss": loss, "grads": grads}, f"{out_path}.{rank}")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_tdt_duration_head_grads_summed(tmp_path):
    """The token-and-duration transducer's duration-head gradients take part
    in the weight-gradient exchange like the label head's."""
    world = 2
    out = str(tmp_path / "tdt")
    mp.start_processes(_tdt_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    import oracle
    batch, W_d, b_d = _tdt_batch()
    f, g, W_f, W_g, W_o, b_o = (x.numpy() for x in batch.float64())
    ref = oracle.tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d.double().numpy(), b_d.double().numpy(),
                             batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(), TDT_D,
                             grad_loss=np.linspace(0.5, 1.5, 5))
    seen = []
    for r in range(world):
        d = torch.load(f"{out}.{r}")
        seen += d["idx"]
        np.testing.assert_allclose(d["loss"].numpy(), ref.loss[d["idx"]], rtol=1e-12)
        for k in ("dW_f", "dW_g", "dW_o", "db_o", "dW_d", "db_d"):
            np.testing.assert_allclose(d["grads"][k].numpy(), getattr(ref, k), rtol=1e-10, atol=1e-12)
    assert sorted(seen) == list(range(5))


def _flat_fp32_compute(shard, w):
    """The oracle as the per-rank compute, returning what the library returns
    with wgrad_f32: fp32 weight gradients (here the fp64 values rounded to
    fp32 once) as views of one flat fp32 buffer with 16-byte-aligned segments."""
    loss, grads = _oracle_compute(shard, w)
    keys = ("dW_f", "dW_g", "dW_o", "db_o")
    sizes = [(grads[k].numel() + 3) // 4 * 4 for k in keys]
    flat = torch.zeros(sum(sizes), dtype=torch.float32)
    off = 0
    out = dict(grads)
    for k, n in zip(keys, sizes):
        v = flat[off:off + grads[k].numel()].view(grads[k].shape)
        v.copy_(grads[k].float())
        out[k] = v
        off += n
    return loss, out


def _fp32_worker(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    calls = []
    real = dist.all_reduce

    def counting(*a, **k):
        calls.append(1)
        return real(*a, **k)

    dist.all_reduce = counting
    try:
        batch = synth.make(B=5, T=7, U=4, D_enc=4, D_pred=3, H=6, V=7, dtype="f32", seed=77, T_range=(2, 7),
                           U_range=(0, 4), bias_std=0.3)
        t = {k: getattr(batch, k) for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")}
        w = torch.linspace(0.5, 1.5, 5)
        # fp32 partials reduced in place: one all-reduce, the sum kept in fp32
        idx, _, g32 = rdist.fwd_bwd_sharded(t, _flat_fp32_compute, rank, world, grad_loss=w)
        n_flat = len(calls)
        # separate fp32 partials: packed into one buffer, one all-reduce, the sum rounded once to bf16
        def fp32_compute(shard, ww):
            loss, grads = _oracle_compute(shard, ww)
            return loss, {k: v.float() for k, v in grads.items()}
        _, _, g16 = rdist.fwd_bwd_sharded(t, fp32_compute, rank, world, grad_loss=w, out_dtype=torch.bfloat16)
        n_packed = len(calls) - n_flat
        torch.save({"idx": idx, "g32": g32, "g16": g16, "n_flat": n_flat, "n_packed": n_packed},
                   f"{out_path}.{rank}")
    finally:
        dist.all_reduce = real
        dist.destroy_process_group()


def test_two_gloo_ranks_fp32_partials_one_allreduce(tmp_path):
    """The exchange is one all-reduce of one flat fp32 buffer.  Summing the
    ranks' fp32 partial weight gradients gives the single-device result at fp32
    accumulation (the loss is a sum over utterances, "Sequence Transduction
    with Recurrent Neural Networks", abstract): within fp32 reassociation of
    the single-device gradient rounded to fp32."""
    world = 2
    out = str(tmp_path / "f32")
    mp.start_processes(_fp32_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    import oracle
    batch = synth.make(B=5, T=7, U=4, D_enc=4, D_pred=3, H=6, V=7, dtype="f32", seed=77, T_range=(2, 7),
                       U_range=(0, 4), bias_std=0.3)
    f, g, W_f, W_g, W_o, b_o = (x.numpy() for x in batch.float64())
    ref = oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(),
                         grad_loss=np.linspace(0.5, 1.5, 5))
    for r in range(world):
        d = torch.load(f"{out}.{r}")
        assert d["n_flat"] == 1 and d["n_packed"] == 1, (d["n_flat"], d["n_packed"])
        for k in ("dW_f", "dW_g", "dW_o", "db_o"):
            single = getattr(ref, k).astype(np.float32)        # the single-device fp32 accumulator
            got = d["g32"][k]
            assert got.dtype == torch.float32
            scale = np.abs(single).max()
            np.testing.assert_allclose(got.numpy(), single, rtol=1e-6, atol=1e-6 * scale)
            # summed in fp32, rounded once to bf16: within one bf16 rounding (half a step, 2^-8
            # relative) of the exact sum, plus the fp32 sum's own error
            got16 = d["g16"][k]
            assert got16.dtype == torch.bfloat16
            exact = getattr(ref, k)
            err = np.abs(got16.double().numpy() - exact)
            assert np.all(err <= np.abs(exact) * 2.0 ** -8 + 1e-6 * scale), k
