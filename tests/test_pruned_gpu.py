"""GPU parity of the pruned (banded) lattice against the oracle with the same
bounds, through frnnt_fwd_bwd_pruned (bf16, tensor-core kernels)."""

import numpy as np
import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import GRADS, compare, rel_l2, run_oracle, to_device, weights_for

pytestmark = pytest.mark.gpu


def _call(batch, bounds, S, mode="tiled", grad_loss=None, chunk_cells=0, loss="marginal", check=True):
    d = to_device(batch)
    w = None if grad_loss is None else torch.as_tensor(grad_loss, dtype=torch.float32).cuda()
    bd = torch.as_tensor(np.asarray(bounds), dtype=torch.int32).contiguous().cuda()
    out = frnnt.fwd_bwd_pruned(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                               d["U_len"], bd, S, grad_loss=w, mode=mode, chunk_cells=chunk_cells,
                               blank=batch.blank, loss=loss, check=check)
    torch.cuda.synchronize()
    return out


def _random_bounds(batch, S, seed):
    """Valid bounds with random steps of 0..S-1 (U_len shortened where S cannot reach it)."""
    rng = np.random.default_rng(seed)
    B, T = batch.f.shape[:2]
    out = np.zeros((B, T), dtype=np.int32)
    for b in range(B):
        Tb = int(batch.T_len[b])
        batch.U_len[b] = min(int(batch.U_len[b]), (Tb - 1) * (S - 1) + S - 1)
        Ub = int(batch.U_len[b])
        s = 0
        for t in range(1, Tb):
            lo = max(s, Ub - S + 1 - (Tb - 1 - t) * (S - 1), 0)
            hi = max(min(s + S - 1, Ub), lo)
            s = int(rng.integers(lo, hi + 1))
            out[b, t] = s
        out[b, Tb:] = out[b, Tb - 1]
    return out


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
@pytest.mark.parametrize("S", [2, 3, 5, 8])
def test_ragged_random_bounds(cuda_ok, mode, S):
    batch = synth.make(B=5, T=40, U=12, D_enc=64, D_pred=32, H=128, V=256, dtype="bf16", seed=600 + S,
                       T_range=(8, 40), U_range=(0, 12), bias_std=0.3)
    bounds = _random_bounds(batch, S, seed=S)
    w = np.linspace(0.5, 1.5, 5)
    for loss in ("marginal", "viterbi"):
        l, g = _call(batch, bounds, S, mode=mode, grad_loss=w, chunk_cells=512, loss=loss)
        compare(l, g, run_oracle(batch, grad_loss=w, loss=loss, bounds=bounds, S=S), "bf16",
                extra_note=f"pruned S{S}/{mode}/{loss}")


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_wide_band_32_lane_tiles(cuda_ok, mode):
    """S = 20 rounds up to 32 band positions per tile row: a frame's cells fill
    a whole warp, the one layout where the frame sums run over all 32 lanes."""
    S = 20
    batch = synth.make(B=3, T=24, U=48, D_enc=64, D_pred=32, H=128, V=256, dtype="bf16", seed=620,
                       T_range=(6, 24), U_range=(10, 48), bias_std=0.3)
    bounds = _random_bounds(batch, S, seed=S)
    w = np.linspace(0.5, 1.5, 3)
    l, g = _call(batch, bounds, S, mode=mode, grad_loss=w, chunk_cells=1024)
    compare(l, g, run_oracle(batch, grad_loss=w, bounds=bounds, S=S), "bf16", extra_note=f"pruned S{S}/{mode}")


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_short_diagonal_band(cuda_ok, mode):
    batch = synth.workload("short")
    S = 6
    bounds = synth.diagonal_bounds(batch.T_len, batch.U_len, batch.f.shape[1], S)
    l, g = _call(batch, bounds, S, mode=mode)
    compare(l, g, run_oracle(batch, bounds=bounds.numpy(), S=S), "bf16", extra_note=f"pruned short/{mode}")


def test_full_band_matches_unpruned(cuda_ok):
    """A band as wide as the lattice (S = U+1, every start 0) is the whole lattice."""
    batch = synth.make(B=4, T=30, U=15, D_enc=64, D_pred=64, H=128, V=256, dtype="bf16", seed=88,
                       T_range=(10, 30), U_range=(0, 15))
    S = 16
    bounds = np.zeros((4, 30), dtype=np.int32)
    lp, gp = _call(batch, bounds, S)
    lp, gp = lp.clone(), {k: v.clone() for k, v in gp.items()}
    d = to_device(batch)
    lf, gf = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                           d["U_len"], blank=batch.blank)
    torch.cuda.synchronize()
    assert torch.allclose(lp, lf, rtol=1e-4)
    for k in GRADS:
        assert rel_l2(gp[k].float().cpu().numpy(), gf[k].float().cpu().numpy()) <= 1e-2, k


@pytest.mark.parametrize("case", ["start", "step", "reverse", "end"])
def test_invalid_bounds_set_status(cuda_ok, case):
    batch = synth.workload("short")
    S = 6
    bounds = synth.diagonal_bounds(batch.T_len, batch.U_len, batch.f.shape[1], S).numpy()
    Tb = int(batch.T_len[0])
    if case == "start":
        bounds[0, 0] = 1
    elif case == "step":
        bounds[0, Tb // 2:] += S
    elif case == "reverse":
        bounds[0, Tb // 2] = max(0, bounds[0, Tb // 2 - 1] - 1) if bounds[0, Tb // 2 - 1] > 0 else 0
        bounds[0, Tb // 2 - 1] = bounds[0, Tb // 2] + 1
    elif case == "end":
        bounds[0, :Tb] = 0
    import oracle
    expect = oracle.validate_bounds(S, bounds, batch.T_len.numpy(), batch.U_len.numpy())
    assert expect == frnnt.STATUS_BOUNDS
    with pytest.raises(frnnt.FrnntStatusError) as ei:
        _call(batch, bounds, S)
    assert ei.value.bits & frnnt.STATUS_BOUNDS


@pytest.mark.parametrize("mode", ["tiled", "untiled"])
def test_medium_sampled(cuda_ok, mode):
    batch = synth.workload("medium")
    S = 8
    bounds = synth.diagonal_bounds(batch.T_len, batch.U_len, batch.f.shape[1], S)
    B = batch.f.shape[0]
    pick = [0, B - 1]
    w = weights_for(B, pick, device="cpu").numpy()
    l, g = _call(batch, bounds, S, mode=mode, grad_loss=w)
    ref = run_oracle(batch, grad_loss=w, utterances=pick, bounds=bounds.numpy(), S=S)
    compare(l, g, ref, "bf16", utterances=pick, extra_note=f"pruned medium/{mode}")
