"""Failure detection on the GPU without a fault: a producer that never
announces its first K block (the lose_gemm_loads test setting) leaves a
bounded mbarrier wait to run out.  The kernel must end on its own, report
FRNNT_STATUS_TIMEOUT in the status word, and leave the context usable: the
same work run again afterwards is complete and correct."""

import pytest
import torch

from rnn_joint_network_02_b200 import frnnt, synth
from tests.helpers import compare, run_oracle, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture
def lose_loads():
    prev = frnnt.lose_gemm_loads(0)
    yield frnnt.lose_gemm_loads
    frnnt.lose_gemm_loads(prev)


def _gemm_operands(M, N, K):
    g = torch.Generator(device="cuda").manual_seed(11)
    A = torch.randn(M, K, device="cuda", generator=g).bfloat16()      # K-major A
    B = torch.randn(K, N, device="cuda", generator=g).bfloat16()      # MN-major B ([K][N])
    return A, B, A.float() @ B.float()


@pytest.mark.parametrize("variant", [0, 1])
def test_lost_load_times_out_and_context_survives(cuda_ok, lose_loads, variant):
    """variant 0: one CTA per tile (its MMA issuer's wait runs out); 1: CTA
    pairs (the leader's issuer and the partner's producer both give up)."""
    M, N, K = 512, 256, 512
    A, B, ref = _gemm_operands(M, N, K)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    lose_loads(1)
    frnnt.test_gemm_bf16(A, B, False, True, M, N, K, epi=0, variant=variant, status=status)
    torch.cuda.synchronize()
    assert lose_loads(0) == 0, "the setting is consumed by exactly one launch"
    assert int(status[0]) & frnnt.STATUS_TIMEOUT, int(status[0])

    status.zero_()
    out = frnnt.test_gemm_bf16(A, B, False, True, M, N, K, epi=0, variant=variant, status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    err = (out - ref).norm() / ref.norm()
    assert err.item() <= 1e-5, err.item()


def test_lost_load_inside_a_call_is_reported(cuda_ok, lose_loads):
    """One GEMM of a whole fwd_bwd call loses its load: the call returns, its
    status word carries the timeout (FrnntStatusError from the binding), and the
    next call on the same inputs matches the oracle."""
    batch = synth.workload("short")
    d = to_device(batch)
    args = (d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"], d["U_len"])
    lose_loads(1)
    with pytest.raises(frnnt.FrnntStatusError, match="timed out"):
        frnnt.fwd_bwd(*args, mode="untiled")
    assert lose_loads(0) == 0
    loss, grads = frnnt.fwd_bwd(*args, mode="untiled")
    torch.cuda.synchronize()
    compare(loss, grads, run_oracle(batch), "bf16", extra_note="after a timed-out call")
