"""The tcgen05 tensor-core GEMM (through its C-ABI test hook) against a plain
PyTorch fp32 matmul of the same bf16 operands."""

import pytest
import torch

from rnn_joint_network_02_b200 import frnnt

pytestmark = pytest.mark.gpu


def _operands(M, N, K, a_mn, b_mn, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    A = torch.randn(M, K, device="cuda", generator=g).bfloat16()
    B = torch.randn(K, N, device="cuda", generator=g).bfloat16()
    a_arg = A.t().contiguous() if a_mn else A.contiguous()     # MN-major A is stored [K][M]
    b_arg = B.contiguous() if b_mn else B.t().contiguous()     # K-major B is stored [N][K]
    ref = A.float() @ B.float()
    return a_arg, b_arg, ref


def _check(out, ref, tol=2e-3):
    err = (out.float() - ref).norm() / ref.norm()
    assert err.item() <= tol, err.item()


@pytest.mark.parametrize("variant", [0, 1, 2, 3])
@pytest.mark.parametrize("a_mn", [False, True])
@pytest.mark.parametrize("b_mn", [False, True])
@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (256, 256, 128), (296, 640, 520), (1000, 512, 256), (200, 608, 192),
                                   (312, 448, 128)])
def test_store_f32(cuda_ok, a_mn, b_mn, M, N, K, variant):
    """variant 0: one CTA per 128-row tile; 1: CTA pairs on 256-row tiles (cta_group::2);
    2 / 3: the same with 256-wide N tiles whatever N (a ragged last tile)."""
    A, B, ref = _operands(M, N, K, a_mn, b_mn)
    out = frnnt.test_gemm_bf16(A, B, a_mn, b_mn, M, N, K, epi=0, variant=variant)
    torch.cuda.synchronize()
    _check(out, ref, 1e-5)


@pytest.mark.parametrize("variant", [0, 1])
@pytest.mark.parametrize("a_mn,b_mn", [(False, True), (True, True), (False, False)])
def test_store_bf16(cuda_ok, a_mn, b_mn, variant):
    M, N, K = 384, 256, 640
    A, B, ref = _operands(M, N, K, a_mn, b_mn, seed=1)
    out = frnnt.test_gemm_bf16(A, B, a_mn, b_mn, M, N, K, epi=1, variant=variant)
    torch.cuda.synchronize()
    _check(out, ref, 8e-3)


@pytest.mark.parametrize("variant", [0, 1, 2, 3])
@pytest.mark.parametrize("splits", [1, 3, 7])
def test_split_k_reduce(cuda_ok, splits, variant):
    M, N, K = 1024, 640, 4096 + 64
    A, B, ref = _operands(M, N, K, True, True, seed=2)
    out = torch.full((M, N), 0.5, device="cuda")
    frnnt.test_gemm_bf16(A, B, True, True, M, N, K, epi=2, k_splits=splits, out=out, variant=variant)
    torch.cuda.synchronize()
    _check(out - 0.5, ref, 1e-5)


@pytest.mark.parametrize("variant", [0, 1, 2, 3])
def test_dtanh_epilogue(cuda_ok, variant):
    M, N, K = 512, 640, 1024
    A, B, ref = _operands(M, N, K, False, True, seed=3)
    h = torch.tanh(torch.randn(M, N, device="cuda")).bfloat16()
    out = h.clone()
    frnnt.test_gemm_bf16(A, B, False, True, M, N, K, epi=3, out=out, variant=variant)
    torch.cuda.synchronize()
    expect = ref * (1 - h.float() ** 2)
    _check(out, expect, 8e-3)


@pytest.mark.parametrize("variant", [0, 1, 2, 3])
def test_many_tiles_persistent(cuda_ok, variant):
    """More output tiles than SMs: every CTA walks several tiles and both TMEM buffers."""
    M, N, K = 6400, 640, 512
    A, B, ref = _operands(M, N, K, False, True, seed=4)
    out = frnnt.test_gemm_bf16(A, B, False, True, M, N, K, epi=0, variant=variant)
    torch.cuda.synchronize()
    _check(out, ref, 1e-5)
