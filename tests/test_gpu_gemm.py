"""The tcgen05/TMA GEMM against float64 matmul of the same bf16 operands (and the CUDA-core kernel).

Bound: float32 accumulation of K products, |dC| <= 1e-4 * (|A| |W|^T) elementwise.
"""
import numpy as np
import pytest
import torch

from workloads import TINY
from gpu_util import build_model

pytestmark = pytest.mark.gpu

SHAPES = [
    (32, 6144, 2048),     # 48+48 decoder q/k/v at B=32
    (17, 11264, 2048),    # ragged few-row batch, FFN gate/up width
    (3, 2048, 5632),      # FFN down at B=3
    (512, 3072, 1024),    # 300M-class decoder q/k/v at B=512
    (512, 1024, 4096),    # FFN down
    (64, 2048, 2048),     # small-batch decoder row count
    (1, 256, 128),        # single row
    (300, 200, 136),      # ragged M, N and K (K not a multiple of the 64-wide k-block)
    (4096, 1536, 1024),   # encoder-like
    (129, 40, 64),
    (2, 6144, 2048),      # weight-streaming kernel: two rows
    (4, 11264, 5632),     # four rows, the widest K it takes
    (1, 32000, 1024),     # LM head of the 300M-class model at B=1
    (2000, 3000, 520),    # persistent kernel: ragged M, N and K over several waves
]


@pytest.fixture(scope="module")
def model():
    return build_model(TINY.model, max_pos=8)


@pytest.mark.parametrize("kernel", [0, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16, 17, 18, 19, 20])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_tcgen05_gemm_matches_float64(model, M, N, K, kernel):
    if 11 <= kernel <= 15 and M > 64:
        pytest.skip("the few-row kernel takes M <= 64")
    if kernel == 16 and (M > 4 or N % 32 or K > 6144):
        pytest.skip("the weight-streaming kernel takes M <= 4, N a multiple of 32, K <= 6144")
    g = torch.Generator().manual_seed(M * 7919 + N * 31 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    ref = A.double() @ W.double().T
    bound = A.double().abs() @ W.double().abs().T
    c_tc = model.gemm_bf16(A, W, kernel=kernel).cpu().double()
    torch.cuda.synchronize()
    assert model.last_error() == 0
    err = (c_tc - ref).abs()
    assert bool((err <= 1e-4 * bound + 1e-6).all()), float((err / (bound + 1e-6)).max())
    if kernel == 0:
        c_simt = model.gemm_bf16(A, W, kernel=1).cpu().double()
        assert bool(((c_simt - ref).abs() <= 1e-4 * bound + 1e-6).all())


@pytest.mark.parametrize("kernel", [0, 7, 8, 9, 10, 14, 15, 17, 18, 19, 20])
def test_tcgen05_gemm_is_deterministic(model, kernel):
    g = torch.Generator().manual_seed(5)
    A = torch.randn(64 if 11 <= kernel <= 15 else 512, 1024, generator=g).to(torch.bfloat16)
    W = torch.randn(3072, 1024, generator=g).to(torch.bfloat16)
    a = model.gemm_bf16(A, W, kernel=kernel)
    b = model.gemm_bf16(A, W, kernel=kernel)
    assert torch.equal(a, b)
