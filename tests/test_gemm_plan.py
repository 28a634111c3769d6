"""Projection kernel choice (host logic, CPU): the kernel id rlt_gemm_plan reports for the
workloads' decode and encoder shapes, i.e. the choices the measured timings picked.

Ids as rlt_gemm_bf16 numbers them: 2 + v = row-tile variant v (0: 128x32, 1: 128x64,
2: 128x128 x3 stages, 3: 128x128 x6, 4: 128x256, 5: 128x128 split 2, 6: 128x128 split 4,
7: 128x64 split 2, 8: 128x64 split 4); 11 + s = few-row kernel, s = 1, 2, 3 for a K split of
1, 2, 4.
"""
import pytest

from cross_token_latent_b200.rlt import gemm_plan

PLANS = [
    # 300M-class decoder at B=512 (d=1024, F=4096, V=32000)
    ((512, 1024, 1024), 9, "o / q_c / o_c: 64-wide tiles, K split in two (half the L2 re-reads of 32-wide)"),
    ((512, 3072, 1024), 5, "q/k/v: 128x128 with a deep ring, 96 CTAs"),
    ((512, 8192, 1024), 6, "gate/up: 128x256"),
    ((512, 1024, 4096), 8, "down: 128x128 with K split over four"),
    ((512, 2048, 2048), 7, "gated merge: 128x128 with K split in two"),
    ((512, 32000, 1024), 6, "LM head: more tiles than a wave, widest tile"),
    # 24+24 replay at B=64 (d=2048, F=5632)
    ((64, 2048, 2048), 10, "33..64 rows, narrow output: row tiles, 64 wide, K split over four"),
    ((64, 2048, 5632), 10, "down at B=64"),
    ((64, 6144, 2048), 13, "q/k/v at B=64: the weights fill a wave, few-row kernel, split 2"),
    ((64, 11264, 2048), 12, "gate/up at B=64: few-row kernel, no split"),
    # 48+48 at B=32 and B=1
    ((32, 2048, 2048), 14, "<= 32 rows: few-row kernel, split 4"),
    ((32, 6144, 2048), 13, "q/k/v at B=32"),
    ((32, 2048, 5632), 14, "down at B=32"),
    ((1, 2048, 2048), 14, "B=1"),
    ((1, 11264, 2048), 12, "gate/up at B=1"),
    ((4, 2048, 5632), 14, "down at B=4"),
    # small shapes and the encoder
    ((64, 384, 128), 2, "two k-blocks: narrow row tiles put the most CTAs in flight"),
    ((65536, 3072, 1024), 6, "encoder q/k/v: grids of many waves take the widest tile"),
]


@pytest.mark.parametrize("shape,kernel,why", PLANS, ids=[f"{m}x{n}x{k}" for (m, n, k), _, _ in PLANS])
def test_plan_of_workload_shapes(shape, kernel, why):
    assert gemm_plan(*shape) == kernel, why


def test_plan_rejects_empty_shapes():
    assert gemm_plan(0, 16, 16) == -1
    assert gemm_plan(16, 16, 0) == -1


def test_few_row_kernel_never_plans_eight_way_clusters():
    """8-CTA clusters measured 2.2x slower than 4 (two waves at one CTA per SM)."""
    for M in (1, 7, 16, 17, 32, 48, 64):
        for N in (256, 1024, 2048, 6144, 11264):
            for K in (256, 1024, 2048, 5632, 16384):
                assert gemm_plan(M, N, K) != 15
