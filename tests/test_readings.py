"""Rounding points of the bf16 GPU path that differ from the storage contract's literal
placement (CPU, numpy float64).

The decoder defers its sublayer RMSNorm into the projections: the GEMM input rounded to bf16
is x * g, and 1 / rms multiplies the product's rows, where the contract rounds the normalised
h = x / rms * g.  Both round every input element once with relative error <= 2^-9, so both
products sit within the same bound of the exact product; these tests check that bound on
seeded data shaped like the workloads' activations (a residual stream whose scale grows with
depth), and that without rounding the two forms are the same function.
"""
import numpy as np
import pytest

from oracle import round_bf16

U = 2.0 ** -9          # unit roundoff of bfloat16 (8 significant bits, round to nearest)


def _case(seed: int, B: int, d: int, N: int, scale: float):
    rng = np.random.default_rng([seed, B, d, N])
    x = rng.standard_normal((B, d)) * scale * np.exp(rng.standard_normal((B, 1)))   # rows of varied scale
    g = 1.0 + 0.1 * rng.standard_normal(d)
    W = round_bf16(rng.standard_normal((N, d)) * 0.02)                               # stored weights
    rinv = 1.0 / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-6)
    return x, g, W, rinv


@pytest.mark.parametrize("seed,B,d,N,scale", [(0, 16, 1024, 256, 1.0), (1, 8, 2048, 128, 30.0),
                                              (2, 4, 64, 64, 0.01)])
def test_deferred_norm_is_within_the_contracts_bf16_bound(seed, B, d, N, scale):
    x, g, W, rinv = _case(seed, B, d, N, scale)
    exact = (x * rinv * g) @ W.T
    contract = round_bf16(x * rinv * g) @ W.T                  # round the normalised input
    deferred = (round_bf16(x * g) @ W.T) * rinv                # round x * g, scale the rows after
    # |sum_k (h_k (1 + e_k) - h_k) W_nk| <= U * sum_k |h_k W_nk| for either placement
    bound = U * (np.abs(x * rinv * g) @ np.abs(W).T)
    assert np.all(np.abs(contract - exact) <= bound + 1e-12)
    assert np.all(np.abs(deferred - exact) <= bound * (1 + 1e-9) + 1e-12)
    # and the two differ from each other by at most twice that
    assert np.all(np.abs(deferred - contract) <= 2 * bound + 1e-12)


def test_deferred_norm_without_rounding_is_the_same_function():
    x, g, W, rinv = _case(3, 8, 256, 96, 5.0)
    np.testing.assert_allclose((x * g) @ W.T * rinv, (x * rinv * g) @ W.T, rtol=1e-12, atol=1e-14)
