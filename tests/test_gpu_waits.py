"""Failure detection of the tensor-core kernels: every mbarrier wait is bounded.

rlt_selftest_wait_timeout launches a tensor-core GEMM kernel in a mode that issues no TMA load
and no MMA, with a 1 ms bound on every wait, so the kernel's first wait runs out.  The call
must then report RLT_ETIMEOUT through rlt_last_error, leave its output untouched, and leave the
model and the CUDA context usable: the next calls on the same handle match their references.
No GPU fault, trap or endless loop is involved.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import RLTOracle
from workloads import TINY, make_tokens, make_weights
from gpu_util import build_model, cosine, to_np

pytestmark = pytest.mark.gpu

RLT_ETIMEOUT = 4
WAIT_NS = 1_000_000

# kernel ids as rlt_gemm_bf16 numbers them: 2 + v row-tile variant v, 11 + s few-row kernel,
# 18 + p CTA-pair tiles
CASES = {
    "row-tile 128x64": (3, 256, 512, 512),
    "CTA pair 256x128": (19, 512, 512, 1024),
    "row-tile 128x128 K split over 2 CTAs": (7, 256, 512, 1024),
    "few-row K split over 2 CTAs": (13, 16, 512, 1024),
}


@pytest.mark.parametrize("name", list(CASES))
def test_a_wait_that_runs_out_latches_timeout_and_the_model_stays_usable(name):
    kernel, M, N, K = CASES[name]
    cfg = replace(TINY.model, dtype="bf16", W=3)
    w = make_weights(cfg)
    model = build_model(cfg, max_pos=16, weights=w)
    g = torch.Generator().manual_seed(7)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    Wt = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    C = torch.full((M, N), 7.0, device="cuda")
    assert model.last_error() == 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    model.selftest_wait_timeout(A, Wt, C, kernel, WAIT_NS)
    b.record()
    torch.cuda.synchronize()
    assert model.last_error() == RLT_ETIMEOUT
    assert model.last_error() == 0                         # reported once, then cleared
    assert a.elapsed_time(b) >= 0.9 * WAIT_NS / 1e6          # the wait really ran to its bound
    assert bool((C == 7.0).all())                          # no partial result was stored
    # the same handle still computes: the same kernel normally, then an exact replay
    C2 = model.gemm_bf16(A, Wt, kernel)
    ref = A.double() @ Wt.double().t()
    assert float((C2.double() - ref).abs().max()) <= 1e-3 * float(ref.abs().max())
    tok = make_tokens(TINY)[:, :16]
    score, lp, st = model.replay(torch.from_numpy(tok).cuda(), 6, 1.0, want_logp=True, want_state=True)
    torch.cuda.synchronize()
    assert model.last_error() == 0
    _, lp_r, s_r, _ = RLTOracle(cfg, w).replay(tok, 6, 1.0)
    assert np.abs(to_np(lp) - lp_r).max() <= 5e-2
    assert cosine(to_np(st.s()), s_r[:, -1]).min() >= 0.999
