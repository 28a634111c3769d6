"""Full-size workloads on the GPU vs stored oracle outputs on sampled sequences.

The GPU runs the whole batch at the workload's full size (the launch configuration bench.py
times: full B, e and M for all T tokens); the float32 CPU oracle's outputs for a seeded
sample of sequences and prefixes were written by tests/golden/make_golden.py.  Tolerances
are the bf16 ones: |dlogp| <= 5e-2 nats, cosine(s_t) >= 0.999.
"""
from pathlib import Path

import numpy as np
import pytest
import torch

from workloads import WORKLOADS, make_tokens, make_weights
from gpu_util import build_model, cosine, to_np

pytestmark = pytest.mark.gpu

GOLDEN = Path(__file__).resolve().parent / "golden"
LP_TOL, COS_MIN = 5e-2, 0.999


def golden(workload: str, tag: str) -> dict:
    f = GOLDEN / f"oracle_{workload}_{tag}.npz"
    if not f.exists():
        pytest.fail(f"missing golden file {f.name}: run tests/golden/make_golden.py")
    return dict(np.load(f))


def run_prefix(wl, steps: int, s_idx):
    """Whole batch, e/M over all T tokens, `steps` decoder steps; returns per-step log-prob of the
    next token and LSE [B, steps] and s_t [B, len(s_idx), d] at the 1-based steps s_idx."""
    m = wl.model
    model = build_model(m, max_pos=wl.T, weights=make_weights(m, wl.weight_seed))
    tok = torch.from_numpy(make_tokens(wl)).cuda()
    e, M = model.encode(tok)
    torch.cuda.synchronize()
    model.release_workspaces()
    B = wl.B
    st = model.new_state(B)
    tok_tb = tok.t().contiguous()
    lp = torch.zeros((steps, B), device="cuda")
    lse = torch.zeros((steps, B), device="cuda")
    s_keep = []
    want = set(int(i) for i in s_idx)
    for t in range(steps):
        nxt = t + 1 < wl.T
        model.decode_step(st, e, M, next_tok=tok_tb[t + 1] if nxt else None, tau=wl.tau,
                          logp_tok=lp[t] if nxt else None, lse=lse[t])
        if t + 1 in want:
            s_keep.append(st.s().clone())
    torch.cuda.synchronize()
    assert model.last_error() == 0
    return to_np(lp.t()), to_np(lse.t()), np.stack([to_np(x) for x in s_keep], 1)


def compare(g: dict, lp, lse, s):
    seqs = g["seqs"]
    steps = int(g["steps"])
    d_lp = np.abs(lp[seqs, : steps - 1] - g["logp_tok"][:, : steps - 1]).max()
    d_lse = np.abs(lse[seqs, :steps] - g["lse"]).max()
    cos = cosine(s[seqs], g["s"]).min()
    assert d_lp <= LP_TOL, d_lp
    assert d_lse <= LP_TOL, d_lse
    assert cos >= COS_MIN, cos
    return d_lp, d_lse, cos


def test_300m_b512_sampled_sequences_first_256_steps():
    wl = WORKLOADS["300m-12+12-b512"]
    g = golden(wl.name, "4x256")
    lp, lse, s = run_prefix(wl, int(g["steps"]), g["s_idx"])
    compare(g, lp, lse, s)


def test_300m_b512_one_sequence_full_length():
    wl = WORKLOADS["300m-12+12-b512"]
    g = golden(wl.name, "1x1024")
    lp, lse, s = run_prefix(wl, int(g["steps"]), g["s_idx"])
    compare(g, lp, lse, s)


def test_48_48_b32_sampled_sequences_first_256_steps():
    wl = WORKLOADS["ref-48+48-b32"]
    g = golden(wl.name, "2x256")
    lp, lse, s = run_prefix(wl, int(g["steps"]), g["s_idx"])
    compare(g, lp, lse, s)


def test_48_48_b1_latency_run_first_256_steps():
    """The single-sequence decode of the 48+48 model (few-row GEMMs with K split over CTA
    clusters, cross-attention split along keys) against sequence 0 of the B=32 oracle outputs:
    the B=1 run draws the same first sequence of the same token stream."""
    wl = WORKLOADS["ref-48+48-b1"]
    g = golden("ref-48+48-b32", "2x256")
    assert int(g["seqs"][0]) == 0
    g0 = {k: (v[:1] if k in ("seqs", "logp_tok", "lse", "s", "score") else v) for k, v in g.items()}
    lp, lse, s = run_prefix(wl, int(g0["steps"]), g0["s_idx"])
    compare(g0, lp, lse, s)


def test_replay_24_24_scores_and_per_token_log_probs():
    """rlt_replay over the whole B=64 x 2048 batch at tau 0.8: per-token log-probs of the sampled
    sequences match the oracle (first 256 tokens of four sequences, all 2048 of two), and so do
    their response scores."""
    wl = WORKLOADS["replay-24+24-b64"]
    g_short = golden(wl.name, "4x256")
    g_long = golden(wl.name, "2x2048")
    m = wl.model
    model = build_model(m, max_pos=wl.T, weights=make_weights(m, wl.weight_seed))
    tok = torch.from_numpy(make_tokens(wl)).cuda()
    score, lp, _ = model.replay(tok, wl.prompt_len, wl.tau, want_logp=True)
    torch.cuda.synchronize()
    assert model.last_error() == 0
    lp = to_np(lp)
    for g in (g_short, g_long):
        seqs, steps = g["seqs"], int(g["steps"])
        assert np.abs(lp[seqs, : steps - 1] - g["logp_tok"][:, : steps - 1]).max() <= LP_TOL
    # The score is the float32 sum of the n = T - P scored per-token log-probs (entries P-1 ..
    # T-2).  It can differ from the oracle's by at most the summed per-token differences plus
    # the rounding of the two float32 summations, each within gamma_n * sum|logp| (gamma_n =
    # n u / (1 - n u), u = 2^-24: the standard bound for a recursive sum).
    ref = g_long["score"]
    got = to_np(score)[g_long["seqs"]]
    P, T = wl.prompt_len, wl.T
    n = T - P
    lp_g, lp_r = lp[g_long["seqs"], P - 1:T - 1], g_long["logp_tok"][:, P - 1:T - 1].astype(np.float64)
    u = 2.0 ** -24
    gamma = n * u / (1 - n * u)
    bound = np.abs(lp_g - lp_r).sum(-1) + gamma * (np.abs(lp_g).sum(-1) + np.abs(lp_r).sum(-1))
    assert np.all(np.abs(got - ref) <= bound), (got, ref, bound)
    # and the score is the sum of the log-probs the same call returned
    assert np.all(np.abs(got - lp_g.astype(np.float64).sum(-1)) <= gamma * np.abs(lp_g).sum(-1))
