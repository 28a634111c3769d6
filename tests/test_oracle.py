"""Pins of the CPU oracle against facts other than itself (no GPU needed).

Each test fixes the oracle to a closed form, an invariant the pages state, a
library routine, or a brute-force textbook pass, chosen so that a dropped term,
a wrong sign, a wrong index or a transposed operand fails at least one of them.
"""
import math
from dataclasses import replace

import numpy as np
import pytest
import scipy.special
import torch

from oracle import RLTOracle, round_bf16, rms_norm, rope, sample_token
from workloads import TINY, SMALL, make_tokens, make_weights
import parallel_ref as pref

TINY_M = TINY.model


def tiny_weights(model=TINY_M, **overrides):
    w = make_weights(model)
    for k, v in overrides.items():
        w[k] = v
    return w


def no_feedback(w):
    w = dict(w)
    w["merge_fb"] = np.zeros_like(w["merge_fb"])
    return w


# ---------------------------------------------------------------- elementary ops

def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 100000),
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0, 65504.0,
                                  3.0e38, 1e-30], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    got = round_bf16(x)
    np.testing.assert_array_equal(got, ref)
    # ties go to the even neighbour
    assert round_bf16(np.float64(1 + 2 ** -8)) == 1.0
    assert round_bf16(np.float64(1 + 3 * 2 ** -8)) == 1 + 2 ** -6


def test_rms_norm_closed_forms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 64))
    y = rms_norm(x, np.ones(64), 1e-6)
    ms = np.mean(x * x, -1)
    np.testing.assert_allclose(np.mean(y * y, -1), ms / (ms + 1e-6), rtol=1e-14)
    np.testing.assert_allclose(rms_norm(3.0 * x, np.ones(64), 0.0), rms_norm(x, np.ones(64), 0.0), rtol=1e-14)
    g = rng.standard_normal(64)
    np.testing.assert_allclose(rms_norm(x, g, 1e-6), y * g, rtol=1e-14)
    # constant vector c*1 -> sign(c) / sqrt(1 + eps/c^2)
    c = -2.5
    np.testing.assert_allclose(rms_norm(np.full(8, c), np.ones(8), 1e-6), np.full(8, np.sign(c) / np.sqrt(1 + 1e-6 / c ** 2)))


def test_rope_equals_complex_rotation_and_is_relative():
    rng = np.random.default_rng(2)
    hd, H, T = 16, 3, 7
    x = rng.standard_normal((2, T, H, hd))
    pos = np.arange(T) + 5
    got = rope(x, pos, 10000.0)
    half = hd // 2
    theta = pos[:, None] * 10000.0 ** (-np.arange(half) * 2.0 / hd)
    z = (x[..., :half] + 1j * x[..., half:]) * np.exp(1j * theta)[None, :, None, :]
    np.testing.assert_allclose(got, np.concatenate([z.real, z.imag], -1), atol=1e-13)
    # norm preserved, identity at position 0
    np.testing.assert_allclose(np.linalg.norm(got, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(rope(x, np.zeros(T, int), 10000.0), x, atol=0)
    # q(m).k(n) depends only on m - n
    q, k = rng.standard_normal((1, 1, 1, hd)), rng.standard_normal((1, 1, 1, hd))
    dots = [np.sum(rope(q, np.array([m + s]), 1e4) * rope(k, np.array([2 + s]), 1e4)) for m, s in ((9, 0), (9, 31))]
    assert abs(dots[0] - dots[1]) < 1e-12


# ---------------------------------------------------------------- encoder

@pytest.mark.parametrize("G", [1, 2])
def test_encoder_matches_textbook_causal_transformer(G):
    m = replace(TINY_M, G=G)
    w = make_weights(m)
    tok = make_tokens(TINY)[:, :20]
    e, M = RLTOracle(m, w).encode(tok)
    e_ref, M_ref = pref.encoder(m, w, tok)
    np.testing.assert_allclose(e, e_ref.numpy(), atol=1e-12)
    np.testing.assert_allclose(M, M_ref.numpy(), atol=1e-12)


def test_encoder_is_causal():
    w = make_weights(TINY_M)
    o = RLTOracle(TINY_M, w)
    tok = make_tokens(TINY)[:, :30]
    tok2 = tok.copy()
    tok2[:, 17:] = (tok2[:, 17:] + 11) % TINY_M.V
    e1, M1 = o.encode(tok)
    e2, M2 = o.encode(tok2)
    np.testing.assert_array_equal(e1[:, :17], e2[:, :17])
    assert np.abs(e1[:, 17:] - e2[:, 17:]).max() > 1e-3


# ---------------------------------------------------------------- decoder vs parallel passes

@pytest.mark.parametrize("W,G", [(64, 1), (64, 2), (4, 1), (7, 2), (1, 1)])
def test_decoder_without_feedback_equals_banded_parallel_pass(W, G):
    """Feedback zeroed: the recurrence equals a textbook parallel pass whose self-attention
    mask is causal and W wide (full causal when W >= T)."""
    m = replace(TINY_M, W=W, G=G)
    w = no_feedback(make_weights(m))
    tok = make_tokens(TINY)[:, :24]
    o = RLTOracle(m, w)
    e, M, s, lp = o.run(tok, tau=0.7)
    e_ref, M_ref = pref.encoder(m, w, tok)
    s_ref, lp_ref = pref.decoder_no_feedback(m, w, e_ref, M_ref, tau=0.7)
    np.testing.assert_allclose(s, s_ref.numpy(), atol=1e-11)
    np.testing.assert_allclose(lp, lp_ref.numpy(), atol=1e-11)


def test_parallel_swa_pass_differs_from_recurrence_with_feedback():
    """Model-hardware principle of the news summary: the standard parallel SWA decoder pass
    is not equivalent to the recurrence."""
    w = make_weights(TINY_M)
    tok = make_tokens(TINY)[:, :24]
    _, _, s, lp = RLTOracle(TINY_M, w).run(tok)
    e_ref, M_ref = pref.encoder(TINY_M, w, tok)
    s_ref, lp_ref = pref.decoder_no_feedback(TINY_M, w, e_ref, M_ref)
    assert np.abs(lp - lp_ref.numpy()).max() > 1e-3
    assert np.abs(s - s_ref.numpy()).max() > 1e-3
    # the first step has s_0 = s* but no history: it still differs through the feedback term
    assert np.abs(s[:, 0] - s_ref.numpy()[:, 0]).max() > 1e-6


def test_tokens_older_than_window_do_not_reach_layer1_swa():
    """Feedback zeroed, W < t: inputs x0_j with j <= t-W do not reach layer-1 SWA at t,
    while the oldest in-window token t-W+1 does."""
    m = replace(TINY_M, W=4)
    w = no_feedback(make_weights(m))
    o = RLTOracle(m, w)
    tok = make_tokens(TINY)[:, :12]
    e, M = o.encode(tok)
    t_probe = 10

    def layer1_swa(e_in):
        st = o.init_state(e_in.shape[0])
        for t in range(1, t_probe + 1):
            st, _, parts = o.step(st, e_in[:, t - 1], M, return_parts=True)
        return parts[0]

    base = layer1_swa(e)
    e_old = e.copy()
    e_old[:, : t_probe - m.W] += 0.5          # tokens 1 .. t-W
    np.testing.assert_array_equal(layer1_swa(e_old), base)
    e_edge = e.copy()
    e_edge[:, t_probe - m.W] += 0.5           # token t-W+1 is still in the window
    assert np.abs(layer1_swa(e_edge) - base).max() > 1e-6


def test_window_one_attends_to_self_only():
    m = replace(TINY_M, W=1)
    w = make_weights(m)
    o = RLTOracle(m, w)
    x = np.random.default_rng(3).standard_normal((2, m.d))
    st = o.init_state(2)
    out, kv = o.swa(0, x, st, t=5)
    a = rms_norm(x, w["layers.0.attn_norm"], m.rms_eps)
    np.testing.assert_allclose(out, (a @ w["layers.0.wv"].T) @ w["layers.0.wo"].T, atol=1e-12)


def test_cache_holds_the_newest_w_minus_1_entries():
    m = replace(TINY_M, W=5)
    o = RLTOracle(m, make_weights(m))
    tok = make_tokens(TINY)[:, :9]
    e, M = o.encode(tok)
    st = o.init_state(2)
    pushed = []
    for t in range(1, 10):
        new, _ = o.step(st, e[:, t - 1], M)
        pushed.append(new.cache[0][-1])
        assert len(new.cache[0]) == min(t, m.W - 1)
        for a, b in zip(new.cache[0], pushed[-(m.W - 1):]):
            np.testing.assert_array_equal(a[0], b[0])
        st = new


# ---------------------------------------------------------------- merge

@pytest.mark.filterwarnings("ignore:overflow encountered in exp")
def test_gate_limits():
    w = make_weights(TINY_M)
    rng = np.random.default_rng(4)
    e_t, s = rng.standard_normal((3, 64)), rng.standard_normal((3, 64))
    closed = RLTOracle(TINY_M, dict(w, merge_bias=np.full(64, -1e4, np.float32)))
    np.testing.assert_array_equal(closed.merge(e_t, s), e_t)
    opened = RLTOracle(TINY_M, dict(w, merge_bias=np.full(64, 1e4, np.float32)))
    # an open gate gives the additive feedback form of the teardown's minimal skeleton
    np.testing.assert_allclose(opened.merge(e_t, s), e_t + s @ w["merge_fb"].astype(np.float64).T, atol=1e-13)
    zero_fb = RLTOracle(TINY_M, no_feedback(w))
    np.testing.assert_array_equal(zero_fb.merge(e_t, s), e_t)


def _expit(x: float) -> float:
    return 1.0 / (1.0 + math.exp(-x))


def _merge_model(ge=None, gs=None, fb=None, bias=None, cls=RLTOracle):
    """TINY with chosen merge weights (others as drawn); returns (oracle, d)."""
    w = make_weights(TINY_M)
    d = TINY_M.d
    for name, val in (("merge_ge", ge), ("merge_gs", gs), ("merge_fb", fb), ("merge_bias", bias)):
        if val is not None:
            w[name] = np.asarray(val, np.float32)
    return cls(TINY_M, w), d


def test_merge_interior_gate_reads_e_and_feedback_reads_s(cls=RLTOracle):
    """Gate weights on e only (W_gs = 0), feedback the identity: x0_i = e_i + expit((W_ge e)_i) s_i,
    computed here element by element.  A gate fed s instead of e, or a feedback applied to e,
    gives different values."""
    rng = np.random.default_rng(11)
    d = TINY_M.d
    ge = rng.standard_normal((d, d)) * 0.3
    o, _ = _merge_model(ge=ge, gs=np.zeros((d, d)), fb=np.eye(d), bias=np.zeros(d), cls=cls)
    e_t, s = rng.standard_normal((2, d)), rng.standard_normal((2, d))
    got = o.merge(e_t, s)
    ge32 = ge.astype(np.float32).astype(np.float64)
    for b in range(2):
        for i in range(d):
            pre = sum(ge32[i, j] * e_t[b, j] for j in range(d))
            assert abs(got[b, i] - (e_t[b, i] + _expit(pre) * s[b, i])) < 1e-12


def test_merge_interior_state_gate_and_feedback_projection(cls=RLTOracle):
    """W_ge = 0: x0_i = e_i + expit((W_gs s)_i + b_i) (W_fb s)_i with a nonzero bias and a dense
    W_fb, element by element.  A bias outside the sigmoid or dropped, or W_fb applied to e,
    gives different values."""
    rng = np.random.default_rng(12)
    d = TINY_M.d
    gs = rng.standard_normal((d, d)) * 0.3
    fb = rng.standard_normal((d, d)) * 0.3
    bias = rng.standard_normal(d)
    o, _ = _merge_model(ge=np.zeros((d, d)), gs=gs, fb=fb, bias=bias, cls=cls)
    e_t, s = rng.standard_normal((2, d)), rng.standard_normal((2, d))
    got = o.merge(e_t, s)
    gs32, fb32, b32 = (a.astype(np.float32).astype(np.float64) for a in (gs, fb, bias))
    for b in range(2):
        for i in range(d):
            g = _expit(sum(gs32[i, j] * s[b, j] for j in range(d)) + b32[i])
            u = sum(fb32[i, j] * s[b, j] for j in range(d))
            assert abs(got[b, i] - (e_t[b, i] + g * u)) < 1e-12


def test_merge_interior_single_entry_weights_fix_every_index(cls=RLTOracle):
    """One nonzero entry per merge matrix pins which input component reaches which output:
    W_ge[0, 1] = 2, W_gs[0, 2] = -1, W_fb[0, 3] = 1.5, bias b_0 = log 3 (so the gate of an
    all-zero pre-activation is 3/4).  Output 0 is e_0 + expit(2 e_1 - s_2 + log 3) * 1.5 s_3;
    every other output i has gate expit(b_i) = 1/2 times a zero feedback, i.e. e_i.  A
    transposed operand moves the nonzero terms to other components."""
    d = TINY_M.d
    ge, gs, fb = np.zeros((d, d)), np.zeros((d, d)), np.zeros((d, d))
    ge[0, 1], gs[0, 2], fb[0, 3] = 2.0, -1.0, 1.5
    bias = np.zeros(d)
    bias[0] = math.log(3.0)
    o, _ = _merge_model(ge=ge, gs=gs, fb=fb, bias=bias, cls=cls)
    rng = np.random.default_rng(13)
    e_t, s = rng.standard_normal((3, d)), rng.standard_normal((3, d))
    got = o.merge(e_t, s)
    b0 = float(np.float32(math.log(3.0)))
    for b in range(3):
        want0 = e_t[b, 0] + _expit(2.0 * e_t[b, 1] - s[b, 2] + b0) * 1.5 * s[b, 3]
        assert abs(got[b, 0] - want0) < 1e-12
        np.testing.assert_array_equal(got[b, 1:], e_t[b, 1:])
    # with every weight zero the gate is expit(b_0) = 3/4 on a zero feedback: x0 = e
    o0, _ = _merge_model(ge=np.zeros((d, d)), gs=np.zeros((d, d)), fb=np.eye(d), bias=bias, cls=cls)
    got0 = o0.merge(e_t, s)
    np.testing.assert_allclose(got0[:, 0], e_t[:, 0] + 0.75 * s[:, 0], atol=1e-7)
    np.testing.assert_allclose(got0[:, 1:], e_t[:, 1:] + 0.5 * s[:, 1:], atol=1e-15)


class _SwappedGateInputs(RLTOracle):       # s_{t-1} fed to W_ge and e_t to W_gs
    def merge(self, e_t, s_prev):
        s_in = self.rnd(s_prev)
        g = 1 / (1 + np.exp(-(s_in @ self.w["merge_ge"].T + e_t @ self.w["merge_gs"].T + self.w["merge_bias"])))
        return e_t + g * (s_in @ self.w["merge_fb"].T)


class _FeedbackOnE(RLTOracle):             # W_fb applied to e_t
    def merge(self, e_t, s_prev):
        s_in = self.rnd(s_prev)
        g = 1 / (1 + np.exp(-(e_t @ self.w["merge_ge"].T + s_in @ self.w["merge_gs"].T + self.w["merge_bias"])))
        return e_t + g * (e_t @ self.w["merge_fb"].T)


class _BiasOutsideGate(RLTOracle):         # b_g added after the sigmoid
    def merge(self, e_t, s_prev):
        s_in = self.rnd(s_prev)
        g = 1 / (1 + np.exp(-(e_t @ self.w["merge_ge"].T + s_in @ self.w["merge_gs"].T))) + self.w["merge_bias"]
        return e_t + g * (s_in @ self.w["merge_fb"].T)


class _TransposedFeedback(RLTOracle):      # W_fb^T instead of W_fb
    def merge(self, e_t, s_prev):
        s_in = self.rnd(s_prev)
        g = 1 / (1 + np.exp(-(e_t @ self.w["merge_ge"].T + s_in @ self.w["merge_gs"].T + self.w["merge_bias"])))
        return e_t + g * (s_in @ self.w["merge_fb"])


@pytest.mark.parametrize("wrong", [_SwappedGateInputs, _FeedbackOnE, _BiasOutsideGate, _TransposedFeedback])
def test_merge_pins_catch_planted_mistakes(wrong):
    """Each plausible mistake, planted in a copy of the oracle, fails at least one merge pin."""
    failed = 0
    for pin in (test_merge_interior_gate_reads_e_and_feedback_reads_s,
                test_merge_interior_state_gate_and_feedback_projection,
                test_merge_interior_single_entry_weights_fix_every_index):
        try:
            pin(cls=wrong)
        except AssertionError:
            failed += 1
    assert failed >= 1


# ---------------------------------------------------------------- head

def test_head_is_log_softmax_at_temperature():
    w = make_weights(TINY_M)
    o = RLTOracle(TINY_M, w)
    s = np.random.default_rng(5).standard_normal((4, 64))
    for tau in (1.0, 0.8, 3.0):
        lp = o.head(s, tau)
        z = s @ w["unembed"].astype(np.float64).T
        np.testing.assert_allclose(lp, scipy.special.log_softmax(z / tau, axis=-1), atol=1e-12)
        np.testing.assert_allclose(np.exp(lp).sum(-1), 1.0, atol=1e-12)
    # infinite temperature -> uniform
    np.testing.assert_allclose(o.head(s, 1e12), -np.log(TINY_M.V), atol=1e-9)


# ---------------------------------------------------------------- sampler (reading R12)

def _lp(p):
    return np.log(np.asarray(p, np.float64))


def test_sampler_inverse_cdf_on_a_known_distribution():
    """p = (0.1, 0.2, 0.3, 0.4): the CDF in id order is 0.1, 0.3, 0.6, 1.0, so u picks the first
    id whose cumulative mass exceeds u; the behaviour log-prob is log p."""
    lp = _lp([0.1, 0.2, 0.3, 0.4])
    for u, want in ((0.0, 0), (0.05, 0), (0.11, 1), (0.29, 1), (0.31, 2), (0.59, 2), (0.61, 3), (0.999, 3)):
        tok, blp = sample_token(lp, u)
        assert tok == want, (u, tok)
        assert blp == pytest.approx(math.log([0.1, 0.2, 0.3, 0.4][want]), abs=1e-12)


def test_sampler_top_k_and_top_p_renormalise_the_kept_tokens():
    lp = _lp([0.1, 0.2, 0.3, 0.4])
    # top-k 2 keeps ids 2, 3 (0.3, 0.4): renormalised CDF 3/7, 1
    assert sample_token(lp, 0.42, top_k=2) == (2, pytest.approx(math.log(3 / 7), abs=1e-12))
    assert sample_token(lp, 0.43, top_k=2) == (3, pytest.approx(math.log(4 / 7), abs=1e-12))
    # top-p 0.5: id 3 has no more-probable mass, id 2 has 0.4 < 0.5, id 1 has 0.7: kept {2, 3}
    assert sample_token(lp, 0.0, top_p=0.5)[0] == 2
    assert sample_token(lp, 0.9, top_p=0.5) == (3, pytest.approx(math.log(4 / 7), abs=1e-12))
    # top-p 0.4: id 2 has exactly 0.4 more-probable mass, not below 0.4: only id 3 is kept
    assert sample_token(lp, 0.0, top_p=0.4) == (3, pytest.approx(0.0, abs=1e-12))
    # top-k 3 then top-p 0.5 of the kept mass 0.9: ids 3 (0 < 0.45), 2 (0.4 < 0.45), 1 (0.7): {2, 3}
    assert sample_token(lp, 0.0, top_k=3, top_p=0.5)[0] == 2
    # top-k 3 then top-p 0.4 of 0.9 = 0.36: id 2 has 0.4 >= 0.36: only id 3
    assert sample_token(lp, 0.0, top_k=3, top_p=0.4)[0] == 3


def test_sampler_keeps_every_token_tied_at_the_boundary():
    lp = _lp([0.25, 0.25, 0.25, 0.25])
    # top-k 1: no token has a strictly more probable one, so all four stay: uniform
    assert [sample_token(lp, u, top_k=1)[0] for u in (0.1, 0.3, 0.6, 0.9)] == [0, 1, 2, 3]
    assert sample_token(lp, 0.3, top_k=1)[1] == pytest.approx(math.log(0.25), abs=1e-12)
    lp2 = _lp([0.1, 0.3, 0.3, 0.3])
    # top-k 2: the three 0.3 ties stay, 0.1 goes (three tokens are more probable than it)
    assert sample_token(lp2, 0.0, top_k=2)[0] == 1
    assert sample_token(lp2, 0.0, top_k=2)[1] == pytest.approx(math.log(1 / 3), abs=1e-12)


def test_sampler_frequencies_match_the_truncated_distribution():
    """Over 20000 evenly spaced uniforms the token counts equal the kept probabilities
    (renormalised) within one count per token."""
    rng = np.random.default_rng(21)
    z = rng.standard_normal(40) * 2
    lp = z - scipy.special.logsumexp(z)
    p = np.exp(lp)
    order = np.argsort(-p)
    kept = np.zeros(40, bool)
    kept[order[:7]] = True                       # top-k 7 (no ties in a continuous draw)
    n = 20000
    counts = np.zeros(40)
    for j in range(n):
        counts[sample_token(lp, (j + 0.5) / n, top_k=7)[0]] += 1
    want = np.where(kept, p, 0) / p[kept].sum() * n
    assert np.all(np.abs(counts - want) <= 1.0 + 1e-9)


def _sample_by_definition(logp, u, top_k=0, top_p=1.0):
    """Reading R12 written out token by token (quadratic; tiny vocabularies only)."""
    p = np.exp(np.asarray(logp, np.float64))
    V = len(p)
    keep = [top_k <= 0 or sum(1 for j in range(V) if p[j] > p[i]) < top_k for i in range(V)]
    if top_p < 1.0:
        z1 = sum(p[i] for i in range(V) if keep[i])
        keep = [keep[i] and sum(p[j] for j in range(V) if keep[j] and p[j] > p[i]) < top_p * z1 for i in range(V)]
    z = sum(p[i] for i in range(V) if keep[i])
    acc, last = 0.0, -1
    for i in range(V):
        if keep[i]:
            acc += p[i]
            last = i
            if acc > u * z:
                return i, math.log(p[i] / z)
    return last, math.log(p[last] / z)


def test_sampler_equals_its_definition_by_brute_force():
    """400 random small rows (a third with exact ties), random top-k / top-p / uniform."""
    rng = np.random.default_rng(22)
    for trial in range(400):
        V = int(rng.integers(2, 40))
        z = rng.standard_normal(V) * rng.uniform(0.3, 3)
        if trial % 3 == 0:
            z = np.round(z * 2) / 2
        lp = z - scipy.special.logsumexp(z)
        u = float(rng.random())
        k = int(rng.integers(0, V + 2)) if trial % 2 else 0
        tp = float(rng.uniform(0.05, 1.0)) if trial % 4 < 2 else 1.0
        tok, blp = sample_token(lp, u, k, tp)
        want_tok, want_blp = _sample_by_definition(lp, u, k, tp)
        assert tok == want_tok, (trial, tok, want_tok)
        assert blp == pytest.approx(want_blp, abs=1e-12)


# ---------------------------------------------------------------- replay contract

@pytest.fixture(scope="module")
def tiny_replay():
    w = make_weights(TINY_M)
    o = RLTOracle(TINY_M, w)
    tok = make_tokens(TINY)
    return o, tok, o.replay(tok, TINY.prompt_len, 1.0)


def test_replay_rms_and_normalisation(tiny_replay):
    o, tok, (score, lp_tok, s, _) = tiny_replay
    ms = np.mean(s * s, -1)                      # = mean(x^2) / (mean(x^2) + eps) with unit gains
    assert np.all(ms < 1.0) and np.all(ms > 1.0 - 1e-4)
    assert np.all(lp_tok[:, :-1] < 0) and np.all(lp_tok[:, -1] == 0)


def test_incremental_encoding_equals_replay(tiny_replay):
    """One transition serves prefill, generation and replay: stepping with e and M from a
    per-token recomputation of the causal encoder equals the full replay."""
    o, tok, (score, lp_tok, s, _) = tiny_replay
    B, T = tok.shape
    st = o.init_state(B)
    for t in range(1, T + 1):
        e, M = o.encode(tok[:, :t])
        st, lp = o.step(st, e[:, t - 1], M)
        np.testing.assert_allclose(st.s, s[:, t - 1], atol=1e-12)
        if t < T:
            np.testing.assert_allclose(lp[np.arange(B), tok[:, t]], lp_tok[:, t - 1], atol=1e-12)


def test_proposition_3_1_split_invariance(tiny_replay):
    """Moving the prompt/response split leaves every per-token output unchanged; the scores
    differ exactly by the moved terms."""
    o, tok, (score24, lp24, s24, _) = tiny_replay
    for P in (8, 40, 1, 64):
        score, lp, s, _ = o.replay(tok, P, 1.0)
        np.testing.assert_array_equal(lp, lp24)
        np.testing.assert_array_equal(s, s24)
        lo, hi = sorted((P, 24))
        moved = lp24[:, lo - 1:hi - 1].sum(-1)
        np.testing.assert_allclose(score - score24, moved if P < 24 else -moved, atol=1e-10)


def test_replay_score_sums_response_log_probs(tiny_replay):
    o, tok, (score, lp_tok, s, _) = tiny_replay
    _, _, s_run, lp_run = o.run(tok)
    B, T = tok.shape
    expect = np.zeros(B)
    for b in range(B):
        for i in range(TINY.prompt_len + 1, T + 1):        # response tokens x_{P+1..T}, 1-based
            expect[b] += lp_run[b, i - 2, tok[b, i - 1]]
    np.testing.assert_allclose(score, expect, atol=1e-10)
    np.testing.assert_array_equal(s_run, s)


def test_future_tokens_do_not_change_the_past(tiny_replay):
    o, tok, (score, lp_tok, s, _) = tiny_replay
    tok2 = tok.copy()
    tok2[:, 40:] = (tok2[:, 40:] * 7 + 3) % TINY_M.V
    _, lp2, s2, _ = o.replay(tok2, TINY.prompt_len, 1.0)
    np.testing.assert_array_equal(s2[:, :40], s[:, :40])
    np.testing.assert_array_equal(lp2[:, :39], lp_tok[:, :39])
    assert np.abs(s2[:, 40:] - s[:, 40:]).max() > 1e-4


def test_no_reset_at_the_prompt_boundary(tiny_replay):
    """The state after the prompt is carried into the response: resetting it to H_0 at the
    boundary changes the response log-probs."""
    o, tok, (score, lp_tok, s, _) = tiny_replay
    from oracle import DecoderState
    P = TINY.prompt_len
    e, M = o.encode(tok)
    fresh = o.init_state(2)
    st = DecoderState(s=fresh.s, cache=fresh.cache, t=P)   # s and caches reset, position kept
    for t in range(P + 1, P + 4):
        st = o.step(st, e[:, t - 1], M)[0]
    assert np.abs(st.s - s[:, P + 2]).max() > 1e-3


# ---------------------------------------------------------------- precision

def test_float32_oracle_agrees_with_float64():
    w = make_weights(TINY_M)
    tok = make_tokens(TINY)
    s64 = RLTOracle(TINY_M, w, np.float64).replay(tok, 24)[2]
    s32 = RLTOracle(TINY_M, w, np.float32).replay(tok, 24)[2]
    assert np.abs(s64 - s32).max() < 1e-5


def test_bf16_storage_contract_values_are_representable():
    m = SMALL.model
    o = RLTOracle(m, make_weights(m))
    tok = make_tokens(SMALL, range(2))[:, :20]
    e, M = o.encode(tok)
    np.testing.assert_array_equal(round_bf16(e), e)
    np.testing.assert_array_equal(round_bf16(M), M)
    st = o.init_state(2)
    for t in range(1, 6):
        st, lp = o.step(st, e[:, t - 1], M)
    for k, v in st.cache[2]:
        np.testing.assert_array_equal(round_bf16(k), k)
        np.testing.assert_array_equal(round_bf16(v), v)
    for k in ("layers.1.wq", "unembed", "s_star"):
        np.testing.assert_array_equal(round_bf16(o.w[k]), o.w[k])
    assert not np.array_equal(round_bf16(st.s), st.s)      # s_t itself stays full precision
