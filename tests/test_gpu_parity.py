"""GPU path vs the CPU oracle on identical seeded inputs, through the C ABI.

Tolerances: float32 models max|ds_t| <= 1e-4 and |dlogp| <= 1e-4; bf16 models
|dlogp| <= 5e-2 nats and cosine(s_t) >= 0.999.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from cross_token_latent_b200 import RLTError
from oracle import RLTOracle
from workloads import TINY, SMALL, make_tokens, make_weights
from gpu_util import build_model, cosine, gpu_run, to_np

pytestmark = pytest.mark.gpu

F32_S_TOL, F32_LP_TOL = 1e-4, 1e-4
BF16_LP_TOL, BF16_COS_MIN = 5e-2, 0.999


def m_layout(M_gpu: torch.Tensor, T: int) -> np.ndarray:
    """[G, 2, B, H, T_alloc, hd] -> [G, 2, B, T, d] like the oracle."""
    G, two, B, H, Ta, hd = M_gpu.shape
    return to_np(M_gpu[:, :, :, :, :T].permute(0, 1, 2, 4, 3, 5).reshape(G, 2, B, T, H * hd))


def check(cfg, s_gpu, lp_gpu, s_ref, lp_ref, lp_tok_gpu=None, lp_tok_ref=None):
    if cfg.dtype == "f32":
        assert np.abs(s_gpu - s_ref).max() <= F32_S_TOL
        assert np.abs(lp_gpu - lp_ref).max() <= F32_LP_TOL
    else:
        assert cosine(s_gpu, s_ref).min() >= BF16_COS_MIN
        assert np.abs(lp_gpu - lp_ref).max() <= BF16_LP_TOL
    if lp_tok_gpu is not None:
        tol = F32_LP_TOL if cfg.dtype == "f32" else BF16_LP_TOL
        assert np.abs(lp_tok_gpu - lp_tok_ref).max() <= tol


# ------------------------------------------------------------------ tiny float32 workload

@pytest.fixture(scope="module")
def tiny():
    cfg = TINY.model
    w = make_weights(cfg)
    tok = make_tokens(TINY)
    model = build_model(cfg, max_pos=TINY.T, weights=w)
    ora = RLTOracle(cfg, w)
    e_r, M_r, s_r, lp_r = ora.run(tok)
    return cfg, w, tok, model, ora, (e_r, M_r, s_r, lp_r)


def test_tiny_encoder_parity(tiny):
    cfg, w, tok, model, ora, (e_r, M_r, _, _) = tiny
    e, M = model.encode(torch.from_numpy(tok).cuda())
    assert np.abs(to_np(e) - e_r).max() <= 1e-5
    assert np.abs(m_layout(M, tok.shape[1]) - M_r).max() <= 1e-5


def test_tiny_decode_parity_every_step(tiny):
    cfg, w, tok, model, ora, (_, _, s_r, lp_r) = tiny
    _, _, s, lp, lp_tok, st = gpu_run(model, tok)
    check(cfg, s, lp, s_r, lp_r)
    B, T = tok.shape
    ref_tok = np.array([[lp_r[b, t, tok[b, t + 1]] for t in range(T - 1)] for b in range(B)])
    assert np.abs(lp_tok[:, :-1] - ref_tok).max() <= F32_LP_TOL
    assert st.position == T


def test_tiny_replay_parity_and_incremental_equality(tiny):
    cfg, w, tok, model, ora, _ = tiny
    score_r, lp_tok_r, s_r, _ = ora.replay(tok, TINY.prompt_len, 1.0)
    score, lp_tok, st = model.replay(torch.from_numpy(tok).cuda(), TINY.prompt_len, 1.0, want_logp=True,
                                     want_state=True)
    torch.cuda.synchronize()
    assert np.abs(to_np(lp_tok) - lp_tok_r).max() <= F32_LP_TOL
    assert np.abs(to_np(score) - score_r).max() <= F32_LP_TOL * TINY.T
    assert np.abs(to_np(st.s()) - s_r[:, -1]).max() <= F32_S_TOL
    # one transition for prefill and replay: stepping equals the replay bit for bit
    _, _, s_step, _, lp_step, _ = gpu_run(model, tok, full=False)
    np.testing.assert_array_equal(lp_step, to_np(lp_tok))
    np.testing.assert_array_equal(s_step[:, -1], to_np(st.s()))


def test_gpu_proposition_3_1(tiny):
    cfg, w, tok, model, ora, _ = tiny
    tt = torch.from_numpy(tok).cuda()
    s24, lp24, _ = model.replay(tt, 24, 1.0, want_logp=True)
    for P in (8, 40):
        s, lp, _ = model.replay(tt, P, 1.0, want_logp=True)
        np.testing.assert_array_equal(to_np(lp), to_np(lp24))
        lo, hi = sorted((P, 24))
        moved = to_np(lp24)[:, lo - 1:hi - 1].sum(-1)
        np.testing.assert_allclose(to_np(s) - to_np(s24), moved if P < 24 else -moved, atol=1e-3)


def test_temperature_and_lse(tiny):
    cfg, w, tok, model, ora, _ = tiny
    tt = torch.from_numpy(tok).cuda()
    e, M = model.encode(tt)
    st = model.new_state(2)
    lse = torch.empty(2, device="cuda")
    full = torch.empty(2, cfg.V, device="cuda")
    gat = torch.empty(2, device="cuda")
    nxt = tt[:, 1].contiguous()
    model.decode_step(st, e, M, next_tok=nxt, tau=0.8, logp_tok=gat, lse=lse, logp_full=full)
    _, _, _, lp_r = ora.run(tok[:, :1], tau=0.8)
    lp = to_np(full)
    assert np.abs(lp - lp_r[:, 0]).max() <= F32_LP_TOL
    np.testing.assert_allclose(np.exp(lp).sum(-1), 1.0, atol=1e-5)
    np.testing.assert_array_equal(to_np(gat), lp[np.arange(2), tok[:, 1]])


# ------------------------------------------------------------------ shape variants (ragged, edge cases)

VARIANTS = {
    "W1": dict(W=1),
    "W_ge_T": dict(W=64),
    "W7_G2": dict(W=7, G=2),
    "hd32": dict(n_heads=2, head_dim=32),
    "hd64": dict(n_heads=1, head_dim=64),
    "hd128": dict(d=128, n_heads=1, head_dim=128, F=384),
    "bf16": dict(dtype="bf16"),
    "bf16_hd64_W5": dict(dtype="bf16", n_heads=1, head_dim=64, W=5),
    "bf16_hd16_G2": dict(dtype="bf16", G=2, W=3),
    "bf16_hd128": dict(dtype="bf16", d=128, n_heads=1, head_dim=128, F=384, W=9),
    # d not a multiple of 64: the decoder's sublayer norms run as kernels of their own instead
    # of being deferred into the projections
    "bf16_d96_norm_kernels": dict(dtype="bf16", d=96, n_heads=3, head_dim=32, F=256, W=4),
}


@pytest.mark.parametrize("name", list(VARIANTS))
@pytest.mark.parametrize("B,T", [(3, 37), (1, 70)])
def test_variant_parity(name, B, T):
    cfg = replace(TINY.model, **VARIANTS[name])
    w = make_weights(cfg, seed=7)
    tok = np.random.default_rng([11, B, T]).integers(0, cfg.V, size=(B, T)).astype(np.int32)
    model = build_model(cfg, max_pos=T + 5, weights=w)
    _, _, s, lp, lp_tok, _ = gpu_run(model, tok, tau=0.9, T_alloc=T + 3)
    _, _, s_r, lp_r = RLTOracle(cfg, w).run(tok, tau=0.9)
    check(cfg, s, lp, s_r, lp_r)


@pytest.mark.parametrize("hd,T", [(64, 300), (128, 300), (64, 129), (128, 257)])
def test_tensor_core_encoder_attention_over_several_key_tiles(hd, T):
    """bf16 head_dim 64/128 encoders run causal attention on the tensor cores in 128x128 tiles:
    several query and key tiles, ragged last tiles, online rescaling across tiles."""
    cfg = replace(TINY.model, dtype="bf16", d=128, n_heads=128 // hd, head_dim=hd, F=256, W=6)
    w = make_weights(cfg, seed=5)
    tok = np.random.default_rng([13, hd, T]).integers(0, cfg.V, size=(2, T)).astype(np.int32)
    model = build_model(cfg, max_pos=T, weights=w)
    e_r, M_r = RLTOracle(cfg, w).encode(tok)
    e, M = model.encode(torch.from_numpy(tok).cuda())
    assert cosine(to_np(e), e_r).min() >= 0.999
    assert cosine(m_layout(M, T), M_r).min() >= 0.999
    steps = 40 if T > 200 else T
    _, _, s, lp, _, _ = gpu_run(model, tok, steps=steps)
    _, _, s_r, lp_r = RLTOracle(cfg, w).run(tok, steps=steps)
    check(cfg, s, lp, s_r, lp_r)


# ------------------------------------------------------------------ small bf16 workload (full batch)

def test_small_bf16_parity_full_batch():
    cfg = SMALL.model
    w = make_weights(cfg)
    tok = make_tokens(SMALL)                           # 64 x 512
    model = build_model(cfg, max_pos=SMALL.T, weights=w)
    _, _, s, _, lp_tok, _ = gpu_run(model, tok, full=False)
    sample = [0, 1, 17, 63]
    _, lp_tok_r, s_r, _ = RLTOracle(cfg, w).replay(tok[sample], SMALL.prompt_len, 1.0)
    assert cosine(s[sample], s_r).min() >= BF16_COS_MIN
    assert np.abs(lp_tok[sample][:, :-1] - lp_tok_r[:, :-1]).max() <= BF16_LP_TOL
    # replay score of the whole batch vs the oracle on the sample
    score, _, _ = model.replay(torch.from_numpy(tok).cuda(), SMALL.prompt_len, 1.0)
    score_r = lp_tok_r[:, SMALL.prompt_len - 1:-1].sum(-1)
    assert np.abs(to_np(score)[sample] - score_r).max() <= BF16_LP_TOL * 4


@pytest.mark.parametrize("B", [259, 256])
def test_large_ragged_batch_matches_the_oracle(B):
    """Batches spanning several 128-row tensor-core tiles (ragged for odd B): sampled sequences
    across the tiles match the oracle, and stepping equals replay bit for bit."""
    cfg = replace(TINY.model, dtype="bf16", W=5, G=2)
    w = make_weights(cfg, seed=3)
    T = 20
    tok = np.random.default_rng([5, B]).integers(0, cfg.V, size=(B, T)).astype(np.int32)
    model = build_model(cfg, max_pos=T, weights=w)
    _, _, s, lp, _, st = gpu_run(model, tok, tau=1.0)
    assert st.position == T
    sample = [0, 1, B // 2 - 1, B // 2, B // 2 + 1, B - 1]
    _, _, s_r, lp_r = RLTOracle(cfg, w).run(tok[sample])
    check(cfg, s[sample], lp[sample], s_r, lp_r)
    # replay over the same batch agrees with stepping
    score, lp_tok, _ = model.replay(torch.from_numpy(tok).cuda(), 8, 1.0, want_logp=True)
    _, _, _, _, lp_step, _ = gpu_run(model, tok, full=False)
    np.testing.assert_array_equal(to_np(lp_tok), lp_step)


@pytest.mark.parametrize("options", [{"row_groups": 2}, {"row_groups": 2, "group_pdl": 1, "attn_ctas_per_sm": 5},
                                     {"attn_ctas_per_sm": 3}])
def test_scheduling_options_keep_parity(options):
    """The scheduling options (two row groups on library streams, a cap on the attention CTAs
    per SM) change only summation order: sampled sequences of a 259-row batch match the oracle
    and the per-token log-probs stay within the bf16 tolerance of the default schedule."""
    cfg = replace(TINY.model, dtype="bf16", W=5, G=2)
    w = make_weights(cfg, seed=3)
    B, T = 259, 20
    tok = np.random.default_rng([5, B]).integers(0, cfg.V, size=(B, T)).astype(np.int32)
    model = build_model(cfg, max_pos=T, weights=w)
    _, _, _, _, lp_default, _ = gpu_run(model, tok, full=False)
    for k, v in options.items():
        model.set_option(k, v)
    _, _, s, lp, lp_tok, _ = gpu_run(model, tok, tau=1.0)
    assert np.abs(lp_tok - lp_default).max() <= BF16_LP_TOL
    sample = [0, 127, 128, 255, 256, 258]
    _, _, s_r, lp_r = RLTOracle(cfg, w).run(tok[sample])
    check(cfg, s[sample], lp[sample], s_r, lp_r)


@pytest.mark.parametrize("B", [40, 7])
def test_few_row_batch_matches_the_oracle_and_replays_bit_for_bit(B):
    """Batches of at most 64 rows take the swapped few-row projections (K split over clusters,
    deferred norms reduced across lanes): sampled sequences match the oracle, and stepping
    twice and replaying give identical bits."""
    cfg = replace(TINY.model, dtype="bf16", d=128, n_heads=4, head_dim=32, F=384, W=6)
    w = make_weights(cfg, seed=9)
    T = 24
    tok = np.random.default_rng([6, B]).integers(0, cfg.V, size=(B, T)).astype(np.int32)
    model = build_model(cfg, max_pos=T, weights=w)
    _, _, s, lp, lp_step, _ = gpu_run(model, tok, tau=1.0)
    sample = sorted({0, B // 2, B - 1})
    _, _, s_r, lp_r = RLTOracle(cfg, w).run(tok[sample])
    check(cfg, s[sample], lp[sample], s_r, lp_r)
    _, _, s2, _, lp_step2, _ = gpu_run(model, tok, full=False)
    np.testing.assert_array_equal(s2, s)
    np.testing.assert_array_equal(lp_step2, lp_step)
    _, lp_tok, _ = model.replay(torch.from_numpy(tok).cuda(), 8, 1.0, want_logp=True)
    np.testing.assert_array_equal(to_np(lp_tok), lp_step)


# ------------------------------------------------------------------ error handling at the boundary

def test_errors_are_reported_not_hung(tiny):
    cfg, w, tok, model, ora, _ = tiny
    tt = torch.from_numpy(tok).cuda()
    e, M = model.encode(tt)
    st = model.new_state(2)
    ws_model = model
    # out-of-range token id in the gather: latched and reported, nothing hangs
    bad = torch.tensor([5, cfg.V + 3], dtype=torch.int32, device="cuda")
    gat = torch.empty(2, device="cuda")
    ws_model.decode_step(st, e, M, next_tok=bad, logp_tok=gat)
    assert model.last_error() == 6
    assert model.last_error() == 0
    # T_alloc smaller than the next position
    with pytest.raises(RLTError) as ex:
        model.decode_step(st, e[:, :1], M[:, :, :, :, :1], logp_tok=None)
    assert ex.value.status == "RLT_EINVAL"
    # stale state after a weight update
    model.set_weight("s_star", w["s_star"])
    from cross_token_latent_b200.rlt import lib
    assert lib().rlt_model_commit(model.handle) == 0
    with pytest.raises(RLTError) as ex:
        model.decode_step(st, e, M)
    assert ex.value.status == "RLT_ESTALE"
    # an unregistered state
    other = model.new_state(2)
    raw = type(other)(model, 2, torch.empty_like(other.buf))
    with pytest.raises(RLTError) as ex:
        model.decode_step(raw, e, M)
    assert ex.value.status == "RLT_ESTATE"
    # bad encoder token ids are latched too
    model.encode(torch.full((1, 4), -1, dtype=torch.int32, device="cuda"))
    assert model.last_error() == 6


def test_state_copy_is_a_prefix_snapshot(tiny):
    cfg, w, tok, model, ora, _ = tiny
    tt = torch.from_numpy(tok).cuda()
    e, M = model.encode(tt)
    st = model.new_state(2)
    for _ in range(10):
        model.decode_step(st, e, M)
    snap = st.copy()
    full = torch.empty(2, cfg.V, device="cuda")
    model.decode_step(st, e, M, logp_full=full)
    a = full.clone()
    model.decode_step(snap, e, M, logp_full=full)
    assert snap.position == st.position == 11
    np.testing.assert_array_equal(to_np(full), to_np(a))
