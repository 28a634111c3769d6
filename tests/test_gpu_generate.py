"""The generation loop on the GPU against the CPU oracle, through the C ABI: the sampler
(rlt_sample), incremental encoding (rlt_encode_prefill / rlt_encode_append) and the whole loop
(sample x_{t+1} from logp_t, encode it, step).

A sampled token is an integer decided by floating point: where the GPU's and the oracle's
cumulative sums differ by rounding, a uniform that falls within a hair of a CDF boundary may
legitimately pick either neighbour.  A draw is therefore accepted when it is what the oracle
draws at u, u - delta or u + delta.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from oracle import RLTOracle, sample_token
from workloads import TINY, SMALL, make_tokens, make_weights
from gpu_util import build_model, cosine, gpu_run, to_np

pytestmark = pytest.mark.gpu


def valid_draw(lp_row, u, top_k, top_p, tok, delta):
    return tok in {sample_token(lp_row, min(max(x, 0.0), 1.0 - 1e-12), top_k, top_p)[0]
                   for x in (u, u - delta, u + delta)}


def log_softmax32(z):
    z = z.astype(np.float64)
    z = z - z.max(-1, keepdims=True)
    return (z - np.log(np.exp(z).sum(-1, keepdims=True))).astype(np.float32)


SAMPLER_CASES = [
    # V, top_k, top_p, logit scale, quantised logits (ties)
    (512, 0, 1.0, 3.0, False),
    (512, 20, 1.0, 3.0, False),
    (512, 0, 0.9, 3.0, False),
    (512, 50, 0.8, 2.0, False),
    (512, 7, 1.0, 1.0, True),
    (512, 0, 0.5, 1.0, True),
    (32000, 0, 1.0, 4.0, False),
    (32000, 40, 0.95, 4.0, False),
    (32000, 0, 0.9, 2.0, False),
]


@pytest.mark.parametrize("V,top_k,top_p,scale,ties", SAMPLER_CASES)
def test_sampler_matches_the_oracle(V, top_k, top_p, scale, ties):
    cfg = replace(TINY.model, V=V)
    model = build_model(cfg, max_pos=8)
    rng = np.random.default_rng([31, V, top_k])
    B = 48
    z = rng.standard_normal((B, V)) * scale
    if ties:
        z = np.round(z * 2) / 2                    # many exactly equal logits
    lp = log_softmax32(z)
    u = rng.random(B).astype(np.float32)
    u[:4] = [0.0, 0.5, 0.999, 0.25]
    tok = torch.empty(B, dtype=torch.int32, device="cuda")
    blp = torch.empty(B, dtype=torch.float32, device="cuda")
    model.sample(torch.from_numpy(lp).cuda(), torch.from_numpy(u).cuda(), top_k, top_p, out=tok, behaviour_logp=blp)
    torch.cuda.synchronize()
    assert model.last_error() == 0
    tok, blp = tok.cpu().numpy(), to_np(blp)
    same = 0
    for b in range(B):
        ref_tok, ref_blp = sample_token(lp[b], float(u[b]), top_k, top_p)
        assert valid_draw(lp[b], float(u[b]), top_k, top_p, int(tok[b]), 1e-6), (b, tok[b], ref_tok)
        if tok[b] == ref_tok:
            same += 1
            assert abs(blp[b] - ref_blp) <= 1e-5, (b, blp[b], ref_blp)
    assert same >= B - 1


ENC_CASES = {
    "tiny-f32": (TINY.model, 2, 20, 44),
    "small-bf16": (SMALL.model, 8, 100, 140),
    "hd64-bf16": (replace(TINY.model, dtype="bf16", d=256, n_heads=4, head_dim=64, F=512, W=8), 5, 30, 150),
    "hd128-bf16-G2": (replace(TINY.model, dtype="bf16", d=256, n_heads=2, head_dim=128, F=512, W=8, G=2), 3, 1, 40),
}


@pytest.mark.parametrize("name", list(ENC_CASES))
def test_incremental_encoding_equals_token_parallel_encoding(name):
    """Prefill P tokens with a cache, then append the rest one position at a time: e and M equal
    the token-parallel encoding of the whole sequence and the oracle's."""
    cfg, B, P, T = ENC_CASES[name]
    w = make_weights(cfg)
    model = build_model(cfg, max_pos=T, weights=w)
    tok = np.random.default_rng([5, B, T]).integers(0, cfg.V, size=(B, T)).astype(np.int32)
    tt = torch.from_numpy(tok).cuda()
    e_full, M_full = model.encode(tt)
    e, M, cache = model.encode_prefill(tt[:, :P], T_alloc=T, T_max=T)
    tt_tb = tt.t().contiguous()
    for p in range(P, T):
        model.encode_append(tt_tb[p], p, cache, T, e, M)
    torch.cuda.synchronize()
    assert model.last_error() == 0
    e_o, M_o = RLTOracle(cfg, w).encode(tok)
    M_np = to_np(M).transpose(0, 1, 2, 4, 3, 5).reshape(cfg.G, 2, B, T, cfg.d)
    if cfg.dtype == "f32":
        assert np.abs(to_np(e) - to_np(e_full)).max() <= 1e-5
        assert np.abs(to_np(M) - to_np(M_full)).max() <= 1e-5
        assert np.abs(to_np(e) - e_o).max() <= 1e-5
        assert np.abs(M_np - M_o).max() <= 1e-5
    else:
        assert cosine(to_np(e).reshape(-1, cfg.d), to_np(e_full).reshape(-1, cfg.d)).min() >= 0.999
        assert cosine(to_np(e).reshape(-1, cfg.d), e_o.reshape(-1, cfg.d)).min() >= 0.999
        assert cosine(M_np.reshape(-1, cfg.d), M_o.reshape(-1, cfg.d)).min() >= 0.999


def test_generation_loop_tiny_f32_matches_the_oracle():
    """Float32 model: every generated token is the oracle's draw from the oracle's next-token
    distribution over the tokens so far (teacher-forced on the GPU's tokens), and the behaviour
    and prompt log-probs agree within 1e-4."""
    cfg = TINY.model
    w = make_weights(cfg)
    model = build_model(cfg, max_pos=TINY.T, weights=w)
    P, n_new, tau, top_k, top_p = 24, 40, 0.9, 20, 0.95
    prompt = torch.from_numpy(make_tokens(TINY)[:, :P]).cuda()
    B = prompt.shape[0]
    u = torch.from_numpy(np.random.default_rng(41).random((n_new, B)).astype(np.float32)).cuda()
    toks, blp, lp_prompt, st = model.generate(prompt, n_new, u, tau, top_k, top_p)
    torch.cuda.synchronize()
    assert model.last_error() == 0
    toks, blp, lp_prompt, u = toks.cpu().numpy(), to_np(blp), to_np(lp_prompt), u.cpu().numpy()
    assert np.array_equal(toks[:, :P], prompt.cpu().numpy())
    ora = RLTOracle(cfg, w)
    _, _, s_o, lp_o = ora.run(toks, tau=tau)
    for b in range(B):
        for t in range(1, P):
            assert abs(lp_prompt[b, t - 1] - lp_o[b, t - 1, toks[b, t]]) <= 1e-4
        for j in range(n_new):
            t = P + j                               # column t holds x_{t+1}, drawn from logp_t
            row = lp_o[b, t - 1]
            assert valid_draw(row, float(u[j, b]), top_k, top_p, int(toks[b, t]), 1e-4), (b, t)
            ref_tok, ref_blp = sample_token(row, float(u[j, b]), top_k, top_p)
            if ref_tok == toks[b, t]:
                assert abs(blp[b, j] - ref_blp) <= 1e-4
    assert st.position == P + n_new
    assert np.abs(to_np(st.s()) - s_o[:, -1]).max() <= 1e-4


def test_generation_loop_small_bf16():
    """bf16 model: (1) the loop's wiring: re-running the same calls teacher-forced on the
    generated tokens (prefill, decoder steps, resample each full log-prob row with the same
    uniform, append the token) reproduces every token bit for bit, so each draw came from the
    step's own row and uniform; (2) on sampled sequences the oracle, teacher-forced on the GPU's
    tokens, gives the same prompt and behaviour log-probs within the bf16 tolerance."""
    cfg = SMALL.model
    w = make_weights(cfg)
    model = build_model(cfg, max_pos=192, weights=w)
    B, P, n_new, tau, top_k, top_p = 64, 128, 64, 0.8, 0, 0.9
    T = P + n_new
    prompt = torch.from_numpy(make_tokens(SMALL)[:B, :P]).cuda()
    u = torch.from_numpy(np.random.default_rng(42).random((n_new, B)).astype(np.float32)).cuda()
    toks, blp, lp_prompt, st = model.generate(prompt, n_new, u, tau, top_k, top_p)
    torch.cuda.synchronize()
    assert model.last_error() == 0
    toks_np = toks.cpu().numpy()
    assert np.array_equal(toks_np[:, :P], prompt.cpu().numpy())
    # (1) the same calls, teacher-forced
    tt = torch.from_numpy(np.ascontiguousarray(toks_np.T)).cuda()          # row t = x_{t+1}
    e, M, cache = model.encode_prefill(prompt.contiguous(), T_alloc=T, T_max=T)
    st2 = model.new_state(B)
    row = torch.empty((B, cfg.V), device="cuda")
    redraw = torch.empty(B, dtype=torch.int32, device="cuda")
    blp2 = torch.empty(B, device="cuda")
    for t in range(1, T):
        if t < P:
            model.decode_step(st2, e, M, next_tok=tt[t], tau=tau)
            continue
        model.decode_step(st2, e, M, tau=tau, logp_full=row)
        model.sample(row, u[t - P], top_k, top_p, out=redraw, behaviour_logp=blp2)
        assert torch.equal(redraw, tt[t]), t
        assert torch.equal(blp2, blp[:, t - P]), t
        model.encode_append(tt[t], t, cache, T, e, M)
    # (2) oracle, teacher-forced, on four sequences
    seqs = [0, 1, 17, 63]
    _, _, _, lp_o = RLTOracle(cfg, w).run(toks_np[seqs], tau=tau)
    blp, lp_prompt = to_np(blp), to_np(lp_prompt)
    u_np = u.cpu().numpy()
    for i, b in enumerate(seqs):
        for t in range(1, P):
            assert abs(lp_prompt[b, t - 1] - lp_o[i, t - 1, toks_np[b, t]]) <= 5e-2
        for j in range(n_new):
            t = P + j
            ref_tok, ref_blp = sample_token(lp_o[i, t - 1], float(u_np[j, b]), top_k, top_p)
            if ref_tok == toks_np[b, t]:
                assert abs(blp[b, j] - ref_blp) <= 5e-2
