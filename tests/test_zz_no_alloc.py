"""The allocation-free decode step against the regular one, through the C ABI.

Some callers cannot allocate device memory (a host runtime that owns the whole device pool,
or a serving loop that must not touch an allocator once running); they call
rlt_decode_step_noalloc, whose scratch is the library's static 32 MiB device array instead of
a caller workspace.  This file is collected last so that a run stopping at its first failure
has already run every other test.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from cross_token_latent_b200 import RLTError
from workloads import TINY, SMALL, make_tokens, make_weights
from gpu_util import build_model, cosine, to_np

pytestmark = pytest.mark.gpu

CASES = {
    # model, batch, tolerance on log-probs, on s (float32: max abs; bf16: cosine)
    "tiny-f32": (TINY.model, 2, 1e-4),
    "small-bf16": (SMALL.model, 64, 5e-2),
    "tiny-bf16-wide-batch": (replace(TINY.model, dtype="bf16", W=5), 300, 5e-2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_step_matches_decode_step_on_two_calls(name):
    cfg, B, tol = CASES[name]
    T = 16
    model = build_model(cfg, max_pos=T, weights=make_weights(cfg, seed=4))
    tok = np.random.default_rng([9, B]).integers(0, cfg.V, size=(B, T)).astype(np.int32)
    tt = torch.from_numpy(tok).cuda()
    e, M = model.encode(tt)
    st_ref, st_na = model.new_state(B), model.new_state(B)
    for step in range(2):                                  # two calls in a row
        nxt = tt[:, step + 1].contiguous()
        out = {}
        for key, st, call in (("ref", st_ref, model.decode_step), ("noalloc", st_na, model.decode_step_noalloc)):
            lp = torch.empty(B, device="cuda")
            lse = torch.empty(B, device="cuda")
            full = torch.empty(B, cfg.V, device="cuda")
            call(st, e, M, next_tok=nxt, tau=0.9, logp_tok=lp, lse=lse, logp_full=full)
            torch.cuda.synchronize()
            out[key] = (to_np(lp), to_np(lse), to_np(full), to_np(st.s()))
        assert model.last_error() == 0
        (lp_a, lse_a, full_a, s_a), (lp_b, lse_b, full_b, s_b) = out["ref"], out["noalloc"]
        assert np.abs(full_a - full_b).max() <= tol
        assert np.abs(lp_a - lp_b).max() <= tol and np.abs(lse_a - lse_b).max() <= tol
        if cfg.dtype == "f32":
            assert np.abs(s_a - s_b).max() <= 1e-4
        else:
            assert cosine(s_a, s_b).min() >= 0.999
        assert st_na.position == st_ref.position == step + 1


def test_noalloc_step_rejects_batches_beyond_the_static_scratch():
    cfg = SMALL.model
    model = build_model(cfg, max_pos=8, weights=make_weights(cfg))
    e, M = model.alloc_encoder_outputs(1, 8)
    st = model.new_state(1)
    big = type(st)(model, 16384, st.buf)                  # workspace for 16384 rows exceeds 32 MiB
    with pytest.raises(RLTError) as ex:
        model.decode_step_noalloc(big, e, M)
    assert ex.value.status == "RLT_EUNSUPPORTED"
