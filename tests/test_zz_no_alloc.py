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
from gpu_util import build_model, to_np

pytestmark = pytest.mark.gpu

def ring_view(st, cfg) -> np.ndarray:
    """The SWA ring of a state buffer, [L_D, B, 2, n_heads, W - 1, head_dim] (layout of
    rlt_state_bytes: a 256-byte header, s [B, d] float32, then the ring 256-byte aligned)."""
    off = (256 + st.B * cfg.d * 4 + 255) // 256 * 256
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = (cfg.L_D, st.B, 2, cfg.n_heads, cfg.W - 1, cfg.head_dim)
    n = int(np.prod(shape)) * (2 if cfg.dtype == "bf16" else 4)
    return to_np(st.buf[off:off + n].view(dt).view(shape))


CASES = {
    # model, batch
    "tiny-f32": (TINY.model, 2),
    "small-bf16": (SMALL.model, 64),
    "tiny-bf16-wide-batch": (replace(TINY.model, dtype="bf16", W=5), 300),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_step_matches_decode_step_on_two_calls(name):
    """Both entry points launch the same deterministic kernels on the same inputs; only the
    scratch address differs, so every output is identical bit for bit."""
    cfg, B = CASES[name]
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
        for a, b in zip(out["ref"], out["noalloc"]):
            np.testing.assert_array_equal(a, b)
        # the ring slots written so far (the others still hold whatever the buffers held)
        n = min(step + 1, cfg.W - 1)
        np.testing.assert_array_equal(ring_view(st_ref, cfg)[..., :n, :], ring_view(st_na, cfg)[..., :n, :])
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


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2, reason="needs two devices")
def test_noalloc_step_rejects_a_current_device_other_than_the_models():
    cfg = TINY.model
    model = build_model(cfg, max_pos=8, weights=make_weights(cfg))
    e, M = model.alloc_encoder_outputs(1, 8)
    st = model.new_state(1)
    with torch.cuda.device(1):
        with pytest.raises(RLTError) as ex:
            model.decode_step_noalloc(st, e, M)
    assert ex.value.status == "RLT_EINVAL"
