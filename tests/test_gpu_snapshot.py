"""Prefix snapshots and per-sequence positions on the GPU, through the C ABI.

A sequence is saved with rlt_snapshot_save (s_t, its SWA ring, M_{<=t} and its encoder cache)
and loaded into a row of another batch state with rlt_snapshot_load; rows of one state may
then stand at different positions, and every decoder step advances each of them by one token
at its own position.  Each row must follow the CPU oracle's run of its own sequence.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from cross_token_latent_b200 import RLTError
from oracle import RLTOracle
from workloads import TINY, SMALL, make_weights
from gpu_util import build_model, cosine, to_np

pytestmark = pytest.mark.gpu

CASES = {"tiny-f32": (TINY.model, 1e-4), "small-bf16": (SMALL.model, 5e-2)}
T = 48


def seqs_for(cfg, n, seed=17):
    return np.random.default_rng([seed, cfg.V]).integers(0, cfg.V, size=(n, T)).astype(np.int32)


class Batch:
    """e, M, encoder cache and decoder state of B rows with capacity T (prefilled with `tok`)."""

    def __init__(self, model, tok: np.ndarray, P: int):
        self.model = model
        self.tok = torch.from_numpy(tok).cuda()
        self.B = tok.shape[0]
        self.e, self.M, self.cache = model.encode_prefill(self.tok[:, :P].contiguous(), T_alloc=T, T_max=T)
        self.st = model.new_state(self.B)
        self.pref = P                    # tokens 0..P-1 of every row are encoded

    def step(self, tok_rows: np.ndarray | None = None):
        """One decoder step of every row at its own position p_b: encode its token p_b if it is
        not encoded yet, then step, gathering the log-prob of token p_b + 1.  Returns (logp [B],
        s [B, d], positions before the step)."""
        m = self.model
        pos = np.array(self.st.positions())
        tok = self.tok if tok_rows is None else torch.from_numpy(tok_rows).cuda()
        cur = torch.from_numpy(np.ascontiguousarray(tok.cpu().numpy()[np.arange(self.B), pos])).cuda()
        nxt = torch.from_numpy(np.ascontiguousarray(tok.cpu().numpy()[np.arange(self.B), np.minimum(pos + 1, T - 1)])).cuda()
        if (pos >= self.pref).any():
            m.encode_append(cur, int(pos.max()), self.cache, T, self.e, self.M, positions=self.st.positions_device())
        lp = torch.empty(self.B, device="cuda")
        m.decode_step(self.st, self.e, self.M, next_tok=nxt, logp_tok=lp)
        torch.cuda.synchronize()
        return to_np(lp), to_np(self.st.s()).copy(), pos


@pytest.mark.parametrize("name", list(CASES))
def test_rows_loaded_from_snapshots_at_different_positions_follow_the_oracle(name):
    cfg, tol = CASES[name]
    w = make_weights(cfg, seed=3)
    model = build_model(cfg, max_pos=T, weights=w)
    seqs = seqs_for(cfg, 3)
    # sequence 0 runs 13 steps, sequence 1 runs 5 steps, each in its own batch, then is saved
    snaps = []
    for k, n in ((0, 13), (1, 5)):
        bt = Batch(model, seqs[k:k + 1], P=n)
        for _ in range(n):
            bt.step()
        assert bt.st.positions() == [n]
        snaps.append(model.snapshot_save(bt.st, 0, bt.M, bt.cache, T))
    # a batch of three rows: row 0 <- sequence 1 (t=5), row 1 <- sequence 0 (t=13), row 2 fresh
    rows = np.stack([seqs[1], seqs[0], seqs[2]])
    bt = Batch(model, rows, P=1)
    model.snapshot_load(snaps[1], bt.st, 0, bt.M, bt.cache, T)    # sequence 1 at t = 5
    model.snapshot_load(snaps[0], bt.st, 1, bt.M, bt.cache, T)    # sequence 0 at t = 13
    assert bt.st.positions() == [5, 13, 0]
    got_lp, got_s, got_pos = [], [], []
    for _ in range(20):
        lp, s, pos = bt.step()
        got_lp.append(lp); got_s.append(s); got_pos.append(pos)
    assert model.last_error() == 0
    assert bt.st.positions() == [25, 33, 20]
    ora = RLTOracle(cfg, w)
    for row, k in enumerate((1, 0, 2)):
        _, _, s_o, lp_o = ora.run(seqs[k:k + 1], steps=34)
        for i in range(20):
            p = got_pos[i][row]                     # the step consumed token p and predicts p + 1
            ref_lp = lp_o[0, p, seqs[k, p + 1]]
            assert abs(got_lp[i][row] - ref_lp) <= tol, (row, i, got_lp[i][row], ref_lp)
            if cfg.dtype == "f32":
                assert np.abs(got_s[i][row] - s_o[0, p]).max() <= 1e-4
            else:
                assert cosine(got_s[i][row][None], s_o[0, p][None]).min() >= 0.999


def test_snapshot_round_trip_continues_like_the_uninterrupted_run():
    cfg = TINY.model
    model = build_model(cfg, max_pos=T, weights=make_weights(cfg, seed=5))
    seqs = seqs_for(cfg, 2, seed=23)
    a = Batch(model, seqs, P=9)
    for _ in range(9):
        a.step()
    snap = model.snapshot_save(a.st, 1, a.M, a.cache, T)
    ref = [a.step() for _ in range(12)]
    b = Batch(model, seqs[1:2], P=1)
    model.snapshot_load(snap, b.st, 0, b.M, b.cache, T)
    got = [b.step() for _ in range(12)]
    for (lp_r, s_r, _), (lp_g, s_g, _) in zip(ref, got):
        assert abs(lp_r[1] - lp_g[0]) <= 1e-5
        assert np.abs(s_r[1] - s_g[0]).max() <= 1e-5


def test_reset_row_restarts_one_sequence():
    cfg = replace(TINY.model, dtype="bf16", W=5)
    w = make_weights(cfg, seed=6)
    model = build_model(cfg, max_pos=T, weights=w)
    seqs = seqs_for(cfg, 2, seed=29)
    bt = Batch(model, seqs, P=T)
    for _ in range(7):
        bt.step()
    bt.st.reset_row(1)
    assert bt.st.positions() == [7, 0]
    outs = [bt.step() for _ in range(6)]
    _, _, s_o, lp_o = RLTOracle(cfg, w).run(seqs[1:2], steps=8)
    for i, (lp, s, pos) in enumerate(outs):
        assert pos[1] == i
        assert abs(lp[1] - lp_o[0, i, seqs[1, i + 1]]) <= 5e-2
        assert cosine(s[1][None], s_o[0, i][None]).min() >= 0.999


def test_a_snapshot_from_replaced_weights_is_stale():
    cfg = TINY.model
    w = make_weights(cfg, seed=7)
    model = build_model(cfg, max_pos=T, weights=w)
    bt = Batch(model, seqs_for(cfg, 1, seed=31), P=4)
    for _ in range(4):
        bt.step()
    snap = model.snapshot_save(bt.st, 0, bt.M, bt.cache, T)
    model.load_weights(w)                          # a new model version
    fresh = Batch(model, seqs_for(cfg, 1, seed=31), P=1)
    with pytest.raises(RLTError) as ex:
        model.snapshot_load(snap, fresh.st, 0, fresh.M, fresh.cache, T)
    assert ex.value.status == "RLT_ESTALE"
