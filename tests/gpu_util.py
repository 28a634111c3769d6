"""Helpers shared by the GPU tests: build a library model from seeded weights and run it."""
from __future__ import annotations

import numpy as np
import torch

from cross_token_latent_b200 import RLTModel
from workloads import make_weights


def build_model(cfg, max_pos: int, weights: dict | None = None, seed: int = 0) -> RLTModel:
    m = RLTModel(cfg, max_pos=max_pos)
    m.load_weights(make_weights(cfg, seed) if weights is None else weights)
    return m


def gpu_run(model: RLTModel, tokens: np.ndarray, steps: int | None = None, tau: float = 1.0,
            full: bool = True, T_alloc: int | None = None):
    """Encode `tokens` then take `steps` decoder steps.

    Returns e, M (device), s [B, n, d] float32 (host), logp_full [B, n, V] (host, or None)
    and logp_tok [B, n] (host; entry t-1 = log p(x_{t+1}), 0 for the last token)."""
    tok = torch.from_numpy(np.ascontiguousarray(tokens, np.int32)).cuda()
    B, T = tok.shape
    n = T if steps is None else steps
    e, M = model.encode(tok, T_alloc=T_alloc)
    st = model.new_state(B)
    d, V = model.cfg.d, model.cfg.V
    s_all = torch.empty((B, n, d), dtype=torch.float32, device="cuda")
    lp_all = torch.empty((B, n, V), dtype=torch.float32, device="cuda") if full else None
    lp_tok = torch.zeros((B, n), dtype=torch.float32, device="cuda")
    row = torch.empty((B, V), dtype=torch.float32, device="cuda") if full else None
    gat = torch.empty(B, dtype=torch.float32, device="cuda")
    for t in range(n):
        nxt = tok[:, t + 1].contiguous() if t + 1 < T else None
        model.decode_step(st, e, M, next_tok=nxt, tau=tau, logp_tok=gat if nxt is not None else None,
                          logp_full=row)
        s_all[:, t] = st.s()
        if full:
            lp_all[:, t] = row
        if nxt is not None:
            lp_tok[:, t] = gat
    torch.cuda.synchronize()
    model.check_device_errors()
    return (e, M, s_all.cpu().numpy(), None if lp_all is None else lp_all.cpu().numpy(),
            lp_tok.cpu().numpy(), st)


def cosine(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    return (a * b).sum(-1) / (np.linalg.norm(a, axis=-1) * np.linalg.norm(b, axis=-1))


def to_np(x: torch.Tensor) -> np.ndarray:
    return x.float().cpu().numpy()
