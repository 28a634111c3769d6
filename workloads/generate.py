"""Seeded synthetic inputs: model weights and token batches.

Both the CPU oracle and the CUDA path draw their inputs from here, so that a
parity test compares the two on identical data.  Nothing here computes any part
of the method; it only draws random numbers.

Weights: every matrix and the learned start state s* are N(0, 0.02) in float32,
each tensor from its own counter-based stream keyed by (weight_seed, crc32(name)),
so any subset can be regenerated alone.  Norm gains start at 1 and the merge-gate
bias at 0.  For bf16 models the float32 draws are handed over as they are; each
side rounds them to bfloat16 (round to nearest even) itself.

Tokens (one stream per sequence, keyed by (token_seed, b), so a subset of the
batch regenerates identically):
  uniform  i.i.d. uniform over the vocabulary
  markov2  an order-2 Markov chain; the row for context (a, b) is Dirichlet(alpha)
           drawn lazily from the stream (2, a, b) as normalised Gamma(alpha)
           variates; the first two tokens are uniform
  zipf     P(rank r) proportional to r^-s over r = 1..V, ranks mapped to ids by a
           permutation drawn from stream (3, V)
"""
from __future__ import annotations

import zlib

import numpy as np

from .configs import ModelConfig, Workload

INIT_STD = 0.02


def weight_shapes(m: ModelConfig) -> dict[str, tuple[int, ...]]:
    """Canonical weight layout: a linear map y = x @ W.T stores W as [out, in]."""
    d, F, V = m.d, m.F, m.V
    shapes: dict[str, tuple[int, ...]] = {"embed": (V, d)}
    for l in range(m.L_E):
        shapes.update({
            f"layers.{l}.attn_norm": (d,),
            f"layers.{l}.wq": (d, d),
            f"layers.{l}.wk": (d, d),
            f"layers.{l}.wv": (d, d),
            f"layers.{l}.wo": (d, d),
            f"layers.{l}.ffn_norm": (d,),
            f"layers.{l}.w_gate": (F, d),
            f"layers.{l}.w_up": (F, d),
            f"layers.{l}.w_down": (d, F),
        })
    shapes["enc_norm"] = (d,)
    shapes["mem_k"] = (m.G, d, d)
    shapes["mem_v"] = (m.G, d, d)
    for l in range(m.L_D):
        shapes.update({
            f"dec.{l}.xattn_norm": (d,),
            f"dec.{l}.w_qc": (d, d),
            f"dec.{l}.w_oc": (d, d),
        })
    shapes.update({
        "merge_ge": (d, d),
        "merge_gs": (d, d),
        "merge_fb": (d, d),
        "merge_bias": (d,),
        "s_star": (d,),
        "dec_norm": (d,),
        "unembed": (V, d),
    })
    return shapes


def _is_gain(name: str) -> bool:
    return name.endswith("_norm")


def make_weight(m: ModelConfig, name: str, seed: int = 0) -> np.ndarray:
    shape = weight_shapes(m)[name]
    if _is_gain(name):
        return np.ones(shape, np.float32)
    if name == "merge_bias":
        return np.zeros(shape, np.float32)
    rng = np.random.default_rng([seed, zlib.crc32(name.encode())])
    w = rng.standard_normal(shape, dtype=np.float32)
    w *= np.float32(INIT_STD)
    return w


def make_weights(m: ModelConfig, seed: int = 0) -> dict[str, np.ndarray]:
    return {name: make_weight(m, name, seed) for name in weight_shapes(m)}


def _zipf_tables(V: int, s: float):
    ranks = np.arange(1, V + 1, dtype=np.float64)
    p = ranks ** (-s)
    cdf = np.cumsum(p)
    cdf /= cdf[-1]
    perm = np.random.default_rng([3, V]).permutation(V)
    return cdf, perm


def make_tokens(w: Workload, seqs=None) -> np.ndarray:
    """Token ids int32 [len(seqs), T]; seqs defaults to range(B)."""
    seqs = range(w.B) if seqs is None else list(seqs)
    V, T = w.model.V, w.T
    out = np.empty((len(seqs), T), np.int32)
    if w.tokens == "uniform":
        for i, b in enumerate(seqs):
            out[i] = np.random.default_rng([w.token_seed, b]).integers(0, V, size=T)
    elif w.tokens == "zipf":
        cdf, perm = _zipf_tables(V, w.zipf_s)
        for i, b in enumerate(seqs):
            u = np.random.default_rng([w.token_seed, b]).random(T)
            r = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1)
            out[i] = perm[r]
    elif w.tokens == "markov2":
        rows: dict[tuple[int, int], np.ndarray] = {}
        for i, b in enumerate(seqs):
            rng = np.random.default_rng([w.token_seed, b])
            seq = np.empty(T, np.int64)
            first = rng.integers(0, V, size=min(2, T))
            seq[: len(first)] = first
            for t in range(2, T):
                ctx = (int(seq[t - 2]), int(seq[t - 1]))
                cum = rows.get(ctx)
                if cum is None:
                    g = np.random.default_rng([2, ctx[0], ctx[1]]).gamma(w.dirichlet_alpha, size=V)
                    cum = np.cumsum(g)
                    cum /= cum[-1]
                    rows[ctx] = cum
                seq[t] = min(int(np.searchsorted(cum, rng.random(), side="right")), V - 1)
            out[i] = seq
    else:
        raise ValueError(f"unknown token distribution {w.tokens}")
    return out
