"""Independent token-parallel references built from library routines (torch, float64).

These are NOT the oracle.  They restate two special cases of the method as
textbook transformer passes, so that the oracle's step-by-step recurrence can be
checked against something other than itself:

* the causal encoder is a standard pre-norm causal transformer: attention via
  torch.nn.functional.scaled_dot_product_attention(is_causal=True), RMSNorm via
  torch.nn.functional.rms_norm, rotary embedding via complex multiplication;
* with the feedback projection zeroed (W_fb = 0) the gated merge returns e_t, so
  the decoder no longer depends on s_{t-1} and collapses to a parallel pass with
  a banded causal self-attention mask of width W (full causal when W >= T) plus
  causal cross-attention to M.  ("Recurrent Looped Transformer" news summary,
  model-hardware principle: the standard parallel SWA pass is NOT equivalent once
  the feedback is on, which the tests also check.)
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as Fn


def _t(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.float64)


def rope_complex(x: torch.Tensor, pos: torch.Tensor, base: float) -> torch.Tensor:
    """x [B, H, T, hd]: rotate the complex number x_i + j x_{i+hd/2} by pos*base^(-2i/hd)."""
    hd = x.shape[-1]
    half = hd // 2
    inv = base ** (-torch.arange(half, dtype=torch.float64) * 2.0 / hd)
    ang = pos.to(torch.float64)[:, None] * inv[None, :]
    z = torch.complex(x[..., :half], x[..., half:]) * torch.polar(torch.ones_like(ang), ang)
    return torch.cat([z.real, z.imag], dim=-1)


def _split(x, H):
    B, T, d = x.shape
    return x.view(B, T, H, d // H).transpose(1, 2)


def _join(x):
    B, H, T, hd = x.shape
    return x.transpose(1, 2).reshape(B, T, H * hd)


def encoder(cfg, w: dict, tokens) -> tuple[torch.Tensor, torch.Tensor]:
    """Textbook causal pre-norm transformer; returns e [B,T,d], M [G,2,B,T,d]."""
    tok = torch.as_tensor(np.asarray(tokens), dtype=torch.long)
    B, T = tok.shape
    H, eps = cfg.n_heads, cfg.rms_eps
    pos = torch.arange(T)
    h = _t(w["embed"])[tok]
    for l in range(cfg.L_E):
        p = f"layers.{l}."
        a = Fn.rms_norm(h, (cfg.d,), _t(w[p + "attn_norm"]), eps)
        q = rope_complex(_split(a @ _t(w[p + "wq"]).T, H), pos, cfg.rope_base)
        k = rope_complex(_split(a @ _t(w[p + "wk"]).T, H), pos, cfg.rope_base)
        v = _split(a @ _t(w[p + "wv"]).T, H)
        o = Fn.scaled_dot_product_attention(q, k, v, is_causal=True)
        h = h + _join(o) @ _t(w[p + "wo"]).T
        f = Fn.rms_norm(h, (cfg.d,), _t(w[p + "ffn_norm"]), eps)
        h = h + (Fn.silu(f @ _t(w[p + "w_gate"]).T) * (f @ _t(w[p + "w_up"]).T)) @ _t(w[p + "w_down"]).T
    e = Fn.rms_norm(h, (cfg.d,), _t(w["enc_norm"]), eps)
    M = torch.stack([torch.stack([e @ _t(w["mem_k"][g]).T, e @ _t(w["mem_v"][g]).T])
                     for g in range(cfg.G)])
    return e, M


def decoder_no_feedback(cfg, w: dict, e: torch.Tensor, M: torch.Tensor, tau: float = 1.0):
    """Parallel decoder pass with x0 = e (feedback zeroed).  Returns s [B,T,d], logp [B,T,V]."""
    B, T, d = e.shape
    H, eps = cfg.n_heads, cfg.rms_eps
    pos = torch.arange(T)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    band = (j <= i) & (j > i - cfg.W)             # window of W tokens including the current one
    x = e.clone()
    for l in range(cfg.L_D):
        p, pd = f"layers.{l}.", f"dec.{l}."
        g = 0 if cfg.G == 1 else l
        a = Fn.rms_norm(x, (d,), _t(w[p + "attn_norm"]), eps)
        q = rope_complex(_split(a @ _t(w[p + "wq"]).T, H), pos, cfg.rope_base)
        k = rope_complex(_split(a @ _t(w[p + "wk"]).T, H), pos, cfg.rope_base)
        v = _split(a @ _t(w[p + "wv"]).T, H)
        o = Fn.scaled_dot_product_attention(q, k, v, attn_mask=band)
        x = x + _join(o) @ _t(w[p + "wo"]).T
        c = Fn.rms_norm(x, (d,), _t(w[pd + "xattn_norm"]), eps)
        qc = _split(c @ _t(w[pd + "w_qc"]).T, H)
        o = Fn.scaled_dot_product_attention(qc, _split(M[g, 0], H), _split(M[g, 1], H), is_causal=True)
        x = x + _join(o) @ _t(w[pd + "w_oc"]).T
        f = Fn.rms_norm(x, (d,), _t(w[p + "ffn_norm"]), eps)
        x = x + (Fn.silu(f @ _t(w[p + "w_gate"]).T) * (f @ _t(w[p + "w_up"]).T)) @ _t(w[p + "w_down"]).T
    s = Fn.rms_norm(x, (d,), _t(w["dec_norm"]), eps)
    logp = torch.log_softmax((s @ _t(w["unembed"]).T) / tau, dim=-1)
    return s, logp
