"""CPU oracle for the Recurrent Looped Transformer (RLT) decoder transition.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
tests, the smoke check and the benchmark's CPU-baseline leg may run it.  It
shares no code with the CUDA path.

It is a plain, slow, literal restatement of the method, one token step at a
time, in numpy, in float64 by default (float32 on request).  Every function
names the passage it follows.  Sources (web pages about the technical report):

  [news]      "普林斯顿提出 RLT：跨 Token 携带解码器状态的循环 Transformer"
              (feinterview news summary): the encoder/memory paragraph, the
              decoder-state paragraph, the weight-tying paragraph, the three
              design principles (model-hardware; model-RL with Proposition 3.1).
  [teardown]  "技术拆解 009｜RLT" (deepsonar): sections 2.2 (attention pattern),
              2.3 (state and cache), 2.4 (one token's path), 2.5 (one execution
              semantics), section 6 (minimal skeleton).
  [review]    "Recurrent Looped Transformer：路徑變深，就真的更會推理嗎？"
              (alphalab): section 1 (three memories), section 4 (replay contract).

Readings taken where the pages leave a step open (each is a documented choice):
  R1 merge      x0 = e_t + sigmoid(W_ge e_t + W_gs s_{t-1} + b_g) * (W_fb s_{t-1});
                [news] says "gated merge" of e_t with s_{t-1}; [teardown] 2.4 and
                section 6 give the additive "feedback projection plus input" form,
                which an open gate reduces to.
  R2 memory     M^g = (e W_K^g, e W_V^g), g = 1..G, projected from the final
                encoder output e ([news] encoder paragraph).
  R3 SWA k/v    k_t, v_t come from the same normed sublayer input as q_t; the
                current token attends to itself; the window is [t-W+1, t] and the
                cache keeps the W-1 newest past entries ([teardown] 2.2, 2.3).
  R4 cross-attn over M_{<=t}, positions 1..t, no rotary embedding.
  R5 RoPE       rotate-half pairing (i, i + hd/2), base 10000, 0-based position
                t-1, on encoder and decoder self-attention q and k; keys are
                cached after rotation.
  R6 norms      RMSNorm y = x / sqrt(mean(x^2) + eps) * gain, pre-norm.  The
                decoder's self-attention and FFN norms are tied with the encoder
                layer like their weights; the cross-attention norm is its own.
  R7 head       untied W_U; z = W_U s_t / tau; logp_t = z - logsumexp(z)
                predicts x_{t+1}; s_t = RMSNorm(final decoder output).
  R8 bf16       storage contract for bf16 models: weights, e, M, cached k/v (and
                the current k/v), encoder q/k/v, and every GEMM input activation
                (normed h, attention output o, SiLU(g)*u, s fed to merge and head)
                are rounded to bfloat16 (round to nearest even).  The residual
                stream, norms, decoder queries, softmax and its probabilities,
                s_t, the log-sum-exp and logp stay in full precision.
  R12 sampling  top-k and top-p keep every token tied at their boundary; the kept tokens
                are renormalised and sampled by inverse CDF in token-id order with a
                caller-given uniform (sample_token).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


# ----------------------------------------------------------------------------------
# elementary operations
# ----------------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 value (8 significant bits), ties to even.

    Written from the definition: x = m * 2^e with 0.5 <= |m| < 1, keep 8 bits of m
    with round-half-even, rescale.  Exact in float64 for the normal range.
    """
    x = np.asarray(x)
    xd = x.astype(np.float64)
    m, e = np.frexp(xd)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    return r.astype(x.dtype)


def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis (reading R6)."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gain


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotary embedding, rotate-half pairing (reading R5).

    x: [..., n_pos, n_heads, hd]; pos: integer positions [n_pos].  Pair i rotates
    (x_i, x_{i+hd/2}) by angle pos * base^(-2i/hd).
    """
    hd = x.shape[-1]
    half = hd // 2
    inv_freq = base ** (-np.arange(half, dtype=np.float64) * 2.0 / hd)
    ang = np.asarray(pos, np.float64)[:, None] * inv_freq[None, :]      # [n_pos, half]
    cos = np.cos(ang)[:, None, :].astype(x.dtype)
    sin = np.sin(ang)[:, None, :].astype(x.dtype)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * cos - b * sin, a * sin + b * cos], axis=-1)


def softmax(s: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(s, axis=axis, keepdims=True)
    p = np.exp(s - m)
    return p / np.sum(p, axis=axis, keepdims=True)


def log_softmax(z: np.ndarray) -> np.ndarray:
    m = np.max(z, axis=-1, keepdims=True)
    return z - (m + np.log(np.sum(np.exp(z - m), axis=-1, keepdims=True)))


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def sample_token(logp: np.ndarray, u: float, top_k: int = 0, top_p: float = 1.0):
    """Draw one token from the next-token distribution with a caller-given uniform u in [0, 1)
    ([teardown] 2.5: generation runs the same transition; [news] model-RL principle: the
    behaviour log-probability is the one of the distribution actually sampled from).

    logp: log-probabilities of one row at the sampling temperature (log_softmax(z / tau)).
    Truncation (reading R12): with p = exp(logp), top-k keeps token i when fewer than k tokens
    are strictly more probable than i (top_k <= 0: no top-k); top-p then keeps i when the
    probability mass of the tokens strictly more probable than i is below top_p times the mass
    top-k kept (top_p >= 1: no top-p).  Tokens tied at a boundary are all kept.  The kept
    tokens are renormalised to total Z and the token is the inverse CDF at u * Z, the kept
    tokens taken in increasing id order: the first id whose cumulative kept mass exceeds u * Z.
    Returns (token, behaviour log-probability log(p_token / Z))."""
    lp = np.asarray(logp, np.float64)
    p = np.exp(lp)
    V = p.shape[0]
    # tokens in decreasing probability; for every token, how many and how much probability
    # mass lie strictly above it (a sort as a library step, then prefix sums)
    desc = np.sort(p)[::-1]
    n_above = np.searchsorted(-desc, -p, side="left")          # count of values > p_i
    keep = np.ones(V, bool)
    if top_k > 0:
        keep = n_above < top_k
    if top_p < 1.0:
        z1 = p[keep].sum()
        mass_above = np.concatenate([[0.0], np.cumsum(desc)])[n_above]   # sum of the values > p_i
        keep = keep & (mass_above < top_p * z1)
    z = p[keep].sum()
    # inverse CDF over the kept tokens in increasing id order
    cdf = np.cumsum(np.where(keep, p, 0.0))
    i = int(np.searchsorted(cdf, u * z, side="right"))
    if i >= V:
        i = int(np.nonzero(keep)[0][-1])
    return i, float(lp[i] - np.log(z))


# ----------------------------------------------------------------------------------
# state
# ----------------------------------------------------------------------------------

@dataclass
class DecoderState:
    """H_t = (s_t, C_t^D) for a batch of independent sequences ([news] decoder-state
    paragraph; [teardown] 2.3).  `cache[l]` is a list of (k, v) pairs, oldest first,
    each [batch, n_heads, hd]; `t` is the number of tokens consumed."""
    s: np.ndarray
    cache: list = field(default_factory=list)
    t: int = 0

    def copy(self) -> "DecoderState":
        return DecoderState(self.s.copy(), [list(c) for c in self.cache], self.t)


# ----------------------------------------------------------------------------------
# the model
# ----------------------------------------------------------------------------------

class RLTOracle:
    """Literal CPU restatement of the RLT encoder, decoder transition and replay.

    cfg: a ModelConfig-like object (V, d, n_heads, head_dim, L_E, L_D, F, W, G,
    dtype, rms_eps, rope_base).  weights: dict of float32 arrays in the canonical
    layout (a linear map y = x @ W.T stores W as [out, in]).
    """

    def __init__(self, cfg, weights: dict, dtype=np.float64):
        self.cfg = cfg
        self.dt = np.dtype(dtype)
        self.bf16 = cfg.dtype == "bf16"
        self.w = {}
        for k, v in weights.items():
            a = np.asarray(v, np.float32)
            if self.bf16:
                a = round_bf16(a)
            self.w[k] = a.astype(self.dt)

    # storage rounding of reading R8 (identity for float32 models)
    def rnd(self, x: np.ndarray) -> np.ndarray:
        return round_bf16(x) if self.bf16 else x

    def _lin(self, x: np.ndarray, W: np.ndarray) -> np.ndarray:
        """The linear map y = x W^T over the last axis.  For a few rows the product is taken
        as (W x^T)^T, which BLAS runs several times faster for the same result."""
        x2 = x.reshape(-1, x.shape[-1])
        y = (W @ x2.T).T if x2.shape[0] <= 64 else x2 @ W.T
        return y.reshape(*x.shape[:-1], W.shape[0])

    def _heads(self, x: np.ndarray) -> np.ndarray:
        return x.reshape(*x.shape[:-1], self.cfg.n_heads, self.cfg.head_dim)

    def _merge_heads(self, x: np.ndarray) -> np.ndarray:
        return x.reshape(*x.shape[:-2], self.cfg.d)

    # ---- encoder: [news] encoder paragraph; [teardown] 2.1; [review] section 1 ----

    def encode(self, tokens: np.ndarray):
        """Causal encoder over one or more sequences.

        tokens: int [B, T].  Returns e [B, T, d] and M [G, 2, B, T, d] where
        M[g, 0] = e W_K^g (keys) and M[g, 1] = e W_V^g (values), reading R2.
        Token-parallel with a causal mask: position i sees positions <= i.
        """
        c, w = self.cfg, self.w
        tokens = np.asarray(tokens)
        B, T = tokens.shape
        hd = c.head_dim
        pos = np.arange(T)
        h = w["embed"][tokens]                                    # [B, T, d]
        causal = np.tril(np.ones((T, T), bool))
        for l in range(c.L_E):
            p = f"layers.{l}."
            a = self.rnd(rms_norm(h, w[p + "attn_norm"], c.rms_eps))
            q = self._heads(self._lin(a, w[p + "wq"]))            # [B, T, H, hd]
            k = self._heads(self._lin(a, w[p + "wk"]))
            v = self._heads(self._lin(a, w[p + "wv"]))
            q = self.rnd(rope(q, pos, c.rope_base))
            k = self.rnd(rope(k, pos, c.rope_base))
            v = self.rnd(v)
            s = np.einsum("bihx,bjhx->bhij", q, k) / np.sqrt(hd)  # [B, H, T, T]
            s = np.where(causal, s, -np.inf)
            o = np.einsum("bhij,bjhx->bihx", softmax(s), v)
            o = self.rnd(self._merge_heads(o))
            h = h + self._lin(o, w[p + "wo"])
            f = self.rnd(rms_norm(h, w[p + "ffn_norm"], c.rms_eps))
            m = self.rnd(silu(self._lin(f, w[p + "w_gate"])) * self._lin(f, w[p + "w_up"]))
            h = h + self._lin(m, w[p + "w_down"])
        e = self.rnd(rms_norm(h, w["enc_norm"], c.rms_eps))
        M = np.stack([np.stack([self.rnd(self._lin(e, w["mem_k"][g])),
                                self.rnd(self._lin(e, w["mem_v"][g]))])
                      for g in range(c.G)])                       # [G, 2, B, T, d]
        return e, M

    # ---- initial state: [news] decoder-state paragraph ("learned s*, empty cache") ----

    def init_state(self, B: int) -> DecoderState:
        s = np.broadcast_to(self.w["s_star"], (B, self.cfg.d)).copy()
        return DecoderState(s=s, cache=[[] for _ in range(self.cfg.L_D)], t=0)

    # ---- one decoder transition: [news] decoder-state paragraph; [teardown] 2.2-2.4 ----

    def merge(self, e_t: np.ndarray, s_prev: np.ndarray) -> np.ndarray:
        """Gated merge of e_t with s_{t-1} (reading R1)."""
        w = self.w
        s_in = self.rnd(s_prev)
        gate = sigmoid(self._lin(e_t, w["merge_ge"]) + self._lin(s_in, w["merge_gs"])
                       + w["merge_bias"])
        return e_t + gate * self._lin(s_in, w["merge_fb"])

    def swa(self, l: int, x: np.ndarray, state: DecoderState, t: int):
        """Causal sliding-window self-attention of decoder layer l at step t.

        Uses encoder layer l's norm and projections (weight tying, [news] tying
        paragraph).  Keys/values: cached entries of tokens max(1, t-W+1) .. t-1 plus
        the current token t (reading R3).  Returns the attention output (already
        projected by W_o) and the current (k, v) to push."""
        c, w = self.cfg, self.w
        p = f"layers.{l}."
        a = self.rnd(rms_norm(x, w[p + "attn_norm"], c.rms_eps))
        pos = np.array([t - 1])
        q = rope(self._heads(self._lin(a, w[p + "wq"]))[:, None], pos, c.rope_base)[:, 0]
        k = rope(self._heads(self._lin(a, w[p + "wk"]))[:, None], pos, c.rope_base)[:, 0]
        k = self.rnd(k)
        v = self.rnd(self._heads(self._lin(a, w[p + "wv"])))
        window = [kv for kv in state.cache[l]] + [(k, v)]
        assert len(window) <= c.W
        K = np.stack([kv[0] for kv in window], axis=2)            # [B, H, n, hd]
        Vv = np.stack([kv[1] for kv in window], axis=2)
        sc = np.einsum("bhx,bhnx->bhn", q, K) / np.sqrt(c.head_dim)
        o = np.einsum("bhn,bhnx->bhx", softmax(sc), Vv)
        o = self.rnd(self._merge_heads(o))
        return self._lin(o, w[p + "wo"]), (k, v)

    def cross_attn(self, l: int, x: np.ndarray, M: np.ndarray, t: int) -> np.ndarray:
        """Cross-attention of decoder layer l to the causal encoder memory M_{<=t}
        (reading R4).  M: [G, 2, B, >=t, d]; group g(l) = 0 if G == 1 else l."""
        c, w = self.cfg, self.w
        p = f"dec.{l}."
        g = 0 if c.G == 1 else l
        a = self.rnd(rms_norm(x, w[p + "xattn_norm"], c.rms_eps))
        q = self._heads(self._lin(a, w[p + "w_qc"]))              # [B, H, hd]
        Km = self._heads(M[g, 0][:, :t])                           # [B, t, H, hd]
        Vm = self._heads(M[g, 1][:, :t])
        sc = np.einsum("bhx,bjhx->bhj", q, Km) / np.sqrt(c.head_dim)
        o = np.einsum("bhj,bjhx->bhx", softmax(sc), Vm)
        o = self.rnd(self._merge_heads(o))
        return self._lin(o, w[p + "w_oc"])

    def ffn(self, l: int, x: np.ndarray) -> np.ndarray:
        """SwiGLU FFN tied to encoder layer l."""
        c, w = self.cfg, self.w
        p = f"layers.{l}."
        f = self.rnd(rms_norm(x, w[p + "ffn_norm"], c.rms_eps))
        m = self.rnd(silu(self._lin(f, w[p + "w_gate"])) * self._lin(f, w[p + "w_up"]))
        return self._lin(m, w[p + "w_down"])

    def head(self, s_t: np.ndarray, tau: float = 1.0) -> np.ndarray:
        """Next-token log-probabilities from s_t at temperature tau (reading R7)."""
        z = self._lin(self.rnd(s_t), self.w["unembed"]) / tau
        return log_softmax(z)

    def step(self, state: DecoderState, e_t: np.ndarray, M: np.ndarray, tau: float = 1.0,
             return_parts: bool = False):
        """H_{t-1}, e_t, M_{<=t} -> H_t, logp_t for every sequence of the batch.

        e_t: [B, d]; M: [G, 2, B, >=t, d] holding at least positions 1..t.
        Returns the new state and logp_t [B, V] (predicting x_{t+1})."""
        c = self.cfg
        t = state.t + 1
        x = self.merge(np.asarray(e_t, self.dt), state.s)
        new_cache = []
        parts = []
        for l in range(c.L_D):
            o, kv = self.swa(l, x, state, t)
            x = x + o
            if return_parts:
                parts.append(o)
            x = x + self.cross_attn(l, x, M, t)
            x = x + self.ffn(l, x)
            # push the current (k, v); keep the W-1 newest ([teardown] 2.3)
            keep = c.W - 1
            entries = state.cache[l] + [kv]
            new_cache.append(entries[max(0, len(entries) - keep):] if keep > 0 else [])
        s_t = rms_norm(x, self.w["dec_norm"], c.rms_eps)
        logp = self.head(s_t, tau)
        out = DecoderState(s=s_t, cache=new_cache, t=t)
        if return_parts:
            return out, logp, parts
        return out, logp

    # ---- exact current-policy replay: [news] model-RL principle; [review] section 4 ----

    def replay(self, tokens: np.ndarray, prompt_len, tau: float = 1.0):
        """Rebuild M, every SWA cache and s_t from the start, then score the
        response.  tokens int [B, T]; prompt_len P (int or [B]); 1 <= P <= T.

        Returns (score [B], logp_tok [B, T], s [B, T, d], final state):
          logp_tok[:, t-1] = log p(x_{t+1} | x_{<=t}) for t = 1..T-1 and 0 at t = T;
          score = sum over t = P .. T-1 of logp_tok[:, t-1]  (response x_{P+1..T}).
        """
        tokens = np.asarray(tokens)
        B, T = tokens.shape
        P = np.broadcast_to(np.asarray(prompt_len), (B,))
        e, M = self.encode(tokens)
        state = self.init_state(B)
        logp_tok = np.zeros((B, T), self.dt)
        s_all = np.zeros((B, T, self.cfg.d), self.dt)
        for t in range(1, T + 1):
            state, logp = self.step(state, e[:, t - 1], M, tau)
            s_all[:, t - 1] = state.s
            if t < T:
                logp_tok[:, t - 1] = logp[np.arange(B), tokens[:, t]]
        steps = np.arange(1, T + 1)
        scored = (steps[None, :] >= P[:, None]) & (steps[None, :] < T)
        score = np.sum(np.where(scored, logp_tok, 0.0), axis=1)
        return score, logp_tok, s_all, state

    def run(self, tokens: np.ndarray, tau: float = 1.0, steps: int | None = None):
        """Encode then step through the first `steps` tokens (default T).

        Returns e, M, s [B, n, d], logp [B, n, V]."""
        tokens = np.asarray(tokens)
        B, T = tokens.shape
        n = T if steps is None else steps
        e, M = self.encode(tokens[:, :n])
        state = self.init_state(B)
        s_all = np.zeros((B, n, self.cfg.d), self.dt)
        lp_all = np.zeros((B, n, self.cfg.V), self.dt)
        for t in range(1, n + 1):
            state, logp = self.step(state, e[:, t - 1], M, tau)
            s_all[:, t - 1] = state.s
            lp_all[:, t - 1] = logp
        return e, M, s_all, lp_all
