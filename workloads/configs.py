"""Model and workload table for the Recurrent Looped Transformer decoder transition.

Only numbers live here: model shapes, window, memory-group count, batch, length,
prompt split, temperature and the token distribution to draw from.  No part of
the method's arithmetic is in this module; both the CPU oracle and the CUDA
library are fed from it.

Shapes follow the notation of "Recurrent Looped Transformer" as summarised on the
feinterview news page (encoder and memory M, decoder state H_t = (s_t, C_t^D),
window W, memory groups G) and the deepsonar teardown (section 2.3, the state and
cache definition).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace


@dataclass(frozen=True)
class ModelConfig:
    """Architecture of one encoder/decoder pair.

    V          vocabulary size
    d          model width
    n_heads    attention heads (no grouped KV)
    head_dim   per-head width, n_heads * head_dim == d
    L_E, L_D   encoder and decoder depths (decoder layer l reuses encoder layer l)
    F          SwiGLU hidden width
    W          sliding window, counting the current token (the cache keeps W-1)
    G          encoder-memory groups: 1 (shared by every decoder layer) or L_D
    dtype      "f32" or "bf16" (storage type of weights, e, M and the SWA cache)
    """

    V: int
    d: int
    n_heads: int
    head_dim: int
    L_E: int
    L_D: int
    F: int
    W: int
    G: int
    dtype: str
    rms_eps: float = 1e-6
    rope_base: float = 10000.0

    def __post_init__(self):
        if self.n_heads * self.head_dim != self.d:
            raise ValueError("n_heads * head_dim must equal d")
        if self.G not in (1, self.L_D):
            raise ValueError("G must be 1 or L_D")
        if self.L_E != self.L_D:
            raise ValueError("weight tying needs L_E == L_D")
        if self.dtype not in ("f32", "bf16"):
            raise ValueError("dtype must be f32 or bf16")
        if self.W < 1 or self.head_dim % 2:
            raise ValueError("W >= 1 and an even head_dim are required")


@dataclass(frozen=True)
class Workload:
    """A model plus the batch it is run on."""

    name: str
    model: ModelConfig
    B: int
    T: int
    prompt_len: int
    tau: float
    tokens: str            # "uniform" | "markov2" | "zipf"
    token_seed: int
    weight_seed: int = 0
    zipf_s: float = 1.1
    dirichlet_alpha: float = 0.1
    notes: str = field(default="", compare=False)

    def with_batch(self, B: int, T: int | None = None) -> "Workload":
        T = self.T if T is None else T
        return replace(self, B=B, T=T, prompt_len=min(self.prompt_len, T))


TINY = Workload(
    name="tiny-f32",
    model=ModelConfig(V=256, d=64, n_heads=4, head_dim=16, L_E=2, L_D=2, F=256,
                      W=4, G=1, dtype="f32"),
    B=2, T=64, prompt_len=24, tau=1.0, tokens="uniform", token_seed=1,
    notes="vocab 256, d=64, 4x16 heads, 2+2 layers, W=4, G=1, fp32")

SMALL = Workload(
    name="small-bf16",
    model=ModelConfig(V=512, d=128, n_heads=4, head_dim=32, L_E=4, L_D=4, F=512,
                      W=16, G=4, dtype="bf16"),
    B=64, T=512, prompt_len=128, tau=1.0, tokens="markov2", token_seed=2,
    notes="vocab 512, d=128, 4x32 heads, 4+4 layers, W=16, G=L_D, order-2 Markov tokens")

RLT_300M = Workload(
    name="300m-12+12-b512",
    model=ModelConfig(V=32000, d=1024, n_heads=16, head_dim=64, L_E=12, L_D=12,
                      F=4096, W=128, G=1, dtype="bf16"),
    B=512, T=1024, prompt_len=1024, tau=1.0, tokens="zipf", token_seed=3,
    notes="300M-class 12+12, B=512 x T=1024, Zipf(1.1) tokens, lockstep decode")

REPLAY_24 = Workload(
    name="replay-24+24-b64",
    model=ModelConfig(V=32768, d=2048, n_heads=16, head_dim=128, L_E=24, L_D=24,
                      F=5632, W=256, G=24, dtype="bf16"),
    B=64, T=2048, prompt_len=512, tau=0.8, tokens="zipf", token_seed=4,
    notes="RL replay scoring: 512 prompt + 1536 response tokens, tau 0.8")

REF_48 = Workload(
    name="ref-48+48-b32",
    model=ModelConfig(V=32768, d=2048, n_heads=16, head_dim=128, L_E=48, L_D=48,
                      F=5632, W=512, G=1, dtype="bf16"),
    B=32, T=4096, prompt_len=2048, tau=1.0, tokens="zipf", token_seed=5,
    notes="tied 48+48 reference model, 2048 prompt + 2048 response")

REF_48_B1 = replace(REF_48, name="ref-48+48-b1", B=1,
                    notes="latency-bound single-sequence decode of the 48+48 model")

WORKLOADS = {w.name: w for w in (TINY, SMALL, RLT_300M, REPLAY_24, REF_48, REF_48_B1)}


def decoder_param_count(m: ModelConfig) -> int:
    """Weights read by one decode step: tied self-attention (4d^2), cross q/o (2d^2),
    SwiGLU (3dF) per layer, the merge (3d^2) and the LM head (V d)."""
    return m.L_D * (6 * m.d * m.d + 3 * m.d * m.F) + 3 * m.d * m.d + m.V * m.d


def total_param_count(m: ModelConfig) -> int:
    enc = m.L_E * (4 * m.d * m.d + 3 * m.d * m.F) + m.V * m.d
    mem = m.G * 2 * m.d * m.d
    dec_extra = m.L_D * 2 * m.d * m.d + 3 * m.d * m.d + m.V * m.d + 2 * m.d
    return enc + mem + dec_extra
