"""Python binding of librlt.so (the C ABI in include/rlt.h).

Argument marshalling only: PyTorch provides device memory and the current CUDA
stream; every step of the encoder, the decoder transition and the replay runs in
the library's kernels.  There is no CPU or PyTorch fallback: if the library is
missing or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import numpy as np
import torch

LIB_PATH = Path(__file__).resolve().parent / "librlt.so"

RLT_F32, RLT_BF16 = 0, 1
STATUS = {0: "RLT_OK", 1: "RLT_EINVAL", 2: "RLT_ECUDA", 3: "RLT_ESTALE", 4: "RLT_ETIMEOUT",
          5: "RLT_EUNSUPPORTED", 6: "RLT_EDEVICE", 7: "RLT_ESTATE"}


class RLTError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        self.status = STATUS.get(code, str(code))
        super().__init__(f"{what}: {self.status}")


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("V", "d", "n_heads", "head_dim", "L_E", "L_D", "F", "W", "G",
                                                "dtype")] + \
               [("rms_eps", ctypes.c_float), ("rope_base", ctypes.c_float), ("max_pos", ctypes.c_int32)]


_lib = None
_EXPORTS = {
    "rlt_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "rlt_weights_bytes": (ctypes.c_size_t, [ctypes.POINTER(Config)]),
    "rlt_model_create": (ctypes.c_int, [ctypes.POINTER(Config), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                        ctypes.POINTER(ctypes.c_void_p)]),
    "rlt_model_destroy": (None, [ctypes.c_void_p]),
    "rlt_model_set_weight": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_char_p, ctypes.c_void_p, ctypes.c_size_t,
                                            ctypes.c_void_p]),
    "rlt_model_commit": (ctypes.c_int, [ctypes.c_void_p]),
    "rlt_model_version": (ctypes.c_uint64, [ctypes.c_void_p]),
    "rlt_encode_workspace_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int]),
    "rlt_encode": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                  ctypes.c_void_p]),
    "rlt_encoder_cache_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int]),
    "rlt_encode_prefill": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "rlt_encode_append_workspace_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int]),
    "rlt_encode_append": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_void_p]),
    "rlt_sample": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                  ctypes.c_float, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "rlt_state_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int]),
    "rlt_state_positions_offset": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int]),
    "rlt_state_positions": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64)]),
    "rlt_state_reset_row": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "rlt_snapshot_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int]),
    "rlt_snapshot_save": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_void_p]),
    "rlt_snapshot_load": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_void_p]),
    "rlt_state_init": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "rlt_state_copy": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "rlt_state_position": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64)]),
    "rlt_state_release": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "rlt_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int]),
    "rlt_decode_step": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_float,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p]),
    "rlt_decode_step_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_float,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_void_p]),
    "rlt_replay_workspace_bytes": (ctypes.c_size_t, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int]),
    "rlt_replay": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                  ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "rlt_last_error": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "rlt_launch_count": (ctypes.c_uint64, [ctypes.c_void_p]),
    "rlt_gemm_bf16": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "rlt_gemm_plan": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "rlt_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_uint64, ctypes.c_void_p]),
    "rlt_set_option": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_char_p, ctypes.c_int64]),
    "rlt_profile_start": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_uint32]),
    "rlt_profile_stop": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_uint64)]),
}

KERNEL_KINDS = ["norm", "merge", "qkv", "swa", "o_proj", "qc_proj", "xattn", "oc_proj", "ffn_up", "ffn_down",
                "final_norm", "head", "lse", "encoder", "small_step", "enc_gemm", "enc_attn", "enc_other"]


def lib() -> ctypes.CDLL:
    """Load librlt.so (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m cross_token_latent_b200.build`")
        h = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in _EXPORTS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def exported_names() -> list[str]:
    return list(_EXPORTS)


def gemm_plan(M: int, N: int, K: int) -> int:
    """Kernel id (as rlt_gemm_bf16 numbers them) the library picks for an M x N x K bf16 product."""
    return lib().rlt_gemm_plan(M, N, K)


def _check(code: int, what: str) -> None:
    if code != 0:
        raise RLTError(code, what)


def _ptr(t) -> ctypes.c_void_p | None:
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def make_config(cfg, max_pos: int) -> Config:
    """cfg: any object with the ModelConfig fields (V, d, n_heads, ..., dtype 'f32'|'bf16')."""
    return Config(cfg.V, cfg.d, cfg.n_heads, cfg.head_dim, cfg.L_E, cfg.L_D, cfg.F, cfg.W, cfg.G,
                  RLT_BF16 if cfg.dtype == "bf16" else RLT_F32, float(cfg.rms_eps), float(cfg.rope_base),
                  int(max_pos))


class RLTState:
    """A caller-owned decoder state buffer H (registered with its model)."""

    def __init__(self, model: "RLTModel", B: int, buf: torch.Tensor):
        self.model, self.B, self.buf = model, B, buf

    @property
    def position(self) -> int:
        t = ctypes.c_int64()
        _check(lib().rlt_state_position(self.model.handle, _ptr(self.buf), ctypes.byref(t)), "rlt_state_position")
        return t.value

    def s(self) -> torch.Tensor:
        """View of s_t [B, d] float32 inside the state buffer."""
        d = self.model.cfg.d
        return self.buf[256:256 + self.B * d * 4].view(torch.float32).view(self.B, d)

    def positions(self) -> list[int]:
        """Tokens consumed by every sequence (host registry)."""
        out = (ctypes.c_int64 * self.B)()
        _check(lib().rlt_state_positions(self.model.handle, _ptr(self.buf), out), "rlt_state_positions")
        return list(out)

    def positions_device(self) -> torch.Tensor:
        """View of the state's int32 [B] device positions (what rlt_encode_append takes)."""
        off = lib().rlt_state_positions_offset(self.model.handle, self.B)
        return self.buf[off:off + 4 * self.B].view(torch.int32)

    def reset_row(self, row: int) -> None:
        _check(lib().rlt_state_reset_row(self.model.handle, _ptr(self.buf), int(row), _stream()), "rlt_state_reset_row")

    def copy(self) -> "RLTState":
        other = torch.empty_like(self.buf)
        _check(lib().rlt_state_copy(self.model.handle, _ptr(other), _ptr(self.buf), _stream()), "rlt_state_copy")
        return RLTState(self.model, self.B, other)

    def __del__(self):
        try:
            if self.model.handle:
                lib().rlt_state_release(self.model.handle, _ptr(self.buf))
        except Exception:
            pass


class RLTModel:
    """One model on one CUDA device: weight arena, encoder, decoder step and replay."""

    def __init__(self, cfg, max_pos: int, device: str | torch.device = "cuda"):
        if not torch.cuda.is_available():
            raise RuntimeError("RLTModel needs a CUDA device")
        self.cfg = cfg
        self.device = torch.device(device)
        self.max_pos = int(max_pos)
        self.sdtype = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        self._c = make_config(cfg, max_pos)
        nbytes = lib().rlt_weights_bytes(ctypes.byref(self._c))
        if nbytes == 0:
            raise RLTError(1, "rlt_weights_bytes (config rejected)")
        self.arena = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        _check(lib().rlt_model_create(ctypes.byref(self._c), _ptr(self.arena), nbytes, _stream(), ctypes.byref(h)),
               "rlt_model_create")
        self.handle = h
        self._ws: dict = {}
        self._destroy = lib().rlt_model_destroy    # held so that teardown at exit still reaches it

    def __del__(self):
        h = getattr(self, "handle", None)
        destroy = getattr(self, "_destroy", None)
        if h and destroy is not None:
            destroy(h)
            self.handle = None

    # ---------------------------------------------------------------- weights
    def set_weight(self, name: str, value) -> None:
        t = torch.as_tensor(np.ascontiguousarray(value, dtype=np.float32) if isinstance(value, np.ndarray) else value)
        t = t.to(device=self.device, dtype=torch.float32).contiguous()
        _check(lib().rlt_model_set_weight(self.handle, name.encode(), _ptr(t), t.numel(), _stream()),
               f"rlt_model_set_weight({name})")
        self._keep = t     # the copy is stream-ordered; keep the source alive until the next call

    def load_weights(self, weights: dict) -> None:
        for name, value in weights.items():
            self.set_weight(name, value)
        _check(lib().rlt_model_commit(self.handle), "rlt_model_commit")
        torch.cuda.current_stream().synchronize()
        self._keep = None

    def set_option(self, name: str, value: int) -> None:
        """Scheduling option of the handle (rlt_set_option): "row_groups", "group_attn_ctas_per_sm",
        "group_pdl"."""
        _check(lib().rlt_set_option(self.handle, name.encode(), int(value)), f"rlt_set_option({name})")

    @property
    def version(self) -> int:
        return lib().rlt_model_version(self.handle)

    @property
    def launch_count(self) -> int:
        return lib().rlt_launch_count(self.handle)

    def _workspace(self, key, nbytes: int) -> torch.Tensor:
        buf = self._ws.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            self._ws[key] = buf
        return buf

    def release_workspaces(self) -> None:
        self._ws.clear()

    # ---------------------------------------------------------------- encoder
    def alloc_encoder_outputs(self, B: int, T_alloc: int):
        c = self.cfg
        e = torch.empty((B, T_alloc, c.d), dtype=self.sdtype, device=self.device)
        M = torch.empty((c.G, 2, B, c.n_heads, T_alloc, c.head_dim), dtype=self.sdtype, device=self.device)
        return e, M

    def encode(self, tokens: torch.Tensor, T_alloc: int | None = None, out=None):
        """tokens int32 [B, T] on the device -> (e [B, T_alloc, d], M [G, 2, B, H, T_alloc, hd])."""
        tokens = tokens.to(device=self.device, dtype=torch.int32).contiguous()
        B, T = tokens.shape
        T_alloc = T if T_alloc is None else T_alloc
        e, M = out if out is not None else self.alloc_encoder_outputs(B, T_alloc)
        nb = lib().rlt_encode_workspace_bytes(self.handle, B, T)
        ws = self._workspace(("enc", B, T), nb)
        _check(lib().rlt_encode(self.handle, _ptr(tokens), B, T, T_alloc, _ptr(e), _ptr(M), _ptr(ws), ws.numel(),
                                _stream()), "rlt_encode")
        return e, M

    # ---------------------------------------------------------------- incremental encoder
    def alloc_encoder_cache(self, B: int, T_max: int) -> torch.Tensor:
        return torch.empty(lib().rlt_encoder_cache_bytes(self.handle, B, T_max), dtype=torch.uint8,
                           device=self.device)

    def encode_prefill(self, tokens: torch.Tensor, T_alloc: int, T_max: int | None = None, out=None, cache=None):
        """rlt_encode_prefill: (e, M, encoder cache) of the first T tokens, capacities T_alloc / T_max."""
        tokens = tokens.to(device=self.device, dtype=torch.int32).contiguous()
        B, T = tokens.shape
        T_max = T_alloc if T_max is None else T_max
        e, M = out if out is not None else self.alloc_encoder_outputs(B, T_alloc)
        cache = self.alloc_encoder_cache(B, T_max) if cache is None else cache
        nb = lib().rlt_encode_workspace_bytes(self.handle, B, T)
        ws = self._workspace(("enc", B, T), nb)
        _check(lib().rlt_encode_prefill(self.handle, _ptr(tokens), B, T, T_alloc, _ptr(e), _ptr(M), _ptr(cache), T_max,
                                        _ptr(ws), ws.numel(), _stream()), "rlt_encode_prefill")
        return e, M, cache

    def encode_append(self, tokens: torch.Tensor, pos: int, cache: torch.Tensor, T_max: int, e: torch.Tensor,
                      M: torch.Tensor, positions: torch.Tensor | None = None) -> None:
        """rlt_encode_append: tokens is an int32 device vector [B] or a column view of a [B, T]
        matrix (its stride is passed through); the token at position pos is encoded, or with
        `positions` (int32 device [B], e.g. RLTState.positions_device()) sequence b's token at
        positions[b] <= pos."""
        B = tokens.shape[0]
        stride = tokens.stride(0)
        nb = lib().rlt_encode_append_workspace_bytes(self.handle, B)
        ws = self._workspace(("app", B), nb)
        _check(lib().rlt_encode_append(self.handle, _ptr(tokens), stride, B, int(pos), _ptr(positions), _ptr(cache),
                                       int(T_max), _ptr(e), _ptr(M), e.shape[1], _ptr(ws), ws.numel(), _stream()),
               "rlt_encode_append")

    # ---------------------------------------------------------------- sequence snapshots
    def snapshot_save(self, state: "RLTState", row: int, M: torch.Tensor, cache: torch.Tensor | None = None,
                      T_max: int = 0) -> torch.Tensor:
        """rlt_snapshot_save of sequence `row` into a new device buffer."""
        t = state.positions()[row]
        buf = torch.empty(lib().rlt_snapshot_bytes(self.handle, t), dtype=torch.uint8, device=self.device)
        _check(lib().rlt_snapshot_save(self.handle, _ptr(state.buf), int(row), _ptr(cache), int(T_max), _ptr(M),
                                       M.shape[4], _ptr(buf), buf.numel(), _stream()), "rlt_snapshot_save")
        return buf

    def snapshot_load(self, snap: torch.Tensor, state: "RLTState", row: int, M: torch.Tensor,
                      cache: torch.Tensor | None = None, T_max: int = 0) -> None:
        _check(lib().rlt_snapshot_load(self.handle, _ptr(snap), _ptr(state.buf), int(row), _ptr(cache), int(T_max),
                                       _ptr(M), M.shape[4], _stream()), "rlt_snapshot_load")

    def sample(self, logp: torch.Tensor, u: torch.Tensor, top_k: int = 0, top_p: float = 1.0,
               out: torch.Tensor | None = None, behaviour_logp: torch.Tensor | None = None) -> torch.Tensor:
        """rlt_sample: one token per row of logp [B, V] with the uniforms u [B]; `out` may be a
        column view of a token matrix (its stride is passed through)."""
        B = logp.shape[0]
        out = torch.empty(B, dtype=torch.int32, device=self.device) if out is None else out
        _check(lib().rlt_sample(self.handle, _ptr(logp), B, _ptr(u), int(top_k), float(top_p), _ptr(out),
                                out.stride(0), _ptr(behaviour_logp), _stream()), "rlt_sample")
        return out

    def generate(self, prompt: torch.Tensor, n_new: int, uniforms: torch.Tensor, tau: float = 1.0, top_k: int = 0,
                 top_p: float = 1.0):
        """Sample n_new tokens after each prompt row (all rows in lockstep): encode the prompt with a
        cache, step the decoder through it, then repeat [sample x_{t+1} from logp_t, encode it
        incrementally, step].  uniforms: float device [n_new, B].  Returns (tokens [B, P + n_new]
        int32, behaviour log-probs [B, n_new], prompt log-probs [B, P - 1] (entry t-1 = log p of
        x_{t+1}), the state after all P + n_new tokens).  Every step of the loop runs in the
        library's kernels; nothing is copied to the host."""
        prompt = prompt.to(device=self.device, dtype=torch.int32).contiguous()
        B, P = prompt.shape
        T = P + n_new
        toks = torch.empty((T, B), dtype=torch.int32, device=self.device)     # row t = x_{t+1}
        toks[:P] = prompt.t()
        e, M, cache = self.encode_prefill(prompt, T_alloc=T, T_max=T)
        st = self.new_state(B)
        blp = torch.empty((n_new, B), dtype=torch.float32, device=self.device)
        lp_prompt = torch.zeros((max(P - 1, 0), B), dtype=torch.float32, device=self.device)
        row = torch.empty((B, self.cfg.V), dtype=torch.float32, device=self.device)
        for t in range(1, T):                      # step t consumes x_t and predicts x_{t+1}
            if t < P:
                self.decode_step(st, e, M, next_tok=toks[t], tau=tau, logp_tok=lp_prompt[t - 1])
                continue
            self.decode_step(st, e, M, tau=tau, logp_full=row)
            self.sample(row, uniforms[t - P], top_k, top_p, out=toks[t], behaviour_logp=blp[t - P])
            self.encode_append(toks[t], t, cache, T, e, M)
        self.decode_step(st, e, M, tau=tau)         # the transition of x_T
        return toks.t().contiguous(), blp.t().contiguous(), lp_prompt.t().contiguous(), st

    # ---------------------------------------------------------------- decoder
    def new_state(self, B: int) -> RLTState:
        buf = torch.empty(lib().rlt_state_bytes(self.handle, B), dtype=torch.uint8, device=self.device)
        _check(lib().rlt_state_init(self.handle, _ptr(buf), B, _stream()), "rlt_state_init")
        return RLTState(self, B, buf)

    def reset_state(self, state: RLTState) -> RLTState:
        _check(lib().rlt_state_init(self.handle, _ptr(state.buf), state.B, _stream()), "rlt_state_init")
        return state

    def decode_step(self, state: RLTState, e: torch.Tensor, M: torch.Tensor, next_tok: torch.Tensor | None = None,
                    tau: float = 1.0, logp_tok: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                    logp_full: torch.Tensor | None = None) -> None:
        """One transition H_{t-1} -> H_t in place; outputs go to the given device tensors."""
        B = state.B
        nb = lib().rlt_decode_workspace_bytes(self.handle, B)
        ws = self._workspace(("dec", B), nb)
        _check(lib().rlt_decode_step(self.handle, _ptr(state.buf), B, _ptr(e), _ptr(M), e.shape[1], _ptr(next_tok),
                                     float(tau), _ptr(logp_tok), _ptr(lse), _ptr(logp_full), _ptr(ws), ws.numel(),
                                     _stream()), "rlt_decode_step")

    def decode_step_noalloc(self, state: RLTState, e: torch.Tensor, M: torch.Tensor,
                            next_tok: torch.Tensor | None = None, tau: float = 1.0,
                            logp_tok: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                            logp_full: torch.Tensor | None = None) -> None:
        """rlt_decode_step without a caller workspace: the step's scratch is the library's static
        device array (see include/rlt.h for its size limit and the rules on overlapping calls)."""
        _check(lib().rlt_decode_step_noalloc(self.handle, _ptr(state.buf), state.B, _ptr(e), _ptr(M), e.shape[1],
                                             _ptr(next_tok), float(tau), _ptr(logp_tok), _ptr(lse), _ptr(logp_full),
                                             _stream()), "rlt_decode_step_noalloc")

    def replay(self, tokens: torch.Tensor, prompt_len, tau: float = 1.0, want_logp: bool = False,
               want_state: bool = False):
        """Exact current-policy replay; returns (score [B], logp_tok [B, T] | None, state | None)."""
        tokens = tokens.to(device=self.device, dtype=torch.int32).contiguous()
        B, T = tokens.shape
        P = torch.as_tensor(prompt_len, dtype=torch.int32).to(self.device).expand(B).contiguous()
        score = torch.empty(B, dtype=torch.float32, device=self.device)
        lp = torch.empty((B, T), dtype=torch.float32, device=self.device) if want_logp else None
        st = None
        if want_state:
            st = RLTState(self, B, torch.empty(lib().rlt_state_bytes(self.handle, B), dtype=torch.uint8,
                                               device=self.device))
        nb = lib().rlt_replay_workspace_bytes(self.handle, B, T)
        ws = self._workspace(("replay", B, T), nb)
        _check(lib().rlt_replay(self.handle, _ptr(tokens), B, T, _ptr(P), float(tau), _ptr(score), _ptr(lp),
                                _ptr(st.buf) if st else None, _ptr(ws), ws.numel(), _stream()), "rlt_replay")
        return score, lp, st

    def gemm_bf16(self, A: torch.Tensor, W: torch.Tensor, kernel: int = 0,
                  out: torch.Tensor | None = None) -> torch.Tensor:
        """C = A W^T (bf16 in, float32 out) with the kernel id of rlt_gemm_bf16 (0: the library's
        choice, 1: CUDA cores, 2 + v: row-tile variant v, 11 + s: few-row kernel, 16: weight
        streaming, 17: persistent, 18 + p: CTA-pair tiles 256 x (64 << p))."""
        A = A.to(self.device, torch.bfloat16).contiguous()
        W = W.to(self.device, torch.bfloat16).contiguous()
        M, K = A.shape
        N = W.shape[0]
        C = torch.empty((M, N), dtype=torch.float32, device=self.device) if out is None else out
        _check(lib().rlt_gemm_bf16(self.handle, _ptr(A), _ptr(W), _ptr(C), M, N, K, kernel, _stream()),
               "rlt_gemm_bf16")
        return C

    def selftest_wait_timeout(self, A: torch.Tensor, W: torch.Tensor, C: torch.Tensor, kernel: int,
                              wait_ns: int) -> None:
        """Launch tensor-core kernel `kernel` in its no-load self-test mode (every wait bounded by
        wait_ns); the next last_error() reports RLT_ETIMEOUT."""
        M, K = A.shape
        N = W.shape[0]
        _check(lib().rlt_selftest_wait_timeout(self.handle, _ptr(A), _ptr(W), _ptr(C), M, N, K, kernel,
                                               int(wait_ns), _stream()), "rlt_selftest_wait_timeout")

    def profile_start(self, kinds=None) -> None:
        """Bracket every launch of the given kernel kinds (names of KERNEL_KINDS) with CUDA events."""
        kinds = KERNEL_KINDS if kinds is None else kinds
        mask = 0
        for k in kinds:
            mask |= 1 << KERNEL_KINDS.index(k)
        _check(lib().rlt_profile_start(self.handle, mask), "rlt_profile_start")

    def profile_stop(self) -> dict:
        """Per kind: (summed milliseconds, bracketed launches)."""
        n = len(KERNEL_KINDS)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_uint64 * n)()
        _check(lib().rlt_profile_stop(self.handle, ms, cnt), "rlt_profile_stop")
        return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS) if cnt[i]}

    def last_error(self) -> int:
        return lib().rlt_last_error(self.handle, _stream())

    def check_device_errors(self) -> None:
        _check(self.last_error(), "device-side check")
