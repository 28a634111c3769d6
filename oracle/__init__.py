"""CPU oracle for the Recurrent Looped Transformer decoder transition.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the library.  It shares no code with the
CUDA path.  See rlt.py for the readings it takes and the passages it follows.
"""
from .rlt import (RLTOracle, DecoderState, round_bf16, rms_norm, rope, softmax, log_softmax,
                  silu, sigmoid, sample_token)

__all__ = ["RLTOracle", "DecoderState", "round_bf16", "rms_norm", "rope", "softmax",
           "log_softmax", "silu", "sigmoid", "sample_token"]
