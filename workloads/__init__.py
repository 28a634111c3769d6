"""Workload table and seeded input generators shared by the oracle, the tests and the bench."""
from .configs import (ModelConfig, Workload, WORKLOADS, TINY, SMALL, RLT_300M, REPLAY_24,
                      REF_48, REF_48_B1, decoder_param_count, total_param_count)
from .generate import weight_shapes, make_weight, make_weights, make_tokens, INIT_STD

__all__ = ["ModelConfig", "Workload", "WORKLOADS", "TINY", "SMALL", "RLT_300M", "REPLAY_24",
           "REF_48", "REF_48_B1", "decoder_param_count", "total_param_count", "weight_shapes",
           "make_weight", "make_weights", "make_tokens", "INIT_STD"]
