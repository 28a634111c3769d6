"""B200-native (sm_100a) library of the Recurrent Looped Transformer decoder transition.

The compute lives in librlt.so (C ABI, include/rlt.h); this package is its thin
Python binding plus the in-tree build script.
"""
from .rlt import (RLTModel, RLTState, RLTError, lib, exported_names, make_config, LIB_PATH,
                  RLT_F32, RLT_BF16)

__all__ = ["RLTModel", "RLTState", "RLTError", "lib", "exported_names", "make_config", "LIB_PATH",
           "RLT_F32", "RLT_BF16"]
