"""The C-ABI library loads and exports every entry point include/rlt.h declares (no GPU)."""
import ctypes
import re
from pathlib import Path

import pytest

from cross_token_latent_b200 import LIB_PATH, exported_names, lib, make_config
from workloads import WORKLOADS, TINY

ROOT = Path(__file__).resolve().parent.parent


def declared_functions():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        text = h.read_text()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(rlt_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_is_built_in_tree():
    assert LIB_PATH.exists() and LIB_PATH.parent.name == "cross_token_latent_b200"


def test_every_declared_symbol_is_exported():
    h = ctypes.CDLL(str(LIB_PATH))
    declared = declared_functions()
    assert len(declared) >= 19
    for name in declared:
        assert hasattr(h, name), name
    # the binding wraps every declared entry point
    assert set(declared) <= set(exported_names()), set(declared) - set(exported_names())


def test_status_strings():
    L = lib()
    for code in range(8):
        assert L.rlt_status_string(code)
    assert L.rlt_status_string(0) == b"ok"


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_weights_bytes_cover_the_model(name):
    w = WORKLOADS[name]
    m = w.model
    c = make_config(m, w.T)
    nbytes = lib().rlt_weights_bytes(ctypes.byref(c))
    esz = 2 if m.dtype == "bf16" else 4
    d, F, V = m.d, m.F, m.V
    mats = V * d * 2 + m.L_E * (4 * d * d + 3 * d * F) + m.G * 2 * d * d + m.L_D * 2 * d * d + 4 * d * d
    assert nbytes >= mats * esz
    assert nbytes < mats * esz * 1.05 + (1 << 24)


def test_invalid_configs_are_rejected_on_the_host():
    m = TINY.model
    bad = [dict(head_dim=24), dict(G=3), dict(W=0), dict(dtype=5), dict(d=60), dict(L_E=3)]
    for kw in bad:
        c = make_config(m, 64)
        for k, v in kw.items():
            setattr(c, k, v)
        assert lib().rlt_weights_bytes(ctypes.byref(c)) == 0, kw
    c = make_config(m, 64)
    c.max_pos = 0
    assert lib().rlt_weights_bytes(ctypes.byref(c)) == 0
    # model creation refuses a NULL arena before touching the device
    out = ctypes.c_void_p()
    c = make_config(m, 64)
    assert lib().rlt_model_create(ctypes.byref(c), None, 1 << 20, None, ctypes.byref(out)) == 1


def test_null_handles_are_rejected():
    L = lib()
    assert L.rlt_decode_workspace_bytes(None, 4) == 0
    assert L.rlt_state_bytes(None, 4) == 0
    assert L.rlt_decode_step(None, None, 1, None, None, 1, None, 1.0, None, None, None, None, 0, None) == 1
    assert L.rlt_replay(None, None, 1, 1, None, 1.0, None, None, None, None, 0, None) == 1
    assert L.rlt_launch_count(None) == 0
    assert L.rlt_encoder_cache_bytes(None, 4, 16) == 0
    assert L.rlt_encode_append_workspace_bytes(None, 4) == 0
    assert L.rlt_encode_prefill(None, None, 1, 1, 1, None, None, None, 1, None, 0, None) == 1
    assert L.rlt_encode_append(None, None, 1, 1, 0, None, None, 1, None, None, 1, None, 0, None) == 1
    assert L.rlt_state_positions_offset(None, 4) == 0
    assert L.rlt_snapshot_bytes(None, 4) == 0
    assert L.rlt_state_reset_row(None, None, 0, None) == 1
    assert L.rlt_snapshot_save(None, None, 0, None, 1, None, 1, None, 0, None) == 1
    assert L.rlt_snapshot_load(None, None, None, 0, None, 1, None, 1, None) == 1
    assert L.rlt_sample(None, None, 1, None, 0, 1.0, None, 1, None, None) == 1
    assert L.rlt_set_option(None, b"row_groups", 1) == 1
    assert L.rlt_selftest_wait_timeout(None, None, None, None, 1, 1, 8, 2, 1000000, None) == 1
    # the GEMM building block: every kernel id (0-20) and one past the last
    for k in (0, 17, 18, 20, 21):
        assert L.rlt_gemm_bf16(None, None, None, None, 8, 8, 8, k, None) == 1
        assert L.rlt_selftest_wait_timeout(None, None, None, None, 8, 8, 8, k, 1000000, None) == 1
