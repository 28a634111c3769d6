"""The benchmark's cost model (CPU): bench.py's per-step roofline against values derived
independently for the five workloads (roofline decoder tokens/s = B*T / run roofline with the
measured 6544 GB/s and 1665.9 TFLOP/s), and the shape of the stricter shared-memory bound."""
import sys
from pathlib import Path

import pytest

sys.path.insert(0, str(Path(__file__).resolve().parents[1]))

import bench  # noqa: E402
from workloads import WORKLOADS  # noqa: E402

PEAKS = {"hbm_gbs": 6544.0, "bf16_tflops": 1665.9}

# roofline decoder tokens/s of each workload, derived by hand from the byte / FLOP formulas
EXPECTED_TOK_S = {
    "small-bf16": 10.9e6,
    "300m-12+12-b512": 203.7e3,
    "replay-24+24-b64": 22.1e3,
    "ref-48+48-b32": 5.55e3,
    "ref-48+48-b1": 950.0,
}


@pytest.mark.parametrize("name", sorted(EXPECTED_TOK_S))
def test_run_roofline_matches_the_derived_table(name):
    wl = WORKLOADS[name]
    tok_s = wl.B * wl.T / bench.run_roofline_s(wl.model, wl.B, wl.T, PEAKS)
    assert tok_s == pytest.approx(EXPECTED_TOK_S[name], rel=6e-3)


def test_step_cost_of_the_300m_workload_by_its_parts():
    """Per-token bytes at t = T for B = 512: weights / B + the full SWA window + M_{<=T} once per
    layer; step FLOPs: 2 per weight and sequence plus the attention terms."""
    wl = WORKLOADS["300m-12+12-b512"]
    m, B, T = wl.model, wl.B, wl.T
    nbytes, flops = bench.step_cost(m, B, T)
    P = 262.4e6                                  # decoder weights read per step
    ring = m.L_D * (m.W - 1) * 2 * m.d * 2       # 127 cached k/v entries per layer
    cur = m.L_D * 2 * m.d * 2                    # the current k/v written
    mem = m.L_D * T * 2 * m.d * 2                # M_{<=T} read by every layer
    per_seq = ring + cur + mem + m.d * 2
    assert nbytes == pytest.approx(P * 2 + B * per_seq, rel=1e-3)
    assert flops == pytest.approx(B * (2 * P + m.L_D * 4 * m.d * (m.W + T)), rel=1e-3)


def test_shared_memory_bound_is_stricter_only_for_a_shared_memory():
    shared = WORKLOADS["300m-12+12-b512"]        # G = 1
    per_layer = WORKLOADS["replay-24+24-b64"]    # G = L_D
    a = bench.run_roofline_s(shared.model, shared.B, shared.T, PEAKS)
    a1 = bench.run_roofline_s(shared.model, shared.B, shared.T, PEAKS, m_once=True)
    assert a1 < a / 3
    b = bench.run_roofline_s(per_layer.model, per_layer.B, per_layer.T, PEAKS)
    b1 = bench.run_roofline_s(per_layer.model, per_layer.B, per_layer.T, PEAKS, m_once=True)
    assert b1 == b


# encoder FLOPs of each workload, derived by hand (linear maps + causal attention), in TFLOP
EXPECTED_ENCODE_TF = {"300m-12+12-b512": 227.0, "replay-24+24-b64": 402.0, "ref-48+48-b32": 754.0,
                      "ref-48+48-b1": 23.6}


@pytest.mark.parametrize("name", sorted(EXPECTED_ENCODE_TF))
def test_encode_flops_match_the_derived_table(name):
    wl = WORKLOADS[name]
    assert bench.encode_flops(wl.model, wl.B, wl.T) / 1e12 == pytest.approx(EXPECTED_ENCODE_TF[name], rel=4e-3)


def test_encode_flops_of_one_token_is_two_per_weight_plus_its_self_attention():
    m = WORKLOADS["tiny-f32"].model
    per_weight = 2.0 * (m.L_E * (4 * m.d * m.d + 3 * m.d * m.F) + m.G * 2 * m.d * m.d)
    assert bench.encode_flops(m, 1, 1) == per_weight + 4.0 * m.L_E * m.d
