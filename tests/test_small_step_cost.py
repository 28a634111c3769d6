"""The bench's algorithmic bytes of the one-launch small-model step equal the step roofline's
bytes summed over the sweep (CPU)."""
import sys
from pathlib import Path

sys.path.insert(0, str(Path(__file__).resolve().parents[1]))

import bench  # noqa: E402
from workloads import WORKLOADS  # noqa: E402


def test_small_step_bytes_are_the_sweeps_step_bytes():
    wl = WORKLOADS["small-bf16"]
    m, B, T = wl.model, wl.B, wl.T
    bound, nbytes = bench.kind_cost("small_step", m, B, T)
    assert bound == "hbm"
    assert nbytes == sum(bench.step_cost(m, B, t)[0] for t in range(1, T + 1))
