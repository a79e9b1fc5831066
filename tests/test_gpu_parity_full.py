"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times, over each workload's whole decode length: one layer per
workload, every row run on the device, sampled rows checked against the oracle
through prefill, the initial pack and every decode step (attention output and
scores every step, tiers, codes and scales at every reassignment).  Each
reassignment interval prints one PARITY line with the largest output and score
errors seen in it and the number of near-cut tokens exempted."""
import pytest

from mixed_precision_kv_arkv_b200 import workloads
from tests.test_gpu_parity import run_scenario

pytestmark = pytest.mark.gpu

CASES = [
    (workloads.LLAMA3_3B, [0, 7]),
    (workloads.LLAMA3_8B, [0, 31]),
    (workloads.QWEN3_8B, [3]),
    (workloads.RAGGED, [0, 133, 255]),
]


@pytest.mark.parametrize("wl,rows", CASES, ids=[w.name for w, _ in CASES])
def test_full_size_whole_decode_length(cuda, wl, rows):
    s = run_scenario(wl, wl.steps, cuda, rows=rows)
    assert len(s["log"]) == wl.steps // wl.reassign_interval
    print(wl.name, {k: v for k, v in s.items() if k != "log"})
