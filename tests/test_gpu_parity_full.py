"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: one layer per workload, every row run on the device, sampled rows
checked against the oracle through prefill, the initial pack and one full
reassignment interval of decode steps."""
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
def test_full_size_sampled_rows(cuda, wl, rows):
    s = run_scenario(wl, wl.reassign_interval, cuda, rows=rows)
    print(wl.name, s)
