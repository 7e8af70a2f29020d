"""The bench's reference arm (CPU): the line it prints carries the keys of the
bench's JSON contract, the same config object as the GPU arm, and a step time
and rate that agree with the sample it describes."""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS  # noqa: E402


def test_reference_line_contract():
    args = argparse.Namespace(workload="prefill_L4096", warmup=1, steps=2, ref_step_s=0.5)
    line = bench.run_reference(args, 1, 0)
    json.loads(json.dumps(line))            # one JSON object
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["config"] == bench.workload_config(WORKLOADS[1], 1)
    assert line["value"] > 0
    # a step is a bounded sample: at least its sampling budget, and at least
    # the time the rate implies for the rows it took
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"]
    assert "query rows of prefill_L4096" in cpu["sample"]
    assert line["ms_per_step"] >= 0.5e3
    e2e = line["e2e"]
    assert e2e == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}


def test_workload_config_names_the_workload():
    for i in (1, 2, 3):
        wl = WORKLOADS[i]
        c = bench.workload_config(wl, 2)
        assert c["workload"] == wl.name and c["L"] == wl.L and c["k"] == wl.k
        assert c["parallelism"] == "replicas x2 (independent sequences)"
        q_gb = wl.L * 128 * 576 * 2 / 1e9
        assert f"{q_gb:.1f} GB" in c["l2"] and q_gb * 1e9 > 126e6   # q alone exceeds L2
