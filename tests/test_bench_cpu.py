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


def _smi(sm, util, reasons=(), mx=1965, power=900):
    """One nvidia-smi line of Clocks.FIELDS (csv, noheader, nounits)."""
    act = ["Active" if n in reasons else "Not Active"
           for n in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")]
    return ", ".join(["0", str(sm), str(mx), str(power), str(util), "0x0"] + act) + "\n"


def test_clock_summary_and_rejection():
    idle = [_smi(345, 0, power=120)] * 3
    # median SM clock under load; idle samples around the timed region ignored
    c = bench.Clocks.parse(idle + [_smi(1965, 100), _smi(1950, 100), _smi(1965, 99)])
    assert c["sm_mhz"] == 1965 and c["sm_max_mhz"] == 1965 and c["reasons"] == []
    assert c["samples_under_load"] == 3 and c["power_w_max"] == 900
    assert not bench.clock_rejected(c)
    # the power cap is kept (and named); slowdowns reject the region
    c = bench.Clocks.parse([_smi(1800, 100, ["sw_power_cap"])] * 4)
    assert c["reasons"] == ["sw_power_cap"] and not bench.clock_rejected(c)
    for why in bench.REJECTING_REASONS:
        c = bench.Clocks.parse([_smi(1965, 100)] * 3 + [_smi(1200, 100, [why])])
        assert why in c["reasons"] and bench.clock_rejected(c), why
    # clocks held well below the maximum with no reason: a lock left behind
    c = bench.Clocks.parse([_smi(1100, 100)] * 5)
    assert c["reasons"] == [] and bench.clock_rejected(c)
    # no samples (no nvidia-smi): nothing to reject
    assert bench.Clocks.parse(["garbage\n"]) is None and not bench.clock_rejected(None)
    assert bench.any_rank(True, 1) and not bench.any_rank(False, 1)
