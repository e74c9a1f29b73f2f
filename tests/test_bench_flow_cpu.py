"""The bench's control flow on the host (no GPU): bench.main() runs in a
subprocess with the library and CUDA faked (tests/host/bench_flow.py), and its
JSON line must carry every key of the contract.  Catches a workload, runner or
key that the flow breaks, before a GPU run does."""

import json
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
FLOW = os.path.join(HERE, "host", "bench_flow.py")
KEYS = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"]
ROOF = ["bound", "achieved", "peak", "unit", "frac", "traffic"]


def _run(*args):
    res = subprocess.run([sys.executable, FLOW, "--steps", "2", "--warmup", "1", "--no-cpu-baseline", *args],
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    return json.loads(res.stdout.strip().splitlines()[-1])


def test_default_line_has_every_key_and_secondary():
    line = _run()
    assert [k for k in KEYS if k not in line] == []
    assert [k for k in ROOF if k not in line["roofline"]] == []
    assert line["config"]["workload"] == "v2_prefill" and line["roofline"]["traffic"] is not None
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert set(line["secondary"]) == {"v1_prefill", "v2_backward", "v1_backward", "v2_decode", "v2_decode_paged",
                                      "v2_decode_serving", "v1_decode", "v1_decode_unfused", "lowrank_prefill",
                                      "snr_sweep"}
    assert line["secondary_cols"] == ["value", "unit", "ms_per_step", "kernel_ms", "frac", "frac_of_8tbs", "sm_mhz"]
    for name, row in line["secondary"].items():
        assert len(row) == 7 and row[1] in ("TFLOP/s", "GB/s"), name
        assert (row[5] is None) == (row[1] == "TFLOP/s"), name
    assert [r[0] for r in line["snr"]] == [1024, 2048]
    # the rows come last and the whole line stays short, so the end of the
    # output a reader keeps (about 3 KB) holds every row
    assert list(line)[-1] == "secondary"
    assert len(json.dumps(line)) < 2800, len(json.dumps(line))


@pytest.mark.parametrize("workload", ["snr_sweep", "lowrank_prefill", "v2_backward", "v2_decode_paged",
                                      "v2_decode_serving"])
def test_other_workloads(workload):
    line = _run("--workload", workload, "--no-secondary")
    assert [k for k in KEYS if k not in line] == []
    assert line["config"]["workload"] == workload
    if workload in ("snr_sweep", "lowrank_prefill", "v2_backward", "v2_decode_serving"):
        assert "unavailable" in line["e2e"]
    if workload == "snr_sweep":
        assert [r[0] for r in line["snr"]] == [1024, 2048]
