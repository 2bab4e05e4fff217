"""The benchmark's JSON line (reference arm, which runs the oracle on the CPU):
every key of the driver's contract, with consistent values."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line_has_the_contract_keys():
    sys.path.insert(0, ROOT)
    import bench

    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3", "--config", "n1_t1_hv8",
                    "--reference-budget-s", "5"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 3
    assert line["higher_is_better"] is False and line["unit"] == "us/call"
    assert abs(line["ms_per_step"] * 1000 - line["value"]) <= 1e-3 * line["value"] + 1e-3
    assert line["config"]["workload"] == "n1_t1_hv8"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_warmup_below_three_is_refused():
    sys.path.insert(0, ROOT)
    import bench
    import pytest

    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1"])
