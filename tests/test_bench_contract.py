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


def test_prefill_roofline_counts():
    """The prefill line's algorithmic flop counts, against a count made here
    chunk by chunk from the chunk form's products (a ragged last chunk counts
    its own tokens for the state recurrence and a whole chunk for the output
    kernel, which multiplies whole 64-row tiles), and the fp32 ALU peak's
    derivation (148 SMs x 128 lanes x 2 flops x 1965 MHz = 74.4 TFLOP/s)."""
    sys.path.insert(0, ROOT)
    import bench

    class W:
        N, T, HV, K, V = 3, 150, 2, 128, 128

    w = W()
    chunks = [64, 64, 22]
    state = sum(2 * tc * w.K * w.V + w.K * w.V + 2 * w.K * tc * w.V + tc * w.V for tc in chunks)
    assert bench.prefill_state_flops(w) == w.N * w.HV * state
    out = sum(2 * 64 * w.K * w.V + 2 * 64 * 64 * w.V for _ in chunks)
    assert bench.prefill_output_flops(w) == w.N * w.HV * out
    assert abs(bench.fp32_alu_peak_tflops(148) - 74.4) < 0.05
    assert abs(bench.fp32_alu_peak_tflops(148, 1000.0) - 37.888) < 1e-9
