"""CPU checks of bench.py's reference arm (the fp64 oracle timed on the host cores): it runs the
requested warm-up and timed steps, each a bounded slice of the workload, and prints the bench's
JSON line with the arm's own cpu_baseline and e2e fields."""
import contextlib
import io
import json

import bench


def test_reference_line_follows_the_contract():
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"]) == 0
    line = json.loads(out.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["steps"] == 3 and line["warmup"] == 3
    assert line["unit"] == "TFLOPS" and line["higher_is_better"] is True
    assert line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["ms_per_step"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "3 timed steps of 256 tokens" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("tiny")
