"""The bench's reference arm on CPU: the float64 oracle timed on the host
cores, printed as one JSON line of the bench contract."""
import contextlib
import io
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    import rlt_inputs as ri
    monkeypatch.setenv("RANK", "0")
    cfg = ri.CONFIGS["tiny_fp32"]
    sample = bench.oracle_sample          # the same leg, on a 2-second sample
    monkeypatch.setattr(bench, "oracle_sample",
                        lambda c, budget_s: sample(c, budget_s=min(budget_s, 2.0)))

    class A:
        steps, warmup, gpus = 1, 0, 2
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(A, cfg)
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["n_gpus"] == 2
    assert line["config"]["global_batch"] == 2 * cfg.batch
    assert line["config"]["workload"].startswith("tiny_fp32")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
