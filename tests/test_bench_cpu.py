"""The bench's reference arm on CPU: the float64 oracle timed on all host
cores (one spawned process per core over rows), printed as one JSON line of
the bench contract."""
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
    # the core count is the number of oracle processes that ran (one per host
    # core unless host memory bounds them), each on one BLAS thread
    assert cb["cores"] == bench.oracle_processes(cfg) <= (os.cpu_count() or 1)
    assert "one process per core" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_clock_summary_parses_nvidia_smi_rows():
    """The clocks record of the JSON line: median SM clock under load, the
    max clock, and every throttle reason seen active."""
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.out = "\n".join([
        "0, 1965, 1965, 650.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 700.3, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ])
    s = c.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    c.out = ""
    assert c.summary() is None


def test_traffic_record_is_used_only_for_the_captured_source(tmp_path):
    """The dominant kernel's ncu traffic is reported only while the kernel's
    source is the one captured; it is scaled by the algorithmic bytes.  The
    committed record, when it matches the current source, shows traffic
    within 1.2x of the algorithmic bytes."""
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "k.cu"
    src.write_bytes(b"kernel source")
    rec = {"source": str(src), "source_sha256": hashlib.sha256(b"kernel source").hexdigest(),
           "dram_bytes": 110, "alg_bytes": 100}
    path = tmp_path / "rec.json"
    path.write_text(json.dumps(rec))
    assert bench.kernel_traffic(200, str(path)) == 220
    src.write_bytes(b"kernel source, edited")
    assert bench.kernel_traffic(200, str(path)) is None
    committed = os.path.join(ROOT, "profiles", "dominant_kernel_traffic.json")
    if os.path.exists(committed):
        c = json.load(open(committed))
        cur = open(os.path.join(ROOT, c["source"]), "rb").read()
        if hashlib.sha256(cur).hexdigest() == c["source_sha256"]:
            assert 1.0 <= c["dram_bytes"] / c["alg_bytes"] < 1.2
        else:
            assert bench.kernel_traffic(c["alg_bytes"]) is None
