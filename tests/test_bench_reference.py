"""The reference arm of bench.py (the CPU oracle timed on the host's cores) on the CPU, for the
workloads that are not covered elsewhere: each prints one JSON line with the same metric and
unit as the GPU arm, `impl: reference`, a `cpu_baseline` that describes the run (its thread
count included), and an `e2e` object with no host<->device bytes."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload,threads", [("blocks", 0), ("prefix_chunk", 2), ("window", 2), ("mqa", 1)])
def test_reference_arm_line(workload, threads):
    """threads > 1: one wave of concurrent oracle calls per step; 1: one thread, --ref-seqs sequences."""
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
           "--workload", workload, "--ref-seqs", "1", "--ref-threads", str(threads)]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench

    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["vs_baseline"] is None and line["data"] == "synthetic" and line["scaling"] == "weak"
    assert line["config"]["workload"] == workload
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["unit"] == line["unit"]
    assert cpu["cores"] == (1 if workload == "blocks" else threads) and isinstance(cpu["sample"], str)
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_wave_reports_a_failed_thread(monkeypatch):
    """A host thread whose oracle call raises ends the wave with that thread's own error
    (the other threads are released from the barriers and joined)."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle

    def failing(*args, **kw):
        raise ValueError("planted failure in one oracle call")

    monkeypatch.setattr(oracle, "paged_decode", failing)
    with pytest.raises(RuntimeError, match="planted failure"):
        bench.cpu_oracle_waves("mqa", steps=1, warmup=0, max_threads=2)
