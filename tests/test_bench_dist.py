"""Multi-process plumbing of bench.py on the CPU (gloo, world size 2): the decode and the
prefill shard by sequence with no exchange, so N GPUs run N independent replicas and the
only collectives are the timing barrier and the max-over-ranks reduction of the elapsed
time.  Checked here: that reduction, the whole-job throughput of the replicas, and the
reference arm (the CPU oracle) printing one JSON line from rank 0 only under torchrun."""
import datetime
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                           timeout=datetime.timedelta(seconds=60))
    import bench

    elapsed = bench.max_over_ranks(10.0 * (rank + 1), torch.device("cpu"))   # rank 1 is the slow one
    thr = bench.job_throughput(100.0, 5, world, elapsed)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, elapsed, thr))


def test_max_over_ranks_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slower rank's time; 2 replicas x 5 steps x 100 units in 20 ms
    assert [r[1] for r in results] == [20.0, 20.0]
    assert all(abs(r[2] - 100.0 * 5 * 2 / 0.020) < 1e-6 for r in results)


def test_max_over_ranks_without_a_process_group_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_throughput(10.0, 2, 1, 1000.0) == 20.0


def test_reference_arm_under_torchrun_prints_from_rank_zero_only():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "3", "--workload", "llama8b", "--ref-seqs", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_clock_summary_of_nvidia_smi_rows():
    sys.path.insert(0, ROOT)
    import bench

    rows = [
        "0, 1965, 1965, 650.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1770, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # unparsable: skipped
        "garbage",
    ]
    got = bench.summarize_clocks(rows)
    assert got == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    slow = bench.summarize_clocks(["0, 1500, 1965, 700, 0x8, Active, Not Active, Active, Not Active"])
    assert slow["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_clocks([]) is None


def test_all_cores_oracle_timing_on_host_threads(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    import oracle

    got = bench.cpu_oracle_all_cores("llama8b", budget_s=0.5, max_threads=2)
    assert set(got) == {"value", "unit", "cores", "sample"}
    assert got["value"] > 0 and got["unit"] == "GB/s" and 1 <= got["cores"] <= 2
    assert bench.cpu_oracle_all_cores("blocks") is None

    def broken(*a, **k):
        raise RuntimeError("planted failure")

    monkeypatch.setattr(oracle, "paged_decode", broken)   # a failing thread ends the measurement, not the bench
    bad = bench.cpu_oracle_all_cores("llama8b", budget_s=0.5, max_threads=2)
    assert "planted failure" in bad["error"]
