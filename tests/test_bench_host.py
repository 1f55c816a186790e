"""Host-side logic of bench.py, on CPU: the reference (oracle) arm's JSON line,
the same arm launched as two ranks (rank 0 alone prints), the clock-sample
window, and the max-over-ranks timing of the replica path over gloo with
world size 2."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, REPO)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _json_lines(out):
    return [json.loads(ln) for ln in out.splitlines() if ln.startswith("{")]


def test_reference_arm_line_on_tiny_workload():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                        "--warmup", "3"], cwd=REPO, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny")


def test_reference_arm_two_ranks_rank0_prints():
    port = _free_port()
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
                        "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       cwd=REPO, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference"


def test_clock_window_keeps_samples_inside_it():
    cs = bench.ClockSampler(0)
    cs.proc = None
    row = "0, {sm}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {cap}"
    cs.lines = [(1.0, row.format(sm=1000, cap="Not Active")), (2.0, row.format(sm=1900, cap="Active")),
                (3.0, row.format(sm=1950, cap="Not Active")), (9.0, row.format(sm=500, cap="Not Active"))]

    class _P:                                       # stands in for the nvidia-smi process
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    class _T:
        def join(self, timeout=None):
            pass

    cs.proc, cs.t = _P(), _T()
    c = cs.stop(1.5, 3.5)
    assert c["samples"] == 2 and c["sm_mhz"] == 1925.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    # a window with no sample inside takes the first sample after it starts
    c = cs.stop(3.2, 3.3)
    assert c["samples"] == 1 and c["sm_mhz"] == 500.0


def _rank_main(rank, world, port, ms_by_rank, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        m = bench.max_over_ranks(ms_by_rank[rank], torch.device("cpu"), world)
        out[rank] = (m, bench.job_throughput(8192, 10, world, m))
    finally:
        dist.destroy_process_group()


def test_replica_timing_is_max_over_ranks_gloo():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    ms = [120.0, 150.0]
    mp.start_processes(_rank_main, args=(world, port, ms, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        m, v = out[r]
        assert m == 150.0
        assert v == pytest.approx(8192 * 10 * 2 / 0.150)
    assert bench.max_over_ranks(42.0, torch.device("cpu"), 1) == 42.0


def test_oracle_baseline_measures_rows_on_their_own():
    """cpu_baseline times the per-query half directly (no difference of two
    timings, no clamp): a positive per-row cost and a rate below the one the
    token-parallel half alone would give."""
    w = bench.synth.workloads()["tiny"]
    tps, info = bench.oracle_baseline(w, budget_s=0.2, chunk=8)
    assert info["rows"] >= 16 and info["per_row_s"] > 0 and info["rows_s"] > 0
    T = sum(w.seqlens)
    assert 0 < tps < T / info["base_s"]
    one = bench.oracle_tiny_one_thread()
    assert one["cores"] == 1 and one["value"] > 0
